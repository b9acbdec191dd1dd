"""GPU parity of fs_decode_splice_gemm: the decode path (M <= 16) with the activation preparation
(FourSight §5.1 "Data preparation": Mask S->0, FP4 Quant, Extract X_S) done by the GEMM kernel
itself.

The kernel writes the same stage bytes that fs_quantize_splice + TMA would have delivered, so its
output must be BIT-IDENTICAL to fs_quantize_splice followed by the decode-path fs_splice_gemm; it
is also held to the oracle's Eq. 5 bound |Y - Y_ref| <= 1e-5 * sum_k |x_hat_k w_hat_k|.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import splice, stats
from tests._util import bf16_tensor, mask_tensor
from tests.test_gpu_gemm import _assert_close, _problem, _ref, nan_output

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _fused_and_unfused(Xt, Wt, P, gA, p, N, K, residual=False, out_bf16=False):
    opts = F.FS_RESIDUAL if residual else 0
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(Wt, mask, p, g, opts=opts)
    plan = F.Plan(N, K, max(p, 1), F.FS_PATH_DECODE | (F.FS_OUT_BF16 if out_bf16 else 0))
    M = Xt.shape[0]
    Yf = F.fs_decode_splice_gemm(plan, Xt, mask, p, g, wq, alpha, xopts=opts, Y=nan_output(M, N, out_bf16))
    xq = F.fs_quantize_splice(Xt, mask, p, g, opts=opts)
    Yu = F.fs_splice_gemm(plan, xq, wq, alpha, Y=nan_output(M, N, out_bf16))
    plan.check()
    return Yf, Yu


@pytest.mark.parametrize("M,N,K,p", [(1, 1024, 4096, 64), (4, 4096, 4096, 64), (16, 1024, 4096, 64),
                                     (16, 4096, 12288, 64), (7, 256, 512, 0), (16, 512, 1024, 256),
                                     (3, 160, 768, 5), (2, 1024, 4096, 17), (1, 24576, 4096, 64),
                                     (1, 256, 12288, 64), (2, 128, 16384, 64)])
def test_fused_decode_matches_unfused_and_oracle(M, N, K, p):
    """One to sixteen tokens, K = 512 .. 12288, P = {}, a ragged 5 or 17, 64 and 256 channels, a
    ragged last weight tile (N = 160) and the 192-tile gate/up width."""
    X, W, Xt, Wt, P, gA = _problem(500 + M + N + p, M, N, K, p)
    Yf, Yu = _fused_and_unfused(Xt, Wt, P, gA, p, N, K)
    assert torch.equal(Yf, Yu), "fused preparation changed the product"
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Yf, Yr, mag)


@pytest.mark.parametrize("M,p", [(5, 64), (16, 256)])
def test_fused_decode_residual_form_and_bf16_output(M, p):
    N, K = 512, 2048
    X, W, Xt, Wt, P, gA = _problem(530 + M, M, N, K, p, residual=True)
    Yf, Yu = _fused_and_unfused(Xt, Wt, P, gA, p, N, K, residual=True)
    assert torch.equal(Yf, Yu)
    Yr, mag = _ref(X, W, P, gA, residual=True)
    _assert_close(Yf, Yr, mag)
    Yf, Yu = _fused_and_unfused(Xt, Wt, P, gA, p, N, K, residual=True, out_bf16=True)
    assert torch.equal(Yf, Yu)
    _assert_close(Yf, Yr, mag, bf16_out=True)


def test_fused_decode_strided_activations():
    """X read through a leading dimension larger than K (rows of a wider buffer)."""
    M, N, K, p = 6, 1024, 2048, 64
    X, W, Xt, Wt, P, gA = _problem(541, M, N, K, p)
    wide = torch.zeros(M, K + 192, dtype=torch.bfloat16, device="cuda")
    wide[:, 64:64 + K] = Xt
    Xv = wide[:, 64:64 + K]
    Yf, Yu = _fused_and_unfused(Xv, Wt, P, gA, p, N, K)
    assert torch.equal(Yf, Yu)
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Yf, Yr, mag)


@pytest.mark.parametrize("M,seg_rows,p", [(1, [4096, 1024, 1024], 64), (16, [12288, 12288], 64),
                                          (3, [512, 256, 256], 256)])
def test_fused_decode_segmented(M, seg_rows, p):
    """Projections sharing X (q/k/v, gate/up) in one fused launch: bit-identical to the segmented
    call on prepared activations, and every projection within its own oracle bound."""
    K = 4096
    x, _ = synth.outlier_activations(551 + M, M, K)
    X = splice.as_f32(x, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq_all, views = F.stacked_packed(seg_rows, K, p)
    alphas = torch.empty(len(seg_rows), device="cuda")
    Ws = []
    for j, (n, view) in enumerate(zip(seg_rows, views)):
        w = synth.gaussian_weights(560 + j, n, K)
        Ws.append(splice.as_f32(w, True))
        F.fs_prepare_weights(bf16_tensor(w), mask, p, g, out=view, alpha=alphas[j:j + 1])
    seg = np.concatenate([[0], np.cumsum(seg_rows)]).tolist()
    plan = F.Plan(seg[-1], K, p)
    Xt = bf16_tensor(x)
    Yf = F.fs_decode_splice_gemm(plan, Xt, mask, p, g, wq_all, alphas, seg_start=seg, Y=nan_output(M, seg[-1]))
    xq = F.fs_quantize_splice(Xt, mask, p, g)
    Yu = F.fs_splice_gemm_segmented(plan, xq, wq_all, alphas, seg, Y=nan_output(M, seg[-1]))
    plan.check()
    assert torch.equal(Yf, Yu)
    for j in range(len(seg_rows)):
        Yr, mag = _ref(X, Ws[j], P, gA)
        _assert_close(Yf[:, seg[j]:seg[j + 1]], Yr, mag)


def test_fused_decode_repeatable_and_argument_errors():
    M, N, K, p = 16, 2048, 4096, 64
    X, W, Xt, Wt, P, gA = _problem(571, M, N, K, p)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(Wt, mask, p, g)
    plan = F.Plan(N, K, p)
    outs = [F.fs_decode_splice_gemm(plan, Xt, mask, p, g, wq, alpha, Y=nan_output(M, N)) for _ in range(3)]
    plan.check()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    # M > 16, a plan forcing the tensor-core path, unknown xopts, p above p_max: rejected, nothing launched
    big = torch.zeros(17, K, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(F.FoursightError):
        F.fs_decode_splice_gemm(plan, big, mask, p, g, wq, alpha)
    with pytest.raises(F.FoursightError):
        F.fs_decode_splice_gemm(F.Plan(N, K, p, F.FS_PATH_TENSOR), Xt, mask, p, g, wq, alpha)
    with pytest.raises(F.FoursightError):
        F.fs_decode_splice_gemm(plan, Xt, mask, p, g, wq, alpha, xopts=F.FS_COMPACT_K)
    with pytest.raises(F.FoursightError):
        F.fs_decode_splice_gemm(plan, Xt, mask, p + 1, g, wq, alpha)
    # an empty batch is a no-op
    empty = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    assert F.fs_decode_splice_gemm(plan, empty, mask, p, g, wq, alpha).shape == (0, N)
