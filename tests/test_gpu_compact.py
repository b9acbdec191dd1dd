"""GPU parity of the compacted-K variant (FS_COMPACT_K) against the oracle's COMPACT mode.

The protected channels are removed from the NVFP4 operand (blocks re-formed over the unprotected
channels, zero padded to a multiple of 256 columns) instead of zeroed in place.  Quantised bytes,
scales and side columns must be bit-exact; the SpliceGEMM of compacted operands (a plan with
K = fs_compact_cols(K, p)) must meet the stated bound |Y - Y_ref| <= 1e-5 sum |x_hat w_hat| on both
kernels.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import nvfp4, splice, stats
from tests._util import bf16_tensor, check_packed, f32_tensor, mask_tensor

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _inputs(seed, M, K, p, dtype):
    x, _ = synth.outlier_activations(seed, M, K, as_bf16=(dtype == "bf16"))
    X = splice.as_f32(x, dtype == "bf16")
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    return x, X, P, stats.next_gain(st, P)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,p", [(8, 512, 64), (130, 576, 5), (300, 4096, 64), (64, 4096, 256), (16, 12288, 256),
                                   (5, 256, 0), (3, 256, 256)])
def test_compact_quantise_bit_exact(dtype, M, K, p):
    x, X, P, gA = _inputs(31 + M + K, M, K, p, dtype)
    T = bf16_tensor(x) if dtype == "bf16" else f32_tensor(x)
    Kc = F.compact_cols(K, p)
    assert Kc == splice.compact_cols(K, p)
    out = F.fs_quantize_splice(T, mask_tensor(stats.protect_mask(P, K)), p,
                               torch.tensor([float(gA)], device="cuda"), opts=F.FS_COMPACT_K)
    torch.cuda.synchronize()
    ref = splice.quantize_splice(X, P, gA, splice.COMPACT)
    if Kc:
        check_packed(out, ref, M, Kc, p)


@pytest.mark.parametrize("N,K,p", [(256, 512, 64), (384, 4096, 256), (128, 12288, 64)])
def test_compact_prepare_weights_bit_exact(N, K, p):
    _, X, P, gA = _inputs(41 + K, 64, K, p, "bf16")
    w = synth.gaussian_weights(42 + N, N, K)
    out, gW, alpha = F.fs_prepare_weights(bf16_tensor(w), mask_tensor(stats.protect_mask(P, K)), p,
                                          torch.tensor([float(gA)], device="cuda"), opts=F.FS_COMPACT_K)
    ref = splice.prepare_weights(splice.as_f32(w, True), P, gA, splice.COMPACT)
    assert gW.item() == float(ref["gW"]) and alpha.item() == float(ref["alpha"])
    check_packed(out, ref, N, F.compact_cols(K, p), p)


@pytest.mark.parametrize("M,N,K,p,path", [(300, 512, 4096, 256, 16), (16, 1024, 4096, 256, 32), (130, 256, 1024, 64, 16),
                                          (8192, 4096, 4096, 256, 0)])
def test_compact_splice_gemm(M, N, K, p, path):
    x, X, P, gA = _inputs(51 + M, M, K, p, "bf16")
    w = synth.gaussian_weights(52 + N, N, K)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, g, opts=F.FS_COMPACT_K)
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g, opts=F.FS_COMPACT_K)
    Kc = F.compact_cols(K, p)
    plan = F.Plan(N, Kc, p, path)
    Y = torch.full((M, N), float("nan"), device="cuda")
    F.fs_splice_gemm(plan, xq, wq, alpha, Y=Y)
    plan.check()
    rows = np.arange(M) if M <= 512 else np.unique(np.concatenate([[0, M - 1], np.arange(5, M, 128)]))
    xr = splice.quantize_splice(X[rows], P, gA, splice.COMPACT)
    wr = splice.prepare_weights(splice.as_f32(w, True), P, gA, splice.COMPACT)
    Yr, mag = splice.splice_gemm(xr, wr, wr["alpha"])
    got = Y[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.all(np.abs(got - Yr) <= 1e-5 * mag)


def test_compact_rejects_the_residual_form():
    _, X, P, gA = _inputs(3, 8, 512, 16, "bf16")
    with pytest.raises(F.FoursightError):
        F.fs_quantize_splice(bf16_tensor(nvfp4.bf16_bits(X)), mask_tensor(stats.protect_mask(P, 512)), 16,
                             torch.tensor([float(gA)], device="cuda"), opts=F.FS_COMPACT_K | F.FS_RESIDUAL)
