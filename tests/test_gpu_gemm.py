"""GPU parity of fs_splice_gemm (both paths) against the oracle's Eq. 5 in float64.

Tolerance (the stated bound): |Y - Y_ref| <= 1e-5 * sum_k |x_hat_k w_hat_k| per element, with the
hats the oracle's dequantised operands; a bf16 output adds its own rounding, 2^-8 |Y_ref|.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import nvfp4, splice, stats
from tests._util import bf16_tensor, f32_tensor, mask_tensor

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")

REL = 1e-5


def _problem(seed, M, N, K, p, dtype="bf16", residual=False, calib_rows=None):
    bf = dtype == "bf16"
    x, _ = synth.outlier_activations(seed, M, K, as_bf16=bf)
    w = synth.gaussian_weights(seed + 1, N, K, as_bf16=bf)
    X, W = splice.as_f32(x, bf), splice.as_f32(w, bf)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P, residual=residual)
    Xt = bf16_tensor(x) if bf else f32_tensor(x)
    Wt = bf16_tensor(w) if bf else f32_tensor(w)
    return X, W, Xt, Wt, P, gA


def nan_output(M, N, bf16=False):
    """Output buffer prefilled with NaN, so that an element the kernel never writes fails the check."""
    return torch.full((M, N), float("nan"), dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")


def _run_gpu(Xt, Wt, P, gA, p, N, K, opts=0, plan_opts=0):
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, gW, alpha = F.fs_prepare_weights(Wt, mask, p, g, opts=opts)
    xq = F.fs_quantize_splice(Xt, mask, p, g, opts=opts)
    plan = F.Plan(N, K, max(p, 1), plan_opts)
    Y = F.fs_splice_gemm(plan, xq, wq, alpha, Y=nan_output(Xt.shape[0], N, bool(plan_opts & F.FS_OUT_BF16)))
    plan.check()
    return Y, plan


def _ref(X, W, P, gA, residual=False, rows=None):
    mode = splice.RESIDUAL if residual else splice.SPLIT
    xq = splice.quantize_splice(X if rows is None else X[rows], P, gA, mode)
    wq = splice.prepare_weights(W, P, gA, mode)
    return splice.splice_gemm(xq, wq, wq["alpha"])


def _assert_close(Y, Yr, mag, bf16_out=False):
    Yg = Y.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(Yg).all(), f"{(~np.isfinite(Yg)).sum()} outputs not finite (unwritten or overflowed)"
    tol = REL * mag + (2.0 ** -8 * np.abs(Yr) if bf16_out else 0.0)
    bad = ~(np.abs(Yg - Yr) <= tol)
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside tolerance; worst excess "
                           f"{np.max(np.abs(Yg - Yr) - tol):.3e} at {np.unravel_index(np.argmax(np.abs(Yg - Yr) - tol), Yr.shape)}")


def test_single_projection_case_both_paths():
    """X 8x512 fp32 with 8 outlier channels x50, W 256x512, P = top-64 variance channels."""
    x, w, _ = synth.single_projection(0)
    st = stats.accumulate(stats.new_state(512), x)
    P = stats.select_topk(st, 64)
    gA = stats.next_gain(st, P)
    Yr, mag = _ref(x, w, P, gA)
    for path in (F.FS_PATH_DECODE, F.FS_PATH_TENSOR):
        Y, _ = _run_gpu(f32_tensor(x), f32_tensor(w), P, gA, 64, 256, 512, plan_opts=path)
        _assert_close(Y, Yr, mag)


@pytest.mark.parametrize("M,N,K,p", [(1, 1024, 4096, 64), (4, 4096, 4096, 64), (16, 1024, 4096, 64),
                                     (16, 4096, 12288, 64), (7, 256, 512, 0), (16, 512, 1024, 256),
                                     (3, 160, 768, 5)])
def test_decode_path(M, N, K, p):
    X, W, Xt, Wt, P, gA = _problem(40 + M + N, M, N, K, p)
    Y, _ = _run_gpu(Xt, Wt, P, gA, p, N, K, plan_opts=F.FS_PATH_DECODE)
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Y, Yr, mag)


@pytest.mark.parametrize("M,N,K,p", [(16, 128, 12288, 64), (5, 384, 4096, 64), (1, 24576, 4096, 64),
                                     (2, 1024, 4096, 256), (9, 144, 256, 16)])
def test_decode_split_k_is_summed_in_order_and_repeatable(M, N, K, p):
    """The decode kernel splits each tile's K range over the CTAs of a cluster and sums their
    partials in rank order (one tile of K = 12288; three tiles; 192 tiles; the BF16 k-tiles of
    P = 256; a ragged last tile): three launches in a row give bit-identical outputs, all within
    the oracle's bound."""
    X, W, Xt, Wt, P, gA = _problem(60 + M + N, M, N, K, p)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(Wt, mask, p, g)
    xq = F.fs_quantize_splice(Xt, mask, p, g)
    plan = F.Plan(N, K, max(p, 1), F.FS_PATH_DECODE)
    outs = []
    for _ in range(3):
        outs.append(F.fs_splice_gemm(plan, xq, wq, alpha, Y=nan_output(M, N)))
    plan.check()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(outs[0], Yr, mag)


@pytest.mark.parametrize("M,N,K,p", [(128, 256, 256, 0), (128, 256, 512, 64), (300, 1024, 4096, 64),
                                     (17, 384, 1024, 64), (1000, 512, 2048, 256), (256, 128, 768, 16),
                                     (200, 768, 4096, 5), (129, 256, 12288, 64)])
def test_tensor_core_path(M, N, K, p):
    X, W, Xt, Wt, P, gA = _problem(70 + M + N + K, M, N, K, p)
    Y, _ = _run_gpu(Xt, Wt, P, gA, p, N, K, plan_opts=F.FS_PATH_TENSOR)
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Y, Yr, mag)


@pytest.mark.parametrize("path", ["decode", "tensor"])
def test_residual_form_and_bf16_output(path):
    M = 8 if path == "decode" else 160
    X, W, Xt, Wt, P, gA = _problem(90, M, 512, 1024, 64, residual=True)
    popts = (F.FS_PATH_DECODE if path == "decode" else F.FS_PATH_TENSOR) | F.FS_OUT_BF16
    Y, _ = _run_gpu(Xt, Wt, P, gA, 64, 512, 1024, opts=F.FS_RESIDUAL, plan_opts=popts)
    assert Y.dtype == torch.bfloat16
    Yr, mag = _ref(X, W, P, gA, residual=True)
    _assert_close(Y, Yr, mag, bf16_out=True)


def test_paths_agree_on_the_same_inputs():
    X, W, Xt, Wt, P, gA = _problem(91, 16, 1024, 4096, 64)
    Yd, _ = _run_gpu(Xt, Wt, P, gA, 64, 1024, 4096, plan_opts=F.FS_PATH_DECODE)
    Yt, _ = _run_gpu(Xt, Wt, P, gA, 64, 1024, 4096, plan_opts=F.FS_PATH_TENSOR)
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Yd, Yr, mag)
    _assert_close(Yt, Yr, mag)


def _row_per_tile(M, seed):
    """One random row in every 128-row tile (first and last rows included): each output tile of
    the launch, and each CTA of a pair, contributes a checked row."""
    rng = np.random.default_rng(seed)
    rows = np.array([t + rng.integers(0, min(128, M - t)) for t in range(0, M, 128)])
    return np.unique(np.concatenate([[0, M - 1], rows]))


def test_full_size_prefill_all_rows_q():
    """The q projection as timed (M = 8192, N = K = 4096, P = 64): every one of the 8192 x 4096
    outputs against the oracle's float64 Eq. 5."""
    M, N, K, p = 8192, 4096, 4096, 64
    X, W, Xt, Wt, P, gA = _problem(7, M, N, K, p)
    Y, _ = _run_gpu(Xt, Wt, P, gA, p, N, K)
    Yr, mag = _ref(X, W, P, gA)
    _assert_close(Y, Yr, mag)


@pytest.mark.parametrize("N,K,p", [(1024, 4096, 64), (12288, 4096, 64), (4096, 12288, 64), (4096, 4096, 256),
                                   (4096, 12288, 256)])
def test_full_size_prefill_rows_of_every_tile(N, K, p):
    """M = 8192 tokens as timed (P = 64, and the P = 256 budget); the oracle checks one row of
    every 128-row tile, so every row tile and both CTAs of every pair are covered."""
    M = 8192
    X, W, Xt, Wt, P, gA = _problem(7, M, N, K, p)
    Y, _ = _run_gpu(Xt, Wt, P, gA, p, N, K)
    rows = _row_per_tile(M, N + K + p)
    Yr, mag = _ref(X, W, P, gA, rows=rows)
    _assert_close(Y[torch.from_numpy(rows).cuda()], Yr, mag)


@pytest.mark.parametrize("M,N,K,p", [(4096, 2048, 1024, 256), (2000, 1536, 2048, 130)])
def test_tensor_core_pairs_several_tiles_sampled_rows(M, N, K, p):
    """More 256 x 256 tiles than CTA pairs, so pairs run several tiles (both accumulator
    positions); p = 256 puts four BF16 k-tiles after every four FP4 k-tiles.  Sampled rows
    include both sides of every 128-row boundary of the first tiles and the ragged end."""
    X, W, Xt, Wt, P, gA = _problem(93 + M, M, N, K, p)
    Y, _ = _run_gpu(Xt, Wt, P, gA, p, N, K, plan_opts=F.FS_PATH_TENSOR)
    rng = np.random.default_rng(M + N)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, 383, 384, M - 1],
                                     rng.choice(M, 40, replace=False)]))
    Yr, mag = _ref(X, W, P, gA, rows=rows)
    _assert_close(Y[torch.from_numpy(rows).cuda()], Yr, mag)


@pytest.mark.parametrize("path,M", [("decode", 8), ("tensor", 300)])
def test_segmented_projections_match_each_projection(path, M):
    """Three projections sharing X and P (a q/k/v-like group), stacked by rows (512, 256, 256),
    each with its own weights and weight gain: one segmented launch reproduces every projection's
    own oracle result in its columns of Y."""
    K, p, seg_rows = 1024, 64, [512, 256, 256]
    x, _ = synth.outlier_activations(201, M, K)
    X = splice.as_f32(x, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g)
    wq_all, views = F.stacked_packed(seg_rows, K, p)
    alphas = torch.empty(len(seg_rows), device="cuda")
    Ws = []
    for j, (n, view) in enumerate(zip(seg_rows, views)):
        w = synth.gaussian_weights(300 + j, n, K)
        Ws.append(splice.as_f32(w, True))
        F.fs_prepare_weights(bf16_tensor(w), mask, p, g, out=view, alpha=alphas[j:j + 1])
    seg = np.concatenate([[0], np.cumsum(seg_rows)]).tolist()
    plan = F.Plan(seg[-1], K, p, F.FS_PATH_DECODE if path == "decode" else F.FS_PATH_TENSOR)
    Y = F.fs_splice_gemm_segmented(plan, xq, wq_all, alphas, seg, Y=nan_output(M, seg[-1]))
    plan.check()
    for j in range(len(seg_rows)):
        Yr, mag = _ref(X, Ws[j], P, gA)
        _assert_close(Y[:, seg[j]:seg[j + 1]], Yr, mag)
    # boundaries must keep every tile inside one segment, start at 0 and end at N
    for bad in ([0, 384, 768, 1024], [0, 512, 768, 1000], [256, 512, 768, 1024]):
        with pytest.raises(F.FoursightError):
            F.fs_splice_gemm_segmented(plan, xq, wq_all, alphas, bad)


@pytest.mark.parametrize("M,seg_rows,p", [(8192, [4096, 1024, 1024], 64), (8192, [12288, 12288], 64),
                                          (16, [4096, 1024, 1024], 64), (8192, [4096, 1024, 1024], 256)])
def test_full_size_segmented_sampled_rows(M, seg_rows, p):
    """The launches bench.py times: M = 8192 tokens (tensor-core path) or 16 (decode path), K =
    4096, the q/k/v (or gate/up) weights stacked in one segmented launch; the oracle checks one
    row of every 128-row tile (all rows at M = 16) of every projection; the qkv launch also at the
    P = 256 budget."""
    K = 4096
    x, _ = synth.outlier_activations(211, M, K)
    X = splice.as_f32(x, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g)
    wq_all, views = F.stacked_packed(seg_rows, K, p)
    alphas = torch.empty(len(seg_rows), device="cuda")
    Ws = []
    for j, (n, view) in enumerate(zip(seg_rows, views)):
        w = synth.gaussian_weights(400 + j, n, K)
        Ws.append(splice.as_f32(w, True))
        F.fs_prepare_weights(bf16_tensor(w), mask, p, g, out=view, alpha=alphas[j:j + 1])
    seg = np.concatenate([[0], np.cumsum(seg_rows)]).tolist()
    plan = F.Plan(seg[-1], K, p)
    Y = F.fs_splice_gemm_segmented(plan, xq, wq_all, alphas, seg, Y=nan_output(M, seg[-1]))
    plan.check()
    rows = np.arange(M) if M <= 40 else _row_per_tile(M, seg[-1])
    rows_t = torch.from_numpy(rows).cuda()
    for j in range(len(seg_rows)):
        Yr, mag = _ref(X, Ws[j], P, gA, rows=rows)
        _assert_close(Y[rows_t, seg[j]:seg[j + 1]], Yr, mag)


def test_empty_batches_are_no_ops():
    """M = 0 tokens (and a grouped call with no routed rows): every call succeeds, reads nothing and
    returns an empty output; the statistics state is untouched."""
    K, N, p = 512, 512, 64
    X, W, Xt, Wt, P, gA = _problem(5, 8, N, K, p)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(Wt, mask, p, g)
    empty = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    st = F.StatsState(1, K)
    F.fs_channel_stats(empty, st)
    assert int(st.n.item()) == 0 and not st.s1.any() and not st.s2.any()
    xq = F.fs_quantize_splice(empty, mask, p, g)
    assert xq.rows == 0
    plan = F.Plan(N, K, p)
    assert F.fs_splice_gemm(plan, xq, wq, alpha).shape == (0, N)
    assert F.fs_splice_gemm_segmented(plan, xq, wq, alpha.repeat(2), [0, 256, N]).shape == (0, N)
    offs = torch.zeros(3, dtype=torch.int64, device="cuda")
    assert F.fs_splice_gemm_grouped(plan, offs, 0, xq, wq, alpha.repeat(2)).shape == (0, N)
    plan.check()


def test_repeatable_and_overwrites_output():
    X, W, Xt, Wt, P, gA = _problem(92, 256, 512, 1024, 64)
    Y1, _ = _run_gpu(Xt, Wt, P, gA, 64, 512, 1024)
    Y2, _ = _run_gpu(Xt, Wt, P, gA, 64, 512, 1024)
    assert torch.equal(Y1, Y2)
    assert torch.isfinite(Y1).all()
