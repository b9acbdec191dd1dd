"""GPU parity of the grouped (mixture-of-experts) path: fs_quantize_splice_grouped and
fs_splice_gemm_grouped against the oracle, expert by expert.

Each expert has its own protected set, activation gain and weights (FourSight §4.2 applies the
protection per projection; §6.3 measures expert projections by tokens per expert).  Experts hold
expert-contiguous routed rows; empty experts and counts around the 128-row tile are included.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import nvfp4, splice, stats
from tests._util import bf16_bits_of, bf16_tensor, mask_tensor, u8

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _build(counts, N, K, p, seed=0):
    E = len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    Xs, Ws, Ps, gAs = [], [], [], []
    for e, n in enumerate(counts):
        x, _ = synth.outlier_activations(seed * 1000 + e, max(int(n), 1), K)
        x = x[: int(n)]
        w = synth.gaussian_weights(seed * 1000 + 500 + e, N, K)
        X = nvfp4.bf16_value(x) if n else np.zeros((0, K), np.float32)
        st = stats.accumulate(stats.new_state(K), X if n else np.zeros((1, K), np.float32))
        P = stats.select_topk(st, p)
        Xs.append(x); Ws.append(w); Ps.append(P); gAs.append(stats.next_gain(st, P))
    return E, offs, Xs, Ws, Ps, gAs


def _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p, plan_opts=0):
    total = int(offs[-1])
    X_all = np.concatenate([x for x in Xs if len(x)]) if total else np.zeros((0, K), np.uint16)
    Xt = bf16_tensor(X_all.reshape(total, K))
    offs_t = torch.from_numpy(offs).cuda()
    masks = mask_tensor(np.stack([stats.protect_mask(P, K) for P in Ps]))
    gA = torch.tensor([float(g) for g in gAs], dtype=torch.float32, device="cuda")
    xq = F.fs_quantize_splice_grouped(Xt, offs_t, masks, p, gA, max_rows=total)
    pp = F.side_cols(p)
    wq_all = torch.empty(E * N, K // 2, dtype=torch.uint8, device="cuda")
    sf_all = torch.empty(F.sf_bytes(E * N, K), dtype=torch.uint8, device="cuda")
    ws_all = torch.zeros(E * N, max(pp, 8), dtype=torch.bfloat16, device="cuda")[:, :pp]
    alpha = torch.empty(E, dtype=torch.float32, device="cuda")
    gW = torch.empty(E, dtype=torch.float32, device="cuda")
    sfb = F.sf_bytes(N, K)
    for e in range(E):
        out = F.Packed(wq_all[e * N:(e + 1) * N], sf_all[e * sfb:(e + 1) * sfb], ws_all[e * N:(e + 1) * N], N, K, p)
        F.fs_prepare_weights(bf16_tensor(Ws[e]), masks[e], p, gA[e:e + 1], out=out, gW=gW[e:e + 1],
                             alpha=alpha[e:e + 1])
    wq = F.Packed(wq_all, sf_all, ws_all, E * N, K, p)
    plan = F.Plan(N, K, max(p, 1), plan_opts)
    # NaN-prefilled output: a row the kernel never writes fails the oracle comparison
    Y = torch.full((max(total, 1), N), float("nan"), device="cuda",
                   dtype=torch.bfloat16 if plan_opts & F.FS_OUT_BF16 else torch.float32)[:total]
    Y = F.fs_splice_gemm_grouped(plan, offs_t, total, xq, wq, alpha, Y=Y)
    plan.check()
    return xq, Y


def _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y, rows_per_expert=None):
    bf16_out = Y.dtype == torch.bfloat16
    Yc = Y.float().cpu().numpy().astype(np.float64)
    for e in range(len(Xs)):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r1 == r0:
            continue
        X = nvfp4.bf16_value(Xs[e])
        W = nvfp4.bf16_value(Ws[e])
        sel = np.arange(r1 - r0) if rows_per_expert is None else np.unique(
            np.linspace(0, r1 - r0 - 1, min(rows_per_expert, r1 - r0)).astype(int))
        xq = splice.quantize_splice(X[sel], Ps[e], gAs[e])
        wq = splice.prepare_weights(W, Ps[e], gAs[e])
        Yr, mag = splice.splice_gemm(xq, wq, wq["alpha"])
        got = Yc[r0 + sel]
        tol = 1e-5 * mag + (2.0 ** -8 * np.abs(Yr) if bf16_out else 0.0)   # + half an ulp of bf16
        assert np.all(np.abs(got - Yr) <= tol), f"expert {e}: outside tolerance"


def test_grouped_small_experts_and_packed_layout():
    counts = [0, 1, 127, 128, 129, 300, 5, 0]
    N, K, p = 256, 512, 16
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=1)
    xq, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p)
    # packed activations: expert e at the padded row offset, padding rows zero
    pad = 0
    q = u8(xq.q)
    sf_tiled = u8(xq.sf)
    side = bf16_bits_of(xq.side)
    for e, n in enumerate(counts):
        if n:
            ref = splice.quantize_splice(nvfp4.bf16_value(Xs[e]), Ps[e], gAs[e])
            assert np.array_equal(q[pad:pad + n], nvfp4.pack_codes(ref["codes"]))
            rr, bb = np.meshgrid(np.arange(n), np.arange(K // 16), indexing="ij")
            assert np.array_equal(sf_tiled[nvfp4.sf_tiled_offset(pad + rr, bb, K)], ref["sf"].astype(np.uint8))
            assert np.array_equal(side[pad:pad + n], nvfp4.bf16_bits(ref["xs"]))
        span = (n + 127) // 128 * 128
        assert not q[pad + n:pad + span].any()
        pad += span
    _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y)


def test_grouped_moe_config_sampled():
    """64 experts, top-8 routing of 4096 tokens with Zipf(1.2) popularity (32768 routed rows),
    up projection 4096 <- 4096 (gate+up) and down projection 4096 <- 2048, P = 64 per expert."""
    counts = synth.moe_routing_counts(0)
    assert counts.sum() == 32768 and counts.max() == 3942
    for (N, K) in ((4096, 4096), (4096, 2048)):
        E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, 64, seed=2)
        _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, 64)
        sub = [0, 1, 7, 31, 63]                     # a few experts, 6 rows each
        Yc = Y.cpu().numpy().astype(np.float64)
        for e in sub:
            r0, r1 = int(offs[e]), int(offs[e + 1])
            sel = np.unique(np.linspace(0, r1 - r0 - 1, 6).astype(int))
            xq = splice.quantize_splice(nvfp4.bf16_value(Xs[e])[sel], Ps[e], gAs[e])
            wq = splice.prepare_weights(nvfp4.bf16_value(Ws[e]), Ps[e], gAs[e])
            Yr, mag = splice.splice_gemm(xq, wq, wq["alpha"])
            assert np.all(np.abs(Yc[r0 + sel] - Yr) <= 1e-5 * mag), f"expert {e} (N={N}, K={K})"


@pytest.mark.parametrize("N", [512, 384])
def test_grouped_more_tiles_than_sms_side_heavy(N):
    """Enough tiles (> 148) that every CTA runs several, with p = 256 so that four BF16 k-tiles
    follow two FP4 k-tiles; N = 512 takes 256-column tiles, N = 384 128-column tiles."""
    counts = [300, 200, 129] * 20
    K, p = 512, 256
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=3)
    _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p)
    _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y, rows_per_expert=6)


@pytest.mark.parametrize("N", [256, 384])
def test_grouped_partial_tiles_bf16_output(N):
    """Experts whose last tile ends inside a 32-row warp group, at a warp boundary and after one
    row, with bf16 output: warps whose rows all belong to the expert store whole boxes, the warp
    holding the expert's last row stores row by row, and nothing spills into the next expert."""
    counts = [1, 127, 129, 32, 0, 64, 95, 160, 31]
    K, p = 512, 16
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=4)
    _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p, plan_opts=F.FS_OUT_BF16)
    assert Y.dtype == torch.bfloat16
    _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y)


# ---------------------------------------------------------------- small experts on the decode kernel
@pytest.mark.parametrize("counts,N,K,p", [
    ([0, 1, 3, 16, 17, 40, 200, 5, 0, 9], 256, 1024, 64),     # mixed: both kernels
    ([1, 0, 4, 2, 5, 0, 3, 1], 384, 2048, 64),                # max_rows <= 16: the decode kernel alone
    ([16, 16, 2, 7], 256, 512, 256),                          # K split over a cluster, four side k-tiles
    ([3, 11, 0, 16, 1], 128, 4096, 0),                        # P = {} (no side k-tiles), one 128-row tile
])
def test_grouped_small_experts_take_the_decode_kernel(counts, N, K, p):
    """FS_PATH_DECODE: experts of 1..16 rows run on the weight-streaming decode kernel (their
    tokens as the 16 MMA columns, read from the expert's padded rows), larger ones on the
    tensor-core kernel.  Every expert's rows are checked against the oracle, and the default
    (every expert on the tensor-core kernel) against it too."""
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=6)
    for opts in (F.FS_PATH_DECODE, 0):
        _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p, plan_opts=opts)
        _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y)


def test_grouped_decode_routing_forced_and_bf16():
    """FS_PATH_DECODE sends the small experts of a large batch to the decode kernel, and
    FS_PATH_TENSOR keeps every expert on the tensor-core kernel; both match the oracle, with bf16
    output on the decode path."""
    counts = [0, 1, 127, 128, 129, 300, 5, 16, 17]
    N, K, p = 256, 512, 16
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=7)
    for opts in (F.FS_PATH_DECODE, F.FS_PATH_TENSOR, F.FS_PATH_DECODE | F.FS_OUT_BF16):
        _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p, plan_opts=opts)
        _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y)


def test_grouped_decode_moe_batch():
    """A decode step of a 64-expert layer: 16 tokens routed top-8 (128 rows, Zipf(1.2) popularity),
    up projection 4096 <- 4096: most experts get 0-4 rows, the popular ones more than 16."""
    rng = np.random.default_rng(11)
    w = 1.0 / np.arange(1, 65) ** 1.2
    counts = rng.multinomial(128, w / w.sum()).tolist()
    assert max(counts) > 16 and min(counts) == 0
    N, K, p = 4096, 4096, 64
    E, offs, Xs, Ws, Ps, gAs = _build(counts, N, K, p, seed=8)
    _, Y = _run_gpu(E, offs, Xs, Ws, Ps, gAs, N, K, p, plan_opts=F.FS_PATH_DECODE)
    _check_expert_outputs(offs, Xs, Ws, Ps, gAs, Y, rows_per_expert=4)
