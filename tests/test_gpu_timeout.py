"""Failure detection of the GEMM kernels: a bounded wait that runs out is reported, not hung on.

Every mbarrier wait in the tensor-core and decode kernels is bounded; when one gives up the kernel
sets the plan's error word, stops issuing work, waits (bounded) for its own copies in flight,
releases its tensor memory and returns, and fs_plan_check reports FS_ERR_TIMEOUT.  The failure is
made on the host side: a plan created with FS_FAULT_NO_COPIES launches kernels whose producers issue
no copies (a "flag that nothing sets") and whose waits are limited to 20 ms.  Nothing is removed
from the kernels; no copy is ever in flight when they abort.  After the timeout the same context
must still compute correct results, which a normal plan then checks against the oracle.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import splice, stats
from tests._util import bf16_tensor, mask_tensor

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _operands(seed, M, N, K, p):
    x, _ = synth.outlier_activations(seed, M, K)
    w = synth.gaussian_weights(seed + 1, N, K)
    X, W = splice.as_f32(x, True), splice.as_f32(w, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, g)
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g)
    xr = splice.quantize_splice(X, P, gA)
    wr = splice.prepare_weights(W, P, gA)
    Yr, mag = splice.splice_gemm(xr, wr, wr["alpha"])
    return xq, wq, alpha, Yr, mag


@pytest.mark.parametrize("path,M,N", [("tensor", 128, 256), ("tensor", 512, 512), ("decode", 4, 256)])
def test_wait_runs_out_then_context_still_computes(path, M, N):
    """One 128-row tile on one CTA, CTA pairs (512 x 512), and the decode kernel (K split over a
    cluster): the starved launch reports FS_ERR_TIMEOUT once, the word is cleared by the check, and
    a normal launch on the same context matches the oracle."""
    K, p = 512, 64
    xq, wq, alpha, Yr, mag = _operands(11 + M, M, N, K, p)
    force = F.FS_PATH_TENSOR if path == "tensor" else F.FS_PATH_DECODE
    starved = F.Plan(N, K, p, force | F.FS_FAULT_NO_COPIES)
    F.fs_splice_gemm(starved, xq, wq, alpha)
    with pytest.raises(F.FoursightError) as exc:
        starved.check()
    assert exc.value.status == 5, str(exc.value)            # FS_ERR_TIMEOUT
    starved.check()                                          # the word was cleared by the report
    good = F.Plan(N, K, p, force)
    Y = torch.full((M, N), float("nan"), device="cuda")
    F.fs_splice_gemm(good, xq, wq, alpha, Y=Y)
    good.check()
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - Yr) <= 1e-5 * mag)


def test_stats_range_flag_is_reported():
    """The other device-side condition: a statistics input out of range raises FS_ERR_RANGE
    through fs_stats_check and adds nothing to the moments."""
    K = 64
    x = np.ones((4, K), np.float32)
    x[2, 5] = 40000.0                                        # >= 2^15
    st = F.StatsState(1, K)
    F.fs_channel_stats(torch.from_numpy(x).cuda(), st)
    with pytest.raises(F.FoursightError) as exc:
        F.fs_stats_check(st)
    assert exc.value.status == 4
    ref = stats.accumulate(stats.new_state(K), x)
    assert ref["flags"] == 1
    assert np.array_equal(st.s1[0].cpu().numpy(), ref["s1"]) and np.array_equal(st.s2[0].cpu().numpy(), ref["s2"])


def test_fused_decode_wait_runs_out_then_context_still_computes():
    """The decode kernel with the activation preparation inside (fs_decode_splice_gemm): with no
    weight copies issued, the MMA thread's waits run out while the preparing warps, which fill the
    first stages and then wait for a stage to be released, give up theirs; the launch reports
    FS_ERR_TIMEOUT and a normal fused launch afterwards matches the oracle.  K = 8192 gives every
    CTA of the cluster four FP4 k-tiles, more than its three stages."""
    M, N, K, p = 4, 256, 8192, 64
    x, _ = synth.outlier_activations(71, M, K)
    w = synth.gaussian_weights(72, N, K)
    X, W = splice.as_f32(x, True), splice.as_f32(w, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    mask = mask_tensor(stats.protect_mask(P, K))
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, g)
    Xt = bf16_tensor(x)
    starved = F.Plan(N, K, p, F.FS_PATH_DECODE | F.FS_FAULT_NO_COPIES)
    F.fs_decode_splice_gemm(starved, Xt, mask, p, g, wq, alpha)
    with pytest.raises(F.FoursightError) as exc:
        starved.check()
    assert exc.value.status == 5, str(exc.value)
    good = F.Plan(N, K, p, F.FS_PATH_DECODE)
    Y = F.fs_decode_splice_gemm(good, Xt, mask, p, g, wq, alpha,
                                Y=torch.full((M, N), float("nan"), device="cuda"))
    good.check()
    xr = splice.quantize_splice(X, P, gA)
    wr = splice.prepare_weights(W, P, gA)
    Yr, mag = splice.splice_gemm(xr, wr, wr["alpha"])
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - Yr) <= 1e-5 * mag)
