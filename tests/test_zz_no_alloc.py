"""fs_splice_gemm_noalloc, the plan-free SpliceGEMM for callers that cannot allocate device memory
(allocator callbacks, arena-only runtimes, plugins that forbid allocations after start-up).

Called through the C ABI and compared with fs_splice_gemm and with the oracle on the same packed
operands, on two calls in a row (the shared scratch word keeps the previous call's contents and must be
cleared); a call that gives up its waits (the failure-detection test option) must be reported and must
not leak its timeout into the next call.  This file
is collected last so that a run that stops at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import splice, stats
from tests._util import bf16_tensor, mask_tensor

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _packed(seed, M, N, K, p):
    x, _ = synth.outlier_activations(seed, M, K)
    w = synth.gaussian_weights(seed + 1, N, K)
    X = splice.as_f32(x, True)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    mask = mask_tensor(stats.protect_mask(P, K))
    gA = stats.next_gain(st, P)
    g = torch.tensor([float(gA)], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, g)
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g)
    return xq, wq, alpha, (X, splice.as_f32(w, True), P, gA)


def _call(lib, N, K, opts, M, p, xq, wq, alpha, Y, check):
    return lib.fs_splice_gemm_noalloc(N, K, opts, M, p, xq.q.data_ptr(), xq.sf.data_ptr(),
                                      xq.side.data_ptr() if p else None, wq.q.data_ptr(), wq.sf.data_ptr(),
                                      wq.side.data_ptr() if p else None, alpha.data_ptr(), Y.data_ptr(), N,
                                      check, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K,p", [(8, 512, 1024, 64), (300, 1024, 4096, 64), (129, 384, 512, 0)])
def test_noalloc_matches_planned_call_twice(M, N, K, p):
    lib = F.load()
    xq, wq, alpha, (X, W, P, gA) = _packed(5 + M, M, N, K, p)
    plan = F.Plan(N, K, max(p, 1))
    Y_ref = F.fs_splice_gemm(plan, xq, wq, alpha)
    plan.check()
    ref = Y_ref.cpu().numpy().astype(np.float64)
    xr = splice.quantize_splice(X, P, gA)
    wr = splice.prepare_weights(W, P, gA)
    Yo, mag_o = splice.splice_gemm(xr, wr, wr["alpha"])
    # the two calls run the same kernels; both are held to the bound every GEMM test uses,
    # 1e-5 * sum_k |x_hat_k w_hat_k|, against the oracle and against each other
    mag = mag_o
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = _call(lib, N, K, 0, M, p, xq, wq, alpha, Y, 1)
        assert st == 0, lib.fs_last_error()
        got = Y.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= 2e-5 * mag), f"call {call} differs from fs_splice_gemm"
        # and within the oracle's bound, like every other GEMM parity test
        assert np.all(np.abs(got - Yo) <= 1e-5 * mag_o), f"call {call} outside the oracle bound"


@pytest.mark.parametrize("path", [0, 32])        # tensor-core kernel (M = 300), decode kernel (M = 8)
def test_noalloc_timeout_is_reported_and_cleared(path):
    """The shared scratch word keeps the last call's contents.  A call with FS_FAULT_NO_COPIES (the
    failure-detection test option: no copies issued, 20 ms wait limit) sets it and reports
    FS_ERR_TIMEOUT; the next normal call must clear it first and report FS_OK with a correct result."""
    lib = F.load()
    M = 8 if path else 300
    N, K, p = 512, 1024, 64
    xq, wq, alpha, (X, W, P, gA) = _packed(77 + M, M, N, K, p)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    assert _call(lib, N, K, path | F.FS_FAULT_NO_COPIES, M, p, xq, wq, alpha, Y, 1) == 5
    plan = F.Plan(N, K, p, path)
    Y_ref = F.fs_splice_gemm(plan, xq, wq, alpha)
    plan.check()
    assert _call(lib, N, K, path, M, p, xq, wq, alpha, Y, 1) == 0, lib.fs_last_error()
    ref = Y_ref.cpu().numpy().astype(np.float64)
    xr = splice.quantize_splice(X, P, gA)
    wr = splice.prepare_weights(W, P, gA)
    Yo, mag = splice.splice_gemm(xr, wr, wr["alpha"])
    got = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - Yo) <= 1e-5 * mag) and np.all(np.abs(got - ref) <= 2e-5 * mag)


def test_noalloc_rejects_unsupported_shapes():
    lib = F.load()
    dummy = 256
    assert lib.fs_splice_gemm_noalloc(100, 4096, 0, 8, 0, dummy, dummy, None, dummy, dummy, None, dummy, dummy,
                                      112, 0, None) == 1
    assert lib.fs_splice_gemm_noalloc(128, 320, 0, 8, 0, dummy, dummy, None, dummy, dummy, None, dummy, dummy,
                                      128, 0, None) == 2
    assert b"K" in lib.fs_last_error()
