"""fs_splice_gemm_noalloc, the plan-free SpliceGEMM for callers that cannot allocate device memory
(allocator callbacks, arena-only runtimes, plugins that forbid allocations after start-up).

Called through the C ABI and compared with fs_splice_gemm on the same packed operands, on two calls
in a row (the shared scratch word keeps the previous call's contents and must be cleared).  This file
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
    g = torch.tensor([float(stats.next_gain(st, P))], device="cuda")
    wq, _, alpha = F.fs_prepare_weights(bf16_tensor(w), mask, p, g)
    xq = F.fs_quantize_splice(bf16_tensor(x), mask, p, g)
    return xq, wq, alpha


@pytest.mark.parametrize("M,N,K,p", [(8, 512, 1024, 64), (300, 1024, 4096, 64), (129, 384, 512, 0)])
def test_noalloc_matches_planned_call_twice(M, N, K, p):
    lib = F.load()
    xq, wq, alpha = _packed(5 + M, M, N, K, p)
    plan = F.Plan(N, K, max(p, 1))
    Y_ref = F.fs_splice_gemm(plan, xq, wq, alpha)
    plan.check()
    ref = Y_ref.cpu().numpy().astype(np.float64)
    s = torch.cuda.current_stream().cuda_stream
    mag = np.abs(ref) + 1e-30
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.fs_splice_gemm_noalloc(N, K, 0, M, p, xq.q.data_ptr(), xq.sf.data_ptr(),
                                        xq.side.data_ptr() if p else None, wq.q.data_ptr(), wq.sf.data_ptr(),
                                        wq.side.data_ptr() if p else None, alpha.data_ptr(), Y.data_ptr(), N,
                                        1, s)
        assert st == 0, lib.fs_last_error()
        got = Y.cpu().numpy().astype(np.float64)
        # same kernels on the same operands: equal up to the 1e-5 relative tolerance the tests use
        assert np.all(np.abs(got - ref) <= 1e-5 * mag), f"call {call} differs from fs_splice_gemm"


def test_noalloc_rejects_unsupported_shapes():
    lib = F.load()
    dummy = 256
    assert lib.fs_splice_gemm_noalloc(100, 4096, 0, 8, 0, dummy, dummy, None, dummy, dummy, None, dummy, dummy,
                                      112, 0, None) == 1
    assert lib.fs_splice_gemm_noalloc(128, 320, 0, 8, 0, dummy, dummy, None, dummy, dummy, None, dummy, dummy,
                                      128, 0, None) == 2
    assert b"K" in lib.fs_last_error()
