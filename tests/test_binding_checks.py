"""The Python binding's extent checks: the C ABI takes plain pointers, so the binding compares the
tensors' shapes with what each call reads or writes and refuses a short or mistyped buffer before
anything is launched.

These run on the CPU: the library's launching entries are replaced by no-ops (the host-only size
helpers stay real), so the bench's own step, with its real buffers, passes through every check,
and each kind of wrong buffer raises ValueError without reaching the library.
"""
import pytest
import torch

import bench
import nvfp4_w4a4_gemm_fs_b200 as F
from nvfp4_w4a4_gemm_fs_b200 import _lib

HOST_ONLY = {"fs_sf_bytes", "fs_side_cols", "fs_grouped_rows", "fs_compact_cols", "fs_status_string",
             "fs_last_error", "fs_version", "fs_ste_backward_work_bytes", "fs_k3_work_bytes"}


@pytest.fixture
def no_launch(monkeypatch):
    real = _lib.load()
    calls = []

    class Fake:
        def __getattr__(self, name):
            if name in HOST_ONLY:
                return getattr(real, name)

            def fn(*args):
                calls.append(name)
                return 0                                        # FS_OK, nothing launched
            return fn
    monkeypatch.setattr(_lib, "load", lambda: Fake())
    monkeypatch.setattr(F.foursight, "stream_handle", lambda stream=None: 0)   # no CUDA stream here
    return calls


@pytest.mark.parametrize("fused,compact,p,out_bf16,fused_prep", [(True, False, 64, False, False),
                                                                 (False, False, 64, False, False),
                                                                 (True, True, 256, False, False),
                                                                 (True, False, 0, True, False),
                                                                 (True, False, 64, False, True)])
def test_the_bench_step_passes_every_check(no_launch, fused, compact, p, out_bf16, fused_prep):
    lay = bench.PrefillLayer(F, 256, p, seed=1, device="cpu", out_bf16=out_bf16, fused=fused, compact=compact,
                             fused_prep=fused_prep)
    lay.step()
    assert "fs_splice_gemm_segmented" in no_launch or "fs_splice_gemm" in no_launch


@pytest.mark.parametrize("M,K,p", [(8, 512, 64), (3, 256, 256), (5, 256, 0), (0, 512, 16), (16, 12288, 256)])
def test_quantise_and_pre_split_outputs_pass_every_check(no_launch, M, K, p):
    """The binding's own outputs in every form: split and compacted K, p = 0, p = K (a compacted
    operand of no NVFP4 columns), an empty batch."""
    mask = torch.zeros((K + 31) // 32, dtype=torch.int32)
    gA = torch.ones(1)
    for opts in (0, F.FS_COMPACT_K):
        F.fs_quantize_splice(torch.zeros(M, K, dtype=torch.bfloat16), mask, p, gA, opts=opts)
        F.fs_quantize_splice(torch.zeros(M, K, dtype=torch.float32), mask, p, gA, opts=opts)
        F.fs_prepare_weights(torch.zeros(max(M, 128), K, dtype=torch.bfloat16), mask, p, gA, opts=opts)
    F.fs_quantize_splice_stats(torch.zeros(M, K, dtype=torch.bfloat16), mask, p, gA, F.StatsState(1, K, device="cpu"))


def test_decode_shaped_calls_pass_every_check(no_launch):
    K, p, M = 4096, 64, 16
    rows = [4096, 1024, 1024]
    wall, views = F.stacked_packed(rows, K, p, "cpu")
    alpha = torch.zeros(3)
    mask = torch.zeros(K // 32, dtype=torch.int32)
    gA = torch.ones(1)
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    plan = F.Plan(sum(rows), K, p)
    xq = F.fs_quantize_splice(X, mask, p, gA)
    F.fs_splice_gemm_segmented(plan, xq, wall, alpha, [0, 4096, 5120, 6144])
    F.fs_decode_splice_gemm(plan, X, mask, p, gA, wall, alpha, seg_start=[0, 4096, 5120, 6144])
    wide = torch.zeros(M, K + 192, dtype=torch.bfloat16)
    F.fs_decode_splice_gemm(F.Plan(4096, K, p), wide[:, 64:64 + K], mask, p, gA, views[0], alpha[:1])


def _gemm_inputs(M=32, N=256, K=512, p=16):
    mask = torch.zeros(K // 32, dtype=torch.int32)
    gA = torch.ones(1)
    xq = F.fs_quantize_splice(torch.zeros(M, K, dtype=torch.bfloat16), mask, p, gA)
    wq, _, alpha = F.fs_prepare_weights(torch.zeros(N, K, dtype=torch.bfloat16), mask, p, gA)
    return xq, wq, alpha, mask, gA


def test_short_or_mistyped_buffers_are_refused(no_launch):
    M, N, K, p = 32, 256, 512, 16
    xq, wq, alpha, mask, gA = _gemm_inputs(M, N, K, p)
    plan = F.Plan(N, K, p)
    plan16 = F.Plan(N, K, p, F.FS_OUT_BF16)
    F.fs_splice_gemm(plan, xq, wq, alpha)                                   # well-formed: accepted
    bad = [
        lambda: F.fs_splice_gemm(plan, xq, wq, alpha, Y=torch.empty(M - 1, N)),             # short Y
        lambda: F.fs_splice_gemm(plan, xq, wq, alpha, Y=torch.empty(M, N - 16)),            # narrow Y
        lambda: F.fs_splice_gemm(plan, xq, wq, alpha, Y=torch.empty(M, N, dtype=torch.bfloat16)),   # dtype
        lambda: F.fs_splice_gemm(plan16, xq, wq, alpha, Y=torch.empty(M, N)),
        lambda: F.fs_splice_gemm(plan, xq, wq, alpha, Y=torch.empty(N, M).t()),             # strided columns
        lambda: F.fs_splice_gemm(F.Plan(2 * N, K, p), xq, wq, alpha),                       # weights too short
        lambda: F.fs_splice_gemm(F.Plan(N, 2 * K, p), xq, wq, alpha),                       # K differs
        lambda: F.fs_splice_gemm(plan, xq, F.Packed(wq.q, wq.sf[:100], wq.side, N, K, p), alpha),   # scales
        lambda: F.fs_splice_gemm(plan, xq, F.Packed(wq.q, wq.sf, wq.side[:, :8], N, K, p), alpha),  # side
        lambda: F.fs_splice_gemm(plan, F.alloc_packed(M, K, 32, "cpu"), wq, alpha),               # p differs
        lambda: F.fs_splice_gemm_segmented(plan, xq, wq, alpha, [0, 128, 256]),             # one alpha, two segments
        lambda: F.fs_decode_splice_gemm(plan, torch.zeros(4, K // 2, dtype=torch.bfloat16), mask, p, gA, wq, alpha),
        lambda: F.fs_decode_splice_gemm(plan, torch.zeros(4, K, dtype=torch.bfloat16), mask[:2], p, gA, wq, alpha),
        lambda: F.fs_quantize_splice(torch.zeros(M, K, dtype=torch.bfloat16), mask, p, gA,
                                     out=F.alloc_packed(M - 1, K, p, "cpu")),                      # short out
        lambda: F.fs_prepare_weights(torch.zeros(N, K, dtype=torch.bfloat16), mask, p, gA,
                                     out=F.alloc_packed(N, 2 * K, p, "cpu")),                      # wrong width
    ]
    for call in bad:
        n = len(no_launch)
        with pytest.raises(ValueError):
            call()
        assert all(name == "fs_plan_create" for name in no_launch[n:]), no_launch[n:]   # nothing launched


def test_refusals_are_library_argument_errors_and_empty_batches_read_nothing(no_launch):
    """A refused buffer raises the library's invalid-argument status (callers that expect the
    library's FoursightError see it), and an empty batch is passed through unchecked, as the
    library reads no operand then."""
    M, N, K, p = 32, 256, 512, 16
    xq, wq, alpha, mask, gA = _gemm_inputs(M, N, K, p)
    with pytest.raises(F.FoursightError) as exc:
        F.fs_splice_gemm(F.Plan(2 * N, K, p), xq, wq, alpha)
    assert exc.value.status == 1                                            # FS_ERR_INVALID_ARGUMENT
    empty = F.fs_quantize_splice(torch.zeros(0, K, dtype=torch.bfloat16), mask, p, gA)
    F.fs_splice_gemm(F.Plan(N, K, p), empty, wq, alpha)
    F.fs_splice_gemm_grouped(F.Plan(N, K, p), torch.zeros(3, dtype=torch.int64), 0, empty, wq, alpha.repeat(2))


def test_grouped_buffers_are_checked(no_launch):
    E, N, K, p, total = 4, 256, 512, 16, 100
    offs = torch.tensor([0, 10, 40, 70, 100], dtype=torch.int64)
    X = torch.zeros(total, K, dtype=torch.bfloat16)
    masks = torch.zeros(E, K // 32, dtype=torch.int32)
    gA = torch.ones(E)
    xq = F.fs_quantize_splice_grouped(X, offs, masks, p, gA)
    wq = F.alloc_packed(E * N, K, p, "cpu")
    alpha = torch.zeros(E)
    plan = F.Plan(N, K, p)
    F.fs_splice_gemm_grouped(plan, offs, total, xq, wq, alpha)              # well-formed: accepted
    with pytest.raises(ValueError):
        F.fs_splice_gemm_grouped(plan, offs, total, F.alloc_packed(total, K, p, "cpu"), wq, alpha)   # not padded
    with pytest.raises(ValueError):
        F.fs_splice_gemm_grouped(plan, offs, total, xq, F.alloc_packed(N, K, p, "cpu"), alpha)       # one expert's rows
    with pytest.raises(ValueError):
        F.fs_splice_gemm_grouped(plan, offs, total, xq, wq, alpha[:2])
    with pytest.raises(ValueError):
        F.fs_splice_gemm_grouped(plan, offs.to(torch.int32), total, xq, wq, alpha)


def _refused(calls, fn):
    n = len(calls)
    with pytest.raises(F.ArgumentError):
        fn()
    assert calls[n:] == [], calls[n:]                                       # nothing reached the library


def test_statistics_selection_and_filter_buffers_are_checked(no_launch):
    K = 256
    st = F.StatsState(2, K, device="cpu")
    X = torch.zeros(10, K, dtype=torch.bfloat16)
    F.fs_channel_stats(X, st, group=1)
    F.fs_channel_stats(X[:0], st)                                           # an empty batch
    F.fs_select_topk(st, 16)
    F.fs_select_topk(st, 0)
    P = torch.empty(2, 16, dtype=torch.int32)
    F.fs_select_topk(st, 16, P=P, mask=torch.empty(2, K // 32, dtype=torch.int32), gA=torch.empty(2))
    _refused(no_launch, lambda: F.fs_channel_stats(torch.zeros(10, 2 * K, dtype=torch.bfloat16), st))   # wider than K
    _refused(no_launch, lambda: F.fs_channel_stats(X, st, group=2))                                 # no such group
    _refused(no_launch, lambda: F.fs_channel_stats(torch.zeros(K, 10, dtype=torch.bfloat16).t(), st))   # strided columns
    _refused(no_launch, lambda: F.fs_select_topk(st, 16, P=torch.empty(1, 16, dtype=torch.int32)))      # one row for two
    _refused(no_launch, lambda: F.fs_select_topk(st, 16, P=torch.empty(2, 32, dtype=torch.int32)[:, :16]))  # pitch
    _refused(no_launch, lambda: F.fs_select_topk(st, 16, mask=torch.empty(2, 4, dtype=torch.int32)))    # short mask
    _refused(no_launch, lambda: F.fs_select_topk(st, 16, gA=torch.empty(1)))
    S, T = 8, 64
    lp = torch.zeros(S, T)
    F.fs_seq_filter(lp, -9.0, 9, 5, lengths=torch.full((S,), T, dtype=torch.int32), G=4, rewards=torch.zeros(S))
    _refused(no_launch, lambda: F.fs_seq_filter(lp.double(), -9.0, 9, 5))
    _refused(no_launch, lambda: F.fs_seq_filter(lp, -9.0, 9, 5, lengths=torch.full((S,), T)))         # int64 lengths
    _refused(no_launch, lambda: F.fs_seq_filter(lp, -9.0, 9, 5, G=4, rewards=torch.zeros(S - 1)))
    _refused(no_launch, lambda: F.fs_seq_filter(lp, -9.0, 9, 5, adv=torch.zeros(S, dtype=torch.float64)))


def test_training_side_buffers_are_checked(no_launch):
    M, N, K = 64, 32, 48
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    plan = F.Plan(256, 256, 1)
    F.fs_gemm_bf16(plan, bf(M, K), bf(N, K), Y=torch.empty(M, N))
    F.fs_transpose_bf16(bf(M, K))
    F.fs_ste_backward(plan, bf(M, N), bf(M, K), bf(N, K))
    S, T = 4, 16
    lp, lo = torch.zeros(S, T), torch.zeros(S, T)
    F.fs_grpo_objective(lp, lo, torch.zeros(S), 0.2, lengths=torch.full((S,), T, dtype=torch.int32))
    F.fs_k3_kl(lp, lo)
    _refused(no_launch, lambda: F.fs_gemm_bf16(plan, bf(M, K), bf(N, K + 16)))                     # K differs
    _refused(no_launch, lambda: F.fs_gemm_bf16(plan, bf(M, K), bf(N, K), Y=torch.empty(M, N - 1)))
    _refused(no_launch, lambda: F.fs_gemm_bf16(plan, bf(M, K), bf(N, K), Y=bf(M, N)))              # dtype of the plan
    _refused(no_launch, lambda: F.fs_transpose_bf16(bf(M, K), dst=bf(K, M - 1)))
    _refused(no_launch, lambda: F.fs_ste_backward(plan, bf(M, N), bf(M - 1, K), bf(N, K)))
    _refused(no_launch, lambda: F.fs_ste_backward(plan, bf(M, N), bf(M, K), bf(N, K), work=torch.empty(8, dtype=torch.uint8)))
    _refused(no_launch, lambda: F.fs_ste_backward(plan, bf(M, N), bf(M, K), bf(N, K), dW=torch.empty(N, K - 1)))
    _refused(no_launch, lambda: F.fs_grpo_objective(lp, torch.zeros(S, 2 * T)[:, :T], torch.zeros(S), 0.2))   # pitch
    _refused(no_launch, lambda: F.fs_grpo_objective(lp, lo, torch.zeros(S - 1), 0.2))
    _refused(no_launch, lambda: F.fs_k3_kl(lp, torch.zeros(S - 1, T)))
