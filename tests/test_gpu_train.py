"""GPU parity of the training-side kernels against the oracle (FourSight §5.2, §4.1 Eq. 4, §6.1).

- fs_gemm_bf16 / fs_ste_backward: the straight-through backward dX = dY W, dW = dY^T X on bf16
  operands; tolerance |err| <= 1e-5 * sum_k |a_k b_k| per element against the float64 product
  (the same bound as the SpliceGEMM tests; the bf16 products are exact in fp32).
- fs_transpose_bf16: bit-exact.
- fs_grpo_objective: fp32 arithmetic (expf of an fp32 difference) against float64; per token the
  ratio carries a few fp32 roundings, so seq_obj and J are compared at 1e-5 of sum |l| / |y_i| and
  the gradient at 1e-5 relative.  At a token whose ratio lies within 1e-5 (relative) of a clip
  boundary both branches are correct results; there the gradient must be 0 or the unclipped value.
- fs_k3_kl: per-sequence and batch means at 1e-5 relative (the small-d branch avoids cancellation).
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4, train

pytestmark = pytest.mark.gpu

F = pytest.importorskip("nvfp4_w4a4_gemm_fs_b200")


def _bf16_np(rng, shape, scale=1.0):
    return nvfp4.bf16_round((rng.standard_normal(shape) * scale).astype(np.float32))


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(300, 256, 512), (128, 384, 104), (17, 1024, 4096), (1000, 512, 2048),
                                   (2048, 4096, 4096)])
def test_gemm_bf16_matches_float64(M, N, K):
    rng = np.random.default_rng(M + N + K)
    A, B = _bf16_np(rng, (M, K)), _bf16_np(rng, (N, K), 0.02)
    plan = F.Plan(256, 256, 1)
    Y = torch.full((M, N), float("nan"), device="cuda")
    F.fs_gemm_bf16(plan, _t(A), _t(B), Y=Y)
    plan.check()
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    mag = np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64)).T
    got = Y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.all(np.abs(got - ref) <= 1e-5 * mag)


@pytest.mark.parametrize("R,C", [(130, 70), (64, 64), (4096, 1024), (1, 9)])
def test_transpose_bit_exact(R, C):
    rng = np.random.default_rng(R * C)
    a = _bf16_np(rng, (R, C))
    out = F.fs_transpose_bf16(_t(a))
    assert torch.equal(out, _t(a.T))


@pytest.mark.parametrize("M,N,K", [(512, 256, 384), (300, 1024, 512), (8192, 1024, 4096)])
def test_ste_backward_matches_oracle(M, N, K):
    rng = np.random.default_rng(7 + M)
    dY, X, W = _bf16_np(rng, (M, N), 1e-3), _bf16_np(rng, (M, K)), _bf16_np(rng, (N, K), 0.02)
    plan = F.Plan(256, 256, 1)
    dX, dW = F.fs_ste_backward(plan, _t(dY), _t(X), _t(W))
    plan.check()
    rX, rW = train.ste_backward(dY, X, W)
    a = lambda v: np.abs(v.astype(np.float64))
    magX = a(dY) @ a(W)
    magW = a(dY).T @ a(X)
    gX, gW = dX.cpu().numpy().astype(np.float64), dW.cpu().numpy().astype(np.float64)
    assert np.isfinite(gX).all() and np.isfinite(gW).all()
    assert np.all(np.abs(gX - rX) <= 1e-5 * magX)
    assert np.all(np.abs(gW - rW) <= 1e-5 * magW)


def _grpo_inputs(seed, S, T):
    rng = np.random.default_rng(seed)
    lo = (-rng.exponential(0.5, (S, T))).astype(np.float32)
    lp = (lo + rng.normal(0, 0.15, (S, T))).astype(np.float32)
    lengths = rng.integers(0, T + 1, S).astype(np.int32)
    lengths[0], lengths[1] = T, 0
    adv = rng.normal(0, 1, S).astype(np.float32)
    adv[rng.random(S) < 0.3] = 0.0                       # sequences dropped by the filter
    return lp, lo, lengths, adv


@pytest.mark.parametrize("S,T", [(16, 64), (64, 1000), (1024, 4096)])
def test_grpo_objective_matches_oracle(S, T):
    lp, lo, lengths, adv = _grpo_inputs(S + T, S, T)
    eps = 0.2
    J, seq, grad = F.fs_grpo_objective(torch.from_numpy(lp).cuda(), torch.from_numpy(lo).cuda(),
                                       torch.from_numpy(adv).cuda(), eps, lengths=torch.from_numpy(lengths).cuda())
    Jr, seqr, gradr = train.grpo_objective(lp, lo, adv, eps, lengths)
    # per-sequence magnitude of the terms: sum |l| / n
    rho = np.exp(lp.astype(np.float64) - lo.astype(np.float64))
    n = np.maximum(lengths, 1)
    pos = np.arange(T)[None, :] < lengths[:, None]
    e = float(np.float32(eps))
    magseq = (np.where(pos, np.maximum(rho, 1 + e) * np.abs(adv)[:, None], 0)).sum(axis=1) / n   # |l| bound
    got = seq.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - seqr) <= 1e-5 * magseq + 1e-30)
    assert abs(J.item() - Jr) <= 1e-5 * magseq.sum() / S + 1e-30
    g = grad.cpu().numpy().astype(np.float64)
    near = (np.abs(rho - (1 + e)) <= 1e-5 * (1 + e)) | (np.abs(rho - (1 - e)) <= 1e-5 * (1 - e))
    far = ~near
    assert np.all(np.abs(g[far] - gradr[far]) <= 1e-5 * np.abs(gradr[far]) + 1e-30)
    unc = rho * adv[:, None] / (S * n[:, None])
    ok_near = (g[near] == 0) | (np.abs(g[near] - unc[near]) <= 1e-5 * np.abs(unc[near]))
    assert ok_near.all()
    assert not g[~pos].any()


@pytest.mark.parametrize("S,T", [(8, 64), (1024, 4096)])
def test_k3_kl_matches_oracle(S, T):
    rng = np.random.default_rng(S)
    roll = (-rng.exponential(0.5, (S, T))).astype(np.float32)
    d = rng.normal(0, 0.05, (S, T))
    d[:, ::7] = rng.normal(0, 1.0, (S, (T + 6) // 7))    # a mix of small and large differences
    d[0, :5] = 0.0
    train_lp = (roll + d).astype(np.float32)
    lengths = rng.integers(0, T + 1, S).astype(np.int32)
    lengths[0] = T
    seq, batch = F.fs_k3_kl(torch.from_numpy(train_lp).cuda(), torch.from_numpy(roll).cuda(),
                            lengths=torch.from_numpy(lengths).cuda())
    seqr, batchr = train.k3_kl(train_lp, roll, lengths)
    got = seq.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - seqr) <= 1e-5 * np.abs(seqr) + 1e-30)
    assert abs(batch.item() - batchr) <= 1e-5 * batchr
