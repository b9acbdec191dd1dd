"""Pins for the training-side oracle (FourSight §5.2 STE backward, §4.1 Eq. 4, §6.1 K3 metric).

Each function is checked against something other than itself: the adjoint identity of the linear
map and a triple loop for the backward; finite differences, hand-built clip cases and the original
denominator for Eq. 4; the exact KL divergence of small categorical distributions (the K3
estimator is unbiased) and its closed-form limits for the metric.
"""
import math

import numpy as np

from oracle import nvfp4, train


def _bf16(a):
    return nvfp4.bf16_round(np.asarray(a, np.float32))


def test_ste_backward_triple_loop_and_adjoint_identity():
    rng = np.random.default_rng(0)
    M, N, K = 5, 3, 4
    dY, X, W = (_bf16(rng.standard_normal(s)) for s in ((M, N), (M, K), (N, K)))
    dX, dW = train.ste_backward(dY, X, W)
    for m in range(M):
        for k in range(K):
            assert dX[m, k] == sum(float(dY[m, n]) * float(W[n, k]) for n in range(N))
    for n in range(N):
        for k in range(K):
            assert dW[n, k] == sum(float(dY[m, n]) * float(X[m, k]) for m in range(M))
    # <dY, X W^T> = <dX, X> = <dW, W>: a transposed operand or swapped role breaks one of them
    Xd, Wd, dYd = X.astype(np.float64), W.astype(np.float64), dY.astype(np.float64)
    lhs = np.sum(dYd * (Xd @ Wd.T))
    assert math.isclose(lhs, np.sum(dX * Xd), rel_tol=1e-12)
    assert math.isclose(lhs, np.sum(dW * Wd), rel_tol=1e-12)


def test_ste_backward_is_the_gradient_of_the_bf16_product():
    """Finite differences of L(X, W) = <dY, X W^T> at bf16 points reproduce dX and dW (the STE
    reading: the quantiser passes the gradient through unchanged)."""
    rng = np.random.default_rng(1)
    dY, X, W = (_bf16(rng.standard_normal(s)) for s in ((4, 3), (4, 5), (3, 5)))
    dX, dW = train.ste_backward(dY, X, W)
    L = lambda x, w: float(np.sum(dY.astype(np.float64) * (x @ w.T)))
    h = 1e-6
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    for (m, k) in ((0, 0), (3, 4), (2, 1)):
        E = np.zeros_like(Xd); E[m, k] = h
        assert math.isclose((L(Xd + E, Wd) - L(Xd - E, Wd)) / (2 * h), dX[m, k], rel_tol=1e-6, abs_tol=1e-9)
    for (n, k) in ((0, 0), (2, 4)):
        E = np.zeros_like(Wd); E[n, k] = h
        assert math.isclose((L(Xd, Wd + E) - L(Xd, Wd - E)) / (2 * h), dW[n, k], rel_tol=1e-6, abs_tol=1e-9)


def test_grpo_on_policy_ratio_one():
    """rho = 1 (logp == logp_old): every token contributes A', J is the mean of A' over all S
    sequences and the gradient is A' / (S |y_i|)."""
    lp = np.full((4, 6), -1.5, np.float32)
    adv = np.array([1.0, -0.5, 0.0, 2.0], np.float32)
    lengths = np.array([6, 3, 6, 1])
    J, seq, grad = train.grpo_objective(lp, lp, adv, 0.2, lengths)
    assert np.allclose(seq, adv) and math.isclose(J, adv.mean())
    for i, n in enumerate(lengths):
        assert np.allclose(grad[i, :n], adv[i] / (4 * n)) and not grad[i, n:].any()


def test_grpo_clip_branches_by_hand():
    """The four sign/ratio cases of the PPO clip with eps = 0.2."""
    lo = np.zeros((1, 4), np.float32)
    lp = np.log(np.array([[1.5, 0.5, 1.5, 0.5]], np.float32)).astype(np.float32)
    rho = np.exp(lp.astype(np.float64))[0]
    e = float(np.float32(0.2))                        # eps is a float32 argument
    for A, want_l, want_active in ((1.0, [1 + e, rho[1], 1 + e, rho[3]], [0, 1, 0, 1]),
                                   (-1.0, [-rho[0], -(1 - e), -rho[2], -(1 - e)], [1, 0, 1, 0])):
        J, seq, grad = train.grpo_objective(lp, lo, np.array([A], np.float32), 0.2)
        assert math.isclose(seq[0], sum(want_l) / 4, rel_tol=1e-12)
        for t in range(4):
            assert (grad[0, t] != 0) == bool(want_active[t])
            if want_active[t]:
                assert math.isclose(grad[0, t], rho[t] * A / 4, rel_tol=1e-12)


def test_grpo_gradient_matches_finite_differences():
    rng = np.random.default_rng(3)
    S, T = 4, 9
    lo = (-rng.exponential(1.0, (S, T))).astype(np.float32)
    lp = (lo + rng.normal(0, 0.1, (S, T))).astype(np.float32)
    adv = np.array([1.0, -1.0, 0.5, 0.0], np.float32)
    lengths = np.array([9, 5, 7, 2])
    J, _, grad = train.grpo_objective(lp, lo, adv, 0.2, lengths)
    h = 1e-7
    for (i, t) in ((0, 0), (1, 4), (2, 6), (3, 1), (0, 8)):
        up = lp.astype(np.float64).copy(); up[i, t] += h
        dn = lp.astype(np.float64).copy(); dn[i, t] -= h
        # evaluate the float64 objective directly on perturbed log-probs
        def Jof(x):
            tot = 0.0
            for r in range(S):
                n = int(lengths[r])
                rho = np.exp(x[r, :n] - lo[r, :n].astype(np.float64))
                tot += np.minimum(rho * adv[r], np.clip(rho, 0.8, 1.2) * adv[r]).sum() / n
            return tot / S
        fd = (Jof(up) - Jof(dn)) / (2 * h)
        assert math.isclose(fd, grad[i, t], rel_tol=1e-5, abs_tol=1e-9)


def test_grpo_keeps_the_original_denominator():
    """Dropping a sequence (its A' becomes 0) leaves the other sequences' contributions, and the
    denominator S = (number of groups) x G, unchanged: surviving gradients are not rescaled."""
    rng = np.random.default_rng(4)
    S, T = 8, 5
    lo = (-rng.exponential(1.0, (S, T))).astype(np.float32)
    lp = (lo + rng.normal(0, 0.05, (S, T))).astype(np.float32)
    adv = rng.normal(0, 1, S).astype(np.float32)
    J, seq, grad = train.grpo_objective(lp, lo, adv, 0.2)
    adv2 = adv.copy(); adv2[[1, 6]] = 0.0
    J2, seq2, grad2 = train.grpo_objective(lp, lo, adv2, 0.2)
    keep = np.ones(S, bool); keep[[1, 6]] = False
    assert np.array_equal(grad2[keep], grad[keep]) and not grad2[~keep].any()
    assert math.isclose(J2, seq[keep].sum() / S, rel_tol=1e-12)


def test_k3_is_unbiased_for_small_categoricals():
    """E_q[k3] = KL(q || p) exactly: enumerate every outcome of small categorical distributions."""
    rng = np.random.default_rng(5)
    for n in (2, 3, 7):
        q = rng.dirichlet(np.ones(n))
        p = rng.dirichlet(np.ones(n))
        est = sum(q[x] * train.k3(math.log(p[x]) - math.log(q[x])) for x in range(n))
        kl = sum(q[x] * math.log(q[x] / p[x]) for x in range(n))
        assert math.isclose(est, kl, rel_tol=1e-12, abs_tol=1e-15)


def test_k3_closed_forms_and_batch_means():
    assert train.k3(0.0) == 0.0
    for d in (1e-9, -1e-6, 1e-3, -0.05, 0.5, -3.0, 8.0):
        v = float(train.k3(d))
        assert v >= 0.0
        assert math.isclose(v, math.exp(d) - 1 - d, rel_tol=1e-6) or abs(d) < 1e-4
        if abs(d) < 1e-3:                                  # d^2/2 + d^3/6 + ...
            assert math.isclose(v, d * d / 2 + d ** 3 / 6, rel_tol=1e-6)
    a = np.array([[0.0, -1.0, -2.0], [-0.5, -0.5, 0.0]], np.float32)
    b = np.array([[0.0, -1.0, -2.0], [-0.25, -1.0, 9.0]], np.float32)
    seq, batch = train.k3_kl(a, b, lengths=[3, 2])
    assert seq[0] == 0.0
    want = (train.k3(-0.25) + train.k3(0.5)) / 2
    assert math.isclose(seq[1], want, rel_tol=1e-15)
    assert math.isclose(batch, (0.0 + 2 * want) / 5, rel_tol=1e-15)   # token mean, position 2 of row 1 ignored
