"""Training side of the FourSight hot path: STE backward, the Eq. 4 objective, the K3 TIM metric.

TEST INFRASTRUCTURE ONLY (see the package docstring).

FourSight §5.2 "System Implementation": the trainer masks sequence advantages with the dual gates
before backpropagation, and backward passes run in BF16 with the straight-through estimator (STE).
§4.1 Eq. 4: the GRPO objective with the filtered advantages A'_i = f_i A_i keeps the original
denominator G (not the number of surviving sequences).  §2.1 defines the clipped token term with
the importance ratio rho = pi_theta / pi_theta_old.  §6.1: TIM is measured with sampled estimates of
the K3 KL divergence between the rollout and training policies.

Readings taken:
* STE: the quantiser's Jacobian is the identity, so the gradients of Y = Q(X) Q(W)^T (+ the BF16
  slice) with respect to X and W are those of Y = X W^T on the BF16 operands:
  dX = dY W and dW = dY^T X (float64 here; bf16 inputs).
* Eq. 4 with S sequences in S/G groups of G: J = mean over groups of (1/G) sum_i (1/|y_i|) sum_t l_it
  = (1/S) sum_i (1/|y_i|) sum_t l_it, with l = min(rho A', clip(rho, 1-eps, 1+eps) A') and
  rho = exp(logp - logp_old) (the log-probs given as float32, the arithmetic in float64).  |y_i| is
  the response length (lengths[i], or T); an empty response contributes 0.
* dJ/dlogp_it = rho A' / (S |y_i|) when the unclipped term is the minimum (rho A' <= clip(rho) A'),
  else 0 (the clipped term does not depend on logp where it is the minimum).
* K3: tokens are drawn by the rollout policy q; with d = logp_train - logp_rollout and r = e^d,
  k3 = (r - 1) - d = e^d - 1 - d >= 0 estimates KL(q || p_train) without bias.  Reported per
  sequence (mean over its tokens) and over the batch (mean over all tokens).
"""
from __future__ import annotations

import numpy as np

from . import nvfp4


def ste_backward(dY, X, W):
    """(dX, dW) = (dY W, dY^T X) in float64 on the bf16-rounded operands (float32 arrays in)."""
    dY = nvfp4.bf16_round(np.asarray(dY, np.float32)).astype(np.float64)
    X = nvfp4.bf16_round(np.asarray(X, np.float32)).astype(np.float64)
    W = nvfp4.bf16_round(np.asarray(W, np.float32)).astype(np.float64)
    return dY @ W, dY.T @ X


def _lengths(lengths, S, T):
    if lengths is None:
        return np.full(S, T, np.int64)
    return np.clip(np.asarray(lengths, np.int64), 0, T)


def grpo_objective(logp, logp_old, adv, eps, lengths=None):
    """Eq. 4: returns (J, seq_obj [S], grad [S,T]) in float64."""
    lp = np.asarray(logp, np.float32).astype(np.float64)
    lo = np.asarray(logp_old, np.float32).astype(np.float64)
    S, T = lp.shape
    L = _lengths(lengths, S, T)
    A = np.asarray(adv, np.float32).astype(np.float64)
    e = float(np.float32(eps))
    seq = np.zeros(S)
    grad = np.zeros((S, T))
    for i in range(S):
        n = int(L[i])
        if n == 0:
            continue
        rho = np.exp(lp[i, :n] - lo[i, :n])
        unc = rho * A[i]
        clp = np.clip(rho, 1.0 - e, 1.0 + e) * A[i]
        active = unc <= clp
        seq[i] = np.where(active, unc, clp).sum() / n
        grad[i, :n] = np.where(active, unc, 0.0) / (S * n)
    return seq.sum() / S, seq, grad


def k3(d):
    """e^d - 1 - d in float64 (expm1 keeps the small-d values accurate)."""
    d = np.asarray(d, np.float64)
    return np.expm1(d) - d


def k3_kl(logp_train, logp_roll, lengths=None):
    """Per-sequence mean K3 over each sequence's tokens, and the batch mean over all tokens."""
    a = np.asarray(logp_train, np.float32).astype(np.float64)
    b = np.asarray(logp_roll, np.float32).astype(np.float64)
    S, T = a.shape
    L = _lengths(lengths, S, T)
    seq = np.zeros(S)
    total, count = 0.0, 0
    for i in range(S):
        n = int(L[i])
        if n == 0:
            continue
        v = k3(a[i, :n] - b[i, :n])
        seq[i] = v.sum() / n
        total += v.sum()
        count += n
    return seq, (total / count if count else 0.0)
