"""TIM-aware dual-gate sequence filter and advantage masking.

TEST INFRASTRUCTURE ONLY (see the package docstring).

FourSight §4.1 "TIM-aware Sequence Filtering": a token is a tail token when its
training probability is at most tau; G1 drops a trajectory with at least K1
tail tokens, G2 one with at least K2 consecutive tail tokens (Eq. 3:
f_i = 1[count < K1 and run < K2]); the advantage becomes f_i * A_i and the GRPO
loss keeps the original 1/G denominator (Eq. 4).  §2.1 gives the group advantage
A_i = (r_i - mu) / sigma.  §6.1: tau = 1e-4, K1 = 0.01 * output_len, K2 = 5.

Readings taken:
* "at most tau" is tested in the log domain, logp <= log_tau, with
  log_tau = fl32(ln(tau)) formed on the host; a NaN log-prob counts as tail;
* positions at or beyond a sequence's length are ignored; runs never cross
  sequences;
* mu and the population sigma are taken over all G rewards of the group
  (filtered sequences included, since filtering is applied after the fact), in
  float64 with sequential sums, then rounded to float32; sigma = 0 gives A = 0;
* a dropped sequence's advantage is +0.0.
"""
from __future__ import annotations

import math

import numpy as np


def log_tau(tau: float) -> np.float32:
    return np.float32(math.log(float(tau)))


def tail_flags(logp, lt) -> np.ndarray:
    lp = np.asarray(logp, dtype=np.float32)
    return (lp <= np.float32(lt)) | np.isnan(lp)


def count_and_run(tail_row) -> tuple[int, int]:
    """Number of tail tokens and the longest run of consecutive ones in a bool vector."""
    t = np.asarray(tail_row, dtype=np.int8)
    if t.size == 0:
        return 0, 0
    padded = np.concatenate(([0], t, [0]))
    d = np.diff(padded)
    starts = np.flatnonzero(d == 1)
    ends = np.flatnonzero(d == -1)
    run = int((ends - starts).max()) if starts.size else 0
    return int(t.sum()), run


def group_advantages(rewards, G: int) -> np.ndarray:
    r = np.asarray(rewards, dtype=np.float32).astype(np.float64)
    if r.size % G:
        raise ValueError("number of sequences must be a multiple of the group size")
    out = np.zeros(r.size, np.float32)
    for g0 in range(0, r.size, G):
        grp = r[g0:g0 + G]
        s = 0.0
        for v in grp:
            s += v
        mu = s / G
        q = 0.0
        for v in grp:
            q += (v - mu) * (v - mu)
        sigma = math.sqrt(q / G)
        for i, v in enumerate(grp):
            out[g0 + i] = np.float32((v - mu) / sigma) if sigma > 0 else np.float32(0.0)
    return out


def seq_filter(logp, lengths, lt, K1: int, K2: int, G: int = 0, rewards=None, adv=None):
    """Dual-gate filter over logp [S,T]; returns dict(keep u8, tail_count i32, max_run i32, adv f32|None)."""
    lp = np.asarray(logp, dtype=np.float32)
    S, T = lp.shape
    L = np.full(S, T, np.int64) if lengths is None else np.asarray(lengths, np.int64)
    tail = tail_flags(lp, lt)
    keep = np.zeros(S, np.uint8)
    cnt = np.zeros(S, np.int32)
    run = np.zeros(S, np.int32)
    for s in range(S):
        c, r = count_and_run(tail[s, : max(0, min(T, L[s]))])
        cnt[s], run[s] = c, r
        keep[s] = 1 if (c < K1 and r < K2) else 0
    out_adv = None
    if rewards is not None:
        base = group_advantages(rewards, G)
        out_adv = np.where(keep == 1, base, np.float32(0.0)).astype(np.float32)
    elif adv is not None:
        out_adv = np.where(keep == 1, np.asarray(adv, np.float32), np.float32(0.0)).astype(np.float32)
    return {"keep": keep, "tail_count": cnt, "max_run": run, "adv": out_adv}
