"""Running channel moments and protected-channel reselection.

TEST INFRASTRUCTURE ONLY (see the package docstring).

FourSight §5.2 "System Implementation": a forward hook uniformly subsamples
token rows, before masking, and accumulates running channel moments in a GPU
buffer; after each optimizer step the protected set is reselected as the top-s
channels by the variance gathered in the previous step.  §4.2 and §9.3
(Prop. 2, Cor. 1) justify variance (or second moment) as the key.  §6.1 uses
s = 64.

Readings taken (the paper gives no formula):
* moments are exact integer fixed-point sums: s1 += rint(x * 2^16) and
  s2 += rint(x^2 * 2^14) (x^2 exact in float64, rint ties to even), so the sum is
  the same for every reduction order; n counts the accumulated rows, taken at
  row indices r = 0, stride, 2*stride, ... of each call;
* amax is the float32 absolute maximum per channel (kept as its bit pattern);
* a range flag is raised for |x| >= 2^15 or a non-finite x, and such an element
  contributes nothing to the sums or the maximum;
* key_j = m2 - m1*m1 with m1 = s1/65536/n, m2 = s2/16384/n in float64, in that
  order (second-moment key: m2); n = 0 gives key 0;
* top-p by (key descending, index ascending), reported in ascending index order;
* next-step activation gain: power-of-two rule on max amax over unprotected
  channels (over all channels in the residual form).
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

S1_SCALE = 2.0 ** 16
S2_SCALE = 2.0 ** 14
RANGE_LIMIT = 2.0 ** 15


def new_state(K: int) -> dict:
    return {"n": 0, "s1": np.zeros(K, np.int64), "s2": np.zeros(K, np.int64),
            "amax": np.zeros(K, np.float32), "flags": 0}


def accumulate(state: dict, X, row_stride: int = 1) -> dict:
    """Add the rows 0, stride, 2*stride, ... of X (float32 [M,K]) to the running moments.

    An element with |x| >= 2^15 or a non-finite one raises the range flag and adds nothing.
    """
    X = np.asarray(X, dtype=np.float32)
    rows32 = X[:: int(row_stride)]
    with np.errstate(invalid="ignore"):
        ok = np.isfinite(rows32) & (np.abs(rows32) < np.float32(RANGE_LIMIT))
    if not np.all(ok):
        state["flags"] |= 1
    rows = np.where(ok, rows32, np.float32(0)).astype(np.float64)
    t1 = np.rint(rows * S1_SCALE).astype(np.int64)
    t2 = np.rint(rows * rows * S2_SCALE).astype(np.int64)
    state["s1"] = state["s1"] + t1.sum(axis=0)
    state["s2"] = state["s2"] + t2.sum(axis=0)
    state["n"] += rows.shape[0]
    if rows.size:
        am = np.abs(rows).max(axis=0).astype(np.float32)
        state["amax"] = np.maximum(state["amax"], am).astype(np.float32)
    return state


def keys(state: dict, second_moment: bool = False) -> np.ndarray:
    n = state["n"]
    if n == 0:
        return np.zeros(len(state["s1"]), np.float64)
    m1 = state["s1"].astype(np.float64) / S1_SCALE / np.float64(n)
    m2 = state["s2"].astype(np.float64) / S2_SCALE / np.float64(n)
    return m2 if second_moment else m2 - m1 * m1


def select_topk(state: dict, p: int, second_moment: bool = False):
    """Top-p channels by (key desc, index asc), returned ascending (int32)."""
    k = keys(state, second_moment)
    order = sorted(range(len(k)), key=lambda j: (-k[j], j))
    return np.array(sorted(order[:p]), dtype=np.int32)


def protect_mask(P, K) -> np.ndarray:
    """Bit j%32 of word j//32 set for every protected channel j."""
    m = np.zeros((K + 31) // 32, np.uint32)
    for j in np.asarray(P, dtype=np.int64):
        m[j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return m


def next_gain(state: dict, P, residual: bool = False, exact: bool = False) -> np.float32:
    amax = state["amax"].copy()
    if not residual and len(P):
        amax[np.asarray(P, np.int64)] = 0
    a = np.float32(amax.max()) if amax.size else np.float32(0)
    return nvfp4.gain_exact(a) if exact else nvfp4.gain_pow2(a)
