"""SpliceGEMM reference: weight pre-split, activation preparation, the output.

TEST INFRASTRUCTURE ONLY (see the package docstring).

FourSight §4.2 "Sparse Precision Compensation", Eq. 5: for Y = X W^T with
X in R^{M x K}, W in R^{N x K} and a protected channel set S,
``Y ~= alpha * (Xq_{~S} Wq_{~S}^T + X_S W'_S^T)`` with ``W'_S = BF16(W_S / alpha)``.
§5.1 "Data preparation": the protected lanes are zeroed in place (K and block
membership are unchanged) before the NVFP4 block scales are computed, and the
protected columns are copied to a compact BF16 side buffer X_S [M, |S|].
§9.3.1 Eq. 7-8 define the same thing with x_R, W_R embedded in the original
K coordinates.  Under power-of-two gains the Eq. 5 form equals the definition
``Y = deq(Q(X[:,~P])) deq(Q(W[:,~P]))^T + X[:,P] W[:,P]^T`` exactly; the tests
pin that identity.

Side buffers are padded to Pp = roundup(p, 16) columns with zeros.

Compacted-K variant (``COMPACT``, the "next" form the pages leave open): the protected columns
are removed from the NVFP4 operand instead of zeroed in place, so the 16-element blocks are
re-formed over the unprotected channels in ascending order; the operand has compact_cols(K, p)
columns (zero padded to a multiple of 256).  Gains, the side buffers and alpha are those of the
split form; only block membership (hence the block scales) changes.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

SPLIT = "split"
RESIDUAL = "residual"
COMPACT = "compact"


def padded_p(p: int) -> int:
    return (int(p) + 15) // 16 * 16


def compact_cols(K: int, p: int) -> int:
    """Columns of the compacted NVFP4 operand: the K - p unprotected channels, padded with zero
    columns to a multiple of 256 (one NVFP4 k-tile of the GEMM kernels)."""
    return (int(K) - int(p) + 255) // 256 * 256


def compact(A, P) -> np.ndarray:
    """A[:, ~P] (unprotected columns in ascending channel order) followed by zero columns up to
    compact_cols(K, p): the compacted-K reading of x_R (§9.3.1), blocks re-formed over ~P."""
    A = np.asarray(A, dtype=np.float32)
    K = A.shape[1]
    keep = keep_vector(P, K)
    out = np.zeros((A.shape[0], compact_cols(K, int((~keep).sum()))), np.float32)
    out[:, : int(keep.sum())] = A[:, keep]
    return out


def keep_vector(P, K) -> np.ndarray:
    keep = np.ones(K, dtype=bool)
    keep[np.asarray(P, dtype=np.int64)] = False
    return keep


def as_f32(a, is_bf16_bits: bool) -> np.ndarray:
    return nvfp4.bf16_value(a) if is_bf16_bits else np.asarray(a, dtype=np.float32)


def quantize_splice(X, P, gA, mode: str = SPLIT):
    """Activation preparation (§5.1 "Data preparation": Mask S->0, FP4 Quant, Extract X_S).

    X: float32 [M,K] (bf16 inputs widened first).  P: protected channels, ascending.
    Returns dict(codes [M,K], sf [M,K/16] row-major codes, xs [M,Pp] float32 holding
    bf16 values (zero padded)).
    """
    X = np.asarray(X, dtype=np.float32)
    M, K = X.shape
    P = np.asarray(P, dtype=np.int64)
    keep = keep_vector(P, K)
    if mode == COMPACT:
        Xc = compact(X, P)
        codes, sf = nvfp4.quantize_blocks(Xc, np.ones(Xc.shape[1], bool), gA)
    else:
        codes, sf = nvfp4.quantize_blocks(X, keep, gA, scale_from_all_lanes=(mode == RESIDUAL))
    xs = np.zeros((M, padded_p(len(P))), np.float32)
    xs[:, : len(P)] = nvfp4.bf16_round(X[:, P])
    return {"codes": codes, "sf": sf, "xs": xs}


def weight_gain(W, P, mode: str = SPLIT, exact: bool = False) -> np.float32:
    """g_W from the absolute maximum of W over the unprotected columns (all columns in residual form)."""
    W = np.asarray(W, dtype=np.float32)
    cols = keep_vector(P, W.shape[1]) if mode != RESIDUAL else np.ones(W.shape[1], bool)
    amax = np.float32(np.abs(W[:, cols]).max()) if cols.any() and W.size else np.float32(0)
    return nvfp4.gain_exact(amax) if exact else nvfp4.gain_pow2(amax)


def prepare_weights(W, P, gA, mode: str = SPLIT, exact_gain: bool = False):
    """Weight pre-split after a policy update (§5.1: NVFP4 pack of W_{~S}, BF16 pack W'_S = BF16(W_S/alpha)).

    Returns dict(codes [N,K], sf [N,K/16], ws [N,Pp] float32 bf16 values, gW, alpha).
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    P = np.asarray(P, dtype=np.int64)
    gW = weight_gain(W, P, mode, exact_gain)
    alpha = nvfp4.alpha_from_gains(gA, gW)
    if mode == COMPACT:
        Wc = compact(W, P)
        codes, sf = nvfp4.quantize_blocks(Wc, np.ones(Wc.shape[1], bool), gW)
    else:
        codes, sf = nvfp4.quantize_blocks(W, keep_vector(P, K), gW, scale_from_all_lanes=(mode == RESIDUAL))
    ws = np.zeros((N, padded_p(len(P))), np.float32)
    wp = nvfp4.bf16_round(W[:, P])
    ws[:, : len(P)] = nvfp4.bf16_round((wp / alpha).astype(np.float32))
    return {"codes": codes, "sf": sf, "ws": ws, "gW": gW, "alpha": alpha}


def splice_gemm(xq, wq, alpha, rows=None):
    """Eq. 5 in float64: Y = alpha * (sum_{k not in S} (q sf)_x (q sf)_w + sum_{j} X_S[:,j] W'_S[:,j]).

    ``xq`` and ``wq`` are the dicts returned above.  The NVFP4 part runs over all K
    lanes (protected lanes hold code 0).  ``rows`` optionally restricts the output to a
    subset of M rows.  Returns (Y float64 [m,N], absolute-product sums float64 [m,N]),
    the latter being sum_k |x_hat_k w_hat_k| for the parity tolerance.  Y itself is
    pinned; the tensor cores' own accumulation error against it is parity unpinned
    (the pages fix no accumulation order or width, so only the stated tolerance,
    1e-5 of this sum, covers it).
    """
    xc, xsf, xs = xq["codes"], xq["sf"], xq["xs"]
    if rows is not None:
        xc, xsf, xs = xc[rows], xsf[rows], xs[rows]
    xv = nvfp4.dequantize(xc, xsf)                       # q*sf, no gain
    wv = nvfp4.dequantize(wq["codes"], wq["sf"])
    a = np.float64(np.float32(alpha))
    xs64 = xs.astype(np.float64)
    ws64 = wq["ws"].astype(np.float64)
    acc = xv @ wv.T + xs64 @ ws64.T
    mag = np.abs(xv) @ np.abs(wv).T + np.abs(xs64) @ np.abs(ws64).T
    return a * acc, a * mag


def reference_definition(X, W, P, gA, gW):
    """The plain definition deq(Q(X[:,~P])) deq(Q(W[:,~P]))^T + bf16(X[:,P]) bf16(W[:,P])^T in float64."""
    X = np.asarray(X, np.float32)
    W = np.asarray(W, np.float32)
    K = X.shape[1]
    keep = keep_vector(P, K)
    cx, sx = nvfp4.quantize_blocks(X, keep, gA)
    cw, sw = nvfp4.quantize_blocks(W, keep, gW)
    xh = nvfp4.dequantize(cx, sx, gA)
    wh = nvfp4.dequantize(cw, sw, gW)
    P = np.asarray(P, np.int64)
    xp = nvfp4.bf16_round(X[:, P]).astype(np.float64)
    wp = nvfp4.bf16_round(W[:, P]).astype(np.float64)
    return xh @ wh.T + xp @ wp.T
