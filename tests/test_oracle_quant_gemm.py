"""Pins for the oracle's block quantiser and SpliceGEMM output.

FourSight §4.2 Eq. 5, §5.1 "Data preparation", §9.3.1 Eq. 7-9, §9.3.2 Lemma 2 and the
neighbour example, §9.3.3 Lemma 3 and Theorem 1.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import bounds, nvfp4, splice, stats


def _read(golden_dir, name):
    out = {}
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            out[k] = [float(x) for x in v]
    return out


# ----------------------------------------------------------------------------- quantiser
def test_exact_round_trip_of_representable_blocks():
    """Blocks that are an E2M1 grid times a UE4M3 scale come back exactly (pow2 gain)."""
    rs = np.random.default_rng(3)
    R, K = 32, 256
    j = 3
    g = nvfp4.gain_pow2(6 * 448 * 2.0 ** -j)          # = 2^j exactly
    assert g == 2.0 ** j
    sf = rs.integers(8, 127, size=(R, K // 16))        # normal scale codes
    q = rs.integers(0, 16, size=(R, K))
    q[:, ::16] = np.where(rs.random((R, K // 16)) < 0.5, 7, 15)   # every block reaches |6|
    x = (nvfp4.e2m1_decode(q) * np.repeat(nvfp4.ue4m3_decode(sf), 16, axis=1) / float(g)).astype(np.float32)
    codes, sf2 = nvfp4.quantize_blocks(x, np.ones(K, bool), g)
    assert np.array_equal(sf2, sf)
    # -0 and +0 both decode to 0; compare values, and the non-zero codes exactly
    assert np.array_equal(nvfp4.dequantize(codes, sf2, g), x.astype(np.float64))
    nz = (q & 7) != 0
    assert np.array_equal(codes[nz], q[nz])


def test_lemma2_per_element_bound_on_random_blocks():
    """|Q(x)-x| <= (17/96) a_b for every block whose scale is normal and not saturated."""
    x, _ = synth.outlier_activations(5, 64, 512, as_bf16=False)
    P = np.arange(0, 512, 37)
    keep = splice.keep_vector(P, 512)
    g = nvfp4.gain_pow2(np.abs(x[:, keep]).max())
    codes, sf = nvfp4.quantize_blocks(x, keep, g)
    xh = nvfp4.dequantize(codes, sf, g)
    xm = np.where(keep, x, 0).astype(np.float64)
    a_b = np.abs(xm).reshape(64, 32, 16).max(axis=2)
    ok = (sf >= 8) & (sf < 126)
    assert ok.mean() > 0.9
    err = np.abs(xh - xm).reshape(64, 32, 16).max(axis=2)
    c = bounds.c_elem()
    assert math.isclose(c, 17 / 96, rel_tol=1e-15)
    assert np.all(err[ok] <= c * a_b[ok] * (1 + 2.0 ** -20))
    assert np.all(xh[:, ~keep] == 0)


def test_lemma3_row_norm_bound():
    x, _ = synth.outlier_activations(6, 64, 1024, as_bf16=False)
    g = nvfp4.gain_pow2(np.abs(x).max())
    codes, sf = nvfp4.quantize_blocks(x, np.ones(1024, bool), g)
    ok_rows = np.all((sf >= 8) & (sf < 126), axis=1)
    dx = nvfp4.dequantize(codes, sf, g) - x
    lhs = np.linalg.norm(dx, axis=1)
    rhs = math.sqrt(16) * bounds.C_ELEM * np.linalg.norm(x.astype(np.float64), axis=1)
    assert ok_rows.sum() > 32
    assert np.all(lhs[ok_rows] <= rhs[ok_rows] * (1 + 1e-6))


def test_neighbour_example_ideal_and_rounded(golden_dir):
    gd = _read(golden_dir, "neighbour_example.txt")
    blk = np.array(gd["block"], np.float64)
    # ideal (unrounded) scale a_b/6, elements rounded to E2M1
    s = blk.max() / 6
    assert s == gd["ideal_scale"][0]
    deq = nvfp4.e2m1_decode(nvfp4.e2m1_encode((blk / s).astype(np.float32))) * s
    assert deq.tolist() == gd["ideal_dequant"]
    masked = blk.copy(); masked[0] = 0
    s2 = masked.max() / 6
    assert math.isclose(s2, gd["protected_ideal_scale"][0], rel_tol=1e-15)
    deq2 = nvfp4.e2m1_decode(nvfp4.e2m1_encode((masked / s2).astype(np.float32))) * s2
    assert np.allclose(deq2, gd["protected_ideal_dequant"], rtol=1e-12)
    # the oracle's quantiser with a UE4M3-rounded scale (g = 1)
    x = blk.astype(np.float32)[None, :]
    c, sf = nvfp4.quantize_blocks(x, np.ones(16, bool), np.float32(1))
    assert nvfp4.ue4m3_decode(sf)[0, 0] == 8.0
    assert nvfp4.dequantize(c, sf).tolist()[0] == gd["ideal_dequant"]
    keep = np.ones(16, bool); keep[0] = False
    c, sf = nvfp4.quantize_blocks(x, keep, np.float32(1))
    assert nvfp4.ue4m3_decode(sf)[0, 0] == 0.171875            # RNE of 1/6 in UE4M3
    d = nvfp4.dequantize(c, sf)[0]
    assert d[0] == 0 and np.all(d[1:] == 1.03125)
    assert np.all(np.abs(d[1:] - 1) <= bounds.C_ELEM * 1.0)     # Lemma 2 for the rounded scale


def test_masked_lanes_cannot_widen_the_block_scale():
    x = np.ones((1, 32), np.float32); x[0, 3] = 1000.0
    keep = np.ones(32, bool); keep[3] = False
    _, sf_split = nvfp4.quantize_blocks(x, keep, np.float32(1))
    _, sf_res = nvfp4.quantize_blocks(x, keep, np.float32(1), scale_from_all_lanes=True)
    assert nvfp4.ue4m3_decode(sf_split)[0, 0] == nvfp4.ue4m3_decode(nvfp4.ue4m3_encode(np.float32(1 / 6)))
    assert nvfp4.ue4m3_decode(sf_res)[0, 0] > 100
    assert sf_split[0, 1] == sf_res[0, 1]


def test_zero_scale_keeps_sign_and_zero_codes():
    x = np.zeros((1, 16), np.float32); x[0, 1] = -0.0; x[0, 2] = 1e-30; x[0, 3] = -1e-30
    c, sf = nvfp4.quantize_blocks(x, np.ones(16, bool), np.float32(1))
    assert sf[0, 0] == 0
    assert c[0, 0] == 0 and c[0, 1] == 8 and c[0, 2] == 0 and c[0, 3] == 8


# ----------------------------------------------------------------------------- GEMM
def _small_problem(seed, M, N, K, p, bf16=True):
    x, _ = synth.outlier_activations(seed, M, K, n_outliers=max(1, K // 64), as_bf16=bf16)
    w = synth.gaussian_weights(seed + 7, N, K, as_bf16=bf16)
    X = splice.as_f32(x, bf16)
    W = splice.as_f32(w, bf16)
    st = stats.accumulate(stats.new_state(K), X)
    P = stats.select_topk(st, p)
    gA = stats.next_gain(st, P)
    return X, W, P, gA


def test_gemm_brute_force_tiny():
    """Exact rational triple loop over the dequantised operands vs the oracle's float64 matmul."""
    X, W, P, gA = _small_problem(11, 5, 6, 64, 5)
    xq = splice.quantize_splice(X, P, gA)
    wq = splice.prepare_weights(W, P, gA)
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    xv = nvfp4.dequantize(xq["codes"], xq["sf"])
    wv = nvfp4.dequantize(wq["codes"], wq["sf"])
    a = Fraction(float(wq["alpha"]))
    for m in range(5):
        for n in range(6):
            acc = Fraction(0)
            for k in range(64):
                acc += Fraction(float(xv[m, k])) * Fraction(float(wv[n, k]))
            for j in range(len(P)):
                acc += Fraction(float(xq["xs"][m, j])) * Fraction(float(wq["ws"][n, j]))
            exact = float(a * acc)
            assert math.isclose(Y[m, n], exact, rel_tol=1e-13, abs_tol=1e-300)


def test_eq5_form_equals_definition_under_pow2_gains():
    X, W, P, gA = _small_problem(12, 16, 24, 256, 16)
    xq = splice.quantize_splice(X, P, gA)
    wq = splice.prepare_weights(W, P, gA)
    Y, mag = splice.splice_gemm(xq, wq, wq["alpha"])
    Yd = splice.reference_definition(X, W, P, gA, wq["gW"])
    assert np.all(np.abs(Y - Yd) <= 1e-14 * mag)
    # W'_S = BF16(W_S / alpha) is exactly W_S * gA * gW for power-of-two gains
    ws = wq["ws"][:, : len(P)]
    assert np.array_equal(ws, nvfp4.bf16_round(W[:, P]) * gA * wq["gW"])


def test_empty_protected_set_is_plain_nvfp4_gemm():
    X, W, _, _ = _small_problem(13, 8, 16, 128, 0)
    gA = nvfp4.gain_pow2(np.abs(X).max())
    xq = splice.quantize_splice(X, [], gA)
    wq = splice.prepare_weights(W, [], gA)
    assert xq["xs"].shape == (8, 0) and wq["ws"].shape == (16, 0)
    cx, sx = nvfp4.quantize_blocks(X, np.ones(128, bool), gA)
    cw, sw = nvfp4.quantize_blocks(W, np.ones(128, bool), wq["gW"])
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    ref = nvfp4.dequantize(cx, sx, gA) @ nvfp4.dequantize(cw, sw, wq["gW"]).T
    assert np.allclose(Y, ref, rtol=1e-13, atol=0)


def test_all_channels_protected_is_exact_bf16_gemm():
    X, W, _, _ = _small_problem(14, 8, 16, 64, 0)
    P = np.arange(64)
    gA = np.float32(4.0)
    xq = splice.quantize_splice(X, P, gA)
    wq = splice.prepare_weights(W, P, gA)
    assert np.all(xq["codes"] == 0) and np.all(wq["codes"] == 0)
    assert np.all(xq["sf"] == 0) and np.all(wq["sf"] == 0)
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    ref = nvfp4.bf16_round(X).astype(np.float64) @ nvfp4.bf16_round(W).astype(np.float64).T
    assert np.allclose(Y, ref, rtol=1e-13, atol=0)


def test_split_equals_residual_when_protected_lanes_never_hold_a_block_max():
    rs = np.random.default_rng(15)
    M, N, K = 8, 16, 128
    X = rs.standard_normal((M, K)).astype(np.float32)
    W = (rs.standard_normal((N, K)) * 0.02).astype(np.float32)
    P = np.array([3, 40, 77, 100])
    X[:, P] *= np.float32(1e-3)
    W[:, P] *= np.float32(1e-3)
    gA = nvfp4.gain_pow2(np.abs(X).max())
    ys = []
    for mode in (splice.SPLIT, splice.RESIDUAL):
        xq = splice.quantize_splice(X, P, gA, mode)
        wq = splice.prepare_weights(W, P, gA, mode)
        ys.append(splice.splice_gemm(xq, wq, wq["alpha"])[0])
    assert np.array_equal(ys[0], ys[1])
    # and they differ once a protected lane is the block maximum
    X2 = X.copy(); X2[:, 3] = 100.0
    y2 = [splice.splice_gemm(splice.quantize_splice(X2, P, gA, m), splice.prepare_weights(W, P, gA, m),
                             splice.prepare_weights(W, P, gA, m)["alpha"])[0] for m in (splice.SPLIT, splice.RESIDUAL)]
    assert not np.array_equal(y2[0], y2[1])


def test_residual_form_identity():
    """Residual form == Q(X)Q(W)^T + (X_P W_P^T - Q(X)_P Q(W)_P^T) with all-lane block scales."""
    X, W, P, _ = _small_problem(16, 8, 12, 128, 8)
    gA = nvfp4.gain_pow2(np.abs(X).max())
    xq = splice.quantize_splice(X, P, gA, splice.RESIDUAL)
    wq = splice.prepare_weights(W, P, gA, splice.RESIDUAL)
    Y, mag = splice.splice_gemm(xq, wq, wq["alpha"])
    gW = wq["gW"]
    cx, sx = nvfp4.quantize_blocks(X, np.ones(128, bool), gA)
    cw, sw = nvfp4.quantize_blocks(W, np.ones(128, bool), gW)
    qx = nvfp4.dequantize(cx, sx, gA)
    qw = nvfp4.dequantize(cw, sw, gW)
    xp = nvfp4.bf16_round(X[:, P]).astype(np.float64)
    wp = nvfp4.bf16_round(W[:, P]).astype(np.float64)
    ref = qx @ qw.T + (xp @ wp.T - qx[:, P] @ qw[:, P].T)
    assert np.all(np.abs(Y - ref) <= 1e-13 * mag)


def test_theorem1_bound_holds_per_row(golden_dir):
    """||y_S - y||^2 <= C ||W||_F^2 ||x_R||^2 per row (Thm. 1 before the expectation), C ~ 3.68."""
    gd = _read(golden_dir, "theorem1_constant.txt")
    C = bounds.theorem1_C(gd["c_num"][0] / gd["c_den"][0], gd["c_num"][0] / gd["c_den"][0], int(gd["B"][0]))
    assert round(C, 2) == gd["C_printed"][0]
    X, W, P, gA = _small_problem(17, 64, 32, 512, 64)
    xq = splice.quantize_splice(X, P, gA)
    wq = splice.prepare_weights(W, P, gA)
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    y = X.astype(np.float64) @ W.astype(np.float64).T
    keep = splice.keep_vector(P, 512)
    lhs = ((Y - y) ** 2).sum(axis=1)
    rhs = C * (W.astype(np.float64) ** 2).sum() * (X[:, keep].astype(np.float64) ** 2).sum(axis=1)
    # rows whose blocks are all normal and unsaturated satisfy the hypothesis of the theorem
    rows_ok = np.all((xq["sf"] >= 8) & (xq["sf"] < 126), axis=1)
    assert np.all((wq["sf"] >= 8) & (wq["sf"] < 126) | (wq["sf"] == 0))
    assert rows_ok.sum() > 0
    assert np.all(lhs[rows_ok] <= rhs[rows_ok])
    # and in expectation over rows, with m_j the empirical second moments
    mj = (X[rows_ok].astype(np.float64) ** 2).mean(axis=0)
    assert lhs[rows_ok].mean() <= C * (W.astype(np.float64) ** 2).sum() * mj[keep].sum()


# ----------------------------------------------------------------------------- compacted K
def test_compact_with_no_protection_is_the_split_form():
    """P = {}: nothing is removed, so the compacted operand is the split operand."""
    rng = np.random.default_rng(20)
    X = rng.standard_normal((6, 512)).astype(np.float32)
    g = nvfp4.gain_pow2(np.abs(X).max())
    a = splice.quantize_splice(X, [], g, splice.COMPACT)
    b = splice.quantize_splice(X, [], g, splice.SPLIT)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["sf"], b["sf"])


def test_compact_with_every_channel_protected_is_the_exact_bf16_gemm():
    """P = all: the NVFP4 operand has no columns and Y is the BF16 product X W^T exactly."""
    rng = np.random.default_rng(21)
    X = nvfp4.bf16_round(rng.standard_normal((4, 64)).astype(np.float32))
    W = nvfp4.bf16_round((rng.standard_normal((8, 64)) * 0.1).astype(np.float32))
    P = np.arange(64)
    assert splice.compact_cols(64, 64) == 0
    xq = splice.quantize_splice(X, P, np.float32(1), splice.COMPACT)
    wq = splice.prepare_weights(W, P, np.float32(1), splice.COMPACT)
    assert xq["codes"].shape == (4, 0)
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    assert np.array_equal(Y, X.astype(np.float64) @ W.astype(np.float64).T)


def test_compact_blocks_are_formed_over_the_unprotected_channels():
    """Channel j holds 2^(j // 16): in original coordinates block b has maximum 2^b; with channels
    0 and 17 protected, compacted block 0 holds channels 1..16 (maximum 2) and block 1 channels
    18..33 (maximum 4), block 2 channels 34..47 and zero padding (maximum 4).  The scale codes follow
    from the pinned UE4M3 encoder at those maxima; the split form keeps 1, 2, 4."""
    K = 48
    X = np.array([[2.0 ** (j // 16) for j in range(K)]], np.float32)
    P = [0, 17]
    g = np.float32(1.0)
    sf_of = lambda a: int(nvfp4.ue4m3_encode(np.float32(np.float32(a * g) / np.float32(6.0))))
    c = splice.quantize_splice(X, P, g, splice.COMPACT)
    assert c["codes"].shape == (1, 256)
    assert c["sf"][0, :3].tolist() == [sf_of(2.0), sf_of(4.0), sf_of(4.0)]
    assert not c["sf"][0, 3:].any() and not c["codes"][0, 46:].any()
    s = splice.quantize_splice(X, P, g, splice.SPLIT)
    assert s["sf"][0].tolist() == [sf_of(1.0), sf_of(2.0), sf_of(4.0)]


def test_compact_lemma2_bound_and_gemm_against_brute_force():
    """Every compacted block obeys Lemma 2's per-element bound, and the SpliceGEMM of compacted
    operands equals a rational triple loop over the dequantised values plus the BF16 slice."""
    from fractions import Fraction
    rng = np.random.default_rng(22)
    M, N, K = 3, 2, 96
    X = rng.standard_normal((M, K)).astype(np.float32)
    X[:, [5, 40, 41]] *= 40
    W = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    P = np.array([5, 40, 41])
    gA = nvfp4.gain_pow2(np.abs(np.delete(X, P, axis=1)).max())
    xq = splice.quantize_splice(X, P, gA, splice.COMPACT)
    wq = splice.prepare_weights(W, P, gA, splice.COMPACT)
    Xc = splice.compact(X, P)
    xh = nvfp4.dequantize(xq["codes"], xq["sf"], gA)
    nb = Xc.shape[1] // 16
    a_b = np.abs(Xc).reshape(M, nb, 16).max(axis=2)
    err = np.abs(xh - Xc).reshape(M, nb, 16).max(axis=2)
    ok = (xq["sf"] >= 8) & (xq["sf"] < 126)          # normal, unsaturated scales (Lemma 2's premise)
    assert ok[:, : (K - 3 + 15) // 16].all()
    assert np.all(err[ok] <= bounds.c_elem() * a_b[ok] * (1 + 2.0 ** -20))
    Y, _ = splice.splice_gemm(xq, wq, wq["alpha"])
    xv = nvfp4.dequantize(xq["codes"], xq["sf"])
    wv = nvfp4.dequantize(wq["codes"], wq["sf"])
    for m in range(M):
        for n in range(N):
            acc = sum(Fraction(float(xv[m, k])) * Fraction(float(wv[n, k])) for k in range(xv.shape[1]))
            acc += sum(Fraction(float(xq["xs"][m, j])) * Fraction(float(wq["ws"][n, j])) for j in range(xq["xs"].shape[1]))
            assert Y[m, n] == float(Fraction(float(np.float32(wq["alpha"]))) * acc)
