"""Pins for the oracle's E2M1 / UE4M3 codecs (FourSight §2.1, §9.3.1 "The NVFP4 format")."""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import nvfp4


def _golden(golden_dir, name):
    out = {}
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            out[k] = [float(x) for x in v]
    return out


def test_e2m1_value_set_matches_paper(golden_dir):
    g = _golden(golden_dir, "e2m1_value_set.txt")
    vals = nvfp4.e2m1_decode(np.arange(16))
    assert sorted(set(vals.tolist())) == sorted(set(g["values"]))
    nonneg = np.unique(vals[vals >= 0])
    assert np.max(np.diff(nonneg)) == g["max_gap"][0]
    assert np.max(np.abs(vals)) == g["max_magnitude"][0]
    # codes 0..7 positive ascending, 8..15 their negatives (code 8 is -0)
    assert np.all(np.diff(vals[:8]) > 0)
    assert np.array_equal(vals[8:], -vals[:8])
    assert np.signbit(vals[8])


def test_ue4m3_unit_roundoff_and_range(golden_dir):
    g = _golden(golden_dir, "ue4m3_facts.txt")
    v = nvfp4.ue4m3_decode(np.arange(127))
    assert np.all(np.diff(v) > 0)
    assert v[-1] == 448.0 and v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6
    assert np.isnan(nvfp4.ue4m3_decode(0x7F))
    normals = v[8:]
    half_gap_rel = (normals[1:] - normals[:-1]) / 2 / normals[:-1]
    assert half_gap_rel.max() == g["unit_roundoff_normal"][0]


def _brute_nearest_even(value, table_vals):
    """Exact nearest code by rational distances; ties to the even code; clamp above the max."""
    fv = Fraction(float(abs(value)))
    if fv >= Fraction(float(table_vals[-1])):
        return len(table_vals) - 1
    best, bestd = None, None
    for c, tv in enumerate(table_vals):
        d = abs(fv - Fraction(float(tv)))
        if best is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    return best


def _probe_points(table_vals):
    pts = []
    t = np.asarray(table_vals, dtype=np.float64)
    mids = (t[1:] + t[:-1]) / 2
    for x in list(t) + list(mids):
        f = np.float32(x)
        pts += [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(0))]
    return np.array(pts, dtype=np.float32)


def test_e2m1_rne_matches_brute_force():
    tv = nvfp4.E2M1_MAGNITUDES
    pts = np.concatenate([_probe_points(tv), np.float32([7.0, 100.0, 1e30])])
    rs = np.random.default_rng(1)
    pts = np.concatenate([pts, rs.uniform(0, 7, 2000).astype(np.float32)])
    for sgn in (1.0, -1.0):
        v = (pts * np.float32(sgn)).astype(np.float32)
        codes = nvfp4.e2m1_encode(v)
        for x, c in zip(v, codes):
            exp = _brute_nearest_even(x, tv) | (8 if np.signbit(x) else 0)
            assert c == exp, (x, c, exp)


def test_e2m1_documented_ties():
    got = nvfp4.e2m1_decode(nvfp4.e2m1_encode(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 6.5])))
    assert got.tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -4.0, 6.0]
    assert nvfp4.e2m1_encode(np.float32(-0.0)) == 8
    assert nvfp4.e2m1_encode(np.float32(0.0)) == 0


def test_ue4m3_rne_matches_brute_force():
    tv = nvfp4.UE4M3_VALUES
    pts = np.concatenate([_probe_points(tv), np.float32([449.0, 463.9, 464.0, 500.0, 1e20, 2.0 ** -11, 0.0])])
    rs = np.random.default_rng(2)
    pts = np.concatenate([pts, (2.0 ** rs.uniform(-12, 9.5, 2000)).astype(np.float32)])
    codes = nvfp4.ue4m3_encode(pts)
    for x, c in zip(pts, codes):
        assert c == _brute_nearest_even(x, tv), (x, c)


def test_pack_low_nibble_is_even_element():
    codes = np.array([[1, 2, 15, 8]])
    packed = nvfp4.pack_codes(codes)
    assert packed.tolist() == [[0x21, 0x8F]]
    assert np.array_equal(nvfp4.unpack_codes(packed), codes)


def test_sf_tiled_layout_is_a_bijection_and_spot_values():
    K = 16 * 12                      # 12 blocks -> 3 groups of 4
    R = 256
    rr, bb = np.meshgrid(np.arange(R), np.arange(K // 16), indexing="ij")
    off = nvfp4.sf_tiled_offset(rr, bb, K).ravel()
    Rp, nbp = nvfp4.sf_tiled_shape(R, K)
    assert sorted(off.tolist()) == list(range(Rp * nbp))
    # row 33, block 5: atom (row group 0, block group 1) -> 512; row 33 -> lane 1, column 1; block 1
    assert nvfp4.sf_tiled_offset(33, 5, K) == 512 + 1 * 16 + 1 * 4 + 1
    # row 128 starts the next row group after 3 atoms
    assert nvfp4.sf_tiled_offset(128, 0, K) == 3 * 512
    sf = np.random.default_rng(0).integers(0, 127, size=(200, 10)).astype(np.uint8)
    t = nvfp4.sf_to_tiled(sf, 160)
    assert np.array_equal(nvfp4.sf_from_tiled(t, 200, 160), sf)
    assert t.size == 256 * 12


def test_bf16_round_ties_to_even():
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9], np.float32)
    assert nvfp4.bf16_round(x).tolist() == [1.0, 1.0 + 2.0 ** -6, 1.0]


@pytest.mark.parametrize("amax", [1.0, 2688.0, 2688.0001, 0.3, 1e-3, 5e4, 448.0 * 6 / 1024])
def test_gain_pow2_is_the_largest_fitting_power(amax):
    g = float(nvfp4.gain_pow2(amax))
    a = float(np.float32(amax))
    assert g == 2.0 ** round(np.log2(g))
    assert Fraction(a) * Fraction(g) <= 2688
    assert Fraction(a) * Fraction(2 * g) > 2688
    assert nvfp4.gain_pow2(0.0) == 1.0


def _fl32(q: Fraction) -> float:
    """The binary32 value nearest to the positive rational q (ties to even), or inf past the
    largest finite one: written from the format's definition (24-bit significands, minimum normal
    exponent -126, subnormal spacing 2^-149), independent of numpy's division."""
    e = q.numerator.bit_length() - q.denominator.bit_length()    # 2^e <= q < 2^(e+2)
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    unit = Fraction(2) ** (max(e, -126) - 23)
    n, r = divmod(q, unit)
    n = int(n)
    if r > unit / 2 or (r == unit / 2 and n % 2 == 1):
        n += 1
    v = n * unit
    return float("inf") if v >= Fraction(2) ** 128 else float(v)


@pytest.mark.parametrize("amax", [1.0, 3.0, 7.0, 2688.0, 0.1, 1e-3, 123.456, 5e4, 1e30, 6.0 * 448 / 1024,
                                  8e-36, 7.9e-36])
def test_gain_exact_is_the_correctly_rounded_quotient(amax):
    """gain_exact(a) is 2688/a rounded once to binary32 (the exact rational quotient, rounded by
    the format's definition), and lies within half an ulp of it."""
    a = float(np.float32(amax))
    g = float(nvfp4.gain_exact(a))
    ref = _fl32(Fraction(2688) / Fraction(a))
    assert ref != float("inf")
    assert g == ref
    ulp = float(np.spacing(np.float32(g)))
    assert abs(Fraction(a) * Fraction(g) - 2688) <= Fraction(a) * Fraction(ulp) / 2


def test_gain_exact_degenerate_inputs():
    """amax = 0 and non-finite amax give g = 1; an amax whose quotient overflows (every subnormal,
    and normals below 2688 / FLT_MAX) saturates to the largest finite float32."""
    fmax = float(np.finfo(np.float32).max)
    assert nvfp4.gain_exact(0.0) == 1.0 and nvfp4.gain_exact(float("inf")) == 1.0 and nvfp4.gain_exact(float("nan")) == 1.0
    for a in (float(np.float32(1e-40)), float(np.float32(2.0 ** -149)), float(np.float32(2.0 ** -126)),
              float(np.float32(7.8e-36))):
        assert _fl32(Fraction(2688) / Fraction(a)) == float("inf")
        assert float(nvfp4.gain_exact(a)) == fmax
    # the smallest amax with a finite quotient is not clamped
    a = float(np.nextafter(np.float32(2688.0 / fmax), np.float32(1)))
    assert float(nvfp4.gain_exact(a)) == _fl32(Fraction(2688) / Fraction(a)) <= fmax
