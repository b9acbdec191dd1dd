"""CPU checks of the arithmetic shortcuts the kernels take, against the plain IEEE definitions.

The kernels replace a few correctly rounded operations by cheaper sequences whose equality with
the definition rests on an argument written beside them in the sources:

- multiply-and-snap (``snap12`` in csrc/common.cuh): for bf16 x, a power-of-two gain g and a UE4M3
  block scale sf, the E2M1 code of snap12(RN(x * RN(g * RN(1/sf)))) equals the code of
  RN(RN(x * g) / sf), the quantiser's element rule;
- Markstein's division with two remainder steps (``div_markstein`` in csrc/common.cuh, fp32;
  ``div_rn_by`` in csrc/stats.cu, fp64): RN(y / d) from r = RN(1/d) and fused multiply-adds;
- the quantiser's row quotient (csrc/quant.cu): trunc(RN(RN(i + 1/2) * RN(1/nb))) == i // nb;
- the bit-level roundings of csrc/common.cuh: ``ue4m3_rne`` (block scale to UE4M3, ties to even,
  saturating) and ``gain_pow2`` (largest power-of-two gain with amax * g <= 2688);
- the statistics' integer moments (csrc/moments.cuh): magic-number roundings give rint(x 2^16) and
  rint(x^2 2^14) for every in-range bf16 x, and raw-bit sums survive 32-bit wrap-around;
- the selection's key map (``order_bits`` in csrc/stats.cu) preserves the order of doubles.

Each is re-derived here with numpy's IEEE float32 / float64 operations, fused multiply-adds
emulated exactly with fractions, and compared with the definition, exhaustively where the domain
is small.  No GPU is needed; the GPU parity tests then hold the kernels to the oracle.
"""
from fractions import Fraction
import math

import numpy as np
import pytest

# ------------------------------------------------------------------------------- helpers
E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float64)   # between the 8 magnitudes


def e2m1_code(v: np.ndarray) -> np.ndarray:
    """E2M1 code (sign in bit 3) of float32 values: round to nearest, ties to the even code,
    saturating at 6; -0 keeps its sign."""
    a = np.abs(v.astype(np.float64))
    k = np.searchsorted(E2M1_MIDS, a, side="left")          # midpoints strictly below a
    tie = (k < len(E2M1_MIDS)) & (a == E2M1_MIDS[np.minimum(k, len(E2M1_MIDS) - 1)])
    idx = np.where(tie & (k % 2 == 1), k + 1, k)             # a tie goes to the even code
    sign = np.signbit(v).astype(np.int64) << 3
    return idx.astype(np.int64) | sign


def ue4m3_values() -> np.ndarray:
    """Values of the UE4M3 codes 1..126 (subnormals m * 2^-9, normals (1 + m/8) 2^(e-7))."""
    out = []
    for c in range(1, 127):
        e, m = c >> 3, c & 7
        out.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(out, np.float32)


def snap12(p: np.ndarray) -> np.ndarray:
    b = p.view(np.uint32)
    return ((b + np.uint32(0x800)) & np.uint32(0xFFFFF000)).view(np.float32)


def all_finite_bf16() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    return x[np.isfinite(x)]


def rn32(q: Fraction) -> np.float32:
    """Correct round-to-nearest-even of a rational to float32 (normal range)."""
    if q == 0:
        return np.float32(0.0)
    s = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    scaled = a * Fraction(2) ** (23 - e)                      # in [2^23, 2^24)
    n, rem = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * rem
    if twice > scaled.denominator or (twice == scaled.denominator and n % 2 == 1):
        n += 1
    return np.float32(s * float(Fraction(n) * Fraction(2) ** (e - 23)))


def fma32(a, b, c) -> np.float32:
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def fma64(a: float, b: float, c: float) -> float:
    return float(Fraction(a) * Fraction(b) + Fraction(c))     # float(Fraction) rounds correctly


# ------------------------------------------------------------------------------- multiply-and-snap
@pytest.mark.parametrize("log2g", [-8, 0, 7])
def test_multiply_and_snap_gives_the_e2m1_code_of_the_two_step_division(log2g):
    """Every finite bf16 x, every UE4M3 scale, power-of-two gains: the fast path's code equals the
    element rule's code wherever the kernel uses it (|x g| <= 2688 = 6 * 448, the encode gain's
    bound, so x g / sf stays finite)."""
    g = np.float32(2.0 ** log2g)
    x = all_finite_bf16()
    x = x[np.abs(x.astype(np.float64) * float(g)) <= 2688.0]
    for sf in ue4m3_values():
        sr = np.float32(1.0) / sf                                  # RN(1/sf)
        exact = (x * g) / sf                                       # RN(RN(x g) / sf)
        fast = snap12(x * (g * sr))                                # RN(g sr) is exact for g = 2^k
        got, want = e2m1_code(fast), e2m1_code(exact)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, f"sf={sf}: x={x[bad[:4]]} codes {got[bad[:4]]} != {want[bad[:4]]}"


def test_e2m1_reference_rounding():
    """The reference rounding above: midpoints go to the even code, values at or above 5 beyond
    the 4..6 midpoint saturate at 6, -0 keeps its sign."""
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.01, 7.0, 1e30, -0.0, -0.26, 0.24], np.float32)
    assert e2m1_code(v).tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 7, 7, 8, 9, 0]


# ------------------------------------------------------------------------------- row quotient
def test_fp32_row_quotient_is_exact():
    """trunc(RN(RN(i + 1/2) * RN(1/nb))) == i // nb for every nb = K/16 with K % 64 == 0 up to
    K = 16384, and every block index i of a chunk (below 2^18)."""
    i = np.arange(1 << 18, dtype=np.int64)
    fi = i.astype(np.float32) + np.float32(0.5)
    for nb in range(4, 1025, 4):
        inv = np.float32(1.0) / np.float32(nb)
        q = (fi * inv).astype(np.int64)                            # float -> int truncates
        assert np.array_equal(q, i // nb), f"nb={nb}"


# ------------------------------------------------------------------------------- Markstein division
def div_markstein32(y, d, r):
    q0 = np.float32(y * r)
    e0 = fma32(-q0, d, y)
    q1 = fma32(e0, r, q0)
    e1 = fma32(-q1, d, y)
    q2 = fma32(e1, r, q1)
    return np.float32(math.copysign(abs(float(q2)), float(y)))


def div_rn_by64(y: float, d: float, r: float) -> float:
    q0 = y * r
    e0 = fma64(-q0, d, y)
    q1 = fma64(e0, r, q0)
    e1 = fma64(-q1, d, y)
    return fma64(e1, r, q1)


def test_markstein_fp32_block_scale_and_element_division():
    """RN(y / d) for the divisors the quantiser uses: d = 6 (block scale t = fl32(a g) / 6) and
    every UE4M3 value (element v = fl32(x g) / sf), on random and near-tie dividends."""
    rng = np.random.default_rng(5)
    divisors = [np.float32(6.0)] + list(ue4m3_values()[::5])
    for d in divisors:
        r = np.float32(1.0) / d
        ys = list(rng.standard_normal(60).astype(np.float32) * np.float32(rng.uniform(0.01, 300)))
        # dividends whose quotient is (next to) a midpoint of float32 values: y = RN(d * m) for
        # m halfway between neighbours
        for m in rng.uniform(0.1, 10.0, 20).astype(np.float32):
            mid = (Fraction(float(m)) + Fraction(float(np.nextafter(m, np.float32(20))))) / 2
            ys.append(rn32(mid * Fraction(float(d))))
        ys += [np.float32(-0.0), np.float32(0.0)]
        for y in ys:
            got = div_markstein32(y, d, r)
            want = rn32(Fraction(float(y)) / Fraction(float(d))) if y != 0 else y
            assert got == want and np.signbit(got) == np.signbit(want), (float(y), float(d))


def test_markstein_fp64_selection_key_division():
    """The selection's m = fl64(fl64(s / 2^k) / n) with n the row count: two remainder steps from
    RN(1/n) give the correctly rounded quotient, on random moments and counts and on exact
    quotients."""
    rng = np.random.default_rng(9)
    cases = []
    for _ in range(3000):
        n = int(rng.integers(1, 1 << 22))
        s = int(rng.integers(-(1 << 62), 1 << 62))
        cases.append((float(s) / 2.0 ** 14, float(n)))
    for _ in range(500):                                           # exact quotients
        n = int(rng.integers(1, 1 << 20))
        q = int(rng.integers(-(1 << 30), 1 << 30))
        cases.append((float(q * n) / 2.0 ** 16, float(n)))
    for y, d in cases:
        r = 1.0 / d                                                # RN(1/d) in IEEE double
        assert div_rn_by64(y, d, r) == float(Fraction(y) / Fraction(d)), (y, d)


# ------------------------------------------------------------------------------- UE4M3 and gain bits
def ue4m3_rne_bits(t: np.ndarray) -> np.ndarray:
    """The block-scale rounding of csrc/common.cuh (``ue4m3_rne``) step by step on float32 bits:
    saturate at 448, subnormals as rint(t * 512), otherwise round the fraction to 3 bits (ties to
    even) with one integer add and rebias the exponent."""
    t = t.astype(np.float32)
    b = t.view(np.uint32).astype(np.int64)
    b = b + 0x7FFFF + ((b >> 20) & 1)
    normal = ((((b >> 23) - 120) << 3) | ((b >> 20) & 7))
    normal = np.minimum(normal, 0x7E)
    sub = np.rint((t * np.float32(512.0)).astype(np.float64)).astype(np.int64)   # rint: ties to even
    return np.where(t >= np.float32(448.0), 0x7E, np.where(t < np.float32(0.015625), sub, normal))


def test_ue4m3_bit_rounding_matches_the_definition_on_every_float32_scale():
    """Every float32 t from 2^-12 up to 2^9 (and 0), binade by binade: the bit-level rounding
    equals round-to-nearest-even onto the UE4M3 values, saturating at 448."""
    from oracle import nvfp4
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(127 - 12, 127 + 9):
        t = ((np.uint32(e) << np.uint32(23)) | mant).view(np.float32)
        assert np.array_equal(ue4m3_rne_bits(t), nvfp4.ue4m3_encode(t)), f"binade 2^{e - 127}"
    z = np.zeros(1, np.float32)
    assert ue4m3_rne_bits(z)[0] == 0 == nvfp4.ue4m3_encode(z)[0]


def gain_pow2_bits(amax: np.ndarray) -> np.ndarray:
    """The encode gain of csrc/common.cuh (``gain_pow2``) on float32 bits, for finite amax > 0."""
    a = amax.astype(np.float32)
    b = a.view(np.uint32).astype(np.int64)
    subn = (b >> 23) == 0
    bias = np.where(subn, 64, 0)
    with np.errstate(over="ignore"):                           # evaluated for normal a too, unused there
        scaled = (a * np.float32(2.0 ** 64)).view(np.uint32).astype(np.int64)
    b = np.where(subn, scaled, b)
    e = (b >> 23) - 126 - bias
    frac = b & 0x7FFFFF
    E = np.where(frac <= 0x280000, 12 - e, 11 - e)
    E = np.clip(E, -126, 127)
    return E


def test_pow2_gain_bits_give_the_largest_fitting_power():
    """For amax over every float32 binade (normal and subnormal) with mantissas at and around
    the 0.65625 boundary plus random ones: g = 2^E is the largest power of two with
    amax * g <= 2688, E clamped to [-126, 127] (products with powers of two are exact in float64)."""
    rng = np.random.default_rng(3)
    mants = np.unique(np.concatenate([
        np.array([0, 1, 0x27FFFF, 0x280000, 0x280001, 0x7FFFFE, 0x7FFFFF, 0x400000], np.int64),
        rng.integers(0, 1 << 23, 64)]))
    amax = []
    for e in range(0, 255):
        for m in mants:
            if e == 0 and m == 0:
                continue
            amax.append((e << 23) | int(m))
    a = np.array(amax, np.uint32).view(np.float32)
    E = gain_pow2_bits(a)
    a64 = a.astype(np.float64)
    fits = a64 * np.exp2(E.astype(np.float64)) <= 2688.0
    next_fits = a64 * np.exp2(E.astype(np.float64) + 1) <= 2688.0
    assert np.all(fits | (E == -126)), "gain too large"
    assert np.all(~next_fits | (E == 127)), "a larger power of two would fit"


# ------------------------------------------------------------------------------- integer moments
MAGIC = np.float32(12582912.0)          # 1.5 * 2^23
MAGIC8 = np.float32(3221225472.0)       # 1.5 * 2^31
MAGIC_BITS, MAGIC8_BITS = 0x4B400000, 0x4F400000


def moment_raw_terms(x: np.ndarray):
    """The four raw-bit terms csrc/moments.cuh (``add_bf16``) adds per in-range element, as
    uint32: fp32 additions with the magic constants round to integers (ties to even); the
    multiply-adds are an exact product plus one rounding, as numpy's float32 add reproduces."""
    x = x.astype(np.float32)
    t1 = x + MAGIC
    frac = x - (t1 - MAGIC)
    b1 = frac * np.float32(65536.0) + MAGIC
    y = x * x
    u = y + MAGIC8
    yl = y - (u - MAGIC8)
    d2 = yl * np.float32(16384.0) + MAGIC
    return [v.view(np.uint32).astype(np.int64) for v in (t1, b1, u, d2)]


def rint_even(num: int, den: int) -> int:
    q, r = divmod(num, den)
    return q + (1 if 2 * r > den or (2 * r == den and q % 2 == 1) else 0)


def test_integer_moment_terms_of_every_bf16_value():
    """For every bf16 x with |x| < 2^15: the recovered terms give s1 = rint(x 2^16) and
    s2 = rint(x^2 2^14) exactly (ties to even), the statistics' fixed-point definition."""
    x = all_finite_bf16()
    x = x[np.abs(x) < 32768.0]
    a1, b1, c2, d2 = moment_raw_terms(x)
    s1 = (a1 - MAGIC_BITS) * 65536 + (b1 - MAGIC_BITS)
    s2 = (c2 - MAGIC8_BITS) * 4194304 + (d2 - MAGIC_BITS)
    for xi, g1, g2 in zip(x.tolist(), s1.tolist(), s2.tolist()):
        f = Fraction(xi)
        assert g1 == rint_even(f.numerator * 65536, f.denominator), xi
        assert g2 == rint_even(f.numerator ** 2 * 16384, f.denominator ** 2), xi


def test_integer_moments_survive_wrapping_32_bit_sums_of_256_rows():
    """Raw-bit terms of 256 rows summed modulo 2^32, minus 256 magic patterns, give the exact sums
    of the terms, for rows at the range limit (the largest terms) and random rows."""
    rng = np.random.default_rng(7)
    cases = [np.full(256, np.float32(32512.0)), np.full(256, np.float32(-32512.0)),
             (rng.standard_normal(256) * 3000).astype(np.float32),
             (rng.standard_normal(256) * 0.01).astype(np.float32)]
    for rows in cases:
        rows = (rows.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)   # bf16 values
        terms = moment_raw_terms(rows)
        magics = (MAGIC_BITS, MAGIC_BITS, MAGIC8_BITS, MAGIC_BITS)
        for t, m in zip(terms, magics):
            wrapped = int(t.sum()) % (1 << 32)
            small = (wrapped - 256 * m) % (1 << 32)
            small = small - (1 << 32) if small >= (1 << 31) else small    # back to int32
            assert small == int((t - m).sum())


def order_bits(k: np.ndarray) -> np.ndarray:
    """The selection's key map of csrc/stats.cu (``order_bits``): -0 folded onto +0, then
    negative doubles' bits inverted and positive ones' sign bit set."""
    k = np.where(k == 0.0, 0.0, k)
    b = k.view(np.uint64)
    return np.where((b >> np.uint64(63)) == 1, ~b, b | np.uint64(1 << 63))


def test_selection_key_map_preserves_the_order_of_doubles():
    """Sorting by the mapped integers sorts the keys (ties exactly where the keys are equal, -0
    equal to +0), over random doubles of both signs and magnitudes and the special values the
    keys can take (zero of both signs, subnormals, the largest finite)."""
    rng = np.random.default_rng(13)
    k = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        np.array([0.0, -0.0, 5e-324, -5e-324, 1.7976931348623157e308,
                                  -1.7976931348623157e308, 1.0, -1.0, 1.0])])
    m = order_bits(k)
    i, j = rng.integers(0, len(k), (2, 200000))
    assert np.array_equal(m[i] < m[j], k[i] < k[j])
    assert np.array_equal(m[i] == m[j], k[i] == k[j])
    sp = k[-9:]                                                    # every pair of the special values
    ms = order_bits(sp)
    assert np.array_equal(ms[:, None] < ms[None, :], sp[:, None] < sp[None, :])
    assert np.array_equal(ms[:, None] == ms[None, :], sp[:, None] == sp[None, :])


# ------------------------------------------------------------------------------- K3 small-|d| branch
def k3_series_like_the_kernel(d: np.float32) -> np.float32:
    """csrc/train.cu ``k3_of`` for |d| < 1/16: d^2/2 (1 + d/3 (1 + d/4 (1 + d/5 (1 + d/6 (1 + d/7)))))
    with fused multiply-adds and float32 products, constants RN(1/k)."""
    one = np.float32(1.0)
    p = fma32(d, np.float32(1.0) / np.float32(7.0), one)
    for k in (6.0, 5.0, 4.0, 3.0):
        p = fma32(np.float32(d * (np.float32(1.0) / np.float32(k))), p, one)
    return np.float32(np.float32(np.float32(np.float32(0.5) * d) * d) * p)


def test_k3_series_branch_is_accurate_to_float32():
    """Against the definition e^d - 1 - d evaluated to 60 digits: relative error below 2^-22 (three
    roundings of at most 2^-24 each and the truncated series, whose first omitted term is below
    2^-38 of the result at |d| = 1/16), and never negative (k3 >= 0).  Observed worst: 2^-22.6.
    This pins accuracy, not the term count: terms to d^5 would already truncate below 2^-28."""
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-40, -4, 3000)).astype(np.float32)
    edge = np.nextafter(np.float32(0.0625), np.float32(0.0), dtype=np.float32)
    ds = np.concatenate([mags, -mags, [edge, -edge, np.float32(2.0 ** -20), np.float32(-(2.0 ** -20))]]).astype(np.float32)
    worst = 0.0
    for d in ds:
        assert abs(float(d)) < 0.0625
        got = k3_series_like_the_kernel(d)
        D = Decimal(float(d))
        exact = D.exp() - 1 - D
        assert got >= 0
        worst = max(worst, float(abs((Decimal(float(got)) - exact) / exact)))
    assert worst < 2.0 ** -22, worst
