"""NVFP4 numerics: codecs, encode gains, the masked block quantiser, packing.

TEST INFRASTRUCTURE ONLY (see the package docstring).

NVFP4 as FourSight uses it (§2.1 "Quantized RL Post-training"; §9.3.1 "The
NVFP4 format", Eq. 9): values are E2M1 with the finite set
{0, ±0.5, ±1, ±1.5, ±2, ±3, ±4, ±6}; tensors are cut along the reduction
dimension K into blocks of B = 16 elements that share one E4M3 scale (unsigned
here, UE4M3: unit roundoff 1/16 for normals); a tensor-wide FP32 encode gain g
sits above the block scales.  Eq. 9 gives the block's physical scale as
``s_b = round_E4M3(g * a_b / 6) / g`` with ``a_b`` the block's absolute maximum
after protected lanes are zeroed.

Readings taken where the paper is silent:
* every rounding is round-to-nearest, ties to the even code; values beyond the
  largest finite code saturate to it (no NaN/Inf is ever produced);
* fp32 operation order: ``t = fl32(fl32(a_b*g)/6)``, ``sf = RNE_UE4M3(t)``, and for
  each element ``v = fl32(fl32(x*g)/sf)``, ``q = RNE_E2M1(v)`` (IEEE divisions);
* the sign of zero is kept (-0 encodes as 0x8); a zero block scale gives every
  element the code 0 with its own sign; masked lanes are +0 (code 0x0);
* the gain: largest power of two g with ``amax*g <= 6*448``, or fl32(2688/amax)
  (saturated to the largest finite float32) under the exact-gain option; amax = 0
  gives g = 1.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 16
E2M1_MAX = 6.0
UE4M3_MAX = 448.0
GAIN_TARGET = E2M1_MAX * UE4M3_MAX          # 2688: the largest representable |q*sf|

# E2M1 magnitudes by 3-bit code (sign is bit 3): {0, .5, 1, 1.5, 2, 3, 4, 6}.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes) -> np.ndarray:
    """4-bit code -> value (float64).  Bit 3 is the sign, bits 0-2 index the magnitude."""
    c = np.asarray(codes, dtype=np.int64)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where((c >> 3) & 1, -mag, mag)


def _ue4m3_table() -> np.ndarray:
    """Values of the finite UE4M3 codes 0x00..0x7E (exponent bias 7, 3 mantissa bits)."""
    vals = np.empty(127)
    for code in range(127):
        e, m = code >> 3, code & 7
        vals[code] = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


UE4M3_VALUES = _ue4m3_table()               # ascending in code order


def ue4m3_decode(codes) -> np.ndarray:
    """8-bit UE4M3 code -> value (float64); 0x7F is NaN, codes >= 0x80 are not UE4M3."""
    c = np.asarray(codes, dtype=np.int64)
    if np.any((c < 0) | (c > 0x7F)):
        raise ValueError("UE4M3 codes are 0..0x7F")
    out = np.where(c == 0x7F, np.nan, UE4M3_VALUES[np.minimum(c, 126)])
    return out


def _rne_to_table(mag, table) -> np.ndarray:
    """Index of the nearest entry of ``table`` (ascending, index == code) to each |value|.

    Ties go to the even index; magnitudes above the last entry saturate to it.
    Differences are formed in float64, exact for float32 inputs and these dyadic tables.
    """
    v = np.asarray(mag, dtype=np.float64)
    lo = np.searchsorted(table, v, side="right") - 1          # largest i with table[i] <= v
    lo = np.clip(lo, 0, len(table) - 1)
    hi = np.minimum(lo + 1, len(table) - 1)
    d_lo = v - table[lo]
    d_hi = table[hi] - v
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    idx = np.where(pick_hi, hi, lo)
    return np.where(v >= table[-1], len(table) - 1, idx).astype(np.int64)


def e2m1_encode(v) -> np.ndarray:
    """float32 value -> 4-bit E2M1 code, round to nearest even, saturating at ±6, sign kept."""
    v = np.asarray(v, dtype=np.float32)
    idx = _rne_to_table(np.abs(v), E2M1_MAGNITUDES)
    sign = np.signbit(v).astype(np.int64)
    return (sign << 3) | idx


def ue4m3_encode(t) -> np.ndarray:
    """Non-negative float32 -> UE4M3 code, round to nearest even, saturating at 448."""
    t = np.asarray(t, dtype=np.float32)
    if np.any(t < 0) or np.any(~np.isfinite(t)):
        raise ValueError("block scale must be finite and non-negative")
    return _rne_to_table(t, UE4M3_VALUES)


# ---------------------------------------------------------------------------------------
# Encode gains (the FP32 tensor-wise scale of §2.1; g_A, g_W of §9.3.1)
# ---------------------------------------------------------------------------------------
def gain_pow2(amax: float) -> np.float32:
    """Largest power of two g with amax*g <= 2688 (exponent clamped to [-126, 127]); 1 if amax == 0.

    Exact integer rule: with amax = f*2^e, f in [0.5, 1) and 2688 = 0.65625*2^12,
    the exponent is 12-e when f <= 0.65625 and 11-e otherwise.
    """
    a = float(np.float32(amax))
    if a == 0.0 or not math.isfinite(a):
        return np.float32(1.0)
    f, e = math.frexp(a)
    E = 12 - e if f <= 0.65625 else 11 - e
    E = max(-126, min(127, E))
    return np.float32(2.0 ** E)


FLOAT32_MAX = np.float32(np.finfo(np.float32).max)


def gain_exact(amax: float) -> np.float32:
    """fl32(2688 / amax), saturated to the largest finite float32; 1 if amax == 0 or not finite.

    The common NVFP4 tensor-scale recipe.  The gain must be a finite FP32 value: for amax below
    2688 / FLT_MAX (every subnormal amax) the IEEE quotient overflows, and the gain saturates, as
    the power-of-two rule clamps its exponent at 127.
    """
    a = np.float32(amax)
    if a == 0 or not np.isfinite(a):
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        q = np.float32(np.float32(GAIN_TARGET) / a)
    return np.float32(min(q, FLOAT32_MAX))


def alpha_from_gains(gA, gW) -> np.float32:
    """alpha = fl32(1 / fl32(gA*gW)), the output scale of Eq. 5."""
    return np.float32(np.float32(1.0) / np.float32(np.float32(gA) * np.float32(gW)))


# ---------------------------------------------------------------------------------------
# Block quantiser (Eq. 9 with the protected lanes zeroed first, §5.1 "Mask S->0")
# ---------------------------------------------------------------------------------------
def quantize_blocks(x, keep, g, scale_from_all_lanes: bool = False):
    """Quantise rows of ``x`` [R, K] (float32) in 16-element blocks along K.

    ``keep`` is a bool [K] vector: False marks a protected channel, whose lane is
    zeroed before anything else (split form), so it can widen no block scale.
    With ``scale_from_all_lanes`` the block maximum is taken before zeroing and
    only the codes are zeroed afterwards (the residual-correction form).
    Returns (codes int64 [R,K], sf codes int64 [R,K/16]).
    """
    x = np.asarray(x, dtype=np.float32)
    R, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    keep = np.asarray(keep, dtype=bool)
    g = np.float32(g)
    xm = np.where(keep[None, :], x, np.float32(0.0)).astype(np.float32)
    src = x if scale_from_all_lanes else xm
    a_b = np.abs(src).reshape(R, K // BLOCK, BLOCK).max(axis=2).astype(np.float32)
    t = (np.float32(a_b * g) / np.float32(6.0)).astype(np.float32)
    sf = ue4m3_encode(t)
    sfv = ue4m3_decode(sf).astype(np.float32)
    sfv_e = np.repeat(sfv, BLOCK, axis=1)
    xg = (xm * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (xg / sfv_e).astype(np.float32)
    codes = e2m1_encode(v)
    zero_scale = sfv_e == 0
    codes = np.where(zero_scale, np.signbit(xm).astype(np.int64) << 3, codes)
    codes = np.where(keep[None, :], codes, 0)
    return codes, sf


def dequantize(codes, sf, g=None):
    """Element values q*sf (float64), divided by g when given: x_hat = q*sf/g."""
    codes = np.asarray(codes)
    sfv = np.repeat(ue4m3_decode(sf), BLOCK, axis=1)
    v = e2m1_decode(codes) * sfv
    return v if g is None else v / np.float64(np.float32(g))


# ---------------------------------------------------------------------------------------
# Storage layouts
# ---------------------------------------------------------------------------------------
def pack_codes(codes) -> np.ndarray:
    """[R,K] 4-bit codes -> [R,K/2] bytes; the even element of each pair is the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.int64)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def sf_tiled_shape(rows: int, K: int):
    """(rows padded to 128, K/16 blocks padded to 4): the extents of the tiled scale array."""
    return ((rows + 127) // 128) * 128, ((K // BLOCK + 3) // 4) * 4


def sf_tiled_offset(r, b, K):
    """Byte offset of the scale of row r, block b in the MMA-ready tiled scale array.

    The array is a sequence of 512-byte atoms, each holding 128 rows x 4 blocks;
    atoms run first along K (all block groups of one 128-row group), then along
    rows.  Inside an atom, row r sits at byte (r%32)*16 + ((r%128)//32)*4 and its
    4 blocks are consecutive bytes.
    """
    r = np.asarray(r, dtype=np.int64)
    b = np.asarray(b, dtype=np.int64)
    kb4 = (K // BLOCK + 3) // 4
    return ((r // 128) * kb4 + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)


def sf_to_tiled(sf_rowmajor, K) -> np.ndarray:
    """Row-major [R, K/16] scale codes -> tiled byte array (padding bytes zero)."""
    sf = np.asarray(sf_rowmajor, dtype=np.uint8)
    R, nb = sf.shape
    Rp, nbp = sf_tiled_shape(R, K)
    out = np.zeros(Rp * nbp, np.uint8)
    rr, bb = np.meshgrid(np.arange(R), np.arange(nb), indexing="ij")
    out[sf_tiled_offset(rr, bb, K)] = sf
    return out


def sf_from_tiled(tiled, R, K) -> np.ndarray:
    """Tiled byte array -> row-major [R, K/16] scale codes."""
    t = np.asarray(tiled, dtype=np.uint8)
    rr, bb = np.meshgrid(np.arange(R), np.arange(K // BLOCK), indexing="ij")
    return t[sf_tiled_offset(rr, bb, K)]


# ---------------------------------------------------------------------------------------
# bf16 (the precision the protected channels keep, §4.2)
# ---------------------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """float32 -> nearest bf16 value (ties to even), returned as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x) -> np.ndarray:
    return (bf16_round(x).view(np.uint32) >> 16).astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
