"""FP8 (E4M3, E5M2) and bf16 codecs, written from the format definitions.

Test infrastructure only (see the package docstring).

The AstrAI commit logs name the two formats only through their use: E4M3
for activations and weights, E5M2 for gradients, and a saturation point of
"about 448" (``astrai/extension/fp8.py @4dc5e923``, the bullet on the amax
bug). The bit layouts therefore come from the OCP 8-bit floating point
specification (OFP8 rev. 1.0):

* E4M3 ("FN" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits. No
  infinities; S.1111.111 is NaN, so the largest finite magnitude is
  S.1111.110 = 1.75 * 2^8 = 448. Subnormals: m * 2^-9.
* E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits, IEEE-like:
  exponent 31 holds +-Inf (m = 0) and NaN (m != 0). Largest finite
  magnitude S.11110.11 = 1.75 * 2^15 = 57344. Subnormals: m * 2^-16.

Encoding reading (the pages ask for round-to-nearest-even with saturation):
the finite code whose value is nearest to the input; on an exact tie the code
with an even bit pattern; any magnitude above the largest finite value
(infinity included) saturates to that value with the input's sign; NaN maps
to 0x7F; the sign of zero is kept (-0 -> 0x80).
"""

import math

import numpy as np

E4M3 = 0
E5M2 = 1

# Largest finite magnitudes (OFP8 rev. 1.0, tables of the two encodings).
FMT_MAX = {E4M3: 448.0, E5M2: 57344.0}
_MAX_CODE = {E4M3: 0x7E, E5M2: 0x7B}
_NAN_CODE = 0x7F


def decode(code: int, fmt: int) -> float:
    """Value of one FP8 code, from the sign / exponent / mantissa fields."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    if fmt == E4M3:
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            return math.nan
        if e == 0:
            return sign * m * 2.0 ** -9
        return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    if fmt == E5M2:
        e = (code >> 2) & 0x1F
        m = code & 0x3
        if e == 0x1F:
            return sign * math.inf if m == 0 else math.nan
        if e == 0:
            return sign * m * 2.0 ** -16
        return sign * (1.0 + m / 4.0) * 2.0 ** (e - 15)
    raise ValueError(f"unknown fp8 format {fmt}")


def decode_table(fmt: int) -> np.ndarray:
    """All 256 decoded values of ``fmt`` as float64 (NaN for NaN codes)."""
    return np.array([decode(c, fmt) for c in range(256)], dtype=np.float64)


def encode(v, fmt: int) -> np.ndarray:
    """fp32 values -> FP8 codes (uint8), nearest-even with saturation.

    ``v`` is any array-like of fp32 values. The search is over the
    non-negative finite codes 0x00 .. max code, whose values increase with
    the code, so the nearest one lies next to the insertion point.
    """
    v = np.asarray(v, dtype=np.float32)
    shape = v.shape
    v = v.reshape(-1).astype(np.float64)
    max_code = _MAX_CODE[fmt]
    table = decode_table(fmt)[: max_code + 1]  # ascending, all finite
    mag = np.abs(v)
    sign = np.signbit(v).astype(np.uint8) << 7
    nan = np.isnan(v)
    mag_safe = np.where(nan, 0.0, mag)

    hi = np.searchsorted(table, mag_safe, side="left")  # table[hi] >= mag
    hi_c = np.minimum(hi, max_code)
    lo_c = np.maximum(hi - 1, 0)
    d_hi = table[hi_c] - mag_safe
    d_lo = mag_safe - table[lo_c]
    pick_hi = d_hi < d_lo
    tie = d_hi == d_lo
    # exact tie between two codes: the even bit pattern wins
    pick_hi = np.where(tie, (hi_c & 1) == 0, pick_hi)
    code = np.where(pick_hi, hi_c, lo_c).astype(np.uint8)
    code = np.where(mag_safe > table[max_code], np.uint8(max_code), code)
    code = (code | sign).astype(np.uint8)
    code = np.where(nan, np.uint8(_NAN_CODE), code).astype(np.uint8)
    return code.reshape(shape)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> their exact fp32 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def bf16_round_from_f64(v) -> np.ndarray:
    """Round fp64 values to bf16 (nearest-even, ONE rounding), as fp32.

    bf16 has an 8-bit significand (7 stored bits), exponent range of fp32
    and subnormals down to 2^-133. Rounding is done on the integer grid of
    the value's own ulp: ``rint`` is ties-to-even and an even integer
    multiple of the ulp is an even mantissa. Rounding through fp32 first
    would round twice, which is why this does not use ``astype(float32)``.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float64)
    flat = v.reshape(-1)
    res = out.reshape(-1)
    finite = np.isfinite(flat)
    a = np.abs(flat)
    nz = finite & (a > 0)
    _, ex = np.frexp(np.where(nz, a, 1.0))  # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -126)  # floor(log2 a), clamped at the subnormal floor
    ulp = np.ldexp(1.0, e - 7)
    r = np.rint(np.where(nz, a, 0.0) / ulp) * ulp
    r = np.where(r >= 2.0 ** 128, np.inf, r)  # rounded past the largest bf16
    res[:] = np.where(finite, np.copysign(r, flat), flat)
    return out.astype(np.float32)
