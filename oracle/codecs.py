"""bf16 and FP8 E4M3 codecs for the oracle, in float64 (test infrastructure only).

Written from the format definitions, not from any library:

* bf16 ("brain float"): the upper half of an IEEE-754 binary32 word. 1 sign bit, 8 exponent
  bits with bias 127, 7 fraction bits; exponent field 0 encodes zero/subnormals
  (value = f/128 * 2**-126), exponent field 255 encodes inf (f == 0) and NaN (f != 0).
* OCP 8-bit floating point, E4M3 variant (the FP8 KV-cache format; the Step-3 pages state
  the whole model runs in FP8, bud-325 summary, "Key claims"): 1 sign bit, 4 exponent bits
  with bias 7, 3 fraction bits. Exponent field 0 encodes zero/subnormals
  (value = f/8 * 2**-6). There is no infinity; the single pattern S.1111.111 is NaN, so the
  largest finite magnitude is 1.75 * 2**8 = 448.

Encoding rounds to nearest, ties to even (the reading taken for every rounding point of the
layer, since the pages do not state one). E4M3 encoding saturates finite and infinite
overflow to +-448 ("satfinite"); NaN stays NaN.

Pinned by: exhaustive decode of all 2**16 bf16 and all 2**8 E4M3 patterns against
independent routes (binary32 reinterpretation, torch's float8 dtype), encode of random,
tie, subnormal and overflow values against torch's conversions, and round-trip of every
code (tests/test_oracle_codecs.py).
"""

import numpy as np

# ----------------------------------------------------------------------------------------
# generic value-grid rounding
# ----------------------------------------------------------------------------------------


def _round_to_grid(a, frac_bits, emin):
    """Round non-negative finite float64 magnitudes ``a`` to the nearest value of a binary
    format with ``frac_bits`` fraction bits and minimum normal exponent ``emin``
    (ties to even, unbounded exponent range above). Exact: the grid spacing is a power of
    two, so ``a / ulp`` is exact in float64 and ``np.rint`` performs the tie-to-even step."""
    a = np.asarray(a, dtype=np.float64)
    _, ex = np.frexp(a)  # a = m * 2**ex, m in [0.5, 1)  =>  floor(log2 a) = ex - 1
    e = np.maximum(ex.astype(np.int64) - 1, emin)
    e = np.where(a == 0, emin, e)
    ulp = np.ldexp(1.0, e - frac_bits)
    return np.rint(a / ulp) * ulp


def _grid_value_to_fields(r, frac_bits, emin, bias):
    """Split exactly representable magnitudes ``r`` into (biased exponent, fraction)."""
    r = np.asarray(r, dtype=np.float64)
    m, ex = np.frexp(r)
    e = ex.astype(np.int64) - 1
    normal = (r != 0) & (e >= emin)
    exp_field = np.where(normal, e + bias, 0)
    frac_normal = np.rint((2.0 * m - 1.0) * (1 << frac_bits))
    frac_sub = np.rint(r / np.ldexp(1.0, emin - frac_bits))
    frac = np.where(normal, frac_normal, frac_sub)
    return exp_field.astype(np.int64), frac.astype(np.int64)


# ----------------------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------------------

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_decode(bits):
    """bf16 bit patterns (any integer dtype, values 0..65535) -> float64 values."""
    b = np.asarray(bits).astype(np.int64) & 0xFFFF
    s = (b >> 15) & 1
    e = (b >> 7) & 0xFF
    f = b & 0x7F
    sign = np.where(s == 1, -1.0, 1.0)
    with np.errstate(over="ignore", invalid="ignore"):
        normal = sign * np.ldexp(1.0 + f / 128.0, e - 127)
        sub = sign * np.ldexp(f / 128.0, -126)
        val = np.where(e == 0, sub, normal)
        special = np.where(f == 0, sign * np.inf, np.nan)
    return np.where(e == 255, special, val)


def bf16_encode(x):
    """float64 values -> bf16 bit patterns (uint16), round to nearest even; overflow -> inf;
    NaN -> 0x7FC0 with the input's sign bit."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64)
    a = np.abs(x)
    finite = np.isfinite(a)
    a_f = np.where(finite, a, 0.0)
    r = _round_to_grid(a_f, 7, -126)
    overflow = r > BF16_MAX
    e, f = _grid_value_to_fields(np.where(overflow, 0.0, r), 7, -126, 127)
    bits = (sign << 15) | (e << 7) | f
    bits = np.where(overflow | np.isinf(a), (sign << 15) | 0x7F80, bits)
    bits = np.where(np.isnan(x), (sign << 15) | 0x7FC0, bits)
    return bits.astype(np.uint16)


def bf16_round(x):
    """float64 -> nearest bf16 value, as float64 (the value a bf16 buffer would hold)."""
    return bf16_decode(bf16_encode(x))


# ----------------------------------------------------------------------------------------
# FP8 E4M3 (OCP)
# ----------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """E4M3 codes (any integer dtype, values 0..255) -> float64 values."""
    c = np.asarray(codes).astype(np.int64) & 0xFF
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    f = c & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    normal = sign * np.ldexp(1.0 + f / 8.0, e - 7)
    sub = sign * np.ldexp(f / 8.0, -6)
    val = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (f == 7), np.nan, val)


def e4m3_encode(x):
    """float64 values -> E4M3 codes (uint8), round to nearest even, saturating to +-448
    (infinities included); NaN -> 0x7F with the input's sign bit."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x).astype(np.int64)
    a = np.abs(x)
    nan = np.isnan(a)
    a_f = np.where(nan, 0.0, np.minimum(a, 2.0 * E4M3_MAX))
    r = np.minimum(_round_to_grid(a_f, 3, -6), E4M3_MAX)
    e, f = _grid_value_to_fields(r, 3, -6, 7)
    codes = (sign << 7) | (e << 3) | f
    codes = np.where(nan, (sign << 7) | 0x7F, codes)
    return codes.astype(np.uint8)


def e4m3_round(x):
    """float64 -> nearest (saturated) E4M3 value, as float64."""
    return e4m3_decode(e4m3_encode(x))
