"""The numeric facts the FP8 attention's e4m3 products rest on, checked exhaustively on the
host with the e4m3 and bf16 codecs written from the format definitions (oracle/codecs.py).

For an FP8 cache the attention's S = K Q^T and O = P V run on e4m3 operands. The cached codes
are used as they are, while Q and P (values that carry more precision) are written as a pair
of e4m3 values with one common power-of-two scale: hi = e4m3(x), lo = e4m3(x - hi). The
kernel computes in f16x2: x is first rounded to f16, the remainder x - hi and the sum hi + lo
are taken in f16. This file checks that those steps are exact where the kernel needs them
exact, that hi + lo is within 2^-8 |x| of x (for |x| >= 1/4; within 2^-10 below), the
size of a bf16 rounding, and that for bf16 inputs (Q) the pair is exact. Q is scaled so that
its largest magnitude lies in [128, 256). P = 2^(s - m + 4), with the running max m raised
once a score exceeds it by more than 4, so P <= 2^8. Neither ever reaches e4m3's largest
value, 448.
"""

import numpy as np

from oracle import codecs


def _f16_values(lo, hi):
    """Every non-negative f16 value in [lo, hi]."""
    bits = np.arange(0, 0x7C00, dtype=np.uint16)
    v = bits.view(np.float16).astype(np.float64)
    return v[(v >= lo) & (v <= hi)]


def _split(x):
    hi = codecs.e4m3_round(x)
    r = x - hi
    lo = codecs.e4m3_round(r)
    return hi, r, lo


def test_pair_error_bound_over_every_f16_value_up_to_256():
    x = _f16_values(0.0, 256.0)
    assert len(x) > 20000
    hi, r, lo = _split(x)
    err = np.abs(x - (hi + lo))
    # hi's error is at most 2^-4 |x|, and the remainder's rounding at most 2^-4 of it, or
    # half of e4m3's subnormal step (2^-10) once the remainder drops below 2^-6: so within
    # 2^-8 |x| from |x| = 1/4 up, and within 2^-10 below
    big = x >= 0.25
    assert (err[big] <= np.ldexp(np.abs(x[big]), -8)).all()
    assert (err[~big] <= 2.0 ** -10).all()
    # no saturation: the parts stay below e4m3's largest finite value
    assert np.abs(hi).max() <= 256.0 and np.abs(lo).max() <= 16.0


def test_pair_steps_are_exact_in_f16():
    # the kernel takes x - hi and hi + lo in f16 arithmetic: both must be exact
    x = _f16_values(2.0 ** -14, 256.0)
    hi, r, lo = _split(x)
    assert np.array_equal(r.astype(np.float16).astype(np.float64), r)
    s = hi + lo
    assert np.array_equal(s.astype(np.float16).astype(np.float64), s)


def test_pair_is_symmetric_in_sign():
    x = _f16_values(0.0, 256.0)
    hp, _, lp = _split(x)
    hn, _, ln = _split(-x)
    assert np.array_equal(hn, -hp) and np.array_equal(ln, -lp)


def test_q_scale_maps_the_largest_magnitude_into_128_256_and_keeps_bf16_values_exact():
    # every positive finite bf16 value as the largest |q| of an item
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    m = codecs.bf16_decode(bits.astype(np.uint16))
    # the kernel's rule: e = floor(log2 m) - 7, but at least -100, so that 2^-e stays a
    # finite float32 even for bf16 subnormals
    e = np.maximum(np.floor(np.log2(m)).astype(np.int64) - 7, -100)
    assert np.isfinite(np.float32(np.ldexp(1.0, 100)))
    scaled = np.ldexp(m, -e)
    regular = m >= 2.0 ** -93
    assert ((scaled[regular] >= 128.0) & (scaled[regular] < 256.0)).all()
    assert (scaled[~regular] < 128.0).all() and (scaled[~regular] > 0).all()
    m, e = m[regular], e[regular]
    # any bf16 value up to the largest, times the same power of two, is exact in f16 unless it
    # falls below f16's normal range (2^-14 of a maximum in [128, 256): no contribution)
    rng = np.random.default_rng(5)
    for i in rng.choice(len(m), 400, replace=False):
        mi, ei = m[i], e[i]
        q = codecs.bf16_round(rng.uniform(-mi, mi, 64))
        qs = np.ldexp(q, -ei)
        normal = np.abs(qs) >= 2.0 ** -14
        assert np.array_equal(qs[normal].astype(np.float16).astype(np.float64), qs[normal])


def test_p_stays_below_2_pow_8_under_the_rescale_threshold():
    # scores are raised to 2^(s - m + 4) and m is raised once s > m + 4
    s_minus_m = np.linspace(-40.0, 4.0, 4001)
    p = np.exp2(s_minus_m + 4.0)
    assert p.max() <= 256.0 < 448.0
    # weights down to 2^-10 of the largest possible stay out of e4m3's subnormal range once
    # scaled: 2^-10 * 2^4 (the smallest largest weight) = 2^-6, e4m3's smallest normal
    assert np.exp2(-10.0 + 4.0) == 2.0 ** -6


def test_q_pair_is_exact_for_bf16_values():
    # q arrives in bf16 (8 significant bits): hi takes the top 4 (rounded), and the remainder
    # always fits e4m3's 4 significant bits, so hi + lo is q itself as long as the remainder's
    # last bit (2^-7 of |q|) is not below e4m3's subnormal step 2^-9, i.e. |q| >= 2^-2 once
    # scaled (q's largest magnitude sits in [128, 256), so that is every q within 2^-10 of it)
    bits = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)
    x = codecs.bf16_decode(bits)
    x = x[(x >= 0.25) & (x <= 256.0)]
    assert len(x) > 1000
    hi, r, lo = _split(x)
    assert np.array_equal(hi + lo, x)
    assert np.array_equal(lo, r)  # the remainder is itself an e4m3 value
