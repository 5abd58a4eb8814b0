"""Pins of the oracle's bf16 / FP8 E4M3 codecs against routes that share nothing with them:
binary32 reinterpretation, torch's dtype conversions, and brute-force nearest-value search
over the full code tables."""

import numpy as np
import pytest
import torch

from oracle import codecs


def _f32_from_bf16_bits(bits):
    # (NaN patterns widen to NaN; numpy warns about the cast of signalling ones)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_bf16_decode_all_patterns_match_binary32_upper_half():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = codecs.bf16_decode(bits)
    ref = _f32_from_bf16_bits(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(ours[0x8000]) and not np.signbit(ours[0])


def test_bf16_encode_roundtrips_every_non_nan_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = codecs.bf16_decode(bits)
    ok = ~np.isnan(vals)
    assert np.array_equal(codecs.bf16_encode(vals[ok]), bits[ok])


def _bf16_finite_table():
    bits = np.arange(0, 0x7F80, dtype=np.int64)  # non-negative finite patterns, ascending
    return bits, _f32_from_bf16_bits(bits.astype(np.uint16))


def _nearest_even(table_bits, table_vals, a):
    """Brute force: nearest table value to magnitude ``a``; ties go to the even code."""
    d = np.abs(table_vals - a)
    best = np.min(d)
    cand = np.nonzero(d == best)[0]
    if len(cand) == 1:
        return int(table_bits[cand[0]])
    even = [i for i in cand if table_bits[i] % 2 == 0]
    assert len(even) == 1
    return int(table_bits[even[0]])


def test_bf16_encode_matches_brute_force_nearest_even():
    tb, tv = _bf16_finite_table()
    rng = np.random.default_rng(7)
    xs = list(rng.standard_normal(300) * 10.0 ** rng.integers(-40, 38, 300))
    # exact ties between neighbours (odd and even lower neighbour), and ties nudged by less
    # than a binary32 ulp (double-rounding traps)
    for i in rng.integers(1, 0x7F00, 200):
        lo, hi = tv[i], tv[i + 1]
        mid = (lo + hi) / 2
        xs += [mid, mid * (1 + 2.0 ** -40), mid * (1 - 2.0 ** -40)]
    # subnormal range
    xs += list(rng.uniform(0, 2.0 ** -126, 100))
    for x in xs:
        a = abs(float(x))
        want = _nearest_even(tb, tv, a)
        got = int(codecs.bf16_encode(np.array([a]))[0])
        assert got == want, (a, hex(got), hex(want))
        neg = int(codecs.bf16_encode(np.array([-a]))[0])
        assert neg == want | 0x8000


def test_bf16_encode_agrees_with_torch_on_float32_inputs():
    rng = np.random.default_rng(11)
    x32 = (rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000)).astype(
        np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codecs.bf16_encode(x32.astype(np.float64)), ref)


def test_bf16_encode_overflow_inf_nan():
    big = codecs.BF16_MAX
    assert codecs.bf16_encode(np.array([big]))[0] == 0x7F7F
    # half an ulp above the largest finite value rounds (to even) up to infinity
    assert codecs.bf16_encode(np.array([big + 2.0 ** 119]))[0] == 0x7F80
    assert codecs.bf16_encode(np.array([big + 2.0 ** 118]))[0] == 0x7F7F
    assert codecs.bf16_encode(np.array([-np.inf]))[0] == 0xFF80
    nan = codecs.bf16_encode(np.array([np.nan]))[0]
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F) != 0


def test_e4m3_decode_all_codes_match_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # closed-form landmarks of the format
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_roundtrip_and_brute_force():
    codes = np.arange(256, dtype=np.uint8)
    vals = codecs.e4m3_decode(codes)
    ok = ~np.isnan(vals)
    assert np.array_equal(codecs.e4m3_encode(vals[ok]), codes[ok])
    tb = np.arange(0, 0x7F, dtype=np.int64)
    tv = codecs.e4m3_decode(tb)
    rng = np.random.default_rng(3)
    xs = list(rng.uniform(0, 448, 2000)) + list(rng.uniform(0, 2.0 ** -5, 500))
    xs += [(tv[i] + tv[i + 1]) / 2 for i in range(len(tv) - 1)]  # every exact tie
    for a in xs:
        want = _nearest_even(tb, tv, a)
        assert int(codecs.e4m3_encode(np.array([a]))[0]) == want, a
        assert int(codecs.e4m3_encode(np.array([-a]))[0]) == want | 0x80, a


def test_e4m3_encode_agrees_with_torch_in_range():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(100000) * 60.0
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codecs.e4m3_encode(x.astype(np.float64)), ref)


@pytest.mark.parametrize("x,code", [(448.0, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (1e9, 0x7E),
                                    (np.inf, 0x7E), (-np.inf, 0xFE), (-500.0, 0xFE)])
def test_e4m3_encode_saturates(x, code):
    assert int(codecs.e4m3_encode(np.array([x]))[0]) == code


def test_e4m3_nan_stays_nan():
    c = int(codecs.e4m3_encode(np.array([np.nan]))[0])
    assert c & 0x7F == 0x7F
