"""Pins of the oracle's BF16 / E4M3 codecs against the format definitions and
against PyTorch's own conversions (an independent library routine)."""
import numpy as np
import pytest
import torch

import oracle


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    got = oracle.bf16_decode(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_bf16_round_matches_torch_on_random_float32():
    rng = np.random.default_rng(0)
    raw = rng.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32)
    v = raw.view(np.float32)
    v = v[np.isfinite(v)]
    got = oracle.bf16_round(v.astype(np.float64))
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is halfway between 1 (even) and 1 + 2^-7 (odd mantissa)
    assert oracle.bf16_round(np.array([1 + 2**-8]))[0] == 0x3F80
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert oracle.bf16_round(np.array([1 + 3 * 2**-8]))[0] == 0x3F82
    # a double just above the tie rounds up (single rounding from FP64)
    assert oracle.bf16_round(np.array([1 + 2**-8 + 2**-40]))[0] == 0x3F81


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    # format facts: largest finite 448, smallest subnormal 2^-9, NaN only at S.1111.111
    assert got[0x7E] == 448.0 and got[0x01] == 2.0**-9 and np.isnan(got[0x7F])
    assert np.sum(np.isnan(got)) == 2


def test_e4m3_round_matches_torch_in_range():
    rng = np.random.default_rng(1)
    mag = np.exp2(rng.uniform(-12, np.log2(464.0), size=60_000))
    v = (mag * rng.choice([-1.0, 1.0], size=mag.size)).astype(np.float32)
    got = oracle.e4m3_round(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_round_closed_forms():
    r = lambda x: int(oracle.e4m3_round(np.array([x]))[0])
    assert r(2.0**-10) == 0x00           # half the smallest subnormal: tie to even (0)
    assert r(3 * 2.0**-10) == 0x02       # 1.5 quanta: tie to even (2 quanta)
    assert r(2.0**-6 - 2.0**-10) == 0x08  # 7.5 quanta rounds up into the first normal
    assert r(1000.0) == 0x7E and r(-1e6) == 0xFE  # saturate, never NaN
    assert r(float("inf")) == 0x7E
    assert r(-0.0) == 0x80 and r(0.0) == 0x00
    assert r(1.0) == 0x38 and r(1.0625) == 0x38 and r(1.1875) == 0x3A  # ties at 1.0625, 1.1875
