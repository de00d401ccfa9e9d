"""Pins of the oracle's E4M3 codec against the format definition, hand-worked
landmarks and torch's own CPU float8_e4m3fn conversion (a library routine)."""

import math

import numpy as np
import pytest
import torch

import oracle


def _val(s):
    return float(s)


def test_decode_landmarks(impl, golden):
    rows = [r for r in golden("e4m3_landmarks.txt") if r[0] == "decode"]
    assert len(rows) >= 10
    for _, code, val in rows:
        got = impl.e4m3_decode(np.array([int(code, 16)], np.uint8))[0]
        want = _val(val)
        if math.isnan(want):
            assert math.isnan(got), code
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), code


def test_encode_landmarks(impl, golden):
    rows = [r for r in golden("e4m3_landmarks.txt") if r[0] == "encode"]
    assert len(rows) >= 10
    for _, val, code in rows:
        v = np.float32(_val(val))
        assert float(v) == _val(val), "landmark must be exact in fp32"
        got = int(impl.e4m3_encode(np.array([v], np.float32))[0])
        assert got == int(code, 16), (val, hex(got), code)


def test_every_finite_code_round_trips(impl):
    codes = np.arange(256, dtype=np.uint8)
    vals = impl.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254  # 0x7F and 0xFF are the only NaNs
    enc = impl.e4m3_encode(vals[finite].astype(np.float32))
    np.testing.assert_array_equal(enc, codes[finite])
    assert np.nanmax(vals) == 448.0 and np.nanmin(vals) == -448.0


def test_midpoints_round_to_even_and_neighbours_round_nearest(impl):
    codes = np.arange(0x00, 0x7E, dtype=np.uint8)   # positive finite, below max
    lo = impl.e4m3_decode(codes)
    hi = impl.e4m3_decode(codes + 1)
    mid = (lo + hi) / 2                               # <= 5 significant bits: exact in fp32
    assert np.all(mid.astype(np.float32).astype(np.float64) == mid)
    got = impl.e4m3_encode(mid.astype(np.float32)).astype(np.int64)
    even = np.where(codes % 2 == 0, codes, codes + 1)
    np.testing.assert_array_equal(got, even)
    # one fp32 ulp either side of the midpoint decides to the nearer neighbour
    below = np.nextafter(mid.astype(np.float32), np.float32(0))
    above = np.nextafter(mid.astype(np.float32), np.float32(np.inf))
    np.testing.assert_array_equal(impl.e4m3_encode(below), codes)
    np.testing.assert_array_equal(impl.e4m3_encode(above), codes + 1)
    # negatives mirror positives with the sign bit
    np.testing.assert_array_equal(impl.e4m3_encode(-mid.astype(np.float32)), even | 0x80)


def test_saturation_and_signed_zero(impl):
    big = np.array([448, 448.5, 463.9, 464, 465, 1e6, 3.4e38, np.inf], np.float32)
    assert np.all(impl.e4m3_encode(big) == 0x7E)
    assert np.all(impl.e4m3_encode(-big) == 0xFE)
    assert impl.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80
    assert impl.e4m3_encode(np.array([0.0], np.float32))[0] == 0x00
    tiny = np.array([1e-30, 2.0 ** -11, 2.0 ** -10], np.float32)
    assert np.all(impl.e4m3_encode(tiny) == 0x00)
    assert np.all(impl.e4m3_encode(-tiny) == 0x80)


def _torch_e4m3(v):
    t = torch.from_numpy(np.asarray(v, np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_matches_torch_cpu_conversion_random_and_boundaries(impl):
    rng = np.random.default_rng(1234)
    # log-uniform magnitudes across the whole E4M3 range and beyond, both signs
    mags = np.exp2(rng.uniform(-14, 11, 400_000)).astype(np.float32)
    signs = np.where(rng.random(mags.size) < 0.5, -1, 1).astype(np.float32)
    v = mags * signs
    # every code's value, its midpoints with the next code, and 1-ulp neighbours
    vals = impl.e4m3_decode(np.arange(256, dtype=np.uint8))
    vals = vals[~np.isnan(vals)]
    srt = np.sort(np.unique(vals))
    mids = ((srt[1:] + srt[:-1]) / 2).astype(np.float32)
    edge = np.concatenate([vals.astype(np.float32), mids,
                           np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(-np.inf))])
    v = np.concatenate([v, edge, rng.standard_normal(100_000).astype(np.float32) * 100])
    np.testing.assert_array_equal(impl.e4m3_encode(v), _torch_e4m3(v))


@pytest.mark.parametrize("seed", [0, 1])
def test_every_fp32_bit_pattern_slice(impl, seed):
    """A strided sweep over fp32 bit patterns (NaN excluded) against torch."""
    rng = np.random.default_rng(seed)
    bits = (np.arange(0, 2 ** 32, 2 ** 12, dtype=np.uint64) +
            rng.integers(0, 2 ** 12, 2 ** 20, dtype=np.uint64)).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[~np.isnan(v)]
    np.testing.assert_array_equal(impl.e4m3_encode(v), _torch_e4m3(v))
