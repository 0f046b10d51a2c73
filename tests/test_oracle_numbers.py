"""Pins for the oracle's number formats: bf16, OCP E4M3 (fn) and the
power-of-two scale, checked against torch's CPU casts (a library routine),
exhaustive enumeration and the formats' definitions."""
import numpy as np
import pytest
import torch

import oracle


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2                                  # 0x7f and 0xff
    assert np.array_equal(mine[~nan], ref[~nan])
    # signed zeros keep their sign
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])
    assert mine[0x7e] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def _e4m3_values():
    v = oracle.e4m3_to_f64(np.arange(0, 0x7f, dtype=np.uint8))   # +0 .. 448
    return np.unique(v)


def _encode_samples():
    rng = np.random.default_rng(1)
    vals = _e4m3_values()
    mids = (vals[:-1] + vals[1:]) / 2                      # exact ties
    mids32 = mids.astype(np.float32)
    around = np.concatenate([np.nextafter(mids32, np.float32(-1)), mids32,
                             np.nextafter(mids32, np.float32(1000))])
    bf16_all = (np.arange(0, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
    bf16_in = bf16_all[bf16_all <= 448]
    rand = rng.uniform(-448, 448, 400_000).astype(np.float32)
    tiny = (rng.uniform(-2 ** -5, 2 ** -5, 200_000)).astype(np.float32)
    logu = (np.sign(rng.standard_normal(200_000)) *
            np.exp2(rng.uniform(-20, 8.8, 200_000))).astype(np.float32)
    x = np.concatenate([around, -around, bf16_in, -bf16_in, rand, tiny, logu,
                        vals.astype(np.float32)])
    return x[np.abs(x) <= 448]


def test_e4m3_encode_matches_torch_in_range():
    x = _encode_samples()
    mine = oracle.f32_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(mine != ref)[0]
    assert bad.size == 0, (x[bad[:5]], mine[bad[:5]], ref[bad[:5]])


def test_e4m3_encode_is_nearest_ties_even_bruteforce():
    # brute force over the 127 non-negative finite values: the chosen code is a
    # nearest one, and on a tie its mantissa is even
    vals = oracle.e4m3_to_f64(np.arange(0, 0x7f, dtype=np.uint8))
    x = np.abs(_encode_samples()[::7]).astype(np.float64)
    codes = oracle.f32_to_e4m3(x.astype(np.float32))
    got = oracle.e4m3_to_f64(codes)
    dist = np.abs(x[:, None] - vals[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - x) == best)
    tie = (np.sort(dist, axis=1)[:, 1] == best)
    assert np.all((codes[tie] & 1) == 0)


def test_e4m3_saturates_and_nan():
    x = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e30, np.inf, -500.0, -np.inf],
                 dtype=np.float32)
    assert list(oracle.f32_to_e4m3(x)) == [0x7e] * 7 + [0xfe, 0xfe]
    assert oracle.f32_to_e4m3(np.array([np.nan], np.float32))[0] & 0x7f == 0x7f
    z = oracle.f32_to_e4m3(np.array([0.0, -0.0, -1e-30, 1e-30], np.float32))
    assert list(z) == [0x00, 0x80, 0x80, 0x00]


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(2)
    a = rng.standard_normal(300_000).astype(np.float32) * np.float32(100)
    bits = rng.integers(0, 2 ** 32, 300_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    ties = ((np.arange(1, 20000, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([a, bits, ties, -ties])
    x = x[np.isfinite(x)]
    mine = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_bf16_decode_is_upper_half():
    b = np.array([0x3f80, 0xbf80, 0x4000, 0x0001, 0x7f7f], np.uint16)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(oracle.bf16_to_f32(b), ref)


@pytest.mark.parametrize("s", [1e-4 / 448, 0.1, 0.25, 1.0, 3.0, 448.0 / 448, 7.1e-3, 2.0 ** -20])
def test_pow2_ceil_definition(s):
    s32 = float(np.float32(s))
    p = oracle.pow2_ceil(s32)
    m, e = np.frexp(p)
    assert m == 0.5                                        # a power of two
    assert s32 <= p < 2 * s32                              # the smallest one >= s
