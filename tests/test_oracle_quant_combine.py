"""Pins for the oracle's quantisation, combine and long-sequence rounds.

Quantisation (use_fp8 / round_scale / use_ue8m0 and use_int8 / quant_size of
the "DeepEP communication library guide v2.1", section 1.3.1 and the
low_latency_dispatch signature; float8_e4m3fn storage in section 7.4 of the
DeepEP V1 vs V2 comparative analysis) is pinned through torch's CPU division
and casts (library routines) and the formats' error bounds.  Combine (the
reverse of dispatch) is pinned by the identity-expert round trip
x * sum(w), exact special cases, and an order-sensitive case worked out by
hand.  Rounds ("ant moving home", DeepEP on Ascend A2) must reproduce the
one-shot result.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, bf16_bits_to_f32, make_workload, make_y


def _rows(n, H, seed, sigma=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n, H)) * sigma).astype(np.float32)
    x[0, :] = 0.0                                  # an all-zero row
    x[1, 5] = 300.0                                # a large outlier
    x[2, :128] = 1e-6                              # a tiny group (subnormal range)
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("round_scale", [False, True])
def test_fp8_group128(round_scale):
    H = 512
    xb = _rows(6, H, 4)
    for r in range(xb.shape[0]):
        q, s = oracle.quantize_row(xb[r], "fp8", 128, round_scale)
        xf = bf16_bits_to_f32(xb[r]).reshape(-1, 128)
        amax = np.maximum(np.abs(xf).max(axis=1), np.float32(1e-4))
        s_plain = amax / np.float32(448.0)
        if round_scale:
            m, _ = np.frexp(s)
            assert np.all(m == 0.5) and np.all(s >= s_plain) and np.all(s < 2 * s_plain)
        else:
            # 448 is the scale's divisor: s * 448 recovers amax to within an ulp
            assert np.allclose(s.astype(np.float64) * 448.0, amax, rtol=2 ** -23, atol=0)
            big = np.abs(xf).argmax(axis=1)
            codes = q.reshape(-1, 128)[np.arange(4), big]
            floored = np.abs(xf).max(axis=1) < np.float32(1e-4)
            assert np.all(((codes & 0x7f) == 0x7e) | floored)
        # each code is torch's RNE cast of the IEEE quotient x / s
        quot = torch.from_numpy(xf) / torch.from_numpy(s)[:, None]
        ref = quot.to(torch.float8_e4m3fn).view(torch.uint8).numpy().ravel()
        assert np.array_equal(q, ref)
        # error bounds of e4m3: 3 mantissa bits -> relative 2^-4, subnormal step 2^-9
        deq = oracle.e4m3_to_f64(q).reshape(-1, 128) * s[:, None]
        err = np.abs(deq - xf)
        sub = np.abs(xf) / s[:, None] < 2.0 ** -6
        assert np.all(err[~sub] <= 2.0 ** -4 * np.abs(xf[~sub]))
        assert np.all(err[sub] <= (s[:, None] * 2.0 ** -10 * np.ones_like(xf))[sub])


def test_zero_group_gets_floor_scale_and_zero_codes():
    q, s = oracle.quantize_row(np.zeros(256, np.uint16), "fp8", 128, False)
    assert np.all(q == 0) and np.all(s == np.float32(1e-4) / np.float32(448.0))
    q, s = oracle.quantize_row(np.zeros(256, np.uint16), "int8", 256, False)
    assert np.all(q == 0) and s[0] == np.float32(1e-4) / np.float32(127.0)


@pytest.mark.parametrize("quant_size", [128, 1024])
def test_int8(quant_size):
    H = 1024
    xb = _rows(5, H, 5, sigma=2.0)
    for r in range(xb.shape[0]):
        q, s = oracle.quantize_row(xb[r], "int8", quant_size, False)
        xf = bf16_bits_to_f32(xb[r]).reshape(-1, quant_size)
        amax = np.maximum(np.abs(xf).max(axis=1), np.float32(1e-4))
        assert np.allclose(s.astype(np.float64) * 127.0, amax, rtol=2 ** -23, atol=0)
        quot = torch.from_numpy(xf) / torch.from_numpy(s)[:, None]
        ref = torch.clamp(torch.round(quot), -127, 127).to(torch.int8).numpy().ravel()
        assert np.array_equal(q.view(np.int8), ref)
        qi = q.view(np.int8).reshape(-1, quant_size).astype(np.float64)
        # half a step, plus the rounding of the fp32 quotient x / s (|x/s| <= 127)
        assert np.all(np.abs(qi * s[:, None] - xf) <= s[:, None] * (0.5 + 127 * 2.0 ** -23))
        floored = np.abs(xf).max(axis=1) < np.float32(1e-4)
        assert np.all((np.abs(qi).max(axis=1) == 127) | floored)


def test_combine_single_expert_weight_one_is_identity():
    y = _rows(4, 256, 6)
    dst = np.array([[2, -1], [0, -1], [-1, 3], [1, -1]], np.int32)
    w = np.array([[1, 0], [1, 0], [0, 1], [1, 0]], np.float32)
    out = oracle.combine_rows(y, dst, w)
    assert np.array_equal(out, y[[2, 0, 3, 1]])


def test_combine_fully_masked_is_positive_zero():
    out = oracle.combine_rows(_rows(3, 128, 7), -np.ones((3, 4), np.int32),
                              np.ones((3, 4), np.float32))
    assert np.all(out == 0)


def test_combine_accumulates_in_k_order():
    # rows hold 1, 2^24, -2^24 (exact in bf16).  In k order fp32 gives
    # (0 + 1 + 2^24) -> 2^24 (the tie rounds to even), then - 2^24 -> 0;
    # summed in the reverse order the result would be 1.
    vals = np.array([1.0, 2.0 ** 24, -(2.0 ** 24)], np.float32)
    y = np.repeat(oracle.f32_to_bf16(vals)[:, None], 8, axis=1)
    w = np.ones((2, 3), np.float32)
    out = oracle.combine_rows(y, np.array([[0, 1, 2], [2, 1, 0]], np.int32), w)
    assert np.all(out[0] == 0x0000)
    assert np.all(out[1] == 0x3f80)                # (-2^24 + 2^24) + 1 = 1.0


@pytest.mark.parametrize("name", ["tiny", "prefill", "qwen3"])
def test_identity_expert_round_trip(name):
    """dispatch -> identity experts -> combine reproduces x * sum_k w (bf16)."""
    cfg = CONFIGS[name]
    cfg = cfg.scaled(num_tokens=256 if cfg.num_tokens > 256 else None,
                     hidden=512 if cfg.hidden > 512 else None, quant="none")
    wl = make_workload(cfg, seed=1)
    d = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    out = oracle.combine_rows(d["recv_x"], d["dst_buffer_slot_idx"], wl.topk_weights)
    wsum = np.where(wl.topk_idx >= 0, wl.topk_weights, 0).astype(np.float64).sum(1)
    ref = bf16_bits_to_f32(wl.x).astype(np.float64) * wsum[:, None]
    got = bf16_bits_to_f32(out).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)


def test_identity_expert_round_trip_quantised():
    cfg = CONFIGS["decode"].scaled(num_tokens=64, hidden=512)
    wl = make_workload(cfg, seed=2)
    d = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks,
                        1, "fp8", 128, False)
    deq = oracle.e4m3_to_f64(d["recv_x"]).reshape(d["recv_x"].shape[0], -1, 128)
    deq = (deq * d["recv_scales"][:, :, None]).reshape(d["recv_x"].shape).astype(np.float32)
    y = oracle.f32_to_bf16(deq)
    out = oracle.combine_rows(y, d["dst_buffer_slot_idx"], wl.topk_weights)
    wsum = np.where(wl.topk_idx >= 0, wl.topk_weights, 0).astype(np.float64).sum(1)
    xf = bf16_bits_to_f32(wl.x).astype(np.float64)
    ref = xf * wsum[:, None]
    got = bf16_bits_to_f32(out).astype(np.float64)
    s_max = d["recv_scales"].max()
    assert np.all(np.abs(got - ref) <= (2.0 ** -4 + 2.0 ** -7) * np.abs(ref) + s_max * 2.0 ** -9)


def test_combine_matches_fp64_within_fp32_error():
    rng = np.random.default_rng(8)
    y = _rows(40, 64, 9)
    dst = rng.integers(-1, 40, (30, 8)).astype(np.int32)
    w = rng.random((30, 8)).astype(np.float32)
    out = bf16_bits_to_f32(oracle.combine_rows(y, dst, w)).astype(np.float64)
    yf = bf16_bits_to_f32(y).astype(np.float64)
    terms = np.where(dst[:, :, None] >= 0, w[:, :, None] * yf[np.maximum(dst, 0)], 0)
    ref = terms.sum(1)
    bound = 8 * 2.0 ** -24 * np.abs(terms).sum(1) + 2.0 ** -9 * np.abs(ref) + 1e-38
    assert np.all(np.abs(out - ref) <= bound * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(ref))


def test_round_tokens_partition():
    T, R, rounds = 8 * 96, 8, 8
    seen = []
    for j in range(rounds):
        tok = oracle.round_tokens(T, R, rounds, j)
        assert tok.size == T // rounds
        # each rank sends its j-th contiguous block of (T/R)/rounds tokens
        blocks = tok.reshape(R, -1)
        assert np.all(np.diff(blocks, axis=1) == 1)
        assert np.array_equal(blocks[:, 0], np.arange(R) * (T // R) + j * (T // R // rounds))
        seen.append(tok)
    assert np.array_equal(np.sort(np.concatenate(seen)), np.arange(T))
    with pytest.raises(oracle.OracleError):
        oracle.round_tokens(100, 8, 8, 0)


@pytest.mark.parametrize("quant,qs", [("int8", None), ("fp8", 128), ("none", 128)])
def test_rounds_equal_one_shot(quant, qs):
    cfg = CONFIGS["longseq"].scaled(num_tokens=8 * 64, hidden=256)
    wl = make_workload(cfg, seed=4)
    qs = qs or cfg.hidden
    a = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1,
                        quant, qs, False, num_rounds=1)
    b = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1,
                        quant, qs, False, num_rounds=8)
    assert np.array_equal(a["recv_x"], b["recv_x"])
    if quant != "none":
        assert np.array_equal(a["recv_scales"], b["recv_scales"])
    y = make_y(a["num_recv_rows"], cfg.hidden, seed=4)
    o1 = oracle.combine(y, a["dst_buffer_slot_idx"], wl.topk_weights)
    o8 = oracle.combine(y, a["dst_buffer_slot_idx"], wl.topk_weights, cfg.num_ranks, 8)
    assert np.array_equal(o1, o8)


def test_infinite_group_maximum():
    """A group holding +-inf has an infinite scale: finite values quantise to
    zero codes, and an infinite value gives inf / inf = NaN, whose sign IEEE
    754 leaves open; the reading taken is the positive FP8 NaN code 0x7f, and
    int8 0."""
    row = np.zeros(128, np.uint16)
    row[0] = 0x7F80           # +inf
    row[1] = 0xFF80           # -inf
    row[2] = 0x3F80           # 1.0
    row[3] = 0xBF80           # -1.0
    q, sc = oracle.quantize_row(row, "fp8", 128, False)
    assert np.isinf(sc[0])
    assert q[0] == 0x7F and q[1] == 0x7F
    assert q[2] == 0x00 and q[3] == 0x80        # +0 and -0
    q, _ = oracle.quantize_row(row, "int8", 128, False)
    assert q[0] == 0 and q[1] == 0 and q[2] == 0 and q[3] == 0
