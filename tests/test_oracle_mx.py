"""Pins for the oracle's MXFP4 dispatch quantisation and UE8M0 scale bytes
(use_mxfp4 with quant_size 32 and use_ue8m0 of "DeepEP communication library
guide v2.1", sections 1.3.3 and the low_latency_dispatch listing).

E2M1 and E8M0 are the OCP Microscaling formats: E2M1 holds +-{0, 0.5, 1, 1.5,
2, 3, 4, 6}; an E8M0 byte b is the power of two 2^(b - 127).  The pins: the
E2M1 value set, brute-force nearest / ties-to-even encoding, torch's E8M0 cast
(a library routine) for every scale byte, the MX scale rule's range property,
element error bounds, and agreement with the already pinned fp32-scale path.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, bf16_bits_to_f32, make_workload

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def test_e2m1_value_set_and_sign():
    v = oracle.e2m1_to_f64(np.arange(16))
    assert np.array_equal(v[:8], E2M1)
    assert np.array_equal(v[8:], -E2M1)
    assert np.signbit(v[8]) and not np.signbit(v[0])


def test_e2m1_encode_is_nearest_ties_even():
    rng = np.random.default_rng(0)
    mids = (E2M1[:-1] + E2M1[1:]) / 2
    m32 = mids.astype(np.float32)
    x = np.concatenate([m32, np.nextafter(m32, np.float32(0)), np.nextafter(m32, np.float32(9)), E2M1,
                        rng.uniform(0, 6, 20000), rng.uniform(0, 0.3, 2000)]).astype(np.float32)
    x = np.concatenate([x, -x])
    codes = oracle.f32_to_e2m1(x)
    got = oracle.e2m1_to_f64(codes)
    a = np.abs(x.astype(np.float64))
    dist = np.abs(a[:, None] - E2M1[None, :])
    best = dist.min(1)
    assert np.all(np.abs(np.abs(got) - a) == best)
    tie = np.sort(dist, 1)[:, 1] == best
    assert np.all((codes[tie] & 1) == 0)
    assert np.array_equal(np.signbit(got), np.signbit(x))


def test_e2m1_saturates():
    assert list(oracle.f32_to_e2m1(np.array([6.0, 6.5, 100.0, -7.0], np.float32))) == [7, 7, 7, 15]


def _rows(seed, H=256):
    rng = np.random.default_rng(seed)
    xf = (rng.standard_normal((4, H)) * rng.uniform(0.01, 50, (4, 1))).astype(np.float32)
    xf[1, :32] = 0.0                      # an all-zero group: amax floored at 1e-4
    xf[2, 40] = 1000.0                    # an outlier
    return torch.from_numpy(xf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("seed", [1, 2])
def test_mxfp4_row(seed):
    xb = _rows(seed)
    for row in xb:
        q, sc = oracle.quantize_row_mx(row, "mxfp4", 32)
        assert q.shape == (128,) and sc.dtype == np.uint8
        xf = bf16_bits_to_f32(row).astype(np.float64).reshape(-1, 32)
        amax = np.maximum(np.abs(xf).max(1), 1e-4)
        X = np.exp2(sc.astype(np.float64) - 127)
        # the MX rule: amax / X lies in [4, 8) (X = 2^(floor(log2 amax) - 2))
        assert np.all((amax / X >= 4) & (amax / X < 8))
        # each scale byte is torch's E8M0 encoding of the power of two X
        ref = torch.from_numpy(X.astype(np.float32)).to(torch.float8_e8m0fnu).view(torch.uint8).numpy()
        assert np.array_equal(sc, ref)
        # unpack: even element in the low nibble
        codes = np.stack([q & 15, q >> 4], 1).reshape(-1, 32)
        deq = oracle.e2m1_to_f64(codes) * X[:, None]
        r = np.abs(xf) / X[:, None]
        # in range: at most half the E2M1 spacing; saturated: below 2 X
        half = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0)) * X[:, None]
        inr = r <= 6
        assert np.all(np.abs(deq - xf)[inr] <= half[inr])
        assert np.all((np.abs(deq) == 6 * X[:, None])[~inr]) and np.all((np.abs(xf - deq) < 2 * X[:, None])[~inr])


def test_ue8m0_scale_bytes_for_fp8_and_int8():
    xb = _rows(3, 512)
    for quant, qs in (("fp8", 128), ("int8", 512)):
        for row in xb:
            q_ref, s_ref = oracle.quantize_row(row, quant, qs, True)
            q, sb = oracle.quantize_row_mx(row, quant, qs, True, True)
            assert np.array_equal(q, q_ref)
            ref = torch.from_numpy(s_ref).to(torch.float8_e8m0fnu).view(torch.uint8).numpy()
            assert np.array_equal(sb, ref)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_row_mx(xb[0], "fp8", 128, False, True)     # bytes need power-of-two scales


def test_dispatch_rows_mx_agrees_with_fp32_scale_path():
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 6, hidden=512)
    wl = make_workload(cfg, 5)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks)
    dst = s["dst_buffer_slot_idx"]
    n = s["num_recv_rows"]
    for quant, qs in (("none", 128), ("fp8", 128), ("int8", 512)):
        a, sa = oracle.dispatch_rows(wl.x, dst, quant, qs, False, num_rows=n)
        b, sb = oracle.dispatch_rows_mx(wl.x, dst, quant, qs, False, False, num_rows=n)
        assert np.array_equal(a.view(np.uint8).reshape(n, -1), b)
        if sa is not None:
            assert np.array_equal(sa, sb)
    m, ms = oracle.dispatch_rows_mx(wl.x, dst, "mxfp4", 32, num_rows=n)
    assert m.shape == (n, 256) and ms.shape == (n, 16) and ms.dtype == np.uint8
    t, k = np.nonzero(dst >= 0)
    for i in range(0, t.size, 97):
        q, sc = oracle.quantize_row_mx(wl.x[t[i]], "mxfp4", 32)
        assert np.array_equal(m[dst[t[i], k[i]]], q) and np.array_equal(ms[dst[t[i], k[i]]], sc)
