"""Pins for the oracle's low-latency layout and its combine of quantised expert
outputs.

Low-latency layout (DeepEP V1 vs V2 comparative analysis, section 6.3: per-rank
buffers [num_local_experts, num_ranks * num_max_dispatch_tokens_per_rank,
hidden]): the entry (t,k) for expert e from source rank r lands in row
e*R*M + r*M + p, p its position among that rank's entries for e in (t,k) order.
Combine of quantised outputs (combine-side int8 / fp8 of "DeepEP communication
library guide v2.1", section 1.3.1; the shared-expert combine of lmdeploy PR
#4783): value = decode(code) * scale, then the same k-order fma chain.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, bf16_bits_to_f32, make_workload, make_y


def test_ll_hand_worked_example():
    # T=4 (tokens 0,1 on rank 0; 2,3 on rank 1), E=4 (L=2), K=2, M=2
    ti = np.array([[1, 2], [0, 1], [3, -1], [1, 3]], np.int64)
    w = np.array([[.6, .4], [.7, .3], [1., 0.], [.55, .45]], np.float32)
    s = oracle.ll_slots(ti, w, 4, 2, 2)
    # e0: (1,0)->row 0 | e1: (0,0)->4, (1,1)->5, (3,0)->4+2 | e2: (0,1)->8 | e3: (2,0)->12+2, (3,1)->15
    assert s["dst_buffer_slot_idx"].tolist() == [[4, 8], [0, 5], [14, -1], [6, 15]]
    assert s["recv_count"].tolist() == [1, 3, 1, 2]
    rng = s["layout_range"]
    assert [(int(v) >> 32, int(v) & 0xffffffff) for v in rng.ravel()] == [
        (0, 1), (2, 0), (0, 2), (2, 1), (0, 1), (2, 0), (0, 0), (2, 2)]
    assert s["recv_src_metadata"][14].tolist() == [2, 0]
    assert s["recv_topk_idx"][8].tolist() == [-1, 0]        # e2 is rank 1's local expert 0
    assert np.all(s["recv_src_metadata"][[1, 2, 3, 7, 9]] == -7)   # unused rows untouched


def _ll_by_sort(ti, E, R, M):
    """Rows from numpy's stable lexsort of (expert, source rank, token, k)."""
    T, K = ti.shape
    tpr = T // R
    t, k = np.nonzero(ti >= 0)
    e = ti[t, k]
    r = t // tpr
    order = np.lexsort((k, t, r, e))
    grp = e[order] * R + r[order]
    first = np.concatenate([[0], np.nonzero(np.diff(grp))[0] + 1])
    start = np.zeros(order.size, np.int64)
    start[first] = first
    start = np.maximum.accumulate(start)
    p = np.arange(order.size) - start
    dst = -np.ones((T, K), np.int64)
    dst[t[order], k[order]] = (e[order] * R + r[order]) * M + p
    return dst, p.max(initial=-1)


@pytest.mark.parametrize("name", ["decode", "qwen3", "tiny"])
def test_ll_matches_sort_and_invariants(name):
    cfg = CONFIGS[name]
    T = min(cfg.num_tokens, 16 * 40)
    T -= T % cfg.num_ranks
    wl = make_workload(cfg.scaled(num_tokens=T), seed=2, with_x=False)
    E, R = cfg.num_experts, cfg.num_ranks
    M = T // R
    s = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    dst, pmax = _ll_by_sort(wl.topk_idx, E, R, M)
    assert np.array_equal(s["dst_buffer_slot_idx"], dst) and pmax < M
    assert np.array_equal(s["recv_count"], np.bincount(wl.topk_idx[wl.topk_idx >= 0], minlength=E))
    rng = s["layout_range"]
    assert np.array_equal(rng >> 32, np.tile(np.arange(R) * M, (E, 1)))
    assert np.array_equal((rng & 0xffffffff).sum(1), s["recv_count"])
    t, k = np.nonzero(wl.topk_idx >= 0)
    rows = s["dst_buffer_slot_idx"][t, k]
    assert np.array_equal(s["recv_src_metadata"][rows], np.stack([t, k], 1))


def test_ll_capacity():
    ti = np.array([[0], [0], [0], [1]], np.int64)     # rank 0 sends three entries to expert 0
    s = oracle.ll_slots(ti, np.ones((4, 1), np.float32), 2, 1, 3)  # M = 3 fits
    assert s["recv_count"].tolist() == [3, 1]
    with pytest.raises(oracle.OracleError) as e:
        oracle.ll_slots(ti, np.ones((4, 1), np.float32), 2, 1, 2)  # M = 2 does not
    assert e.value.status == oracle.CAPACITY


def test_combine_q_shared_only_and_plain_equivalence():
    rng = np.random.default_rng(3)
    y = make_y(24, 64, 5)
    shared = make_y(6, 64, 6)
    dst = rng.integers(-1, 24, (6, 4)).astype(np.int32)
    w = rng.random((6, 4)).astype(np.float32)
    # with all weights zero the result is the shared row itself
    assert np.array_equal(oracle.combine_rows_q(y, None, "none", 64, dst, np.zeros_like(w), shared), shared)
    # without a shared row, bf16 input is the plain combine
    assert np.array_equal(oracle.combine_rows_q(y, None, "none", 64, dst, w), oracle.combine_rows(y, dst, w))


@pytest.mark.parametrize("quant,qs", [("fp8", 128), ("int8", 512)])
def test_combine_q_identity_round_trip(quant, qs):
    """dispatch (quantised) -> identity experts -> quantised combine ~= x * sum(w)."""
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 8, hidden=512)
    wl = make_workload(cfg, seed=4)
    d = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1, quant, qs, False)
    out = oracle.combine_rows_q(d["recv_x"], d["recv_scales"], quant, qs, d["dst_buffer_slot_idx"], wl.topk_weights)
    xf = bf16_bits_to_f32(wl.x).astype(np.float64)
    wsum = np.where(wl.topk_idx >= 0, wl.topk_weights, 0).astype(np.float64).sum(1, keepdims=True)
    ref = xf * wsum
    got = bf16_bits_to_f32(out).astype(np.float64)
    smax = d["recv_scales"].max()
    rel = 2.0 ** -4 if quant == "fp8" else 0.0
    assert np.all(np.abs(got - ref) <= (rel + 2.0 ** -7) * np.abs(ref) + smax * (2.0 ** -9 if quant == "fp8" else 0.5) * wsum)


def test_combine_q_single_value_is_scaled_code():
    # one entry of weight 1: out = bf16(+0 + decode(code) * scale), computed by torch
    # (the accumulator starts at +0, so the -0 code gives +0)
    codes = np.arange(0, 256, dtype=np.uint8).reshape(2, 128)
    codes[codes == 0x7f] = 0x7e
    codes[codes == 0xff] = 0xfe
    scales = np.array([[0.75], [3.0]], np.float32)
    dst = np.array([[0], [1]], np.int32)
    out = oracle.combine_rows_q(codes, scales, "fp8", 128, dst, np.ones((2, 1), np.float32))
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).float() * torch.from_numpy(scales) + 0.0
    ref = dec.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, ref)
