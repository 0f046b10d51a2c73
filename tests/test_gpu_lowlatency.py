"""GPU parity of the low-latency (fixed-capacity) dispatch and of the combine of
quantised expert outputs / with a shared expert, against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y

from gpu_parity import to_dev, u16, u8

pytestmark = pytest.mark.gpu


def _ll(cfg, wl, M, dev):
    x, ti, tw = to_dev(wl, dev)
    q = None if cfg.quant == "none" else cfg.quant
    res = ep.ep_dispatch_low_latency(x, ti, tw, M, cfg.num_experts, cfg.num_ranks, q, quant_size=cfg.quant_size,
                                     round_scale=cfg.round_scale)
    torch.cuda.synchronize()
    return res, (x, ti, tw)


def _check_ll(cfg, wl, M, res):
    (recv_x, recv_scales, count, layout_range, h) = res
    E, R = cfg.num_experts, cfg.num_ranks
    ref = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    dst = ref["dst_buffer_slot_idx"]
    assert h.read_error() == ep.EP_OK
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), dst)
    assert np.array_equal(count.cpu().numpy(), ref["recv_count"])
    assert np.array_equal(h.num_recv_tokens_per_expert.cpu().numpy(), ref["recv_count"])
    assert np.array_equal(layout_range.cpu().numpy(), ref["layout_range"])
    used = np.unique(dst[dst >= 0])
    meta = h.recv_src_metadata.cpu().numpy()
    assert np.array_equal(meta[used], ref["recv_src_metadata"][used])
    rows = E * R * M
    got_x = (u16(recv_x) if cfg.quant == "none" else u8(recv_x)).reshape(rows, -1)
    ref_x, ref_s = oracle.dispatch_rows(wl.x, dst, cfg.quant, cfg.quant_size, cfg.round_scale, num_rows=rows)
    assert np.array_equal(got_x[used], ref_x[used])
    if cfg.quant != "none":
        gs = recv_scales.reshape(rows, -1).cpu().numpy()
        assert np.array_equal(gs[used].view(np.uint32), ref_s[used].view(np.uint32))
    return ref, ref_x, ref_s


def test_low_latency_decode_fp8_and_quantised_combine(cuda_device):
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 40, hidden=1024)
    wl = make_workload(cfg, 0)
    M = 48
    res, (x, ti, tw) = _ll(cfg, wl, M, cuda_device)
    ref, ref_x, ref_s = _check_ll(cfg, wl, M, res)
    recv_x, recv_scales, _, _, h = res
    # identity experts: combine the FP8 rows themselves
    out = ep.ep_combine(recv_x, h, tw, y_scales=recv_scales.reshape(-1, recv_scales.shape[-1]), quant_size=128)
    torch.cuda.synchronize()
    ref_out = oracle.combine_rows_q(ref_x, ref_s, "fp8", 128, ref["dst_buffer_slot_idx"], wl.topk_weights)
    assert np.array_equal(u16(out), ref_out)


def test_low_latency_bf16_combine_and_cached(cuda_device):
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg, 1)
    M = cfg.num_tokens // cfg.num_ranks + 3
    res, (x, ti, tw) = _ll(cfg, wl, M, cuda_device)
    ref, _, _ = _check_ll(cfg, wl, M, res)
    _, _, _, _, h = res
    rows = cfg.num_experts * cfg.num_ranks * M
    y_np = make_y(rows, cfg.hidden, 1)
    y = torch.from_numpy(y_np.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    out = ep.ep_combine(y, h, tw)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), oracle.combine_rows(y_np, ref["dst_buffer_slot_idx"], wl.topk_weights))
    # cached dispatch on a low-latency handle: no padding rows, same rows as the oracle
    wl2 = make_workload(cfg, 2)
    x2 = torch.from_numpy(wl2.x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    bufs = ep.alloc_dispatch_buffers(cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                                     1, None, recv_capacity=rows, device=cuda_device)
    bufs.recv_x.view(torch.uint8).fill_(0x33)
    rx, _, _, _, _ = ep.ep_dispatch(x2, buffers=bufs, handle=h)
    torch.cuda.synchronize()
    dst = ref["dst_buffer_slot_idx"]
    used = np.unique(dst[dst >= 0])
    ref_x2, _ = oracle.dispatch_rows(wl2.x, dst, num_rows=rows)
    got = u16(rx)
    assert np.array_equal(got[used], ref_x2[used])
    unused = np.setdiff1d(np.arange(rows), used)
    assert np.all(got[unused].view(np.uint8) == 0x33)       # the fixed-capacity layout has no padding


def test_int8_per_token_combine_with_shared_expert(cuda_device):
    cfg = CONFIGS["longseq"].scaled(num_tokens=8 * 8 * 5, hidden=1024)
    wl = make_workload(cfg, 3)
    x, ti, tw = to_dev(wl, cuda_device)
    recv_x, recv_scales, _, _, h = ep.ep_dispatch(x, ti, tw, 1, "int8", num_experts=cfg.num_experts,
                                                  num_ranks=cfg.num_ranks, quant_size=cfg.hidden,
                                                  num_rounds=cfg.num_rounds)
    shared_np = make_y(cfg.num_tokens, cfg.hidden, 9)
    shared = torch.from_numpy(shared_np.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    out = ep.ep_combine(recv_x.contiguous(), h, tw, y_scales=recv_scales.contiguous(), quant_size=cfg.hidden,
                        shared=shared)
    torch.cuda.synchronize()
    d = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1, "int8", cfg.hidden)
    ref = oracle.combine_rows_q(d["recv_x"], d["recv_scales"], "int8", cfg.hidden, d["dst_buffer_slot_idx"],
                                wl.topk_weights, shared_np)
    assert np.array_equal(u16(out), ref)


def test_low_latency_overflow_sets_capacity(cuda_device):
    cfg = CONFIGS["tiny"].scaled(num_tokens=8 * 4)
    wl = make_workload(cfg, 0)
    wl.topk_idx[:4] = [[3, 3]] * 4                  # rank 0: 8 entries for expert 3
    M = 4
    x, ti, tw = to_dev(wl, cuda_device)
    _, _, count, _, h = ep.ep_dispatch_low_latency(x, ti, tw, M, cfg.num_experts, cfg.num_ranks)
    torch.cuda.synchronize()
    assert h.read_error() == ep.EP_ERR_CAPACITY
    with pytest.raises(oracle.OracleError):
        oracle.ll_slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, M)


def test_low_latency_no_tokens(cuda_device):
    cfg = CONFIGS["decode"].scaled(num_tokens=0, hidden=256)
    wl = make_workload(cfg, 0)
    res, _ = _ll(cfg, wl, 8, cuda_device)
    _, _, count, layout_range, h = res
    assert h.read_error() == ep.EP_OK
    assert torch.all(count == 0) and torch.all((layout_range & 0xffffffff) == 0)
