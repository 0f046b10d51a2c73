"""GPU parity at the workloads' full sizes for the launch modes the benchmark
times besides the default one: the low-latency layout, cached dispatch, the
combine of quantised expert outputs, MXFP4 dispatch and UE8M0 scale bytes.

As in test_gpu_fullsize, everything is compared in full and bit for bit
against the oracle's OpenMP build on every host core: the routing, and the
rows, scales and combined tokens of every token.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

from gpu_parity import assert_combine_close, to_dev, u8, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def threaded_oracle():
    oracle.use_threads(len(os.sched_getaffinity(0)))
    yield
    oracle.use_threads(1)


def _sample(T):
    """Every token (the rows below are compacted to those the tokens use)."""
    return np.arange(T, dtype=np.int32)


def _compact(dst, tok):
    """Rows of the sampled tokens, renumbered 0..n-1 (the oracle's row table)."""
    sub = dst[tok]
    used = np.unique(sub[sub >= 0])
    remap = -np.ones(int(dst.max(initial=0)) + 2, np.int64)
    remap[used] = np.arange(used.size)
    cdst = np.full_like(dst, -1)
    cdst[tok] = np.where(sub >= 0, remap[np.maximum(sub, 0)], -1)
    return used, cdst


def _rows(t, used, dev):
    return t.index_select(0, torch.from_numpy(used.astype(np.int64)).to(dev))


def test_full_size_low_latency_decode(cuda_device):
    """Low-latency layout [E, R*M, H] with M = T/R, FP8 g128, then the combine
    of the FP8 rows themselves (identity experts) with their scales."""
    dev = cuda_device
    cfg = CONFIGS["decode"]
    T, H, E, R = cfg.num_tokens, cfg.hidden, cfg.num_experts, cfg.num_ranks
    M = T // R
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, dev)
    recv_x, recv_scales, count, layout_range, h = ep.ep_dispatch_low_latency(x, ti, tw, M, E, R, "fp8",
                                                                             quant_size=128)
    torch.cuda.synchronize()
    h.check()
    ref = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    dst = ref["dst_buffer_slot_idx"]
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), dst)
    assert np.array_equal(count.cpu().numpy(), ref["recv_count"])
    assert np.array_equal(layout_range.cpu().numpy(), ref["layout_range"])
    rows = E * R * M
    flat_x, flat_s = recv_x.reshape(rows, -1), recv_scales.reshape(rows, -1)
    tok = _sample(T)
    used, cdst = _compact(dst, tok)
    ref_x, ref_s = oracle.dispatch_rows(wl.x, cdst, "fp8", 128, False, tokens=tok, num_rows=used.size)
    assert np.array_equal(u8(_rows(flat_x, used, dev)), ref_x)
    assert np.array_equal(_rows(flat_s, used, dev).cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    out = ep.ep_combine(recv_x, h, tw, y_scales=flat_s, quant_size=128)
    torch.cuda.synchronize()
    h.check()
    ref_out = oracle.combine_rows_q(ref_x, ref_s, "fp8", 128, cdst, wl.topk_weights, tokens=tok)
    got = u16(_rows(out, tok, dev))
    assert_combine_close(got, ref_out)
    assert np.array_equal(got, ref_out)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_full_size_cached_dispatch(name, cuda_device):
    """A second dispatch with new activations and the first call's handle:
    every token's rows are the oracle's rows of the new x at the first
    routing's slots; every padding row is zero again."""
    dev = cuda_device
    cfg = CONFIGS[name]
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    q = None if cfg.quant == "none" else cfg.quant
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, dev)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, q, cfg.quant_size, cfg.num_rounds, device=dev)
    kw = dict(quant_size=cfg.quant_size, round_scale=cfg.round_scale, num_rounds=cfg.num_rounds, buffers=bufs)
    ep.ep_dispatch(x, ti, tw, A, q, num_experts=E, num_ranks=R, do_cpu_sync=False, **kw)
    x2 = torch.from_numpy(make_workload(cfg, 1).x.view(np.int16)).view(torch.bfloat16).to(dev)
    x2_np = x2.view(torch.int16).cpu().numpy().view(np.uint16)
    bufs.recv_x.view(torch.uint8).fill_(0x5A)
    ep.ep_dispatch(x2, quant=q, handle=bufs.handle, **kw)
    torch.cuda.synchronize()
    bufs.handle.check()
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    tok = _sample(T)
    used, cdst = _compact(s["dst_buffer_slot_idx"], tok)
    ref_x, ref_s = oracle.dispatch_rows(x2_np, cdst, cfg.quant, cfg.quant_size, cfg.round_scale, tokens=tok,
                                        num_rows=used.size)
    got = _rows(bufs.recv_x, used, dev)
    assert np.array_equal(u16(got) if q is None else u8(got), ref_x)
    if q is not None:
        assert np.array_equal(_rows(bufs.recv_scales, used, dev).cpu().numpy().view(np.uint32),
                              ref_s.view(np.uint32))
    pad = np.nonzero(s["recv_src_metadata"][:, 0] < 0)[0]
    if pad.size:
        assert torch.all(_rows(bufs.recv_x, pad, dev).view(torch.uint8) == 0)


@pytest.mark.parametrize("quant,qs,rs,ue8", [("mxfp4", 32, False, False), ("fp8", 128, True, True)])
def test_full_size_decode_mxfp4_and_ue8m0(quant, qs, rs, ue8, cuda_device):
    """Decode with MXFP4 codes and UE8M0 scale bytes, or with FP8 codes and
    power-of-two scales stored as UE8M0 bytes."""
    dev = cuda_device
    cfg = CONFIGS["decode"]
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, dev)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, 1, quant, qs, device=dev, scale_ue8m0=ue8)
    ep.ep_dispatch(x, ti, tw, 1, quant, num_experts=E, num_ranks=R, quant_size=qs, round_scale=rs,
                   do_cpu_sync=False, buffers=bufs, scale_ue8m0=ue8)
    torch.cuda.synchronize()
    bufs.handle.check()
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R)
    assert np.array_equal(bufs.handle.dst_buffer_slot_idx.cpu().numpy(), s["dst_buffer_slot_idx"])
    tok = _sample(T)
    used, cdst = _compact(s["dst_buffer_slot_idx"], tok)
    ref_x, ref_s = oracle.dispatch_rows_mx(wl.x, cdst, quant, qs, rs, ue8, tokens=tok, num_rows=used.size)
    assert np.array_equal(u8(_rows(bufs.recv_x, used, dev)).reshape(used.size, -1), ref_x)
    got_s = _rows(bufs.recv_scales, used, dev).cpu().numpy()
    assert got_s.dtype == ref_s.dtype and np.array_equal(got_s.view(np.uint8), ref_s.view(np.uint8))


def test_full_size_prefill_fp8_quantised_combine(cuda_device):
    """Prefill with FP8 g128 dispatch, then the combine of the FP8 rows with
    their scales (identity experts), padding rows included in the layout."""
    dev = cuda_device
    cfg = CONFIGS["prefill"].scaled(quant="fp8", quant_size=128)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, dev)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, "fp8", 128, device=dev)
    ep.ep_dispatch(x, ti, tw, A, "fp8", num_experts=E, num_ranks=R, quant_size=128, do_cpu_sync=False,
                   buffers=bufs)
    out = ep.ep_combine(bufs.recv_x, bufs.handle, tw, y_scales=bufs.recv_scales, quant_size=128)
    torch.cuda.synchronize()
    bufs.handle.check()
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    tok = _sample(T)
    used, cdst = _compact(s["dst_buffer_slot_idx"], tok)
    ref_x, ref_s = oracle.dispatch_rows(wl.x, cdst, "fp8", 128, False, tokens=tok, num_rows=used.size)
    assert np.array_equal(u8(_rows(bufs.recv_x, used, dev)), ref_x)
    assert np.array_equal(_rows(bufs.recv_scales, used, dev).cpu().numpy().view(np.uint32),
                          ref_s.view(np.uint32))
    ref_out = oracle.combine_rows_q(ref_x, ref_s, "fp8", 128, cdst, wl.topk_weights, tokens=tok)
    got = u16(_rows(out, tok, dev))
    assert_combine_close(got, ref_out)
    assert np.array_equal(got, ref_out)
