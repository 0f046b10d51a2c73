"""Seeded random configurations: the CUDA path against the oracle, bit for bit.

Each case draws ranks, experts per rank, top-k, tokens per rank (0 included),
hidden size, expert alignment, masking, x's magnitude, the number of rounds
and the dispatch quantisation (none, FP8 / int8 with groups of 16-512 or per
token, with or without power-of-two scales and UE8M0 bytes, MXFP4), then
compares layout, slots, metadata, rows, codes, scales and the combine of
seeded expert outputs (with and without a shared expert's row).  Some cases
also run the low-latency layout.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y

from gpu_parity import assert_layout_equal, assert_slots_equal, to_dev, u8, u16

pytestmark = pytest.mark.gpu

N_CASES = 96


def _draw(i):
    rng = np.random.default_rng(1000 + i)
    R = int(rng.choice([1, 2, 3, 4, 6, 8, 16]))
    L = int(rng.choice([1, 2, 3, 4, 8]))
    E = R * L
    K = int(rng.integers(1, min(16, E) + 1))
    tpr = int(rng.choice([0, 1, 5, 16, 17, 40]))
    H = int(rng.choice([64, 128, 384, 1024, 1536, 2048]))
    A = int(rng.choice([1, 1, 2, 3, 8, 64]))
    quant = str(rng.choice(["none", "fp8", "int8", "mxfp4"]))
    if quant == "mxfp4":
        qs, rs, ue8 = 32, False, False
    elif quant == "none":
        qs, rs, ue8 = 128, False, False
    else:
        qs = int(rng.choice([g for g in (16, 32, 64, 128, 256, 512) if H % g == 0] + [H]))
        rs = bool(rng.integers(2))
        ue8 = rs and bool(rng.integers(2))
    rounds = int(rng.choice([d for d in (1, 2, 4) if tpr % d == 0]))
    cfg = CONFIGS["tiny"].scaled(num_tokens=R * tpr, hidden=H, num_ranks=R, num_experts=E, num_topk=K,
                                 expert_alignment=A, quant=quant, quant_size=qs, round_scale=rs,
                                 mask_frac=float(rng.choice([0.0, 0.1, 0.5])),
                                 x_sigma=float(rng.choice([1.0, 1e-3, 100.0])), num_rounds=rounds)
    return cfg, ue8


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_configuration(i, cuda_device):
    dev = cuda_device
    cfg, ue8 = _draw(i)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    q = None if cfg.quant == "none" else cfg.quant
    wl = make_workload(cfg, seed=i)
    x, ti, tw = to_dev(wl, dev)
    lay = (torch.empty(R, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev),
           torch.empty((T, R), dtype=torch.bool, device=dev))
    recv_x, recv_s, rti, rtw, h = ep.ep_dispatch(x, ti, tw, A, q, num_experts=E, num_ranks=R,
                                                 quant_size=cfg.quant_size, round_scale=cfg.round_scale,
                                                 num_rounds=cfg.num_rounds, layout_out=lay, scale_ue8m0=ue8)
    torch.cuda.synchronize()
    h.check()
    assert_layout_equal(lay, oracle.layout(wl.topk_idx, E, R))
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    assert_slots_equal(h, rti, rtw, s)
    n = s["num_recv_rows"]
    ref_x, ref_s = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], cfg.quant, cfg.quant_size,
                                           cfg.round_scale, ue8, num_rows=n)
    if n:
        got_x = u16(recv_x).view(np.uint8).reshape(n, -1) if q is None else u8(recv_x).reshape(n, -1)
        assert np.array_equal(got_x, ref_x.reshape(n, -1))
    if q is not None and n:
        got_s = recv_s.contiguous().cpu().numpy()
        assert np.array_equal(got_s.view(np.uint8), ref_s.view(np.uint8))
    # combine of seeded bf16 expert outputs, per round as dispatched
    y_np = make_y(n, H, i)
    y = torch.from_numpy(y_np.view(np.int16)).view(torch.bfloat16).to(dev)
    out = ep.ep_combine(y, h, tw)
    torch.cuda.synchronize()
    h.check()
    ref_out = oracle.combine(y_np, s["dst_buffer_slot_idx"], wl.topk_weights, R, cfg.num_rounds)
    assert np.array_equal(u16(out), ref_out)
    if i % 2 == 0:
        # the same combine seeded with a shared expert's bf16 output
        shared_np = make_y(T, H, i + 3)
        shared = torch.from_numpy(shared_np.view(np.int16)).view(torch.bfloat16).to(dev)
        out = ep.ep_combine(y, h, tw, shared=shared)
        torch.cuda.synchronize()
        h.check()
        ref_sh = oracle.combine_rows_q(y_np, None, "none", 0, s["dst_buffer_slot_idx"], wl.topk_weights, shared_np)
        assert np.array_equal(u16(out), ref_sh)


@pytest.mark.parametrize("i", range(0, N_CASES, 3))
def test_random_configuration_low_latency(i, cuda_device):
    dev = cuda_device
    cfg, _ = _draw(i)
    cfg = cfg.scaled(expert_alignment=1, num_rounds=1, quant="fp8" if cfg.quant != "none" else "none",
                     quant_size=128 if cfg.hidden % 128 == 0 else cfg.hidden, round_scale=False)
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    M = T // R + (i % 3)
    if M == 0:
        pytest.skip("no tokens and no slack: an empty layout")
    q = None if cfg.quant == "none" else cfg.quant
    wl = make_workload(cfg, seed=i)
    x, ti, tw = to_dev(wl, dev)
    recv_x, recv_s, count, layout_range, h = ep.ep_dispatch_low_latency(x, ti, tw, M, E, R, q,
                                                                        quant_size=cfg.quant_size)
    torch.cuda.synchronize()
    h.check()
    ref = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    dst = ref["dst_buffer_slot_idx"]
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), dst)
    assert np.array_equal(count.cpu().numpy(), ref["recv_count"])
    assert np.array_equal(layout_range.cpu().numpy(), ref["layout_range"])
    rows = E * R * M
    used = np.unique(dst[dst >= 0])
    if used.size == 0:
        return
    ref_x, ref_s = oracle.dispatch_rows(wl.x, dst, cfg.quant, cfg.quant_size, False, num_rows=rows)
    got = (u16(recv_x) if q is None else u8(recv_x)).reshape(rows, -1)
    assert np.array_equal(got[used], ref_x[used])
    if q is not None:
        gs = recv_s.reshape(rows, -1).cpu().numpy()
        assert np.array_equal(gs[used].view(np.uint32), ref_s[used].view(np.uint32))


@pytest.mark.parametrize("i", range(1, N_CASES, 2))
def test_random_cached_dispatch_and_quantised_combine(i, cuda_device):
    """On the same draws: the layout call alone; a cached dispatch of new
    activations with the first call's routing; and, for FP8 / int8 codes with
    fp32 scales, the combine of the received codes with a shared-expert row."""
    dev = cuda_device
    cfg, ue8 = _draw(i)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    q = None if cfg.quant == "none" else cfg.quant
    wl = make_workload(cfg, seed=i)
    x, ti, tw = to_dev(wl, dev)
    assert_layout_equal(ep.ep_get_dispatch_layout(ti, E, R), oracle.layout(wl.topk_idx, E, R))
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, q, cfg.quant_size, cfg.num_rounds, device=dev,
                                     scale_ue8m0=ue8)
    kw = dict(quant_size=cfg.quant_size, round_scale=cfg.round_scale, num_rounds=cfg.num_rounds, buffers=bufs,
              scale_ue8m0=ue8)
    ep.ep_dispatch(x, ti, tw, A, q, num_experts=E, num_ranks=R, **kw)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    n = s["num_recv_rows"]
    wl2 = make_workload(cfg, seed=i + 500)
    x2 = torch.from_numpy(wl2.x.view(np.int16)).view(torch.bfloat16).to(dev)
    rx, rs, _, _, _ = ep.ep_dispatch(x2, quant=q, handle=bufs.handle, **kw)
    torch.cuda.synchronize()
    bufs.handle.check()
    if n == 0:
        return
    ref_x, ref_s = oracle.dispatch_rows_mx(wl2.x, s["dst_buffer_slot_idx"], cfg.quant, cfg.quant_size,
                                           cfg.round_scale, ue8, num_rows=n)
    got = u16(rx).view(np.uint8).reshape(n, -1) if q is None else u8(rx).reshape(n, -1)
    assert np.array_equal(got, ref_x.reshape(n, -1))
    if q in ("fp8", "int8") and not ue8:
        shared_np = make_y(T, H, i + 7)
        shared = torch.from_numpy(shared_np.view(np.int16)).view(torch.bfloat16).to(dev)
        out = ep.ep_combine(bufs.recv_x, bufs.handle, tw, y_scales=bufs.recv_scales, quant_size=cfg.quant_size,
                            shared=shared)
        torch.cuda.synchronize()
        bufs.handle.check()
        ref_out = oracle.combine_rows_q(ref_x.reshape(n, -1), ref_s, cfg.quant, cfg.quant_size,
                                        s["dst_buffer_slot_idx"], wl.topk_weights, shared_np)
        assert np.array_equal(u16(out), ref_out)


@pytest.mark.parametrize("i", range(0, N_CASES, 4))
def test_random_error_paths(i, cuda_device):
    """On the same draws: an out-of-range expert id is reported as
    EP_ERR_BAD_EXPERT_ID (dispatch and layout call), and a receive capacity a
    few rows short of what the routing needs is reported as EP_ERR_CAPACITY
    with nothing written at or past the capacity."""
    dev = cuda_device
    cfg, ue8 = _draw(i)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    if T == 0:
        pytest.skip("no tokens: no entry to corrupt, no row to overflow")
    q = None if cfg.quant == "none" else cfg.quant
    rng = np.random.default_rng(7000 + i)
    wl = make_workload(cfg, seed=i)
    kw = dict(num_experts=E, num_ranks=R, quant_size=cfg.quant_size, round_scale=cfg.round_scale,
              num_rounds=cfg.num_rounds, scale_ue8m0=ue8)
    need = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)["num_recv_rows"]

    bad = wl.topk_idx.copy()
    bad[int(rng.integers(T)), int(rng.integers(K))] = int(rng.choice([E, E + 5, -2]))
    x, _, tw = to_dev(wl, dev)
    ti_bad = torch.from_numpy(bad).to(dev)
    _, _, _, _, h = ep.ep_dispatch(x, ti_bad, tw, A, q, do_cpu_sync=False, **kw)
    torch.cuda.synchronize()
    assert h.read_error() == ep.EP_ERR_BAD_EXPERT_ID
    with pytest.raises(ep.EPError) as e:
        ep.ep_get_dispatch_layout(ti_bad, E, R)
    assert e.value.status == ep.EP_ERR_BAD_EXPERT_ID

    if need == 0:
        return
    cap = int(rng.integers(max(0, need - 40), need))
    full = ep.alloc_dispatch_buffers(T, H, K, E, R, A, q, cfg.quant_size, cfg.num_rounds, recv_capacity=need + 64,
                                     device=dev, scale_ue8m0=ue8)
    tails = [full.recv_x, full.recv_topk_idx, full.recv_topk_weights, full.handle.recv_src_metadata]
    if full.recv_scales is not None:
        tails.append(full.recv_scales)
    for t in tails:
        t.view(torch.uint8).fill_(0xA5)
    short = ep.DispatchBuffers(full.recv_x[:cap], None if full.recv_scales is None else full.recv_scales[:cap],
                               full.recv_topk_idx[:cap], full.recv_topk_weights[:cap], full.handle, full.workspace,
                               q, cfg.quant_size)
    ti = torch.from_numpy(wl.topk_idx).to(dev)
    ep.ep_dispatch(x, ti, tw, A, q, buffers=short, do_cpu_sync=False, **kw)
    torch.cuda.synchronize()
    assert full.handle.read_error() == ep.EP_ERR_CAPACITY
    for t in tails:
        assert torch.all(t[cap:].contiguous().view(torch.uint8) == 0xA5)
