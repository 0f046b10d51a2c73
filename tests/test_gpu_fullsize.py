"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (capacity-bound buffers, no host sync inside dispatch).

Everything is compared in full, against the oracle's OpenMP build on every
host core: the layout and every slot, every received row and scale of every
token, and every combined token.  In addition two properties are checked on
every row: padding rows are all zero, and for bf16 dispatch every received
row equals its source token's row.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

from gpu_parity import assert_combine_close, assert_layout_equal, to_dev, u8, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def threaded_oracle():
    oracle.use_threads(len(os.sched_getaffinity(0)))
    yield
    oracle.use_threads(1)


@pytest.mark.parametrize("name", ["prefill", "decode", "qwen3", "longseq", "tiny"])
def test_full_size(name, cuda_device):
    dev = cuda_device
    cfg = CONFIGS[name]
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    wl = make_workload(cfg, seed=0)
    x, ti, tw = to_dev(wl, dev)
    q = None if cfg.quant == "none" else cfg.quant
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, cfg.expert_alignment, q, cfg.quant_size,
                                     cfg.num_rounds, device=dev)
    lay = (torch.empty(R, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev),
           torch.empty((T, R), dtype=torch.bool, device=dev))
    for _ in range(2):   # the second call runs on dirty buffers, as in the timed loop
        ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, q, num_experts=E, num_ranks=R,
                       quant_size=cfg.quant_size, round_scale=cfg.round_scale, num_rounds=cfg.num_rounds,
                       do_cpu_sync=False, buffers=bufs, layout_out=lay)
    torch.cuda.synchronize()
    h = bufs.handle
    h.check()

    ref_lay = oracle.layout(wl.topk_idx, E, R)
    assert_layout_equal(lay, ref_lay)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, cfg.expert_alignment)
    n = s["num_recv_rows"]
    assert np.array_equal(h.psum_num_recv_tokens_per_expert.cpu().numpy(), s["psum_num_recv_tokens_per_expert"])
    assert np.array_equal(h.num_recv_tokens_per_expert.cpu().numpy(), s["num_recv_tokens_per_expert"])
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), s["dst_buffer_slot_idx"])
    assert np.array_equal(h.recv_src_metadata[:n].cpu().numpy(), s["recv_src_metadata"])
    assert np.array_equal(bufs.recv_topk_idx[:n].cpu().numpy(), s["recv_topk_idx"])
    assert np.array_equal(bufs.recv_topk_weights[:n].cpu().numpy().view(np.uint32),
                          s["recv_topk_weights"].view(np.uint32))

    # padding rows: zero bytes (and zero scales)
    meta = s["recv_src_metadata"]
    pad = torch.from_numpy(np.nonzero(meta[:, 0] < 0)[0]).to(dev)
    if pad.numel():
        assert torch.all(bufs.recv_x.index_select(0, pad).view(torch.uint8) == 0)
        if bufs.recv_scales is not None:
            assert torch.all(bufs.recv_scales.index_select(0, pad) == 0)
    # bf16: every received row is its token's row
    if q is None:
        rows = np.nonzero(meta[:, 0] >= 0)[0]
        for c in range(0, rows.size, 32768):
            r = torch.from_numpy(rows[c:c + 32768]).to(dev)
            t = torch.from_numpy(meta[rows[c:c + 32768], 0].astype(np.int64)).to(dev)
            assert torch.equal(bufs.recv_x.index_select(0, r).view(torch.int16),
                               x.index_select(0, t).view(torch.int16))

    # every token's rows and scales against the oracle
    tok = np.arange(T, dtype=np.int32)
    dst = s["dst_buffer_slot_idx"]
    sub = dst[tok]
    used = np.unique(sub[sub >= 0])
    remap = -np.ones(n + 1, np.int64)
    remap[used] = np.arange(used.size)
    cdst = np.full_like(dst, -1)
    cdst[tok] = np.where(sub >= 0, remap[np.maximum(sub, 0)], -1)
    ref_x, ref_s = oracle.dispatch_rows(wl.x, cdst, cfg.quant, cfg.quant_size, cfg.round_scale,
                                        tokens=tok, num_rows=used.size)
    ridx = torch.from_numpy(used).to(dev)
    got = bufs.recv_x.index_select(0, ridx)
    got = u16(got) if q is None else u8(got)
    assert np.array_equal(got, ref_x)
    if q is not None:
        gs = bufs.recv_scales.index_select(0, ridx).cpu().numpy()
        assert np.array_equal(gs.view(np.uint32), ref_s.view(np.uint32))

    # combine of every token on seeded expert outputs y
    g = torch.Generator(device=dev)
    g.manual_seed(99)
    y = torch.randn((bufs.recv_x.shape[0], H), generator=g, device=dev, dtype=torch.bfloat16)
    out = ep.ep_combine(y, h, tw)
    torch.cuda.synchronize()
    h.check()
    y_sub = u16(y.index_select(0, ridx))
    ref_out = oracle.combine_rows(y_sub, cdst, wl.topk_weights, tokens=tok)
    got_out = u16(out.index_select(0, torch.from_numpy(tok.astype(np.int64)).to(dev)))
    assert_combine_close(got_out, ref_out)
    assert np.array_equal(got_out, ref_out)
