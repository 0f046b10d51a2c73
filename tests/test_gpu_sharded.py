"""The multi-GPU expert-parallel path's local steps on a real GPU.

This run has one GPU, so the G GPUs of a sharded batch are emulated as G
virtual GPUs in one process on that device: each runs the CUDA local steps
(routing and packing of its own tokens with a token offset, the padding rows
of its receive layout, the k-order reduction of its returned rows), and the
point-to-point messages of the exchange plan are replaced by device copies
between the virtual GPUs' buffers, one virtual GPU after another (no kernel
waits on another).  Every virtual GPU's received rows, metadata, counts and
combined tokens must equal the single-GPU oracle's, restricted to it, bit
for bit.  A world of one real process (NCCL, one rank) runs ShardedEP end to
end.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep, sharded
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y

pytestmark = pytest.mark.gpu


def _case(quant, A, mask, qs=128, hidden=512, tokens=8 * 32):
    return CONFIGS["decode"].scaled(num_tokens=tokens, hidden=hidden, num_experts=64, num_ranks=8, num_topk=8,
                                    expert_alignment=A, quant=quant, quant_size=qs, mask_frac=mask)


def _oracle_all(cfg, wl):
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, cfg.expert_alignment)
    gx, gs = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], cfg.quant, cfg.quant_size, cfg.round_scale,
                                     False, num_rows=s["num_recv_rows"])
    y = make_y(s["num_recv_rows"], cfg.hidden, 3)
    out = oracle.combine_rows(y, s["dst_buffer_slot_idx"], wl.topk_weights)
    return s, gx, gs, y, out


def _bytes(t):
    return t.contiguous().view(torch.uint8).cpu().numpy().reshape(t.shape[0], -1)


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("quant,A,mask,qs", [("none", 1, 0.0, 128), ("none", 8, 0.1, 128), ("fp8", 4, 0.0, 128),
                                             ("int8", 1, 0.1, 512), ("mxfp4", 2, 0.0, 32)])
def test_virtual_gpus(G, quant, A, mask, qs, cuda_device):
    cfg = _case(quant, A, mask, qs)
    wl = make_workload(cfg, seed=G)
    E, R, K, T, H = cfg.num_experts, cfg.num_ranks, cfg.num_topk, cfg.num_tokens, cfg.hidden
    s, gx, gs, y, gout = _oracle_all(cfg, wl)
    ops = sharded.CudaLocalOps(cuda_device)
    Tg, Eg = T // G, E // G
    q = None if quant == "none" else quant
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    ti = torch.from_numpy(wl.topk_idx).to(cuda_device)
    tw = torch.from_numpy(wl.topk_weights).to(cuda_device)
    # 1. every virtual GPU routes and packs its own tokens
    st = [ops.send_dispatch(x[g * Tg:(g + 1) * Tg].contiguous(), ti[g * Tg:(g + 1) * Tg].contiguous(),
                            tw[g * Tg:(g + 1) * Tg].contiguous(), E, R, q, qs, False, False, g * Tg)
          for g in range(G)]
    # 2. the count matrix; 3. the plans
    C = np.stack([t.counts.cpu().numpy() for t in st]).astype(np.int64)
    plans = [sharded.make_plan(C, g, A) for g in range(G)]
    psum = s["psum_num_recv_tokens_per_expert"]
    recv = []
    for d in range(G):
        rows = int(plans[d].rows[d])
        bufs = [ops.empty_like_rows(t, rows) for t in (st[d].send_x, st[d].send_scales, st[d].send_topk_idx,
                                                       st[d].send_topk_weights, st[d].send_meta)]
        for b in bufs:
            if b is not None:
                b.view(torch.uint8).fill_(0x5A)       # every byte must be written by the exchange or the padding
        # 4. the messages into virtual GPU d, as device copies from each source's send buffer
        _, recvs = sharded.dispatch_messages(plans[d])
        for src, e, row, n in recvs:
            srow = int(plans[src].send_off[e])
            for sa, ra in zip((st[src].send_x, st[src].send_scales, st[src].send_topk_idx,
                               st[src].send_topk_weights, st[src].send_meta), bufs):
                if sa is not None:
                    ra[row:row + n].copy_(sa[srow:srow + n])
        # 5. padding rows
        ops.write_padding(plans[d].my_psum(), plans[d].my_counts(), bufs)
        torch.cuda.synchronize()
        lo = int(psum[d * Eg - 1]) if d else 0
        hi = int(psum[(d + 1) * Eg - 1])
        rx, rs, ri, rw, rm = bufs
        assert rx.shape[0] == hi - lo
        assert np.array_equal(_bytes(rx), gx[lo:hi].reshape(hi - lo, -1))
        if gs is not None:
            assert np.array_equal(_bytes(rs), gs[lo:hi].view(np.uint8).reshape(hi - lo, -1))
        assert np.array_equal(ri.cpu().numpy(), s["recv_topk_idx"][lo:hi])
        assert np.array_equal(rw.cpu().numpy().view(np.uint32), s["recv_topk_weights"][lo:hi].view(np.uint32))
        assert np.array_equal(rm.cpu().numpy(), s["recv_src_metadata"][lo:hi])
        recv.append((lo, hi))
    # combine: each virtual GPU's y rows return to their sources, which reduce them
    yd = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    for g in range(G):
        ret = torch.empty((st[g].send_x.shape[0], H), dtype=torch.bfloat16, device=cuda_device)
        sends, _ = sharded.dispatch_messages(plans[g])
        for dst, e, row, n in sends:
            d_lo = recv[dst][0]
            j = e - dst * Eg
            rrow = int(plans[dst].recv_off[dst, g, j])
            ret[row:row + n].copy_(yd[d_lo + rrow:d_lo + rrow + n])
        out = ops.combine(ret, st[g], tw[g * Tg:(g + 1) * Tg].contiguous())
        torch.cuda.synchronize()
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), gout[g * Tg:(g + 1) * Tg])


def _free_port():
    with socket.socket() as sck:
        sck.bind(("127.0.0.1", 0))
        return sck.getsockname()[1]


def test_one_rank_world_end_to_end(cuda_device):
    import datetime

    import torch.distributed as dist
    cfg = _case("fp8", 4, 0.1)
    wl = make_workload(cfg, seed=9)
    s, gx, gs, y, gout = _oracle_all(cfg, wl)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=cuda_device)
    try:
        sep = sharded.ShardedEP(cfg.num_experts, cfg.num_ranks, cfg.expert_alignment, "fp8", 128,
                                device=cuda_device)
        x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
        ti = torch.from_numpy(wl.topk_idx).to(cuda_device)
        tw = torch.from_numpy(wl.topk_weights).to(cuda_device)
        rx, rs, ri, rw, h = sep.dispatch(x, ti, tw)
        torch.cuda.synchronize()
        assert np.array_equal(_bytes(rx), gx)
        assert np.array_equal(rs.cpu().numpy().view(np.uint32), gs.view(np.uint32))
        assert np.array_equal(h.recv_src_metadata.cpu().numpy(), s["recv_src_metadata"])
        assert np.array_equal(h.psum_num_recv_tokens_per_expert.cpu().numpy(), s["psum_num_recv_tokens_per_expert"])
        out = sep.combine(torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).to(cuda_device), h, tw)
        torch.cuda.synchronize()
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), gout)
    finally:
        dist.destroy_process_group()


def test_padding_rows_kernel(cuda_device):
    # segments with padding at their ends; rows past the capacity untouched
    psum = torch.tensor([4, 4, 12, 16], dtype=torch.int32, device=cuda_device)
    cnt = torch.tensor([1, 0, 8, 3], dtype=torch.int32, device=cuda_device)
    rx = torch.full((15, 32), 7, dtype=torch.uint8, device=cuda_device)
    rs = torch.full((15, 3), 7, dtype=torch.uint8, device=cuda_device)
    ri = torch.full((15, 2), 7, dtype=torch.int32, device=cuda_device)
    rw = torch.full((15, 2), 7.0, dtype=torch.float32, device=cuda_device)
    rm = torch.full((15, 2), 7, dtype=torch.int32, device=cuda_device)
    ep.ep_write_padding_rows(psum, cnt, rx, rs, ri, rw, rm)
    torch.cuda.synchronize()
    pad = [1, 2, 3, 15]                     # row 15 is past the capacity of 15 rows
    for r in range(15):
        want = r in pad
        assert bool((rx[r] == 0).all()) == want and bool((rs[r] == 0).all()) == want
        assert bool((ri[r] == -1).all()) == want and bool((rw[r] == 0).all()) == want
        assert bool((rm[r] == -1).all()) == want
