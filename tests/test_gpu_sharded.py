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


# ------------------------------------------------ the peer-memory data plane

def _dev_rows(t, n):
    return t[:n].contiguous().view(torch.uint8).cpu().numpy().reshape(n, -1)


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("quant,A,mask,qs", [("none", 1, 0.0, 128), ("none", 8, 0.1, 128), ("fp8", 4, 0.0, 128),
                                             ("int8", 1, 0.1, 64)])
def test_peer_plane_on_virtual_gpus(G, quant, A, mask, qs, cuda_device):
    """ep_route + ep_pack_peer + ep_receiver_layout + ep_write_padding_rows +
    ep_combine_peer on G virtual GPUs of one device: the peer pointer tables
    point at the virtual receivers' buffers, so every store and load takes the
    same addressing path as across GPUs; results equal the single-GPU oracle's
    restricted to each virtual GPU, bit for bit."""
    cfg = _case(quant, A, mask, qs)
    wl = make_workload(cfg, seed=10 + G)
    E, R, K, T, H = cfg.num_experts, cfg.num_ranks, cfg.num_topk, cfg.num_tokens, cfg.hidden
    s, gx, gs, y, gout = _oracle_all(cfg, wl)
    Tg, Eg = T // G, E // G
    q = None if quant == "none" else quant
    dev = cuda_device
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(dev)
    ti = torch.from_numpy(wl.topk_idx).to(dev)
    tw = torch.from_numpy(wl.topk_weights).to(dev)
    cap = T * K + Eg * (A - 1)
    bufs = []
    for d in range(G):
        rx, rs = ep._recv_tensors(cap, H, q, qs, False, dev)
        rx.view(torch.uint8).fill_(0x5A)
        if rs is not None:
            rs.view(torch.uint8).fill_(0x5A)
        bufs.append(dict(x=rx, s=rs, i=torch.full((cap, K), 77, dtype=torch.int32, device=dev),
                         w=torch.full((cap, K), 7.0, dtype=torch.float32, device=dev),
                         m=torch.full((cap, 2), 77, dtype=torch.int32, device=dev),
                         y=torch.empty((cap, H), dtype=torch.bfloat16, device=dev)))
    tab = {k: ep.pointer_table([b[k] for b in bufs], dev) for k in ("x", "s", "i", "w", "m", "y")}
    routes = [ep.ep_route(ti[g * Tg:(g + 1) * Tg].contiguous(), tw[g * Tg:(g + 1) * Tg].contiguous(), E, R, H, 1,
                          token_offset=g * Tg) for g in range(G)]
    counts_all = torch.stack([r[2].num_recv_tokens_per_expert for r in routes])
    for g, (rti, rtw, h) in enumerate(routes):
        ep.ep_pack_peer(x[g * Tg:(g + 1) * Tg].contiguous(), h, rti, rtw, counts_all, G, g, A, tab["x"],
                        tab["s"] if q else None, tab["i"], tab["w"], tab["m"], cap, q, qs)
    psum = s["psum_num_recv_tokens_per_expert"]
    for d in range(G):
        p_d, c_d = ep.ep_receiver_layout(counts_all, G, d, A)
        lo = int(psum[d * Eg - 1]) if d else 0
        hi = int(psum[(d + 1) * Eg - 1])
        n = hi - lo
        b = bufs[d]
        ep.ep_write_padding_rows(p_d, c_d, b["x"][:n], None if b["s"] is None else b["s"][:n], b["i"][:n],
                                 b["w"][:n], b["m"][:n])
        torch.cuda.synchronize()
        assert np.array_equal(p_d.cpu().numpy(), psum[d * Eg:(d + 1) * Eg] - lo)
        assert np.array_equal(c_d.cpu().numpy(), s["num_recv_tokens_per_expert"][d * Eg:(d + 1) * Eg])
        assert np.array_equal(_dev_rows(b["x"], n), gx[lo:hi].reshape(n, -1))
        if gs is not None:
            assert np.array_equal(_dev_rows(b["s"], n), gs[lo:hi].view(np.uint8).reshape(n, -1))
        assert np.array_equal(b["i"][:n].cpu().numpy(), s["recv_topk_idx"][lo:hi])
        assert np.array_equal(b["w"][:n].cpu().numpy().view(np.uint32), s["recv_topk_weights"][lo:hi].view(np.uint32))
        assert np.array_equal(b["m"][:n].cpu().numpy(), s["recv_src_metadata"][lo:hi])
        b["y"][:n].copy_(torch.from_numpy(y[lo:hi].view(np.int16)).view(torch.bfloat16))
    for g, (rti, rtw, h) in enumerate(routes):
        out = ep.ep_combine_peer(tab["y"], h, counts_all, G, g, A, tw[g * Tg:(g + 1) * Tg].contiguous(), cap)
        torch.cuda.synchronize()
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), gout[g * Tg:(g + 1) * Tg])
        assert h.read_error() == ep.EP_OK


def _peer_worker(rank, world, port, q):
    import datetime
    import traceback

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        cfg = _case("fp8", 4, 0.1)
        wl = make_workload(cfg, seed=21)
        s, gx, gs, y, gout = _oracle_all(cfg, wl)
        E, R, K, T, H = cfg.num_experts, cfg.num_ranks, cfg.num_topk, cfg.num_tokens, cfg.hidden
        Tg, Eg = T // world, E // world
        sl = slice(rank * Tg, (rank + 1) * Tg)
        sep = sharded.PeerShardedEP(E, R, H, K, Tg, cfg.expert_alignment, "fp8", 128, device=dev)
        x = torch.from_numpy(wl.x[sl].view(np.int16)).view(torch.bfloat16).to(dev)
        ti = torch.from_numpy(wl.topk_idx[sl]).to(dev)
        tw = torch.from_numpy(wl.topk_weights[sl]).to(dev)
        for _ in range(2):   # the second step reuses every buffer
            rx, rs, ri, rw, h = sep.dispatch(x, ti, tw)
            torch.cuda.synchronize()
            psum = s["psum_num_recv_tokens_per_expert"]
            lo = int(psum[rank * Eg - 1]) if rank else 0
            hi = int(psum[(rank + 1) * Eg - 1])
            assert h["rows"] == hi - lo
            assert np.array_equal(_dev_rows(rx, hi - lo), gx[lo:hi].reshape(hi - lo, -1))
            assert np.array_equal(rs.cpu().numpy().view(np.uint32), gs[lo:hi].view(np.uint32))
            assert np.array_equal(sep.recv_meta[:hi - lo].cpu().numpy(), s["recv_src_metadata"][lo:hi])
            sep.y[:hi - lo].copy_(torch.from_numpy(y[lo:hi].view(np.int16)).view(torch.bfloat16))
            out = sep.combine(h, tw)
            torch.cuda.synchronize()
            assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), gout[sl])
        sep.close()
        q.put((rank, "ok"))
    except Exception:
        q.put((rank, traceback.format_exc()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(600)
def test_peer_plane_two_processes_through_cuda_ipc(cuda_device):
    """PeerShardedEP end to end in two processes that share this GPU: each maps
    the other's receive layout and expert outputs through CUDA IPC, exchanges
    the counts over gloo, and orders the steps by device syncs and barriers
    (no kernel waits on the other process)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=500) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    for r in range(2):
        assert res[r] == "ok", f"rank {r}:\n{res[r]}"
