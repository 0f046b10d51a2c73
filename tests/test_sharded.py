"""Expert parallelism over several GPUs (one process per GPU), on CPU ranks.

The exchange plan, the point-to-point messages and the reverse exchange of
combine_topk_idx_rank_b200.sharded run for real over gloo with 2 and 4 ranks;
the local steps on each rank (route and pack of its own tokens, padding rows,
the k-order reduction) are done by the oracle here, standing in for the GPU.
Every rank's received rows, metadata, per-expert counts and combined tokens
must equal the single-GPU oracle's, restricted to that rank, bit for bit.

Also: the plan itself, checked against a brute-force placement.
"""
import os
import socket
import sys
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from combine_topk_idx_rank_b200 import sharded
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ------------------------------------------------------------- plan checks

def test_plan_places_rows_in_single_gpu_order():
    rng = np.random.default_rng(0)
    for G, E, A in ((2, 8, 1), (4, 16, 4), (3, 12, 3), (1, 4, 2)):
        C = rng.integers(0, 5, size=(G, E))
        C[rng.random((G, E)) < 0.2] = 0
        # brute force: the single-GPU layout of all rows, sorted by (expert, source GPU, i)
        rows = []
        for e in range(E):
            for src in range(G):
                rows += [(e, src, i) for i in range(C[src, e])]
            pad = -(-C[:, e].sum() // A) * A - C[:, e].sum()
            rows += [(e, -1, i) for i in range(pad)]
        Eg = E // G
        for g in range(G):
            plan = sharded.make_plan(C, g, A)
            mine = [r for r in rows if g * Eg <= r[0] < (g + 1) * Eg]
            assert plan.rows[g] == len(mine)
            assert plan.my_psum()[-1] == len(mine)
            for src in range(G):
                for j in range(Eg):
                    e = g * Eg + j
                    if C[src, e]:
                        assert mine.index((e, src, 0)) == plan.recv_off[g, src, j]
            # sender side: rows of expert e start after all rows of lower experts
            assert list(plan.send_off) == list(np.concatenate([[0], np.cumsum(C[g])[:-1]]))
            sends, recvs = sharded.dispatch_messages(plan)
            assert sum(n for *_, n in sends) == C[g].sum()
            assert sum(n for *_, n in recvs) == C[:, g * Eg:(g + 1) * Eg].sum()


# ------------------------------------------------- oracle as the local steps

class OracleLocalOps:
    """The local steps of one rank, done by the oracle on CPU tensors."""

    def send_dispatch(self, x, topk_idx, topk_weights, E, R, quant, quant_size, round_scale, scale_ue8m0,
                      token_offset):
        xn = x.numpy().view(np.uint16)
        ti, tw = topk_idx.numpy(), topk_weights.numpy()
        s = oracle.slots(ti, tw, E, R, 1)
        n = s["num_recv_rows"]
        rx, rs = oracle.dispatch_rows_mx(xn, s["dst_buffer_slot_idx"], quant or "none", quant_size, round_scale,
                                         scale_ue8m0, num_rows=n)
        meta = s["recv_src_metadata"].copy()
        meta[:, 0] += token_offset
        st = sharded.SendState(torch.from_numpy(rx), None if rs is None else torch.from_numpy(rs),
                               torch.from_numpy(s["recv_topk_idx"]), torch.from_numpy(s["recv_topk_weights"]),
                               torch.from_numpy(meta), torch.from_numpy(s["num_recv_tokens_per_expert"]),
                               s["dst_buffer_slot_idx"])
        return st

    def empty_like_rows(self, t, rows):
        if t is None:
            return None
        return torch.full((rows,) + tuple(t.shape[1:]), 0x5A, dtype=torch.uint8).view(t.dtype) \
            if t.dtype == torch.uint8 else torch.empty((rows,) + tuple(t.shape[1:]), dtype=t.dtype)

    def write_padding(self, psum, counts, bufs):
        rx, rs, ri, rw, rm = bufs
        lo = 0
        for e in range(psum.shape[0]):
            a, b = lo + int(counts[e]), int(psum[e])
            rx[a:b] = 0
            if rs is not None:
                rs[a:b] = 0
            ri[a:b] = -1
            rw[a:b] = 0
            rm[a:b] = -1
            lo = b
        return psum, counts

    def combine(self, ret_y, st, topk_weights):
        y = ret_y.numpy().view(np.uint16)
        return torch.from_numpy(oracle.combine_rows(y, st.handle, topk_weights.numpy()).view(np.int16))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    "bf16_a1": dict(quant="none", A=1, mask=0.0),
    "bf16_a4_masked": dict(quant="none", A=4, mask=0.15),
    "fp8_g16": dict(quant="fp8", A=1, mask=0.1, quant_size=16),
    "int8_token": dict(quant="int8", A=2, mask=0.0, quant_size=64),
    "mxfp4": dict(quant="mxfp4", A=1, mask=0.0, quant_size=32),
    "fp8_ue8m0_bytes": dict(quant="fp8", A=1, mask=0.0, quant_size=32, round_scale=True, ue8m0=True),
}


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        c = CASES[case]
        qs = c.get("quant_size", 128)
        cfg = CONFIGS["tiny"].scaled(num_tokens=8 * 16, hidden=64, num_experts=32, num_ranks=8, num_topk=4,
                                     expert_alignment=c["A"], quant=c["quant"], quant_size=qs,
                                     round_scale=c.get("round_scale", False), mask_frac=c["mask"])
        wl = make_workload(cfg, seed=11)
        E, R, A, K = cfg.num_experts, cfg.num_ranks, cfg.expert_alignment, cfg.num_topk
        T, H = cfg.num_tokens, cfg.hidden
        ue8 = c.get("ue8m0", False)
        quant = None if cfg.quant == "none" else cfg.quant
        # the single-GPU oracle over the whole batch
        s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
        gx, gs = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], cfg.quant, qs, cfg.round_scale, ue8,
                                         num_rows=s["num_recv_rows"])
        y = make_y(s["num_recv_rows"], H, 5)
        gout = oracle.combine_rows(y, s["dst_buffer_slot_idx"], wl.topk_weights)
        # this rank's share
        Tg, Eg = T // world, E // world
        sl = slice(rank * Tg, (rank + 1) * Tg)
        psum = s["psum_num_recv_tokens_per_expert"]
        lo = int(psum[rank * Eg - 1]) if rank else 0
        hi = int(psum[(rank + 1) * Eg - 1])
        ep = sharded.ShardedEP(E, R, A, quant, qs, cfg.round_scale, ue8, local_ops=OracleLocalOps())
        x = torch.from_numpy(wl.x[sl].view(np.int16))
        rx, rs, ri, rw, h = ep.dispatch(x, torch.from_numpy(wl.topk_idx[sl]), torch.from_numpy(wl.topk_weights[sl]))
        assert rx.shape[0] == hi - lo
        assert np.array_equal(rx.numpy(), gx[lo:hi])
        if gs is not None:
            assert np.array_equal(rs.numpy().view(np.uint8), gs[lo:hi].view(np.uint8))
        assert np.array_equal(ri.numpy(), s["recv_topk_idx"][lo:hi])
        assert np.array_equal(rw.numpy().view(np.uint32), s["recv_topk_weights"][lo:hi].view(np.uint32))
        assert np.array_equal(h.recv_src_metadata.numpy(), s["recv_src_metadata"][lo:hi])
        assert np.array_equal(h.num_recv_tokens_per_expert,
                              s["num_recv_tokens_per_expert"][rank * Eg:(rank + 1) * Eg])
        assert np.array_equal(h.psum_num_recv_tokens_per_expert, psum[rank * Eg:(rank + 1) * Eg] - lo)
        # combine: this rank's expert outputs are its slice of y
        out = ep.combine(torch.from_numpy(y[lo:hi].view(np.int16)), h, torch.from_numpy(wl.topk_weights[sl]))
        assert np.array_equal(out.numpy().view(np.uint16), gout[sl])
        q.put((rank, "ok"))
    except Exception:
        q.put((rank, traceback.format_exc()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    for r in range(world):
        assert res[r] == "ok", f"rank {r}:\n{res[r]}"


@pytest.mark.timeout(600)
@pytest.mark.parametrize("case", list(CASES))
def test_two_ranks(case):
    _run(2, case)


@pytest.mark.timeout(600)
@pytest.mark.parametrize("case", ["bf16_a4_masked", "fp8_g16", "int8_token"])
def test_four_ranks(case):
    _run(4, case)
