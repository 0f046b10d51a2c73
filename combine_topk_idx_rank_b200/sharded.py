"""Expert parallelism over several GPUs, one process per GPU.

G processes share the R logical EP ranks of one batch.  GPU g holds logical
ranks [g R/G, (g+1) R/G): their tokens (the T/G consecutive tokens
[g T/G, (g+1) T/G)) and their experts (the E/G consecutive experts
[g E/G, (g+1) E/G)).  Every GPU ends with the single-GPU result restricted to
itself: its received rows are the rows of its experts in the deterministic
(expert, token, k) order with each expert padded to expert_alignment
("DeepEP V1 vs V2 comparative analysis", sections 3.1 and 8.4), and combine
returns its own tokens.

Dispatch follows the normal mode's phases (same page, section 6.1: layout /
notify, then the data; section 3.2: the host reads the counts):

1. local: this GPU's tokens are routed and packed into a send buffer ordered
   by (expert, token, k) with alignment 1 -- ``ep_dispatch`` with the
   logical ranks, and ``token_offset`` so that the metadata names tokens of
   the whole batch.  The quantisation happens here, once per token.
2. counts: an all-gather of every GPU's per-expert counts, C [G, E] (the
   layout exchange); the host reads C.
3. plan (host): on receiver d, expert e's segment starts at the exclusive
   prefix of the aligned totals sum_g C[g, e] over d's experts; within it,
   source g's rows follow those of every source g' < g.  Because tokens are
   ordered by GPU, this is exactly the (expert, token, k) order.
4. exchange: each (source, expert) block is contiguous in the source's send
   buffer and in the receiver's layout, so it moves with one point-to-point
   message per array, straight into place (no permutation pass).
5. the receiver writes its padding rows (``ep_write_padding_rows``).

Combine runs the exchange in reverse: receiver d returns each source's y rows
into that source's send-buffer order, and the source reduces them with its
send handle (``ep_combine``: the k-order fp32 weighted sum).

The arithmetic of every step runs in the local operations (the CUDA library
for ``CudaLocalOps``); this module computes the plan and moves rows with
``torch.distributed`` point-to-point messages (NCCL between GPUs; the tests
run it on CPU ranks over gloo).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

__all__ = ["ExchangePlan", "make_plan", "dispatch_messages", "combine_messages", "ShardedEP", "ShardedHandle",
           "CudaLocalOps", "SendState"]


# ---------------------------------------------------------------------- plan

@dataclasses.dataclass
class ExchangePlan:
    """Where every row goes, computed from the all-gathered counts C [G, E]."""
    G: int
    g: int                     # this GPU
    E: int
    A: int                     # expert alignment
    counts: np.ndarray         # [G, E] int64: rows from GPU g' for expert e
    send_off: np.ndarray       # [E]: first row of expert e in this GPU's send buffer
    seg_start: np.ndarray      # [G, E/G]: first row of each receiver's expert segments
    recv_off: np.ndarray       # [G, G, E/G]: [d, g', j] first row on receiver d of source g''s rows of
                               # d's j-th expert
    rows: np.ndarray           # [G]: rows of each receiver's layout (padding included)

    @property
    def experts_per_gpu(self) -> int:
        return self.E // self.G

    def my_psum(self) -> np.ndarray:
        """Inclusive prefix of this GPU's aligned per-expert counts (int32)."""
        tot = self.counts.sum(axis=0)[self.g * self.experts_per_gpu:(self.g + 1) * self.experts_per_gpu]
        return np.cumsum(-(-tot // self.A) * self.A).astype(np.int32)

    def my_counts(self) -> np.ndarray:
        """This GPU's unaligned per-expert counts (int32)."""
        return self.counts.sum(axis=0)[self.g * self.experts_per_gpu:(self.g + 1) * self.experts_per_gpu].astype(
            np.int32)


def make_plan(counts: np.ndarray, g: int, A: int) -> ExchangePlan:
    C = np.asarray(counts, np.int64)
    G, E = C.shape
    if E % G:
        raise ValueError("experts must split evenly over the GPUs")
    Eg = E // G
    send_off = np.concatenate([[0], np.cumsum(C[g])[:-1]]).astype(np.int64)
    totals = C.sum(axis=0).reshape(G, Eg)
    aligned = -(-totals // A) * A
    seg_start = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(aligned, axis=1)[:, :-1]], axis=1)
    # rows of earlier sources inside each segment
    before = np.concatenate([np.zeros((1, E), np.int64), np.cumsum(C, axis=0)[:-1]], axis=0)   # [G src, E]
    recv_off = seg_start[:, None, :] + before.reshape(G, G, Eg).transpose(1, 0, 2)
    return ExchangePlan(G, g, E, A, C, send_off, seg_start, recv_off, aligned.sum(axis=1))


def dispatch_messages(plan: ExchangePlan):
    """(sends, recvs) of this GPU's dispatch, as (peer, expert, row, n).

    Sends: every expert with rows from this GPU, in expert order, to its
    owner; recvs: for each source GPU in order, each of this GPU's experts in
    order.  For any ordered pair of GPUs both sides list their messages in
    expert order, so point-to-point messages match in order."""
    G, g, Eg = plan.G, plan.g, plan.experts_per_gpu
    sends = [(e // Eg, e, int(plan.send_off[e]), int(plan.counts[g, e]))
             for e in range(plan.E) if plan.counts[g, e] > 0]
    recvs = [(src, g * Eg + j, int(plan.recv_off[g, src, j]), int(plan.counts[src, g * Eg + j]))
             for src in range(G) for j in range(Eg) if plan.counts[src, g * Eg + j] > 0]
    return sends, recvs


def combine_messages(plan: ExchangePlan):
    """(sends, recvs) of the reverse exchange: the dispatch messages with the
    roles swapped (receivers return rows to their sources)."""
    sends, recvs = dispatch_messages(plan)
    return recvs, sends


def exchange(group, me: int, E: int, pairs, sends, recvs):
    """Moves rows: for each (send_array, recv_array) in `pairs`, every send
    (peer, expert, row, n) ships send_array[row:row+n] to `peer`, and every
    recv (peer, expert, row, n) lands in recv_array[row:row+n].  Messages to
    this GPU itself are local copies.  The tag of a message is its array
    index times E plus its expert, so messages match on every backend."""
    ops = []
    for i, (sa, ra) in enumerate(pairs):
        for peer, e, row, n in sends:
            if peer != me:
                ops.append(dist.P2POp(dist.isend, sa[row:row + n], peer, group, tag=i * E + e))
        for peer, e, row, n in recvs:
            if peer != me:
                ops.append(dist.P2POp(dist.irecv, ra[row:row + n], peer, group, tag=i * E + e))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    mine = {e: (row, n) for peer, e, row, n in sends if peer == me}
    for peer, e, row, n in recvs:
        if peer == me:
            srow, sn = mine[e]
            assert sn == n
            for sa, ra in pairs:
                ra[row:row + n].copy_(sa[srow:srow + n])


# ------------------------------------------------------------- local ops

@dataclasses.dataclass
class SendState:
    """This GPU's tokens routed and packed in (expert, token, k) order."""
    send_x: torch.Tensor            # [n, ...] rows (bf16 or codes)
    send_scales: Optional[torch.Tensor]
    send_topk_idx: torch.Tensor     # [n, K] int32
    send_topk_weights: torch.Tensor  # [n, K] fp32
    send_meta: torch.Tensor         # [n, 2] int32: (global token, k)
    counts: torch.Tensor            # [E] int32 on the transport's device
    handle: object                  # what combine needs to reduce the returned rows


class CudaLocalOps:
    """The local steps on this GPU, through libep.so."""

    def __init__(self, device):
        from . import ep
        self.ep = ep
        self.device = torch.device(device)

    def send_dispatch(self, x, topk_idx, topk_weights, E, R, quant, quant_size, round_scale, scale_ue8m0,
                      token_offset) -> SendState:
        recv_x, recv_s, rti, rtw, h = self.ep.ep_dispatch(
            x, topk_idx, topk_weights, 1, quant, num_experts=E, num_ranks=R, quant_size=quant_size,
            round_scale=round_scale, scale_ue8m0=scale_ue8m0, token_offset=token_offset, do_cpu_sync=True)
        n = h.num_recv_rows
        return SendState(recv_x, recv_s, rti, rtw, h.recv_src_metadata[:n], h.num_recv_tokens_per_expert, h)

    def empty_like_rows(self, t: Optional[torch.Tensor], rows: int):
        if t is None:
            return None
        return torch.empty((rows,) + tuple(t.shape[1:]), dtype=t.dtype, device=self.device)

    def write_padding(self, psum: np.ndarray, counts: np.ndarray, bufs):
        ps = torch.from_numpy(psum).to(self.device)
        cn = torch.from_numpy(counts).to(self.device)
        rx, rs, ri, rw, rm = bufs
        if rx.shape[0]:
            self.ep.ep_write_padding_rows(ps, cn, rx, rs, ri, rw, rm)
        return ps, cn

    def combine(self, ret_y, st: SendState, topk_weights):
        return self.ep.ep_combine(ret_y, st.handle, topk_weights)


# ---------------------------------------------------------------- the API

@dataclasses.dataclass
class ShardedHandle:
    plan: ExchangePlan
    send: SendState
    psum_num_recv_tokens_per_expert: object    # [E/G] inclusive aligned prefix (this GPU's experts)
    num_recv_tokens_per_expert: object         # [E/G] unaligned counts
    recv_src_metadata: torch.Tensor            # [rows, 2]: (global token, k); (-1, -1) on padding
    hidden: int


class ShardedEP:
    """Dispatch / combine of one batch whose logical EP ranks are spread over
    the GPUs of a process group (one process per GPU)."""

    def __init__(self, num_experts: int, num_ranks: int, expert_alignment: int = 1, quant: Optional[str] = None,
                 quant_size: int = 128, round_scale: bool = False, scale_ue8m0: bool = False, group=None,
                 local_ops=None, device=None):
        self.group = group
        self.G = dist.get_world_size(group)
        self.g = dist.get_rank(group)
        if num_experts % num_ranks or num_ranks % self.G:
            raise ValueError("num_ranks must divide num_experts and be a multiple of the GPU count")
        self.E, self.R, self.A = num_experts, num_ranks, expert_alignment
        self.quant = None if quant in (None, "none") else quant
        self.quant_size, self.round_scale, self.scale_ue8m0 = quant_size, round_scale, scale_ue8m0
        self.ops = local_ops if local_ops is not None else CudaLocalOps(device or torch.cuda.current_device())

    def gather_counts(self, counts: torch.Tensor) -> np.ndarray:
        parts = [torch.empty_like(counts) for _ in range(self.G)]
        dist.all_gather(parts, counts, group=self.group)
        return torch.stack(parts).cpu().numpy().astype(np.int64)     # the host reads the layout

    def dispatch(self, x, topk_idx, topk_weights):
        """This GPU's tokens x [T/G, H], topk_idx [T/G, K] (global expert ids),
        topk_weights [T/G, K] -> (recv_x, recv_scales, recv_topk_idx,
        recv_topk_weights, handle) of this GPU's experts."""
        Tg = x.shape[0]
        st = self.ops.send_dispatch(x, topk_idx, topk_weights, self.E, self.R, self.quant, self.quant_size,
                                    self.round_scale, self.scale_ue8m0, token_offset=self.g * Tg)
        plan = make_plan(self.gather_counts(st.counts), self.g, self.A)
        rows = int(plan.rows[self.g])
        rx = self.ops.empty_like_rows(st.send_x, rows)
        rs = self.ops.empty_like_rows(st.send_scales, rows)
        ri = self.ops.empty_like_rows(st.send_topk_idx, rows)
        rw = self.ops.empty_like_rows(st.send_topk_weights, rows)
        rm = self.ops.empty_like_rows(st.send_meta, rows)
        pairs = [(st.send_x, rx), (st.send_topk_idx, ri), (st.send_topk_weights, rw), (st.send_meta, rm)]
        if st.send_scales is not None:
            pairs.append((st.send_scales, rs))
        sends, recvs = dispatch_messages(plan)
        exchange(self.group, self.g, self.E, pairs, sends, recvs)
        psum, cnt = self.ops.write_padding(plan.my_psum(), plan.my_counts(), (rx, rs, ri, rw, rm))
        h = ShardedHandle(plan, st, psum, cnt, rm, x.shape[1])
        return rx, rs, ri, rw, h

    def combine(self, y, handle: ShardedHandle, topk_weights):
        """y [rows, H]: this GPU's expert outputs in its received-row order ->
        the combined rows of this GPU's tokens [T/G, H]."""
        st = handle.send
        n = st.send_x.shape[0]
        ret = self.ops.empty_like_rows(y, n)
        sends, recvs = combine_messages(handle.plan)
        exchange(self.group, self.g, self.E, [(y, ret)], sends, recvs)
        return self.ops.combine(ret, st, topk_weights)


# ------------------------------------------------- peer-memory data plane

class PeerShardedEP:
    """The same split of one batch over G GPUs (one process per GPU), with the
    rows moving through peer memory instead of messages: each GPU routes its
    own tokens (``ep_route``), the per-expert counts are all-gathered into
    device memory, and ``ep_pack_peer`` stores every row (bf16 or quantised
    once) and its per-row metadata straight into its receiver's layout through
    peer pointers; ``ep_combine_peer`` loads each token's rows from the
    receivers' expert outputs and reduces them in k order.  No host reads the
    counts on the way.

    Every GPU allocates its receive layout (and its expert-output buffer ``y``)
    at the worst-case capacity and maps the other GPUs' through CUDA IPC once.
    Steps are ordered across processes by a collective on the stream (NCCL) or
    by a device sync and a host barrier (other backends)."""

    def __init__(self, num_experts: int, num_ranks: int, hidden: int, num_topk: int, tokens_per_gpu: int,
                 expert_alignment: int = 1, quant: Optional[str] = None, quant_size: int = 128,
                 round_scale: bool = False, scale_ue8m0: bool = False, group=None, device=None):
        from . import ep
        self.ep = ep
        self.group = group
        self.G, self.g = dist.get_world_size(group), dist.get_rank(group)
        if num_experts % num_ranks or num_ranks % self.G:
            raise ValueError("num_ranks must divide num_experts and be a multiple of the GPU count")
        self.E, self.R, self.H, self.K, self.A = num_experts, num_ranks, hidden, num_topk, expert_alignment
        self.Tg = tokens_per_gpu
        self.quant = None if quant in (None, "none") else quant
        self.quant_size, self.round_scale, self.scale_ue8m0 = quant_size, round_scale, scale_ue8m0
        self.dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.nccl = dist.get_backend(group) == "nccl"
        # every row of the batch could land on one GPU
        self.cap = self.Tg * self.G * self.K + (self.E // self.G) * (self.A - 1)
        rx, rs = ep._recv_tensors(self.cap, hidden, self.quant, quant_size, scale_ue8m0, self.dev)
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.recv_x, self.recv_scales = rx, rs
        self.recv_topk_idx = torch.empty((self.cap, self.K), **i32)
        self.recv_topk_weights = torch.empty((self.cap, self.K), dtype=torch.float32, device=self.dev)
        self.recv_meta = torch.empty((self.cap, 2), **i32)
        self.y = torch.empty((self.cap, hidden), dtype=torch.bfloat16, device=self.dev)
        self._imported = []
        bufs = [self.recv_x, self.recv_scales, self.recv_topk_idx, self.recv_topk_weights, self.recv_meta, self.y]
        tables = [self._peer_addresses(b) for b in bufs]
        (self.t_x, self.t_scales, self.t_topk_idx, self.t_topk_weights, self.t_meta, self.t_y) = [
            ep.pointer_table(t, self.dev) for t in tables]
        self._flag = torch.zeros((1,), **i32)

    def _peer_addresses(self, t):
        """Every GPU's address of the same buffer, in this process."""
        if t is None:
            return [0] * self.G
        torch.cuda.synchronize(self.dev)
        mine = self.ep.ipc_export(t) if self.G > 1 else (b"", 0)
        allh = [None] * self.G
        dist.all_gather_object(allh, mine, group=self.group)
        out = []
        for q, (h, off) in enumerate(allh):
            if q == self.g:
                out.append(t.data_ptr())
            else:
                addr = self.ep.ipc_import(h, off, self.dev)
                self._imported.append(addr - off)
                out.append(addr)
        return out

    def _order(self):
        """Every GPU has finished the work it queued before this point."""
        if self.nccl:
            dist.all_reduce(self._flag, group=self.group)
        else:
            torch.cuda.synchronize(self.dev)
            dist.barrier(group=self.group)

    def _gather_counts(self, counts):
        if self.nccl:
            out = torch.empty((self.G, self.E), dtype=torch.int32, device=self.dev)
            dist.all_gather_into_tensor(out, counts, group=self.group)
            return out
        parts = [torch.empty((self.E,), dtype=torch.int32) for _ in range(self.G)]
        dist.all_gather(parts, counts.cpu(), group=self.group)
        return torch.stack(parts).to(self.dev)

    def dispatch(self, x, topk_idx, topk_weights):
        """This GPU's tokens -> (recv_x, recv_scales, recv_topk_idx,
        recv_topk_weights, handle) of its experts (views of its layout)."""
        ep = self.ep
        rti, rtw, h = ep.ep_route(topk_idx, topk_weights, self.E, self.R, self.H, 1, token_offset=self.g * self.Tg)
        counts_all = self._gather_counts(h.num_recv_tokens_per_expert)
        self._order()                     # the receivers are done with their previous rows
        ep.ep_pack_peer(x, h, rti, rtw, counts_all, self.G, self.g, self.A, self.t_x, self.t_scales,
                        self.t_topk_idx, self.t_topk_weights, self.t_meta, self.cap, self.quant, self.quant_size,
                        self.round_scale, self.scale_ue8m0)
        self._order()                     # every GPU's rows have landed
        psum, cnt = ep.ep_receiver_layout(counts_all, self.G, self.g, self.A)
        rows = int(psum[-1].item()) if psum.numel() else 0
        ep.ep_write_padding_rows(psum, cnt, self.recv_x[:rows],
                                 None if self.recv_scales is None else self.recv_scales[:rows],
                                 self.recv_topk_idx[:rows], self.recv_topk_weights[:rows], self.recv_meta[:rows])
        handle = dict(route=h, counts_all=counts_all, psum=psum, counts=cnt, rows=rows)
        rs = None if self.recv_scales is None else self.recv_scales[:rows]
        return self.recv_x[:rows], rs, self.recv_topk_idx[:rows], self.recv_topk_weights[:rows], handle

    def combine(self, handle, topk_weights):
        """After the experts wrote this GPU's outputs into ``self.y`` (received
        order): this GPU's tokens, combined."""
        self._order()                     # every receiver's y is written
        out = self.ep.ep_combine_peer(self.t_y, handle["route"], handle["counts_all"], self.G, self.g, self.A,
                                      topk_weights, self.cap)
        self._order()                     # no receiver overwrites y while it is read
        return out

    def close(self):
        for base in self._imported:
            self.ep._lib.ep_ipc_close(C_void_p(base))
        self._imported = []


def C_void_p(v):
    import ctypes
    return ctypes.c_void_p(v)
