"""ep_dispatch_noalloc: dispatch for callers that cannot allocate device memory.

Such callers (code that may not call cudaMalloc, plugins that only receive
their input and output pointers, runtimes without an allocator) pass no
workspace; the library keeps the routing scratch in a static 2 MiB device
array instead.  These tests call it through the C ABI and check that its
results equal ep_dispatch's with a caller workspace, bit for bit, on two
calls in a row (the second runs on the scratch the first left behind), and
that oversized problems are refused before anything runs.

This file is named to be collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

SCRATCH_BYTES = 2 << 20


def _noalloc():
    f = ep._lib.ep_dispatch_noalloc
    p, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
    f.argtypes = [p, i32, i32, p, p, i32, i32, i32, C.POINTER(ep._Opts), p, p, p, p, i64,
                  C.POINTER(ep._Handle), p, p, p, p]
    f.restype = C.c_int
    return f


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _call_noalloc(cfg, x, ti, tw, bufs, lay):
    q = None if cfg.quant == "none" else cfg.quant
    opts = ep._Opts(cfg.expert_alignment, ep._QUANT[q], cfg.quant_size if q else 0, int(cfg.round_scale),
                    cfg.num_rounds, 0, None, None, None)
    h = bufs.handle
    h.num_rounds = cfg.num_rounds
    ch = h._c()
    T, H = x.shape
    st = _noalloc()(_ptr(x), T, H, _ptr(ti), _ptr(tw), ti.shape[1], cfg.num_experts, cfg.num_ranks,
                    C.byref(opts), _ptr(bufs.recv_x), _ptr(bufs.recv_scales), _ptr(bufs.recv_topk_idx),
                    _ptr(bufs.recv_topk_weights), bufs.recv_x.shape[0], C.byref(ch), _ptr(lay[0]),
                    _ptr(lay[1]), _ptr(lay[2]),
                    C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _outputs(bufs, lay, n):
    h = bufs.handle
    out = [bufs.recv_x[:n].contiguous().view(torch.uint8), bufs.recv_topk_idx[:n], bufs.recv_topk_weights[:n].view(torch.int32),
           h.psum_num_recv_tokens_per_expert, h.num_recv_tokens_per_expert, h.dst_buffer_slot_idx,
           h.recv_src_metadata[:n], h.topk_idx, lay[0], lay[1], lay[2]]
    if bufs.recv_scales is not None:
        out.append(bufs.recv_scales[:n].view(torch.int32))
    return [o.cpu() for o in out]


def _case(cfg, seed, dev):
    wl = make_workload(cfg, seed)
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(dev)
    ti = torch.from_numpy(wl.topk_idx).to(dev)
    tw = torch.from_numpy(wl.topk_weights).to(dev)
    return x, ti, tw


def _lay(cfg, T, dev):
    return (torch.empty(cfg.num_ranks, dtype=torch.int32, device=dev),
            torch.empty(cfg.num_experts, dtype=torch.int32, device=dev),
            torch.empty((T, cfg.num_ranks), dtype=torch.bool, device=dev))


@pytest.mark.gpu
def test_noalloc_matches_dispatch_on_two_calls_in_a_row(cuda_device):
    dev = cuda_device
    cases = [CONFIGS["prefill"].scaled(num_tokens=8 * 520, hidden=1024),
             CONFIGS["decode"].scaled(num_tokens=16 * 72, hidden=1024)]
    for i, cfg in enumerate(cases):
        T = cfg.num_tokens
        assert ep.workspace_bytes(T, cfg.num_topk, cfg.num_experts, cfg.num_ranks) <= SCRATCH_BYTES
        x, ti, tw = _case(cfg, 10 + i, dev)
        q = None if cfg.quant == "none" else cfg.quant
        # the existing entry point, with a caller workspace
        ref_bufs = ep.alloc_dispatch_buffers(T, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                                             cfg.expert_alignment, q, cfg.quant_size, device=dev)
        ref_lay = _lay(cfg, T, dev)
        ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, q, num_experts=cfg.num_experts,
                       num_ranks=cfg.num_ranks, quant_size=cfg.quant_size, round_scale=cfg.round_scale,
                       buffers=ref_bufs, layout_out=ref_lay, do_cpu_sync=True)
        n = ref_bufs.handle.num_recv_rows
        ref = _outputs(ref_bufs, ref_lay, n)
        # the no-allocation entry point; its buffers hold no workspace of their own
        bufs = ep.alloc_dispatch_buffers(T, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                                         cfg.expert_alignment, q, cfg.quant_size, device=dev)
        lay = _lay(cfg, T, dev)
        assert _call_noalloc(cfg, x, ti, tw, bufs, lay) == ep.EP_OK
        torch.cuda.synchronize()
        assert bufs.handle.read_error() == ep.EP_OK
        got = _outputs(bufs, lay, n)
        assert len(got) == len(ref)
        for g, r in zip(got, ref):
            assert torch.equal(g, r)


@pytest.mark.gpu
def test_noalloc_rows_feed_combine(cuda_device):
    dev = cuda_device
    cfg = CONFIGS["qwen3"].scaled(num_tokens=16 * 40, quant="none")
    x, ti, tw = _case(cfg, 3, dev)
    bufs = ep.alloc_dispatch_buffers(cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts,
                                     cfg.num_ranks, cfg.expert_alignment, None, device=dev)
    lay = _lay(cfg, cfg.num_tokens, dev)
    assert _call_noalloc(cfg, x, ti, tw, bufs, lay) == ep.EP_OK
    out = ep.ep_combine(bufs.recv_x, bufs.handle, tw)
    ref_rx, _, _, _, ref_h = ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, None, num_experts=cfg.num_experts,
                                            num_ranks=cfg.num_ranks)
    ref_out = ep.ep_combine(ref_rx.contiguous(), ref_h, tw)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # checked on the host before any CUDA call: no GPU needed
    T, K, E, R = 8 * 262144, 8, 1024, 8
    assert ep.workspace_bytes(T, K, E, R) > SCRATCH_BYTES
    opts = ep._Opts(1, 0, 0, 0, 1, 0, None, None, None)
    h = ep._Handle()
    p = C.c_void_p
    st = _noalloc()(p(None), T, 7168, p(None), p(None), K, E, R, C.byref(opts), p(None), p(None), p(None),
                    p(None), 0, C.byref(h), p(None), p(None), p(None), p(None))
    assert st == ep.EP_ERR_INVALID_ARG
