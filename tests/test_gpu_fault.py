"""The routing kernel's bounded wait, made to run out on the GPU.

The test-only entry points of include/ep_testing.h raise the first grid
barrier's target past the number of CTAs, so no CTA can pass it: every CTA
gives up after its 2 s limit, the status word reports EP_ERR_TIMEOUT, the pack
kernel packs nothing (the handle's rows were never written), and the context
stays usable -- the next call on the same buffers is exact again.  No fault,
trap or endless wait is involved.  The product calls (ep_dispatch and the
layout call) take no switch of any kind into this path.
"""
import ctypes as C
import time

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

from gpu_parity import assert_rows_equal, assert_slots_equal, to_dev

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stalled_dispatch(x, ti, tw, A, E, R, bufs):
    f = ep._lib.ep_testing_dispatch_stalled
    p, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    f.argtypes = [p, i32, i32, p, p, i32, i32, i32, C.POINTER(ep._Opts), p, p, p, p, i64, C.POINTER(ep._Handle),
                  p, p, p, p, sz, p]
    f.restype = C.c_int
    T, H = x.shape
    K = ti.shape[1]
    opts = ep._Opts(A, 0, 0, 0, 1, 0, None, None, None)
    ch = bufs.handle._c()
    st = f(_ptr(x), T, H, _ptr(ti), _ptr(tw), K, E, R, C.byref(opts), _ptr(bufs.recv_x), None,
           _ptr(bufs.recv_topk_idx), _ptr(bufs.recv_topk_weights), bufs.recv_x.shape[0], C.byref(ch), None, None,
           None, _ptr(bufs.workspace), bufs.workspace.numel(), ep._stream(x.device))
    assert st == ep.EP_OK


def _stalled_layout(ti, E, R, ws, err):
    f = ep._lib.ep_testing_get_dispatch_layout_stalled
    p, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
    f.argtypes = [p, i32, i32, i32, i32, p, p, p, p, p, sz, p]
    f.restype = C.c_int
    T, K = ti.shape
    st = f(_ptr(ti), T, K, E, R, None, None, None, _ptr(err), _ptr(ws), ws.numel(), ep._stream(ti.device))
    assert st == ep.EP_OK


@pytest.mark.parametrize("A", [1, 8])
def test_route_timeout_is_reported_and_the_context_survives(A, cuda_device):
    cfg = CONFIGS["tiny"].scaled(expert_alignment=A)
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, cuda_device)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, device=cuda_device)
    bufs.recv_x.view(torch.uint8).fill_(0x5A)

    t0 = time.time()
    _stalled_dispatch(x, ti, tw, A, E, R, bufs)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert bufs.handle.read_error() == ep.EP_ERR_TIMEOUT
    assert 1.5 < waited < 60
    assert torch.all(bufs.recv_x.view(torch.uint8) == 0x5A)       # nothing was packed

    err = torch.zeros((1,), dtype=torch.int32, device=cuda_device)  # the layout call reports it too
    _stalled_layout(ti, E, R, bufs.workspace, err)
    torch.cuda.synchronize()
    assert int(err.item()) == ep.EP_ERR_TIMEOUT

    # the product calls on the same buffers are exact again
    recv_x, _, rti, rtw, h = ep.ep_dispatch(x, ti, tw, A, None, num_experts=E, num_ranks=R, buffers=bufs)
    assert h.read_error() == ep.EP_OK
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, E, R, A)
    assert_slots_equal(h, rti, rtw, ref)
    assert_rows_equal(cfg, recv_x, None, ref["recv_x"], None)
    assert np.array_equal(h.psum_num_recv_tokens_per_expert.cpu().numpy(), ref["psum_num_recv_tokens_per_expert"])
    ntpr, ntpe, _ = ep.ep_get_dispatch_layout(ti, E, R, workspace=bufs.workspace)
    lay = oracle.layout(wl.topk_idx, E, R)
    assert np.array_equal(ntpe.cpu().numpy(), lay["num_tokens_per_expert"])
    assert np.array_equal(ntpr.cpu().numpy(), lay["num_tokens_per_rank"])
