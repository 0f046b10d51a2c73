"""The routing kernel's bounded wait, made to run out on the GPU.

EP_TEST_STALL_BARRIER=1 raises the first grid barrier's target past the number
of CTAs, so no CTA can pass it: every CTA gives up after its 2 s limit, the
status word reports EP_ERR_TIMEOUT, the pack kernel packs nothing (the handle's
rows were never written), and the context stays usable -- the next call on the
same buffers is exact again.  No fault, trap or endless wait is involved.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

from gpu_parity import assert_rows_equal, assert_slots_equal, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("A", [1, 8])
def test_route_timeout_is_reported_and_the_context_survives(A, cuda_device, monkeypatch):
    cfg = CONFIGS["tiny"].scaled(expert_alignment=A)
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, cuda_device)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, device=cuda_device)
    bufs.recv_x.view(torch.uint8).fill_(0x5A)

    monkeypatch.setenv("EP_TEST_STALL_BARRIER", "1")
    t0 = time.time()
    ep.ep_dispatch(x, ti, tw, A, None, num_experts=E, num_ranks=R, buffers=bufs, do_cpu_sync=False)
    torch.cuda.synchronize()
    waited = time.time() - t0
    assert bufs.handle.read_error() == ep.EP_ERR_TIMEOUT
    assert 1.5 < waited < 60
    assert torch.all(bufs.recv_x.view(torch.uint8) == 0x5A)       # nothing was packed
    with pytest.raises(ep.EPError) as e:                            # the layout call reports it too
        ep.ep_get_dispatch_layout(ti, E, R)
    assert e.value.status == ep.EP_ERR_TIMEOUT

    monkeypatch.delenv("EP_TEST_STALL_BARRIER")
    recv_x, _, rti, rtw, h = ep.ep_dispatch(x, ti, tw, A, None, num_experts=E, num_ranks=R, buffers=bufs)
    assert h.read_error() == ep.EP_OK
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, E, R, A)
    assert_slots_equal(h, rti, rtw, ref)
    assert_rows_equal(cfg, recv_x, None, ref["recv_x"], None)
    assert np.array_equal(h.psum_num_recv_tokens_per_expert.cpu().numpy(), ref["psum_num_recv_tokens_per_expert"])
