"""Dispatch and combine captured in a CUDA graph (GPU).

A step -- the routing kernel's memset and cooperative launch, the pack and
combine kernels with their programmatic dependent launches -- is captured
once and replayed on new inputs copied into the captured buffers; every
replay must give exactly what eager calls give on the same inputs.
"""
import numpy as np
import pytest
import torch

from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

from gpu_parity import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["decode", "qwen3", "prefill"])
def test_step_replays_from_a_cuda_graph(name, cuda_device):
    dev = cuda_device
    cfg = CONFIGS[name].scaled(num_tokens={"decode": 16 * 40, "qwen3": 16 * 40, "prefill": 8 * 136}[name],
                               hidden=1024)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    q = None if cfg.quant == "none" else cfg.quant
    x, ti, tw = to_dev(make_workload(cfg, 0), dev)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, q, cfg.quant_size, device=dev)
    y = torch.randn((bufs.recv_x.shape[0], H), device=dev, dtype=torch.bfloat16,
                    generator=torch.Generator(device=dev).manual_seed(3))
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    kw = dict(num_experts=E, num_ranks=R, quant_size=cfg.quant_size, round_scale=cfg.round_scale, buffers=bufs,
              do_cpu_sync=False)

    def step():
        ep.ep_dispatch(x, ti, tw, A, q, **kw)
        ep.ep_combine(y, bufs.handle, tw, out=out)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()                                   # warm-up outside the capture
    torch.cuda.current_stream(dev).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (1, 2):
        x2, ti2, tw2 = to_dev(make_workload(cfg, seed), dev)
        x.copy_(x2), ti.copy_(ti2), tw.copy_(tw2)
        out.fill_(0)
        g.replay()
        torch.cuda.synchronize()
        assert bufs.handle.read_error() == ep.EP_OK
        got_out, got_rows = out.clone(), bufs.recv_x.clone()
        got_slots = bufs.handle.dst_buffer_slot_idx.clone()
        step()                                   # eager, same inputs
        torch.cuda.synchronize()
        assert torch.equal(got_slots, bufs.handle.dst_buffer_slot_idx)
        assert torch.equal(got_rows.view(torch.uint8), bufs.recv_x.view(torch.uint8))
        assert torch.equal(got_out.view(torch.int16), out.view(torch.int16))
