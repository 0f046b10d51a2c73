"""GPU parity of group-limited gating (the routing generator upstream of
dispatch, "DeepEP V1 vs V2 comparative analysis", section 8.1) against the
oracle, through the C ABI.

Expert ids are compared bit for bit.  Weights: both sides compute each weight
in binary64 (exp of the logit minus the largest, over the sum of the K terms
in output order), each to within a few units of 2^-52 relative, then round to
binary32; two binary64 values that close round to the same binary32 value or
to neighbours, so the bar is one binary32 ulp (and in practice every weight is
equal; the test also reports that).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_router_logits, make_workload

from gpu_parity import assert_rows_equal, assert_slots_equal, u16

pytestmark = pytest.mark.gpu


def run_gate(lg, n_group, topk_group, per_group, dev):
    t = torch.from_numpy(lg).to(dev)
    idx, w = ep.ep_group_limited_gating(t, n_group, topk_group, per_group)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def assert_gate_equal(lg, n_group, topk_group, per_group, dev):
    idx, w = run_gate(lg, n_group, topk_group, per_group, dev)
    ridx, rw = oracle.group_limited_gating(lg, n_group, topk_group, per_group)
    assert idx.dtype == np.int64 and idx.shape == ridx.shape
    assert np.array_equal(idx, ridx)
    assert np.all(np.abs(w.astype(np.float64) - rw) <= np.spacing(rw))
    return float(np.mean(w.view(np.uint32) == rw.view(np.uint32)))


@pytest.mark.parametrize("T", [2048, 32768])
def test_deepseek_v3_shapes(T, cuda_device):
    # decode (16 ranks x 128 tokens) and prefill (8 ranks x 4096 tokens): 256 experts, 32 groups of 8,
    # top-4 groups, top-2 per group
    for seed in (0, 1):
        lg = make_router_logits(T, 256, seed)
        assert assert_gate_equal(lg, 32, 4, 2, cuda_device) == 1.0


@pytest.mark.parametrize("E,n_group,topk_group,per_group,T", [
    (128, 8, 4, 2, 1003),      # ragged token count (not a multiple of 8 warps)
    (64, 1, 1, 8, 517),        # one group: plain top-8
    (36, 6, 3, 2, 300),        # groups of 6 (scalar loads)
    (1024, 32, 2, 8, 257),     # K = 16, groups of 32
    (256, 16, 16, 1, 64),      # every group kept, one expert each (K = 16)
    (96, 32, 5, 3, 129),       # every expert of a kept group
    (12, 3, 2, 2, 1),
])
def test_other_group_shapes(E, n_group, topk_group, per_group, T, cuda_device):
    lg = make_router_logits(T, E, seed=E + T)
    assert_gate_equal(lg, n_group, topk_group, per_group, cuda_device)


def test_ties(cuda_device):
    # logits on a coarse grid: many equal logits and equal group scores, which the
    # lower id must win on both sides; also +0 / -0
    lg = np.round(make_router_logits(4096, 256, seed=5) * 2) / 2
    lg[::3] = 0.0
    lg[1::7, ::2] = -0.0
    assert_gate_equal(lg.astype(np.float32), 32, 4, 2, cuda_device)
    # extreme finite values: group sums overflow to +inf and tie
    big = np.full((64, 256), 3.0e38, np.float32)
    big[:, ::5] = -3.0e38
    assert_gate_equal(big, 32, 4, 2, cuda_device)


def test_no_tokens(cuda_device):
    idx, w = run_gate(np.zeros((0, 256), np.float32), 32, 4, 2, cuda_device)
    assert idx.shape == (0, 8) and w.shape == (0, 8)


def test_nonfinite_logits_are_reported(cuda_device):
    for bad in (np.nan, np.inf, -np.inf):
        lg = make_router_logits(300, 256, seed=7)
        lg[17, 3] = bad
        lg[250, 200] = bad
        t = torch.from_numpy(lg).to(cuda_device)
        with pytest.raises(ep.EPError) as e:
            ep.ep_group_limited_gating(t, 32, 4, 2)
        assert e.value.status == ep.EP_ERR_NONFINITE
        idx, _ = ep.ep_group_limited_gating(t, 32, 4, 2, check=False)
        idx = idx.cpu().numpy()
        assert idx.min() >= 0 and idx.max() < 256            # still in range and distinct
        assert all(len(set(r.tolist())) == 8 for r in idx)
    # the next call on finite logits is clean
    assert_gate_equal(make_router_logits(64, 256, 8), 32, 4, 2, cuda_device)


def test_host_validation(cuda_device):
    t = torch.zeros((4, 256), dtype=torch.float32, device=cuda_device)
    for args in ((3, 1, 1), (64, 4, 2), (32, 33, 1), (32, 4, 9), (32, 4, 0), (8, 8, 3)):
        with pytest.raises(ep.EPError) as e:
            ep.ep_group_limited_gating(t, *args)
        assert e.value.status == ep.EP_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_gating_feeds_dispatch_and_combine(name, cuda_device):
    """Gating -> dispatch -> combine on the device equals the oracle's gating ->
    dispatch -> combine, bit for bit (DeepSeek-V3 shapes, smaller token count
    and hidden size)."""
    cfg = CONFIGS[name].scaled(num_tokens=CONFIGS[name].num_ranks * 64, hidden=1024)
    wl = make_workload(cfg, seed=2)
    lg = make_router_logits(cfg.num_tokens, cfg.num_experts, seed=2)
    ridx, rw = oracle.group_limited_gating(lg, 32, 4, 2)
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    ti, tw = ep.ep_group_limited_gating(torch.from_numpy(lg).to(cuda_device))
    E, R = cfg.num_experts, cfg.num_ranks
    recv_x, recv_s, rti, rtw, h = ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, cfg.quant, num_experts=E,
                                                 num_ranks=R, quant_size=cfg.quant_size, round_scale=cfg.round_scale)
    y = recv_x if cfg.quant == "none" else None
    out = ep.ep_combine(y, h, tw) if y is not None else ep.ep_combine(recv_x, h, tw, y_scales=recv_s,
                                                                      quant_size=cfg.quant_size)
    torch.cuda.synchronize()
    ref = oracle.dispatch(wl.x, ridx, rw, E, R, cfg.expert_alignment, cfg.quant, cfg.quant_size, cfg.round_scale)
    assert_slots_equal(h, rti, rtw, ref)
    assert_rows_equal(cfg, recv_x, recv_s, ref["recv_x"], ref["recv_scales"])
    if cfg.quant == "none":
        ref_out = oracle.combine_rows(ref["recv_x"], ref["dst_buffer_slot_idx"], rw)
    else:
        ref_out = oracle.combine_rows_q(ref["recv_x"], ref["recv_scales"], cfg.quant, cfg.quant_size,
                                        ref["dst_buffer_slot_idx"], rw)
    assert np.array_equal(u16(out), ref_out)
