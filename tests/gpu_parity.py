"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle element by element.

Integer, index and byte outputs must match bit for bit; so must combine (both
sides accumulate fp32 fused multiply-adds in k order), although its contract
is 1e-2 relative, which ``assert_combine_close`` also checks.
"""
import numpy as np
import torch

import oracle
from combine_topk_idx_rank_b200 import ep


def to_dev(wl, dev):
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(dev)
    ti = torch.from_numpy(wl.topk_idx).to(dev)
    tw = torch.from_numpy(wl.topk_weights).to(dev)
    return x, ti, tw


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.uint8).cpu().numpy()


def gpu_dispatch(cfg, wl, dev, num_rounds=None, buffers=None, do_cpu_sync=True):
    x, ti, tw = to_dev(wl, dev)
    R, E = cfg.num_ranks, cfg.num_experts
    T = wl.topk_idx.shape[0]
    lay = (torch.empty(R, dtype=torch.int32, device=dev), torch.empty(E, dtype=torch.int32, device=dev),
           torch.empty((T, R), dtype=torch.bool, device=dev))
    res = ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, cfg.quant, num_experts=E, num_ranks=R,
                         quant_size=cfg.quant_size, round_scale=cfg.round_scale,
                         num_rounds=cfg.num_rounds if num_rounds is None else num_rounds,
                         buffers=buffers, layout_out=lay, do_cpu_sync=do_cpu_sync)
    return res, lay, (x, ti, tw)


def assert_layout_equal(lay, ref):
    ntpr, ntpe, itr = lay
    assert np.array_equal(ntpr.cpu().numpy(), ref["num_tokens_per_rank"])
    assert np.array_equal(ntpe.cpu().numpy(), ref["num_tokens_per_expert"])
    assert np.array_equal(itr.cpu().numpy(), ref["is_token_in_rank"])


def assert_slots_equal(h, rti, rtw, ref):
    n = ref["num_recv_rows"]
    assert h.num_recv_rows == n
    assert np.array_equal(h.psum_num_recv_tokens_per_expert.cpu().numpy(), ref["psum_num_recv_tokens_per_expert"])
    assert np.array_equal(h.num_recv_tokens_per_expert.cpu().numpy(), ref["num_recv_tokens_per_expert"])
    assert h.num_recv_tokens_per_expert_list == list(ref["num_recv_tokens_per_expert"])
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), ref["dst_buffer_slot_idx"])
    assert np.array_equal(h.recv_src_metadata[:n].cpu().numpy(), ref["recv_src_metadata"])
    assert np.array_equal(rti[:n].cpu().numpy(), ref["recv_topk_idx"])
    # weights are copies: compare bits
    assert np.array_equal(rtw[:n].cpu().numpy().view(np.uint32), ref["recv_topk_weights"].view(np.uint32))


def assert_rows_equal(cfg, recv_x, recv_scales, ref_x, ref_scales, rows=None):
    gx = u16(recv_x) if cfg.quant == "none" else u8(recv_x)
    if rows is not None:
        gx = gx[rows]
    assert gx.shape == ref_x.shape
    bad = np.nonzero((gx != ref_x).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:8]}"
    if cfg.quant != "none":
        gs = recv_scales.cpu().numpy()
        if rows is not None:
            gs = gs[rows]
        assert np.array_equal(gs.view(np.uint32), ref_scales.view(np.uint32))


def assert_combine_close(got_u16, ref_u16):
    """The combine contract: per token ||out - ref||_2 <= 1e-2 ||ref||_2 and per
    element |out - ref| <= 1e-2 (|ref| + mean |ref row|)."""
    g = (got_u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref_u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.linalg.norm(g - r, axis=1) <= 1e-2 * np.linalg.norm(r, axis=1) + 1e-30)
    assert np.all(np.abs(g - r) <= 1e-2 * (np.abs(r) + np.abs(r).mean(axis=1, keepdims=True)) + 1e-30)
