"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Sizes the oracle finishes in seconds that still span several 128-token chunks
and a ragged last chunk, on every workload shape, seeds 0-2; plus the edge
cases (no tokens, all entries masked, K=1, one expert per rank, minimum
hidden, duplicate ids, group sizes 16..512, per-token FP8, power-of-two int8
scales).  Bit-exact for layout, slots, metadata, rows, codes and scales;
combine is bit-exact too and also meets the 1e-2 relative contract.
"""
import copy

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y

from gpu_parity import (assert_combine_close, assert_layout_equal, assert_rows_equal, assert_slots_equal,
                        gpu_dispatch, to_dev, u8, u16)

pytestmark = pytest.mark.gpu


def _small(name):
    cfg = CONFIGS[name]
    R = cfg.num_ranks
    # a token count that is a multiple of R (and of the rounds) but not of 128
    T = {"tiny": 256, "decode": 16 * 40, "prefill": 8 * 136, "qwen3": 16 * 40, "longseq": 8 * 8 * 17}[name]
    H = {"tiny": 512, "decode": 1024, "prefill": 1536, "qwen3": 2048, "longseq": 1024}[name]
    return cfg.scaled(num_tokens=T, hidden=H)


def run_and_compare(cfg, seed, dev, num_rounds=None):
    wl = make_workload(cfg, seed)
    (recv_x, recv_scales, rti, rtw, h), lay, (x, ti, tw) = gpu_dispatch(cfg, wl, dev, num_rounds)
    ref_lay = oracle.layout(wl.topk_idx, cfg.num_experts, cfg.num_ranks)
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks,
                          cfg.expert_alignment, cfg.quant, cfg.quant_size, cfg.round_scale,
                          cfg.num_rounds if num_rounds is None else num_rounds)
    assert_layout_equal(lay, ref_lay)
    assert_slots_equal(h, rti, rtw, ref)
    assert_rows_equal(cfg, recv_x, recv_scales, ref["recv_x"], ref["recv_scales"])
    # combine over expert outputs y (bf16, received-row order)
    y_np = make_y(ref["num_recv_rows"], cfg.hidden, seed)
    y = torch.from_numpy(y_np.view(np.int16)).view(torch.bfloat16).to(dev)
    out = ep.ep_combine(y, h, tw)
    torch.cuda.synchronize()
    h.check()
    ref_out = oracle.combine(y_np, ref["dst_buffer_slot_idx"], wl.topk_weights, cfg.num_ranks,
                             cfg.num_rounds if num_rounds is None else num_rounds)
    got = u16(out)
    assert_combine_close(got, ref_out)
    assert np.array_equal(got, ref_out)
    return wl, ref, h


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("name", list(CONFIGS))
def test_parity_small(name, seed, cuda_device):
    run_and_compare(_small(name), seed, cuda_device)


def test_identity_expert_round_trip(cuda_device):
    cfg = _small("prefill")
    wl = make_workload(cfg, 0)
    (recv_x, _, _, _, h), _, (x, ti, tw) = gpu_dispatch(cfg, wl, cuda_device)
    out = ep.ep_combine(recv_x.contiguous(), h, tw).float()
    wsum = torch.where(ti >= 0, tw, torch.zeros_like(tw)).double().sum(1, keepdim=True)
    ref = x.double() * wsum
    assert torch.all((out.double() - ref).abs() <= 2.0 ** -8 * ref.abs() + 1e-30)


def test_rounds_match_one_shot_on_gpu(cuda_device):
    cfg = _small("longseq")
    wl = make_workload(cfg, 1)
    a, _, _ = gpu_dispatch(cfg, wl, cuda_device, num_rounds=1)
    a = [t.clone() if t is not None else None for t in a[:4]]
    b, _, _ = gpu_dispatch(cfg, wl, cuda_device, num_rounds=8)
    for u, v in zip(a, b[:4]):
        if u is not None:
            assert torch.equal(u.view(torch.uint8), v.view(torch.uint8))


def test_deterministic_repeat(cuda_device):
    cfg = _small("qwen3")
    wl = make_workload(cfg, 2)
    a, _, _ = gpu_dispatch(cfg, wl, cuda_device)
    a = [t.clone() for t in a[:4]]
    b, _, _ = gpu_dispatch(cfg, wl, cuda_device)
    for u, v in zip(a, b[:4]):
        assert torch.equal(u.view(torch.uint8), v.view(torch.uint8))


@pytest.mark.parametrize("quant,qs,rs", [("fp8", 16, False), ("fp8", 32, True), ("fp8", 64, False),
                                         ("fp8", 256, True), ("fp8", 512, False), ("fp8", 1024, False),
                                         ("fp8", 1024, True), ("int8", 128, False), ("int8", 128, True),
                                         ("int8", 1024, True), ("int8", 512, False)])
def test_quant_variants(quant, qs, rs, cuda_device):
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 9, hidden=1024, quant=quant, quant_size=qs,
                                   round_scale=rs, expert_alignment=4)
    run_and_compare(cfg, 0, cuda_device)


@pytest.mark.parametrize("quant,qs,H", [("fp8", 128, 16384), ("int8", 64, 24576), ("mxfp4", 32, 16384),
                                        ("fp8", 512, 40960)])
def test_group_quant_rows_of_several_passes(quant, qs, H, cuda_device):
    """Group quantisation of rows longer than one pass of the group kernel
    (512 threads x 16 channels = 8192 channels): 2, 3 and 5 passes per row,
    with padding rows."""
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 3, hidden=H, quant=quant, quant_size=qs, expert_alignment=4)
    if quant != "mxfp4":
        run_and_compare(cfg, 1, cuda_device)
        return
    wl = make_workload(cfg, 1)
    x, ti, tw = to_dev(wl, cuda_device)
    recv_x, recv_scales, _, _, h = ep.ep_dispatch(x, ti, tw, 4, quant, num_experts=cfg.num_experts,
                                                  num_ranks=cfg.num_ranks, quant_size=qs)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 4)
    n = s["num_recv_rows"]
    ref_x, ref_s = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], quant, qs, num_rows=n)
    assert np.array_equal(recv_x.contiguous().view(torch.uint8).cpu().numpy().reshape(n, -1), ref_x)
    assert np.array_equal(recv_scales.contiguous().cpu().numpy(), ref_s)


@pytest.mark.parametrize("quant,H", [("int8", 16384), ("fp8", 24576), ("int8", 65536)])
def test_per_token_quant_large_hidden(quant, H, cuda_device):
    """Per-token quantisation of long rows: up to 1024 units of 16 channels
    run two units per thread in blocks of up to 512, up to 2048 in blocks of
    1024, longer rows four units per thread."""
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 3, hidden=H, quant=quant, quant_size=H, expert_alignment=4)
    run_and_compare(cfg, 0, cuda_device)


def test_edge_shapes(cuda_device):
    base = CONFIGS["tiny"]
    cases = [
        base.scaled(num_tokens=8, num_topk=1),                               # K = 1
        base.scaled(num_tokens=8 * 33, num_experts=8, num_topk=3),           # one expert per rank
        base.scaled(num_tokens=8 * 20, hidden=8),                            # minimum hidden
        base.scaled(num_tokens=8 * 50, hidden=8 * 7, expert_alignment=64),   # hidden not a power of 2
        base.scaled(num_tokens=4 * 64, num_ranks=4, num_experts=1024, num_topk=16, hidden=64,
                    expert_alignment=3),                                      # largest E and K
        base.scaled(num_tokens=256 * 2, num_ranks=256, num_experts=256, num_topk=4, hidden=64),  # R = 256
        base.scaled(num_tokens=8 * 12, hidden=12000, expert_alignment=5),    # rows of 2 bulk chunks
        base.scaled(num_tokens=8 * 6, hidden=20008),                          # 3 unequal bulk chunks
        base.scaled(num_tokens=8 * 2, hidden=65536, num_topk=3),              # largest hidden
    ]
    for cfg in cases:
        run_and_compare(cfg, 0, cuda_device)


@pytest.mark.parametrize("quant,qs", [("none", 128), ("fp8", 128), ("mxfp4", 32)])
def test_no_tokens(quant, qs, cuda_device):
    # with no tokens and alignment 1 the receive capacity is zero: empty outputs, no scales array needed
    cfg = CONFIGS["prefill"].scaled(num_tokens=0, hidden=256, quant=quant, quant_size=qs,
                                    expert_alignment=1 if quant != "none" else 128)
    wl = make_workload(cfg, 0)
    (recv_x, _, rti, rtw, h), lay, _ = gpu_dispatch(cfg, wl, cuda_device)
    assert h.num_recv_rows == 0
    assert torch.all(h.psum_num_recv_tokens_per_expert == 0)
    assert torch.all(lay[0] == 0) and torch.all(lay[1] == 0)


def test_more_chunks_than_resident_ctas(cuda_device):
    """8 ranks x 16384 tokens: 512 routing chunks of 256 tokens, more than the
    cooperative grid holds at once (3 CTAs per SM), so each CTA routes several
    chunks and phase 3 reloads their ids and ranks from global memory; normal
    and low-latency layouts, hidden 64 to keep the rows small."""
    cfg = CONFIGS["prefill"].scaled(num_tokens=8 * 16384, hidden=64, expert_alignment=16)
    wl, _, _ = run_and_compare(cfg, 6, cuda_device)
    x, ti, tw = to_dev(wl, cuda_device)
    T, E, R = cfg.num_tokens, cfg.num_experts, cfg.num_ranks
    M = T // R
    _, _, count, layout_range, h = ep.ep_dispatch_low_latency(x, ti, tw, M, E, R)
    torch.cuda.synchronize()
    h.check()
    ref = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), ref["dst_buffer_slot_idx"])
    assert np.array_equal(count.cpu().numpy(), ref["recv_count"])
    assert np.array_equal(layout_range.cpu().numpy(), ref["layout_range"])


def test_all_masked_and_duplicates(cuda_device):
    cfg = CONFIGS["tiny"].scaled(num_tokens=8 * 30, expert_alignment=4)
    wl = make_workload(cfg, 0)
    wl.topk_idx[:] = -1
    wl.topk_weights[:] = 0
    wl.topk_idx[3] = [5, 5]          # duplicate ids in one row: each (t, k) gets a row
    wl.topk_weights[3] = [0.25, 0.75]
    (recv_x, _, rti, rtw, h), lay, (x, ti, tw) = gpu_dispatch(cfg, wl, cuda_device)
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 4)
    assert_slots_equal(h, rti, rtw, ref)
    assert_rows_equal(cfg, recv_x, None, ref["recv_x"], None)
    out = ep.ep_combine(recv_x.contiguous(), h, tw)
    ref_out = oracle.combine_rows(ref["recv_x"], ref["dst_buffer_slot_idx"], wl.topk_weights)
    assert np.array_equal(u16(out), ref_out)
    assert np.all(ref_out[np.arange(ref_out.shape[0]) != 3] == 0)


def test_e4m3_and_int8_conversion_exhaustive_over_bf16(cuda_device):
    """Every bf16 value |v| <= 448 goes through the FP8 path with its group's
    scale pinned to exactly 1 (each group holds 448), and every |v| <= 127
    through the int8 path with scale 1 (each group holds 127)."""
    for quant, top in (("fp8", 448.0), ("int8", 127.0)):
        allv = (np.arange(0, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
        v = allv[allv <= top]
        v = np.concatenate([v, -v]).astype(np.float32)
        per = 127
        ngroups = -(-v.size // per)
        v = np.concatenate([v, np.zeros(ngroups * per - v.size, np.float32)]).reshape(ngroups, per)
        g = np.concatenate([np.full((ngroups, 1), top, np.float32), v], axis=1)   # [ngroups, 128]
        H = 1024
        R = 8
        T = -(-ngroups * 128 // H)
        T = -(-T // R) * R
        flat = np.zeros(T * H, np.float32)
        flat[:g.size] = g.ravel()
        flat[g.size:] = top
        cfg = CONFIGS["tiny"].scaled(num_tokens=T, hidden=H, quant=quant, quant_size=128)
        wl = make_workload(cfg, 0)
        wl.x = torch.from_numpy(flat.reshape(T, H)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        (recv_x, recv_scales, rti, rtw, h), _, _ = gpu_dispatch(cfg, wl, cuda_device)
        ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1,
                              quant, 128, False)
        assert np.all(ref["recv_scales"] == 1.0)
        assert_rows_equal(cfg, recv_x, recv_scales, ref["recv_x"], ref["recv_scales"])


def _groups_over_every_scale(seed):
    """One 128-channel group per finite positive bf16 group maximum A (all
    32640 of them, subnormal and huge included): channel 0 holds A, so the
    group's scale is max(A, 1e-4) / qmax, and channels 1..127 hold x values
    with |x| <= A -- 64 significands at A's exponent, 32 one binade lower, 24
    at random lower exponents (down into the fp32 subnormals), zeros, and the
    smallest bf16 subnormal -- with random signs."""
    rng = np.random.default_rng(seed)
    amax = np.arange(1, 0x7f80, dtype=np.uint32)                      # bf16 bit patterns, +0 excluded
    G = amax.size
    e = (amax >> 7).astype(np.int64)                                  # exponent field (0: subnormal)
    xs = np.zeros((G, 127), np.int64)
    sig = rng.integers(0, 128, (G, 120))
    expo = np.empty((G, 120), np.int64)
    expo[:, :64] = e[:, None]
    expo[:, 64:96] = np.maximum(e[:, None] - 1, 0)
    expo[:, 96:] = (rng.random((G, 24)) * (e[:, None] + 1)).astype(np.int64)
    xs[:, :120] = (expo << 7) | sig
    xs[:, 120:124] = 0
    xs[:, 124:] = 1                                                   # smallest subnormal
    xs = np.minimum(xs, amax[:, None].astype(np.int64))               # keep |x| <= A
    xs |= (rng.random((G, 127)) < 0.5).astype(np.int64) << 15         # signs
    g = np.concatenate([amax[:, None].astype(np.int64), xs], axis=1).astype(np.uint16)
    return g                                                          # [G, 128] bf16 bits


@pytest.mark.parametrize("quant", ["fp8", "int8"])
def test_quotients_over_every_group_scale(quant, cuda_device):
    """Every scale a 128-group can have, each against a spread of x values:
    codes and scales bit for bit against the oracle's IEEE fp32 division."""
    g = _groups_over_every_scale(11 if quant == "fp8" else 12)
    H, R = 1024, 8
    per = H // 128
    T = -(-g.shape[0] // per)
    T = -(-T // R) * R
    flat = np.zeros((T * per, 128), np.uint16)
    flat[:g.shape[0]] = g
    cfg = CONFIGS["tiny"].scaled(num_tokens=T, hidden=H, quant=quant, quant_size=128)
    wl = make_workload(cfg, 0)
    wl.x = flat.reshape(T, H)
    (recv_x, recv_scales, _, _, h), _, _ = gpu_dispatch(cfg, wl, cuda_device)
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 1, quant, 128, False)
    assert_rows_equal(cfg, recv_x, recv_scales, ref["recv_x"], ref["recv_scales"])


def test_bad_expert_id_sets_status(cuda_device):
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg, 0)
    wl.topk_idx[17, 1] = cfg.num_experts          # out of range
    (recv_x, _, _, _, h), _, _ = gpu_dispatch(cfg, wl, cuda_device, do_cpu_sync=False)
    torch.cuda.synchronize()
    assert h.read_error() == ep.EP_ERR_BAD_EXPERT_ID
    wl.topk_idx[17, 1] = -5
    (_, _, _, _, h), _, _ = gpu_dispatch(cfg, wl, cuda_device, do_cpu_sync=False)
    assert h.read_error() == ep.EP_ERR_BAD_EXPERT_ID
    with pytest.raises(ep.EPError):
        gpu_dispatch(cfg, wl, cuda_device, do_cpu_sync=True)
    # the layout call reports it too
    _, ti, _ = to_dev(wl, cuda_device)
    with pytest.raises(ep.EPError) as e:
        ep.ep_get_dispatch_layout(ti, cfg.num_experts, cfg.num_ranks)
    assert e.value.status == ep.EP_ERR_BAD_EXPERT_ID


def test_capacity_overflow_sets_status_and_writes_nothing_past_it(cuda_device):
    cfg = CONFIGS["tiny"].scaled(expert_alignment=8)
    wl = make_workload(cfg, 0)
    ref = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 8)
    need = ref["num_recv_rows"]
    cap = need - 50
    full = ep.alloc_dispatch_buffers(cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts,
                                     cfg.num_ranks, 8, recv_capacity=need + 64, device=cuda_device)
    for t in (full.recv_x, full.recv_topk_idx, full.recv_topk_weights, full.handle.recv_src_metadata):
        t.view(torch.uint8).fill_(0xA5)
    short = ep.DispatchBuffers(full.recv_x[:cap], None, full.recv_topk_idx[:cap], full.recv_topk_weights[:cap],
                               full.handle, full.workspace, None, 128)
    (_, _, _, _, h), _, _ = gpu_dispatch(cfg, wl, cuda_device, buffers=short, do_cpu_sync=False)
    torch.cuda.synchronize()
    assert h.read_error() == ep.EP_ERR_CAPACITY
    for t in (full.recv_x, full.recv_topk_idx, full.recv_topk_weights, full.handle.recv_src_metadata):
        assert torch.all(t[cap:].contiguous().view(torch.uint8) == 0xA5)


def test_layout_call_matches_oracle(cuda_device):
    for name in CONFIGS:
        cfg = _small(name)
        wl = make_workload(cfg, 5)
        _, ti, _ = to_dev(wl, cuda_device)
        got = ep.ep_get_dispatch_layout(ti, cfg.num_experts, cfg.num_ranks)
        assert_layout_equal(got, oracle.layout(wl.topk_idx, cfg.num_experts, cfg.num_ranks))


def test_cumulative_stats_accumulate(cuda_device):
    cfg = _small("decode")
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, cuda_device)
    stats = torch.zeros(cfg.num_experts, dtype=torch.int32, device=cuda_device)
    for _ in range(3):
        ep.ep_dispatch(x, ti, tw, 1, "fp8", num_experts=cfg.num_experts, num_ranks=cfg.num_ranks,
                       cumulative_local_expert_recv_stats=stats, do_cpu_sync=False)
    ref = oracle.layout(wl.topk_idx, cfg.num_experts, cfg.num_ranks)["num_tokens_per_expert"]
    assert np.array_equal(stats.cpu().numpy(), 3 * ref)


@pytest.mark.parametrize("name", ["prefill", "decode", "qwen3", "longseq"])
def test_cached_dispatch_repacks_new_rows(name, cuda_device):
    """Cached dispatch (handle reuse): new x, routing from the handle; the rows
    equal the oracle's rows of the new x at the cached slots, padding zeroed."""
    cfg = _small(name)
    wl = make_workload(cfg, 0)
    (_, _, _, _, h), _, (x, ti, tw) = gpu_dispatch(cfg, wl, cuda_device)
    rows = h.num_recv_rows
    wl2 = make_workload(cfg, 1)           # a later step: new activations, same routing
    x2 = torch.from_numpy(wl2.x.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    q = None if cfg.quant == "none" else cfg.quant
    bufs = ep.alloc_dispatch_buffers(cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                                     cfg.expert_alignment, q, cfg.quant_size, cfg.num_rounds, h.recv_capacity,
                                     cuda_device)
    bufs.recv_x.view(torch.uint8).fill_(0x5A)              # stale contents must not survive
    if bufs.recv_scales is not None:
        bufs.recv_scales.fill_(7.0)
    rx, rs, rti, rtw, h2 = ep.ep_dispatch(x2, quant=q, quant_size=cfg.quant_size, round_scale=cfg.round_scale,
                                          num_rounds=cfg.num_rounds, buffers=bufs, handle=h)
    torch.cuda.synchronize()
    h.check()
    assert rti is None and rtw is None and h2 is h and rx.shape[0] == rows
    slots = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, cfg.expert_alignment)
    assert slots["num_recv_rows"] == rows
    ref_x, ref_s = oracle.dispatch_rows(wl2.x, slots["dst_buffer_slot_idx"], cfg.quant, cfg.quant_size,
                                        cfg.round_scale, num_rows=rows)
    assert_rows_equal(cfg, rx, rs, ref_x, ref_s)


@pytest.mark.parametrize("quant,qs", [(None, 128), ("fp8", 128), ("int8", 512)])
def test_pack_skips_and_reports_rows_past_capacity(quant, qs, cuda_device):
    """The pack kernels write no row at or past recv_capacity, whatever the
    handle's dst_buffer_slot_idx holds: such entries are skipped and reported
    as EP_ERR_CAPACITY, the others are packed as usual (bulk bf16, group and
    per-token quantisation)."""
    cfg = CONFIGS["tiny"].scaled(hidden=512)
    wl = make_workload(cfg, 4)
    x, ti, tw = to_dev(wl, cuda_device)
    (_, _, _, _, h), _, _ = gpu_dispatch(cfg, wl, cuda_device)
    need = h.num_recv_rows
    full = ep.alloc_dispatch_buffers(cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                                     1, quant, qs, recv_capacity=need + 64, device=cuda_device)
    full.recv_x.view(torch.uint8).fill_(0x5A)
    cut = need - 8                           # rows cut..need-1 now lie past the capacity
    h2 = copy.copy(h)
    h2.recv_capacity = cut
    h2.err = torch.zeros_like(h.err)
    slots = h.dst_buffer_slot_idx.clone()
    slots[5, 0] = cut + 40                   # and a few more, inside the guard rows
    slots[9, 1] = cut + 63
    h2.dst_buffer_slot_idx = slots
    rs = None if full.recv_scales is None else full.recv_scales[:cut]
    short = ep.DispatchBuffers(full.recv_x[:cut], rs, full.recv_topk_idx, full.recv_topk_weights, h2,
                               full.workspace, quant, qs)
    ep.ep_dispatch(x, quant=quant, quant_size=qs, buffers=short, handle=h2)
    torch.cuda.synchronize()
    assert h2.read_error() == ep.EP_ERR_CAPACITY
    assert torch.all(full.recv_x[cut:].contiguous().view(torch.uint8) == 0x5A)
    dst = slots.cpu().numpy()
    ref_x, ref_s = oracle.dispatch_rows(wl.x, np.where(dst < cut, dst, -1), quant or "none", qs, False,
                                        num_rows=cut)
    got = u16(full.recv_x[:cut]) if quant is None else u8(full.recv_x[:cut]).reshape(cut, -1)
    written = np.unique(dst[(dst >= 0) & (dst < cut)])
    assert np.array_equal(got[written], ref_x[written])
    if quant is not None:
        assert np.array_equal(rs.cpu().numpy()[written].view(np.uint32), ref_s[written].view(np.uint32))


def test_cached_dispatch_rejects_routing_args(cuda_device):
    cfg = CONFIGS["tiny"]
    wl = make_workload(cfg, 0)
    (_, _, _, _, h), _, (x, ti, tw) = gpu_dispatch(cfg, wl, cuda_device)
    with pytest.raises(ValueError):
        ep.ep_dispatch(x, ti, tw, handle=h)


@pytest.mark.parametrize("quant,qs,rs,ue8", [("mxfp4", 32, False, False), ("fp8", 128, True, True),
                                             ("int8", 1024, True, True), ("fp8", 1024, True, True),
                                             ("int8", 64, True, True)])
def test_mxfp4_and_ue8m0_scale_bytes(quant, qs, rs, ue8, cuda_device):
    """MXFP4 (use_mxfp4, groups of 32) and UE8M0 scale bytes (use_ue8m0),
    bit for bit against the oracle, padding rows included."""
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 9, hidden=1024, quant=quant, quant_size=qs, round_scale=rs,
                                   expert_alignment=4)
    wl = make_workload(cfg, 0)
    x, ti, tw = to_dev(wl, cuda_device)
    recv_x, recv_scales, _, _, h = ep.ep_dispatch(x, ti, tw, 4, quant, num_experts=cfg.num_experts,
                                                  num_ranks=cfg.num_ranks, quant_size=qs, round_scale=rs,
                                                  scale_ue8m0=ue8)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, 4)
    n = s["num_recv_rows"]
    assert h.num_recv_rows == n
    ref_x, ref_s = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], quant, qs, rs, ue8, num_rows=n)
    got_x = recv_x.contiguous().view(torch.uint8).cpu().numpy().reshape(n, -1)
    assert np.array_equal(got_x, ref_x)
    got_s = recv_scales.contiguous().cpu().numpy()
    assert got_s.dtype == ref_s.dtype
    assert np.array_equal(got_s.view(np.uint8), ref_s.view(np.uint8))


def test_e2m1_conversion_over_bf16(cuda_device):
    """Every bf16 value |v| <= 6 through the MXFP4 path with the group scale
    pinned to 1 (each 32-group also holds 4.0, so floor(log2 amax) - 2 = 0)."""
    allv = (np.arange(0, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
    v = allv[allv <= 6.0]
    v = np.concatenate([v, -v]).astype(np.float32)
    per = 31
    ng = -(-v.size // per)
    v = np.concatenate([v, np.zeros(ng * per - v.size, np.float32)]).reshape(ng, per)
    g = np.concatenate([np.full((ng, 1), 4.0, np.float32), v], axis=1)
    H, R = 1024, 8
    T = -(-(-(-ng * 32 // H)) // R) * R
    flat = np.full(T * H, 4.0, np.float32)
    flat[:g.size] = g.ravel()
    cfg = CONFIGS["tiny"].scaled(num_tokens=T, hidden=H, quant="mxfp4", quant_size=32)
    wl = make_workload(cfg, 0)
    wl.x = torch.from_numpy(flat.reshape(T, H)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    x, ti, tw = to_dev(wl, cuda_device)
    recv_x, recv_scales, _, _, h = ep.ep_dispatch(x, ti, tw, 1, "mxfp4", num_experts=cfg.num_experts,
                                                  num_ranks=cfg.num_ranks, quant_size=32)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks)
    ref_x, ref_s = oracle.dispatch_rows_mx(wl.x, s["dst_buffer_slot_idx"], "mxfp4", 32,
                                           num_rows=s["num_recv_rows"])
    assert np.all(ref_s == 127)
    assert np.array_equal(recv_x.cpu().numpy(), ref_x)
    assert np.array_equal(recv_scales.cpu().numpy(), ref_s)


def _offset_workspace(nbytes, off, dev):
    """A workspace of nbytes starting `off` bytes into a larger allocation."""
    big = torch.empty((nbytes + 256,), dtype=torch.uint8, device=dev)
    return big[off:off + nbytes]


@pytest.mark.parametrize("name", ["decode", "prefill", "qwen3"])
def test_routing_forms_agree(name, cuda_device):
    """The folded routing form (the per-chunk tables copied whole into shared
    memory after one grid barrier) and the three-phase form (column prefixes
    in the workspace, a second barrier) give the same bits.  The folded form
    needs its workspace tables 16-byte aligned, so a workspace that starts 4
    bytes into an allocation takes the three-phase form on the same shape."""
    dev = cuda_device
    cfg = _small(name)
    T, H, K, E, R, A = (cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks,
                        cfg.expert_alignment)
    q = None if cfg.quant == "none" else cfg.quant
    wl = make_workload(cfg, 3)
    ref = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, E, R, A, cfg.quant, cfg.quant_size, cfg.round_scale,
                          cfg.num_rounds)
    ref_lay = oracle.layout(wl.topk_idx, E, R)
    got = []
    for off in (0, 4):
        bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, A, q, cfg.quant_size, cfg.num_rounds, device=dev)
        bufs.workspace = _offset_workspace(bufs.workspace.numel(), off, dev)
        (recv_x, recv_scales, rti, rtw, h), lay, _ = gpu_dispatch(cfg, wl, dev, buffers=bufs)
        assert_layout_equal(lay, ref_lay)
        assert_slots_equal(h, rti, rtw, ref)
        assert_rows_equal(cfg, recv_x, recv_scales, ref["recv_x"], ref["recv_scales"])
        n = h.num_recv_rows
        got.append([u8(recv_x[:n]), h.dst_buffer_slot_idx.cpu().numpy(), h.recv_src_metadata[:n].cpu().numpy()])
    for a, b in zip(*got):
        assert np.array_equal(a, b)


def test_low_latency_routing_forms_agree(cuda_device):
    """The same for the low-latency layout, whose positions count from each
    source rank's first chunk."""
    dev = cuda_device
    cfg = CONFIGS["decode"].scaled(num_tokens=16 * 40, hidden=1024)
    wl = make_workload(cfg, 4)
    T, K, E, R, M = cfg.num_tokens, cfg.num_topk, cfg.num_experts, cfg.num_ranks, 48
    ref = oracle.ll_slots(wl.topk_idx, wl.topk_weights, E, R, M)
    x, ti, tw = to_dev(wl, dev)
    got = []
    for off in (0, 4):
        ws = _offset_workspace(ep.workspace_bytes(T, K, E, R), off, dev)
        recv_x, recv_scales, count, layout_range, h = ep.ep_dispatch_low_latency(
            x, ti, tw, M, E, R, "fp8", quant_size=128, workspace=ws)
        torch.cuda.synchronize()
        assert h.read_error() == ep.EP_OK
        assert np.array_equal(h.dst_buffer_slot_idx.cpu().numpy(), ref["dst_buffer_slot_idx"])
        assert np.array_equal(count.cpu().numpy(), ref["recv_count"])
        assert np.array_equal(layout_range.cpu().numpy(), ref["layout_range"])
        # the rows that received an entry (the others of the fixed-capacity layout are never written)
        dst = ref["dst_buffer_slot_idx"]
        used = np.unique(dst[dst >= 0])
        rows = E * R * M
        got.append([u8(recv_x).reshape(rows, -1)[used],
                    recv_scales.reshape(rows, -1).cpu().numpy().view(np.uint32)[used]])
    for a, b in zip(*got):
        assert np.array_equal(a, b)
