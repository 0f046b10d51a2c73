"""Every (bf16 value, bf16 group maximum) pair through the quantising pack.

The group kernels divide x by the group's scale s = max(amax, 1e-4) / 448
(FP8) or / 127 (int8) with a corrected reciprocal product (Markstein's
theorem on division with a fused multiply-add, IBM J. Res. Develop. 34(1),
1990) instead of the IEEE division, guarded against underflow.  The codes must
be those of the IEEE quotient, which the oracle computes.  This test runs
every pair: for every non-negative bf16 group maximum m up to +inf, one or
more 128-channel groups hold m and then every bf16 x with |x| <= m of both
signs (0x7F81 * 0x7F82, about 1.07e9 pairs per quantisation), through ep_dispatch with one
expert (each token lands in one row), and compares every code and scale with
the oracle's, bit for bit.  One slice runs at a decode-sized token count so
that the staged pack kernel is covered as well as the streaming one.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from combine_topk_idx_rank_b200 import ep

pytestmark = pytest.mark.gpu

H = 7168                 # 56 groups of 128 channels per token row
GROUPS_PER_ROW = H // 128


def pair_groups(m_lo, m_hi):
    """[n, 128] bf16 bit patterns: for each group maximum pattern m in
    [m_lo, m_hi), groups of (m, then 127 values x with |x| <= m, both signs)."""
    out = []
    for m in range(m_lo, m_hi):
        mag = np.arange(m + 1, dtype=np.uint16)
        xs = np.concatenate([mag, mag | np.uint16(0x8000)])
        ng = -(-xs.size // 127)
        xs = np.concatenate([xs, np.full(ng * 127 - xs.size, m, np.uint16)])
        g = np.empty((ng, 128), np.uint16)
        g[:, 0] = m
        g[:, 1:] = xs.reshape(ng, 127)
        out.append(g)
    return np.concatenate(out)


def run_slice(groups, quant, dev):
    T = -(-groups.shape[0] // GROUPS_PER_ROW)
    rows = np.zeros((T * GROUPS_PER_ROW, 128), np.uint16)
    rows[:groups.shape[0]] = groups
    x_np = rows.reshape(T, H)
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    ti = torch.zeros((T, 1), dtype=torch.int64, device=dev)
    tw = torch.ones((T, 1), dtype=torch.float32, device=dev)
    recv_x, recv_s, _, _, h = ep.ep_dispatch(x, ti, tw, 1, quant, num_experts=1, num_ranks=1, quant_size=128)
    torch.cuda.synchronize()
    got_x = recv_x.contiguous().view(torch.uint8).cpu().numpy()
    got_s = recv_s.cpu().numpy()
    dst = np.arange(T, dtype=np.int32)[:, None]
    ref_x, ref_s = oracle.dispatch_rows(x_np, dst, quant, 128, False, num_rows=T)
    return got_x, got_s, ref_x, ref_s


@pytest.fixture(autouse=True)
def threaded_oracle():
    oracle.use_threads(len(os.sched_getaffinity(0)))
    yield
    oracle.use_threads(1)


@pytest.mark.timeout(1800)
@pytest.mark.parametrize("quant", ["fp8", "int8"])
def test_every_pair(quant, cuda_device):
    total = 0
    bounds = [0, 64, 4096] + list(range(8192, 0x7F81, 4096)) + [0x7F81]   # group maxima up to +inf (0x7F80)
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        g = pair_groups(lo, hi)
        got_x, got_s, ref_x, ref_s = run_slice(g, quant, cuda_device)
        bad = np.nonzero((got_x != ref_x).any(axis=1))[0]
        assert bad.size == 0, f"maxima [{lo:#x}, {hi:#x}): {bad.size} rows differ, first {bad[:4]}"
        assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32))
        total += int(((g[:, 1:] & 0x7FFF) <= g[:, :1]).sum())
    # every pair: sum over maxima patterns p = 0 .. 0x7F80 of 2 (p + 1) = 0x7F81 * 0x7F82, about
    # 1.0655e9 (plus the padding copies of each maximum)
    assert total >= 0x7F81 * 0x7F82


def test_decode_sized_slice_through_the_staged_kernel(cuda_device):
    # 2048 tokens x 56 groups (the decode shape): maxima from 0x3F00 (0.5) up
    g = pair_groups(0x3F00, 0x3F00 + 460)[:2048 * GROUPS_PER_ROW]
    assert g.shape[0] == 2048 * GROUPS_PER_ROW
    for quant in ("fp8", "int8"):
        got_x, got_s, ref_x, ref_s = run_slice(g, quant, cuda_device)
        assert np.array_equal(got_x, ref_x)
        assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32))
