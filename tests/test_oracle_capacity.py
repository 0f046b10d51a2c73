"""The sizing formulas of the "DeepEP on Ascend A2" page (Usage, HCCL_BUFFSIZE;
long-sequence formula) used as capacity checks on the oracle's receive layout.

Non-layered formula: (bs x ep_world_size x min(num_local_experts, topk) x
hidden x 2B + 2MB) x 2 with bs = max tokens per rank: a rank's receive buffer
must hold bs x R x min(L, K) bf16 rows, because each of the R x bs source
tokens brings at most min(L, K) rows to one rank.  With expert alignment each
local expert adds at most A - 1 padding rows.
"""
import numpy as np
import pytest

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

MiB = 1 << 20


def hccl_non_layered_bytes(bs, world, L, K, H):
    return (bs * world * min(L, K) * H * 2 + 2 * MiB) * 2


def per_rank_rows(s, E, R):
    L = E // R
    cnt = s["num_recv_tokens_per_expert"].astype(np.int64).reshape(R, L).sum(1)
    psum = s["psum_num_recv_tokens_per_expert"].astype(np.int64)
    seg = np.diff(np.concatenate([[0], psum])).reshape(R, L).sum(1)
    return cnt, seg


@pytest.mark.parametrize("name", list(CONFIGS))
def test_receive_rows_fit_hccl_formula(name):
    cfg = CONFIGS[name]
    wl = make_workload(cfg, seed=0, with_x=False)
    E, R, K, A, H = cfg.num_experts, cfg.num_ranks, cfg.num_topk, cfg.expert_alignment, cfg.hidden
    L, bs = E // R, cfg.num_tokens // R
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    cnt, seg = per_rank_rows(s, E, R)
    bound_rows = bs * R * min(L, K)
    assert np.all(cnt <= bound_rows)
    assert np.all(seg <= bound_rows + L * (A - 1))
    # bf16 receive bytes per rank against the formula's buffer (one of its two halves)
    assert np.all(seg * H * 2 <= hccl_non_layered_bytes(bs, R, L, K, H) / 2 - 2 * MiB + L * (A - 1) * H * 2)
    # and the total over ranks is what the oracle reports
    assert seg.sum() == s["num_recv_rows"]


def test_formula_bound_is_reached_by_worst_case_routing():
    # every token of every rank picks K experts that all live on rank 0
    R, E, K, bs, H = 4, 32, 4, 16, 128
    L = E // R
    ti = np.tile(np.arange(K, dtype=np.int64), (R * bs, 1))
    s = oracle.slots(ti, np.ones_like(ti, dtype=np.float32), E, R, 1)
    cnt, _ = per_rank_rows(s, E, R)
    assert cnt[0] == bs * R * min(L, K) and cnt[1:].sum() == 0
    assert cnt[0] * H * 2 == hccl_non_layered_bytes(bs, R, L, K, H) / 2 - 2 * MiB


def test_long_sequence_round_fits_per_round_formula():
    # 2 x (102MB + 4MB + PER_ROUND_TOKENS x (hidden x 3) x topk) + PADDING: per
    # round a rank moves at most PER_ROUND_TOKENS x topk rows of
    # hidden x 3 bytes (bf16 + int8 copies of a row).
    cfg = CONFIGS["longseq"]
    wl = make_workload(cfg, seed=0, with_x=False)
    R, rounds, K, H = cfg.num_ranks, cfg.num_rounds, cfg.num_topk, cfg.hidden
    per_round = cfg.num_tokens // R // rounds
    assert 32 <= per_round <= 8192 and 1 <= rounds <= 256
    for j in range(rounds):
        tok = oracle.round_tokens(cfg.num_tokens, R, rounds, j).reshape(R, per_round)
        for r in range(R):
            rows = int((wl.topk_idx[tok[r]] >= 0).sum())
            assert rows <= per_round * K
            assert rows * H * 3 <= 2 * (106 * MiB + per_round * H * 3 * K)
