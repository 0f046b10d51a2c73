"""Pins for the oracle's layout and slot assignment.

The pages print no worked example, so the oracle is pinned by: a small example
worked out by hand from the definitions below, exhaustive brute force on tiny
inputs against numpy library routines (bincount, stable lexsort), and the
invariants the definitions imply.

Definitions followed (DeepEP V1 vs V2 comparative analysis, section 2.1 for the
layout outputs, section 3.1 for the EPHandle fields and expert alignment,
section 8.4 for the deterministic order; DeepEP on Ascend A2, Usage, for
num_local_experts = num_experts / ep_world_size): one received row per
unmasked (token, expert) pair, ordered by (expert, token, k), expert segments
padded to a multiple of expert_alignment.
"""
import itertools

import numpy as np
import pytest

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload


def test_hand_worked_example():
    # T=4 tokens, R=2 ranks, E=4 experts (L=2 per rank), K=2, alignment A=2.
    topk_idx = np.array([[1, 2], [0, 1], [3, -1], [1, 3]], np.int64)
    w = np.array([[.6, .4], [.7, .3], [1., 0.], [.55, .45]], np.float32)
    lay = oracle.layout(topk_idx, 4, 2)
    # expert counts: e0 <- (1,0); e1 <- (0,0),(1,1),(3,0); e2 <- (0,1); e3 <- (2,0),(3,1)
    assert list(lay["num_tokens_per_expert"]) == [1, 3, 1, 2]
    # ranks: e0,e1 on rank 0; e2,e3 on rank 1
    assert lay["is_token_in_rank"].astype(int).tolist() == [[1, 1], [1, 0], [0, 1], [1, 1]]
    assert list(lay["num_tokens_per_rank"]) == [3, 3]
    s = oracle.slots(topk_idx, w, 4, 2, 2)
    # aligned counts 2,4,2,2 -> inclusive prefix sum
    assert list(s["psum_num_recv_tokens_per_expert"]) == [2, 6, 8, 10]
    assert list(s["num_recv_tokens_per_expert"]) == [1, 3, 1, 2]
    assert s["num_recv_rows"] == 10
    # rows: 0=(1,0) 1=pad | 2=(0,0) 3=(1,1) 4=(3,0) 5=pad | 6=(0,1) 7=pad | 8=(2,0) 9=(3,1)
    assert s["dst_buffer_slot_idx"].tolist() == [[2, 6], [0, 3], [8, -1], [4, 9]]
    assert s["recv_src_metadata"].tolist() == [[1, 0], [-1, -1], [0, 0], [1, 1], [3, 0], [-1, -1],
                                               [0, 1], [-1, -1], [2, 0], [3, 1]]
    # recv_topk_idx: local ids (e - r*L) of the token's experts on the receiving rank
    assert s["recv_topk_idx"].tolist() == [[0, 1], [-1, -1], [1, -1], [0, 1], [1, -1], [-1, -1],
                                           [-1, 0], [-1, -1], [1, -1], [-1, 1]]
    rw = s["recv_topk_weights"]
    assert rw[0].tolist() == pytest.approx([.7, .3]) and rw[2].tolist() == pytest.approx([.6, 0])
    assert rw[9].tolist() == pytest.approx([0, .45]) and rw[7].tolist() == [0, 0]


def _expected_by_sort(topk_idx, E, A):
    """Slots from numpy's stable lexsort of the keys (expert, token, k)."""
    T, K = topk_idx.shape
    t, k = np.nonzero(topk_idx >= 0)
    e = topk_idx[t, k]
    order = np.lexsort((k, t, e))          # last key is primary
    counts = np.bincount(e, minlength=E)
    aligned = -(-counts // A) * A
    seg = np.concatenate([[0], np.cumsum(aligned)[:-1]])
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    dst = -np.ones((T, K), np.int64)
    pos = np.empty_like(order)
    pos[order] = np.arange(order.size)
    dst[t, k] = seg[e] + (pos - first[e])
    return dst, np.cumsum(aligned), counts


def test_bruteforce_all_tiny_routings():
    # every topk_idx with T=3, K=2, E=4, R=2 and ids in {-1..3}: 5^6 cases
    E, R, K, T = 4, 2, 2, 3
    w = np.full((T, K), 0.5, np.float32)
    n = 0
    for combo in itertools.product(range(-1, E), repeat=T * K):
        ti = np.array(combo, np.int64).reshape(T, K)
        lay = oracle.layout(ti, E, R)
        valid = ti[ti >= 0]
        assert np.array_equal(lay["num_tokens_per_expert"], np.bincount(valid, minlength=E))
        itr = np.zeros((T, R), bool)
        tt, kk = np.nonzero(ti >= 0)
        itr[tt, ti[tt, kk] // (E // R)] = True
        assert np.array_equal(lay["is_token_in_rank"], itr)
        assert np.array_equal(lay["num_tokens_per_rank"], itr.sum(0))
        for A in (1, 3):
            s = oracle.slots(ti, w, E, R, A)
            dst, psum, cnt = _expected_by_sort(ti, E, A)
            assert np.array_equal(s["dst_buffer_slot_idx"], dst)
            assert np.array_equal(s["psum_num_recv_tokens_per_expert"], psum)
            assert np.array_equal(s["num_recv_tokens_per_expert"], cnt)
        n += 1
    assert n == 5 ** 6


def _check_slot_invariants(ti, w, E, R, A, s):
    T, K = ti.shape
    L = E // R
    dst = s["dst_buffer_slot_idx"]
    meta = s["recv_src_metadata"]
    psum = s["psum_num_recv_tokens_per_expert"].astype(np.int64)
    cnt = s["num_recv_tokens_per_expert"].astype(np.int64)
    n_al = s["num_recv_rows"]
    masked = ti < 0
    # counts sum to T*K minus masked entries
    assert cnt.sum() == T * K - masked.sum()
    # aligned segments: differences are multiples of A and at least the counts
    seg = np.diff(np.concatenate([[0], psum]))
    assert np.all(seg % A == 0) and np.all(seg >= cnt) and np.all(seg - cnt < A)
    assert psum[-1] == n_al
    # masked entries have no row; unmasked ones a row inside their expert's segment
    assert np.all(dst[masked] == -1)
    t, k = np.nonzero(~masked)
    rows = dst[t, k]
    e = ti[t, k]
    lo = np.concatenate([[0], psum[:-1]])[e]
    assert np.all((rows >= lo) & (rows < lo + cnt[e]))
    # bijection: the metadata of a token's row points back to it
    assert np.array_equal(meta[rows, 0], t) and np.array_equal(meta[rows, 1], k)
    assert np.unique(rows).size == rows.size
    # rows not owned by any (t,k) are padding
    pad = np.ones(n_al, bool)
    pad[rows] = False
    assert np.all(meta[pad] == -1)
    assert np.all(s["recv_topk_idx"][pad] == -1) and np.all(s["recv_topk_weights"][pad] == 0)
    # within a segment the (t,k) keys strictly increase
    key = meta[:, 0].astype(np.int64) * K + meta[:, 1]
    starts = np.concatenate([[0], psum[:-1]])
    for ee in range(E):
        kk = key[starts[ee]:starts[ee] + cnt[ee]]
        assert np.all(np.diff(kk) > 0)
    # recv_topk_idx: the row's own k is its expert's local id; entries >= 0 are
    # exactly the token's experts that live on the receiving rank
    rti = s["recv_topk_idx"][rows]
    rtw = s["recv_topk_weights"][rows]
    rdst = e // L
    assert np.array_equal(rti[np.arange(rows.size), k], e - rdst * L)
    same = (ti[t] >= 0) & (ti[t] // L == rdst[:, None])
    assert np.array_equal(rti >= 0, same)
    assert np.all((rti[same] >= 0) & (rti[same] < L))
    assert np.array_equal(rtw[same], w[t][same]) and np.all(rtw[~same] == 0)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_slot_invariants_on_workloads(name):
    cfg = CONFIGS[name]
    T = min(cfg.num_tokens, 1600)
    T -= T % cfg.num_ranks
    wl = make_workload(cfg.scaled(num_tokens=T), seed=3, with_x=False)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks,
                     cfg.expert_alignment)
    _check_slot_invariants(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks,
                           cfg.expert_alignment, s)
    dst, psum, _ = _expected_by_sort(wl.topk_idx, cfg.num_experts, cfg.expert_alignment)
    assert np.array_equal(s["dst_buffer_slot_idx"], dst)


def test_duplicate_ids_each_get_a_row():
    ti = np.array([[2, 2], [2, -1]], np.int64)
    s = oracle.slots(ti, np.ones((2, 2), np.float32), 4, 2, 1)
    assert s["dst_buffer_slot_idx"].tolist() == [[0, 1], [2, -1]]


def test_errors():
    ti = np.array([[0, 4]], np.int64)
    with pytest.raises(oracle.OracleError) as e:
        oracle.layout(ti, 4, 2)
    assert e.value.status == oracle.BAD_EXPERT_ID
    with pytest.raises(oracle.OracleError) as e:
        oracle.slots(np.array([[0, -2]]), np.ones((1, 2), np.float32), 4, 2)
    assert e.value.status == oracle.BAD_EXPERT_ID
    with pytest.raises(oracle.OracleError) as e:
        oracle.layout(np.zeros((1, 1), np.int64), 5, 2)       # E % R != 0
    assert e.value.status == oracle.INVALID_ARG
    with pytest.raises(oracle.OracleError) as e:
        oracle.slots(np.zeros((4, 2), np.int64), np.ones((4, 2), np.float32), 4, 2, 1, capacity=7)
    assert e.value.status == oracle.CAPACITY


def test_empty_and_all_masked():
    s = oracle.slots(np.zeros((0, 8), np.int64), np.zeros((0, 8), np.float32), 16, 8, 4)
    assert s["num_recv_rows"] == 0 and np.all(s["psum_num_recv_tokens_per_expert"] == 0)
    ti = -np.ones((5, 3), np.int64)
    s = oracle.slots(ti, np.zeros((5, 3), np.float32), 8, 4, 4)
    assert s["num_recv_rows"] == 0 and np.all(s["dst_buffer_slot_idx"] == -1)
    lay = oracle.layout(ti, 8, 4)
    assert lay["num_tokens_per_rank"].sum() == 0 and not lay["is_token_in_rank"].any()
