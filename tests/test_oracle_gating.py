"""Pins for the oracle's group-limited gating (the routing generator upstream
of dispatch).

Definition followed ("DeepEP V1 vs V2 comparative analysis", section 8.1,
DeepSeek-V3 group-limited gating): the experts form groups (256 experts, 32
groups of 8); each token keeps its best 4 groups and the best 2 experts inside
each kept group, 8 experts in all.  Readings where the page is silent: the
affinity is the router logit; a group's score is the sum of its best
per-group logits; ties go to the lower id; entries are listed by logit; the
weights are the softmax over the selected logits.

Pinned by: hand-worked tokens (including the case where a group's single
strong expert loses to a group whose two experts add up higher, and exact
ties), brute force over every admissible expert set on tiny shapes (the kept
set maximises the sum of logits subject to the group limit), the special case
of one group (plain top-k, against numpy's lexsort), the case where every
group is kept, the invariants at the DeepSeek-V3 shape, and a check that the
invariant checker rejects planted mistakes.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from combine_topk_idx_rank_b200.workloads import make_router_logits


def softmax64(v):
    v = np.asarray(v, np.float64)
    e = np.exp(v - v.max())
    return (e / e.sum()).astype(np.float32)


def test_hand_worked_tokens():
    # E = 12 experts in 3 groups of 4; keep 2 groups, 2 experts in each: K = 4
    lg = np.array([
        # group 0               group 1                group 2
        [0.5, 3.0, 1.0, -1.0,   2.5, 2.0, 0.0, 0.25,   4.0, -2.0, -3.0, 0.75],
        [0.0] * 12,
        [1.5, 1.5, 0.0, 0.0,    0.0, 2.0, 1.0, 0.0,    2.75, 0.25, 0.0, 0.0],
    ], np.float32)
    idx, w = oracle.group_limited_gating(lg, 3, 2, 2)
    # token 0: group scores 3+1 = 4, 2.5+2 = 4.5, 4+0.75 = 4.75 -> groups 2 and 1;
    # expert 1 (logit 3, the second largest overall) is not kept: its group loses
    assert idx[0].tolist() == [8, 4, 5, 11]
    # softmax of (4, 2.5, 2, 0.75): e^0, e^-1.5, e^-2, e^-3.25 over their sum 1.3972396...
    assert w[0].tolist() == pytest.approx([0.7156968, 0.1596936, 0.0968590, 0.0277506], abs=2e-7)
    # token 1: every logit 0 -> every score 0 -> groups 0, 1 (lower ids), experts 0,1 and 4,5
    assert idx[1].tolist() == [0, 1, 4, 5]
    assert w[1].tolist() == [0.25, 0.25, 0.25, 0.25]
    # token 2: three scores of 3.0 -> groups 0 and 1; group 0's equal logits 1.5, 1.5 both kept;
    # listed by logit: 5 (2.0), 0 (1.5), 1 (1.5, higher id after 0), 6 (1.0)
    assert idx[2].tolist() == [5, 0, 1, 6]
    assert w[2].tolist() == pytest.approx(softmax64([2.0, 1.5, 1.5, 1.0]).tolist(), abs=1e-7)
    e2, e1 = math.exp(0.0), math.exp(-0.5)
    assert w[2][0] == pytest.approx(e2 / (e2 + 2 * e1 + math.exp(-1.0)), abs=1e-7)


def brute_force_set(l, n_group, topk_group, per_group):
    """The admissible expert set (topk_group groups, per_group experts in
    each) with the largest sum of logits, by enumeration."""
    E = l.shape[0]
    S = E // n_group
    best, best_val = None, -np.inf
    for gs in itertools.combinations(range(n_group), topk_group):
        for picks in itertools.product(*[itertools.combinations(range(g * S, (g + 1) * S), per_group)
                                         for g in gs]):
            st = [e for p in picks for e in p]
            v = float(np.sum(l[st].astype(np.float64)))
            if v > best_val:
                best, best_val = set(st), v
    return best


@pytest.mark.parametrize("E,n_group,topk_group,per_group", [
    (16, 4, 2, 2), (16, 4, 1, 3), (16, 4, 3, 1), (12, 3, 2, 2), (16, 8, 3, 2), (8, 2, 1, 2), (9, 3, 2, 3)])
def test_brute_force_tiny(E, n_group, topk_group, per_group):
    lg = make_router_logits(150, E, seed=E * 100 + n_group)
    idx, w = oracle.group_limited_gating(lg, n_group, topk_group, per_group)
    for t in range(lg.shape[0]):
        assert set(idx[t].tolist()) == brute_force_set(lg[t], n_group, topk_group, per_group)


def test_one_group_is_plain_topk():
    lg = make_router_logits(300, 32, seed=3)
    lg[::7, 5] = lg[::7, 9]                      # some exact ties between experts 5 and 9
    idx, w = oracle.group_limited_gating(lg, 1, 1, 8)
    for t in range(lg.shape[0]):
        order = np.lexsort((np.arange(32), -lg[t].astype(np.float64)))[:8]   # larger logit, then lower id
        assert idx[t].tolist() == order.tolist()
        ref = softmax64(lg[t][order])
        assert np.all(np.abs(w[t] - ref) <= np.spacing(ref))


def test_every_group_kept():
    lg = make_router_logits(200, 24, seed=4)
    idx, _ = oracle.group_limited_gating(lg, 6, 6, 2)
    for t in range(lg.shape[0]):
        want = set()
        for g in range(6):
            blk = lg[t, 4 * g:4 * g + 4]
            want |= {4 * g + int(i) for i in np.lexsort((np.arange(4), -blk.astype(np.float64)))[:2]}
        assert set(idx[t].tolist()) == want


def check_gating(lg, idx, w, n_group, topk_group, per_group):
    """Invariants of group-limited gating; returns the first violation or None."""
    T, E = lg.shape
    S = E // n_group
    K = topk_group * per_group
    for t in range(T):
        l = lg[t]
        ids = idx[t]
        if len(set(ids.tolist())) != K or ids.min() < 0 or ids.max() >= E:
            return f"token {t}: ids not {K} distinct experts"
        groups = ids // S
        kept = sorted(set(groups.tolist()))
        if len(kept) != topk_group or any(int(np.sum(groups == g)) != per_group for g in kept):
            return f"token {t}: not {per_group} experts in each of {topk_group} groups"
        score = {}
        for g in range(n_group):
            top = np.sort(l[g * S:(g + 1) * S])[::-1][:per_group]
            sc = np.float32(top[0])
            for v in top[1:]:
                sc = np.float32(sc + v)
            score[g] = sc
        if min(score[g] for g in kept) < max([score[g] for g in range(n_group) if g not in kept], default=-np.inf):
            return f"token {t}: a dropped group scores higher than a kept one"
        for g in kept:
            inside = [e for e in range(g * S, (g + 1) * S)]
            chosen = [e for e in ids if e // S == g]
            if min(l[chosen]) < max([l[e] for e in inside if e not in chosen], default=-np.inf):
                return f"token {t}: a dropped expert of a kept group has a larger logit"
        if np.any(np.diff(l[ids]) > 0):
            return f"token {t}: entries not listed by logit"
        ref = softmax64(l[ids])
        if np.any(np.abs(w[t] - ref) > np.spacing(ref)):
            return f"token {t}: weights are not the softmax of the selected logits"
    return None


def test_deepseek_v3_shape_invariants():
    lg = make_router_logits(2048, 256, seed=0)
    idx, w = oracle.group_limited_gating(lg, 32, 4, 2)
    assert idx.shape == (2048, 8) and idx.dtype == np.int64 and w.dtype == np.float32
    assert check_gating(lg, idx, w, 32, 4, 2) is None
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    # the group limit binds: many tokens' plain top-8 spans more than 4 groups
    plain = np.argsort(-lg, axis=1)[:, :8]
    assert np.mean([len(set((p // 8).tolist())) > 4 for p in plain]) > 0.5


def test_invariant_checker_rejects_planted_mistakes():
    lg = make_router_logits(64, 256, seed=9)
    idx, w = oracle.group_limited_gating(lg, 32, 4, 2)
    assert check_gating(lg, idx, w, 32, 4, 2) is None
    bad = idx.copy()                       # an expert of a dropped group in place of a kept one
    S = 8
    kept = set((bad[0] // S).tolist())
    other = next(g for g in range(32) if g not in kept)
    bad[0, -1] = other * S
    assert check_gating(lg, bad, w, 32, 4, 2) is not None
    bad = idx.copy()                       # swapped order
    bad[1, [0, 1]] = bad[1, [1, 0]]
    assert check_gating(lg, bad, w, 32, 4, 2) is not None
    bad = idx.copy()                       # a worse expert of the same kept group
    g = int(bad[2, 0] // S)
    worse = [e for e in range(g * S, g * S + S) if e not in bad[2]]
    bad[2, 0] = min(worse, key=lambda e: lg[2, e])
    assert check_gating(lg, bad, w, 32, 4, 2) is not None
    ww = w.copy()                          # weights of the unsorted logits
    ww[3] = ww[3][::-1]
    assert check_gating(lg, idx, ww, 32, 4, 2) is not None


def test_errors():
    lg = make_router_logits(4, 16, seed=1)
    with pytest.raises(oracle.OracleError) as e:
        oracle.group_limited_gating(lg, 3, 1, 1)               # 16 experts do not split into 3 groups
    assert e.value.status == oracle.INVALID_ARG
    with pytest.raises(oracle.OracleError):
        oracle.group_limited_gating(lg, 4, 5, 1)               # more groups kept than exist
    with pytest.raises(oracle.OracleError):
        oracle.group_limited_gating(lg, 4, 1, 5)               # more picks than a group holds
    for bad in (np.nan, np.inf, -np.inf):
        l2 = lg.copy()
        l2[2, 7] = bad
        with pytest.raises(oracle.OracleError) as e:
            oracle.group_limited_gating(l2, 4, 2, 2)
        assert e.value.status == oracle.NONFINITE
