"""The oracle reproduces the digests stored in tests/golden/oracle_digests.json
(written by tests/golden/make_golden.py, which calls only the oracle), and the
slot-invariant checker rejects outputs with a planted mistake."""
import json
import os

import numpy as np
import pytest

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_stored_digests():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    with open(mg.OUT) as f:
        stored = json.load(f)
    now = mg.compute()
    assert sorted(now) == sorted(stored)
    for key in stored:
        assert now[key] == stored[key], key


def _planted(s, what):
    s = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in s.items()}
    dst, meta = s["dst_buffer_slot_idx"], s["recv_src_metadata"]
    if what == "swap_within_segment":           # order inside an expert broken
        t, k = np.nonzero(dst >= 0)
        a, b = (t[0], k[0]), None
        for i in range(1, t.size):
            if dst[t[i], k[i]] == dst[a] + 1:
                b = (t[i], k[i])
                break
        ra, rb = dst[a], dst[b]
        dst[a], dst[b] = rb, ra
        meta[[ra, rb]] = meta[[rb, ra]]
    elif what == "psum_off_by_one":
        s["psum_num_recv_tokens_per_expert"][3:] += 1
    elif what == "wrong_local_id":              # transposed expert -> rank mapping
        rti = s["recv_topk_idx"]
        rti[rti >= 0] = (rti[rti >= 0] + 1) % 2
    elif what == "dropped_weight":
        s["recv_topk_weights"][0, :] = 0
    return s


@pytest.mark.parametrize("what", ["swap_within_segment", "psum_off_by_one", "wrong_local_id",
                                  "dropped_weight"])
def test_invariant_checker_catches_planted_mistake(what):
    from test_oracle_layout import _check_slot_invariants
    cfg = CONFIGS["prefill"].scaled(num_tokens=8 * 40)
    wl = make_workload(cfg, seed=5, with_x=False)
    E, R, A = cfg.num_experts, cfg.num_ranks, cfg.expert_alignment
    s = oracle.slots(wl.topk_idx, wl.topk_weights, E, R, A)
    _check_slot_invariants(wl.topk_idx, wl.topk_weights, E, R, A, s)
    with pytest.raises(AssertionError):
        _check_slot_invariants(wl.topk_idx, wl.topk_weights, E, R, A, _planted(s, what))
