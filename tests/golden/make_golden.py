"""Writes tests/golden/oracle_digests.json: SHA-256 digests of the oracle's
outputs on the tiny workload and on scaled-down copies of the other four.

Calls only oracle/ (and the seeded input generators).  The digests guard the
oracle against silent drift: a change to its arithmetic must come with a
regenerated file and a commit message naming the passage that justifies it.

    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_router_logits, make_workload, make_y  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_digests.json")


def cases():
    yield "tiny", CONFIGS["tiny"]
    yield "decode_small", CONFIGS["decode"].scaled(num_tokens=16 * 16, hidden=1024)
    yield "prefill_small", CONFIGS["prefill"].scaled(num_tokens=8 * 100, hidden=1024)
    yield "qwen3_small", CONFIGS["qwen3"].scaled(num_tokens=16 * 24, hidden=512)
    yield "longseq_small", CONFIGS["longseq"].scaled(num_tokens=8 * 64, hidden=1024)


def digest(a) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def compute():
    res = {}
    for name, cfg in cases():
        for seed in (0, 1, 2):
            wl = make_workload(cfg, seed)
            lay = oracle.layout(wl.topk_idx, cfg.num_experts, cfg.num_ranks)
            d = oracle.dispatch(wl.x, wl.topk_idx, wl.topk_weights, cfg.num_experts,
                                cfg.num_ranks, cfg.expert_alignment, cfg.quant,
                                cfg.quant_size, cfg.round_scale, cfg.num_rounds)
            y = make_y(d["num_recv_rows"], cfg.hidden, seed)
            out = oracle.combine(y, d["dst_buffer_slot_idx"], wl.topk_weights,
                                 cfg.num_ranks, cfg.num_rounds)
            entry = {k: digest(v) for k, v in lay.items()}
            for k in ("psum_num_recv_tokens_per_expert", "num_recv_tokens_per_expert",
                      "dst_buffer_slot_idx", "recv_src_metadata", "recv_topk_idx",
                      "recv_topk_weights", "recv_x"):
                entry[k] = digest(d[k])
            if d["recv_scales"] is not None:
                entry["recv_scales"] = digest(d["recv_scales"])
            entry["num_recv_rows"] = int(d["num_recv_rows"])
            entry["combined"] = digest(out)
            res[f"{name}/seed{seed}"] = entry
    # group-limited gating at the DeepSeek-V3 shape (256 experts, 32 groups,
    # top-4 groups, top-2 per group) on 512 tokens of seeded router logits
    for seed in (0, 1, 2):
        idx, w = oracle.group_limited_gating(make_router_logits(512, 256, seed), 32, 4, 2)
        res[f"gating_dsv3_512/seed{seed}"] = {"topk_idx": digest(idx), "topk_weights": digest(w)}
    return res


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(compute(), f, indent=1, sort_keys=True)
    print("wrote", OUT)
