"""Host-side logic of bench.py (CPU only): the algorithmic byte count behind
the roofline, the captured-traffic lookup, and the workload / mode options."""
import argparse
import json
import os

import numpy as np
import pytest

import bench
from combine_topk_idx_rank_b200.workloads import CONFIGS


def _args(**kw):
    d = dict(workload="decode", tokens=0, quant=None, ue8m0=False)
    d.update(kw)
    return argparse.Namespace(**d)


def test_algorithmic_bytes_worked_example():
    # T = 4 tokens, K = 2, E = 4 experts, A = 2, H = 16, bf16: counts (3, 0, 4, 1)
    # -> 8 rows, aligned (4, 0, 4, 2) = 10 rows
    cfg = CONFIGS["tiny"].scaled(num_tokens=4, hidden=16, num_experts=4, num_ranks=2, num_topk=2,
                                 expert_alignment=2)
    ab = bench.algorithmic_bytes(cfg, [3, 0, 4, 1], 4)
    assert ab["rows"] == 8 and ab["rows_aligned"] == 10
    x_read = 4 * 16 * 2                  # every token row once
    rows_written = 10 * 16 * 2           # received rows, padding included
    per_row_meta = 10 * (2 * 2 * 4 + 8)  # recv_topk_idx + recv_topk_weights + recv_src_metadata
    # routing: topk_idx + topk_weights read, the int32 id copy and dst_buffer_slot_idx written,
    # the per-row metadata, psum and counts
    assert ab["route"] == 4 * 2 * (8 + 4 + 4 + 4) + per_row_meta + 2 * 4 * 4
    # pack: x once, dst_buffer_slot_idx read, every received row written
    assert ab["pack"] == x_read + 4 * 2 * 4 + rows_written
    # combine: slots and weights read, each unmasked y row once, out once
    assert ab["combine"] == 4 * 2 * 8 + 8 * 16 * 2 + 4 * 16 * 2
    # FP8 group 8: one byte per element plus an fp32 scale per group; low-latency: no padding rows
    cfg8 = cfg.scaled(quant="fp8", quant_size=8)
    ab8 = bench.algorithmic_bytes(cfg8, [3, 0, 4, 1], 4, low_latency=True)
    assert ab8["rows_aligned"] == 8
    assert ab8["pack"] == x_read + 4 * 2 * 4 + 8 * 16 + 8 * 2 * 4
    # quantised combine reads the codes and their scales instead of bf16 rows
    abq = bench.algorithmic_bytes(cfg8, [3, 0, 4, 1], 4, combine_quant=True)
    assert abq["combine"] == 4 * 2 * 8 + 8 * (16 + 2 * 4) + 4 * 16 * 2


def test_prefill_bytes_match_the_workload_counts():
    cfg = CONFIGS["prefill"]
    from combine_topk_idx_rank_b200.workloads import make_workload
    wl = make_workload(cfg, 0, with_x=False)
    counts = np.bincount(wl.topk_idx[wl.topk_idx >= 0], minlength=cfg.num_experts)
    ab = bench.algorithmic_bytes(cfg, counts, cfg.num_tokens)
    assert ab["rows"] == cfg.num_tokens * cfg.num_topk
    assert ab["rows_aligned"] == int((-(-counts // 128) * 128).sum())
    # x once (0.47 GB) + 8 bf16 copies (3.76 GB) + padding rows: about 4.5 GB
    assert 4.4e9 < ab["pack"] < 4.6e9 and 4.2e9 < ab["combine"] < 4.25e9
    assert 0.02e9 < ab["route"] < 0.03e9


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"dram_bytes_per_launch": 1234, "sources": ["k.cu"], "source_digest": bench.source_digest(["k.cu"])}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k_pack/decode": entry}))
    assert bench.traffic_for("k_pack", "decode") == 1234
    assert bench.traffic_for("k_pack", "prefill") is None          # not captured
    src.write_text("kernel v2")                                     # the kernel changed since
    assert bench.traffic_for("k_pack", "decode") is None
    os.remove(tmp_path / "profiles" / "traffic.json")
    assert bench.traffic_for("k_pack", "decode") is None


def test_workload_options():
    assert bench.workload_config(_args()) == CONFIGS["decode"]
    mx = bench.workload_config(_args(quant="mxfp4"))
    assert mx.quant == "mxfp4" and mx.quant_size == 32
    ue = bench.workload_config(_args(workload="qwen3", ue8m0=True))
    assert ue.round_scale and ue.quant == "fp8"
    fp8 = bench.workload_config(_args(workload="prefill", quant="fp8"))
    assert fp8.quant == "fp8" and fp8.quant_size == 128
    small = bench.workload_config(_args(workload="longseq", tokens=64 * 8))
    assert small.num_tokens == 512 and small.num_rounds == 8
    with pytest.raises(SystemExit):
        bench.workload_config(_args(workload="prefill", ue8m0=True))    # bf16 has no scales
    with pytest.raises(SystemExit):
        bench.workload_config(_args(workload="longseq", tokens=100))     # not ranks x rounds
