"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun
launches them.  Each rank owns an independent problem (its own seed), the
process group carries only the barrier and the max-reduction of timings, the
whole-job value counts every rank's tokens over the slowest rank, and the
reference arm runs on rank 0 only."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    import oracle
    from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload
    try:
        w, r = bench.init_dist("gloo", rank, timeout_s=60)
        assert (w, r) == (world, rank)
        # each rank's own problem, solved locally (the oracle stands in for the GPU step)
        cfg = CONFIGS["tiny"]
        wl = make_workload(cfg, seed=bench.rank_seed(7, r))
        s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks)
        fake_ms = 10.0 + 5.0 * r
        bench.barrier(w)
        slowest = bench.max_over_ranks(fake_ms, w, "cpu")
        value = bench.job_tokens_per_s(w, cfg.num_tokens, slowest)
        out = io.StringIO()
        ns = type("A", (), dict(workload="tiny", seed=0, steps=3, warmup=3, ref_seconds=1.0))()
        with redirect_stdout(out):
            bench.run_reference(ns)
        q.put((r, slowest, value, int(s["num_recv_rows"]), wl.topk_idx.tobytes(), out.getvalue()))
        bench.barrier(w)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    # the slowest rank's time is everyone's time
    assert [x[1] for x in res] == [15.0, 15.0]
    # whole-job throughput: both ranks' 256 tokens over 15 ms
    assert res[0][2] == pytest.approx(2 * 256 / 15e-3)
    # independent problems: different routings on the two ranks
    assert res[0][4] != res[1][4]
    # the reference arm prints one JSON line on rank 0 and nothing elsewhere
    line0 = res[0][5].strip()
    assert json.loads(line0)["impl"] == "reference" and res[1][5] == ""


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.rank_seed(5, 3) == 8
    assert bench.job_tokens_per_s(1, 1000, 2.0) == pytest.approx(5e5)


@pytest.mark.timeout(300)
def test_launcher_starts_one_process_per_gpu():
    """`bench.py --gpus 2` without a torchrun environment starts two ranks
    itself; the reference arm then prints one JSON line (rank 0's) for a
    two-GPU job and the other rank exits 0 without output."""
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3", "--ref-seconds", "2"],
                       capture_output=True, text=True, env=env, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["impl"] == "reference"
    assert rec["config"]["name"] == "tiny" and rec["steps"] == 3
    # the step time is measured: all steps fit in the run's own wall clock
    assert rec["ms_per_step"] * rec["steps"] < 280e3


def test_launch_ranks_reports_a_failing_rank(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    script = tmp_path / "fail_on_rank1.py"
    script.write_text("import os, sys\nsys.exit(3 if os.environ['RANK'] == '1' else 0)\n")
    monkeypatch.setattr(bench, "__file__", str(script))
    assert bench.launch_ranks(2, [], timeout_s=60) == 3
