"""Benchmark: MoE expert-parallel dispatch + combine on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill] [--impl ours|reference]

One step = ep_dispatch (layout histogram, prefix scan + slot assignment,
permute/pack with fused quantisation, per round) + ep_combine (gather + k-order
fp32 weighted reduction) over one batch of synthetic inputs already resident in
HBM.  The default workload is the DeepSeek-V3-shaped prefill: 8 logical ranks x
4096 tokens, hidden 7168, bf16, 256 experts, top-8 Zipf(1.2) routing, expert
alignment 128.  Its inputs (x 470 MB, recv_x and y about 4 GB each) are far
larger than the 126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs its own independent
problem (seed + rank) and there is no data-path collective: weak scaling.
Timing: CUDA events on the launching stream, a barrier and a device sync on
both sides of the timed region, max over ranks.

--impl reference times the CPU oracle (unmodified C; its OpenMP build on every
host core) on bounded token samples of the same workload.

--gpus N without a torchrun environment starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from combine_topk_idx_rank_b200.workloads import CONFIGS, make_router_logits, make_workload  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (fraction of ~8 TB/s) on 1 B200"
UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_DESC = {
    "prefill": "prefill DeepSeek-V3 shape: 8 ranks x 4096 tokens, hidden 7168 bf16, 256 experts top-8 "
               "Zipf(1.2), expert_alignment 128, bf16 dispatch and combine",
    "decode": "decode DeepSeek-V3 shape: 16 ranks x 128 tokens, hidden 7168, 256 experts top-8 uniform, "
              "FP8 e4m3 group-128 dispatch, bf16 combine",
    "qwen3": "Qwen3-30B-A3B EP16 shape: 16 ranks x 512 tokens, hidden 2048, 128 experts top-8 uniform, "
             "10% masked, FP8 group-128 ue8m0 dispatch, bf16 combine",
    "longseq": "long sequence: 65536 tokens (8 ranks, 8 rounds of 8192), hidden 7168 N(0,2), 256 experts "
               "top-8 Zipf(1.0), int8 per-token dispatch, bf16 combine",
    "tiny": "tiny: 256 tokens, hidden 512, 16 experts over 8 ranks, top-2, bf16",
}

REASONS = ["gpu_idle", "applications_clocks_setting", "sw_power_cap", "hw_slowdown", "sync_boost",
           "sw_thermal_slowdown", "hw_thermal_slowdown", "hw_power_brake_slowdown", "display_clock_setting"]


# ----------------------------------------------------------------- helpers

def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(cfg, counts, T, scale_ue8m0=False, combine_quant=False, low_latency=False):
    """Minimum HBM bytes of the three kernels of one step, from the actual counts.

    route (k_route): topk_idx (int64) and topk_weights read once; the int32
    copy of topk_idx and dst_buffer_slot_idx written; for every received row
    (padding included) recv_topk_idx, recv_topk_weights and recv_src_metadata
    written; the per-expert psum and counts written.
    pack: x read once, dst_buffer_slot_idx read, every received row written
    once (padding rows included) with its scales.
    combine: dst_buffer_slot_idx and topk_weights read, each unmasked y row
    read once, out written once."""
    H, K, A, E = cfg.hidden, cfg.num_topk, cfg.expert_alignment, cfg.num_experts
    counts = np.asarray(counts, np.int64)
    n = int(counts.sum())
    n_al = n if low_latency else int((-(-counts // A) * A).sum())
    esize = {"none": 2.0, "fp8": 1.0, "int8": 1.0, "mxfp4": 0.5}[cfg.quant]
    nscales = 0 if cfg.quant == "none" else H // cfg.quant_size
    sbytes = 1 if (scale_ue8m0 or cfg.quant == "mxfp4") else 4
    route = int(T * K * (8 + 4 + 4 + 4) + n_al * (2 * K * 4 + 8) + 2 * E * 4)
    pack = int(T * H * 2 + T * K * 4 + n_al * H * esize + n_al * nscales * sbytes)
    if combine_quant:       # y rows read as 1-byte codes with fp32 scales
        combine = T * K * 8 + n * (H + nscales * 4) + T * H * 2
    else:
        combine = T * K * 8 + n * H * 2 + T * H * 2
    return {"route": route, "pack": pack, "combine": combine, "rows": n, "rows_aligned": n_al}


def source_digest(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of that kernel; else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            tab = json.load(f)
    except Exception:
        return None
    e = tab.get(f"{kernel}/{workload}")
    if not e:
        return None
    if e.get("source_digest") != source_digest(e["sources"]):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""

    def __init__(self, uuid):
        self.uuid = uuid
        self.samples = []
        self.proc = None

    def start(self):
        q = "timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active"
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", self.uuid],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 5:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        sel = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not sel:
            sel = [p for (_, p) in self.samples[-3:]]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(p[1]) for p in sel if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for p in sel if p[2].replace(".", "").isdigit()]
        mask = 0
        for p in sel:
            try:
                mask |= int(p[4], 16)
            except ValueError:
                pass
        reasons = [REASONS[i] for i in range(len(REASONS)) if mask >> i & 1 and REASONS[i] != "gpu_idle"]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sel)}


def workload_config(args):
    """The named workload, optionally with a different token count (--tokens)
    or dispatch quantisation (--quant, --ue8m0)."""
    cfg = CONFIGS[args.workload]
    if getattr(args, "tokens", 0):
        if args.tokens % (cfg.num_ranks * cfg.num_rounds):
            raise SystemExit(f"--tokens must be a multiple of ranks x rounds = {cfg.num_ranks * cfg.num_rounds}")
        cfg = cfg.scaled(num_tokens=args.tokens)
    quant = getattr(args, "quant", None)
    if quant:
        qs = 32 if quant == "mxfp4" else (cfg.quant_size if cfg.quant != "none" else 128)
        cfg = cfg.scaled(quant=quant, quant_size=qs)
    if getattr(args, "ue8m0", False):
        if cfg.quant not in ("fp8", "int8"):
            raise SystemExit("--ue8m0 applies to FP8 / int8 dispatch")
        cfg = cfg.scaled(round_scale=True)
    return cfg


# ------------------------------------------------------- multi-rank plumbing

def dist_env():
    """(world, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, local: int, timeout_s: float = 120.0):
    """Joins the process group when there is more than one rank.  Each rank
    runs an independent problem, so the group carries only barriers and the
    max-reduction of timings, never data."""
    import datetime

    import torch
    import torch.distributed as dist
    world, rank, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank


def rank_seed(seed: int, rank: int) -> int:
    """Every rank draws its own problem."""
    return seed + rank


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: the tokens of all ranks' problems over the
    slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ our arm

def config_dict(args, cfg, world):
    """The `config` object of the JSON line; both arms print the same one."""
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    opt = {"mode": "full", "tokens": 0, "quant": None, "ue8m0": False, "combine_quant": False, "gating": False}
    opt.update({k: getattr(args, k) for k in opt if hasattr(args, k)})
    args = argparse.Namespace(workload=args.workload, **opt)
    ll = args.mode == "ll"
    q = None if cfg.quant == "none" else cfg.quant
    cap = E * R * (T // R) if ll else T * K + E * (cfg.expert_alignment - 1)
    ebytes = 2 if q is None else (0.5 if q == "mxfp4" else 1)
    return {"workload": WORKLOAD_DESC[args.workload] + (f" (scaled to {T} tokens)" if args.tokens else "")
            + (" — cached dispatch (routing reused from the handle)" if args.mode == "cached" else "")
            + (" — low-latency fixed-capacity layout" if ll else "")
            + (f" — dispatch {cfg.quant} g{cfg.quant_size}{' ue8m0 bytes' if args.ue8m0 else ''}"
               if args.quant or args.ue8m0 else "")
            + (" — combine reads the quantised rows" if args.combine_quant else "")
            + (" — routing by group-limited gating (32 groups, top-4 groups, top-2 each) of N(0,1) router "
               "logits, timed in the step" if args.gating else ""),
            "name": args.workload, "mode": args.mode, "tokens": T, "hidden": H,
            "num_experts": E, "num_ranks": R, "topk": K, "expert_alignment": cfg.expert_alignment,
            "quant": cfg.quant, "num_rounds": cfg.num_rounds,
            "parallelism": f"{world} independent EP problems",
            "l2": "no flush: inputs larger than L2 (x %.0f MB, recv_x/y up to %.0f MB each)" % (
                T * H * 2 / 1e6, cap * H * ebytes / 1e6)}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from combine_topk_idx_rank_b200 import ep

    _, _, local = dist_env()
    torch.cuda.set_device(local)
    world, rank = init_dist("nccl", local)
    dev = torch.device("cuda", local)

    cfg = workload_config(args)
    wl = make_workload(cfg, seed=rank_seed(args.seed, rank))
    T, H, K, E, R = cfg.num_tokens, cfg.hidden, cfg.num_topk, cfg.num_experts, cfg.num_ranks
    x = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).to(dev)
    ti = torch.from_numpy(wl.topk_idx).to(dev)
    tw = torch.from_numpy(wl.topk_weights).to(dev)
    q = None if cfg.quant == "none" else cfg.quant
    ue8 = bool(args.ue8m0)
    if args.combine_quant and (q not in ("fp8", "int8") or ue8):
        raise SystemExit("--combine-quant reads FP8 / int8 received rows with fp32 scales")
    ll = args.mode == "ll"
    M = T // R                                  # low-latency capacity per (expert, source rank)
    bufs = ep.alloc_dispatch_buffers(T, H, K, E, R, cfg.expert_alignment, q, cfg.quant_size,
                                     cfg.num_rounds, recv_capacity=(E * R * M if ll else None), device=dev,
                                     scale_ue8m0=ue8)
    if ll:
        if cfg.expert_alignment != 1 or cfg.num_rounds != 1:
            raise SystemExit("--mode ll needs expert_alignment 1 and one round")
        bufs.handle.low_latency = 1
        ll_bufs = {"recv_x": bufs.recv_x, "recv_scales": bufs.recv_scales, "recv_topk_idx": bufs.recv_topk_idx,
                   "recv_topk_weights": bufs.recv_topk_weights,
                   "count": torch.empty((E,), dtype=torch.int32, device=dev),
                   "layout_range": torch.empty((E, R), dtype=torch.int64, device=dev), "handle": bufs.handle}
    if args.gating:
        # the step starts from router logits: group-limited gating produces the routing
        if E % 32 or K != 8 or args.mode != "full":
            raise SystemExit("--gating needs 256-style experts in 32 groups, top-8, and --mode full")
        logits = torch.from_numpy(make_router_logits(T, E, rank_seed(args.seed, rank))).to(dev)
        gerr = torch.zeros((1,), dtype=torch.int32, device=dev)
        ep.ep_group_limited_gating(logits, 32, 4, 2, out=(ti, tw), err=gerr)
    cap = bufs.recv_x.shape[0]
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if args.combine_quant:
        y, y_scales = bufs.recv_x, bufs.recv_scales      # quantised expert outputs (identity experts)
    else:
        g = torch.Generator(device=dev)
        g.manual_seed(1234 + rank)
        y, y_scales = torch.randn((cap, H), generator=g, device=dev, dtype=torch.bfloat16), None

    if args.mode == "cached":       # routing computed once; every step re-packs with the handle
        ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, q, num_experts=E, num_ranks=R,
                       quant_size=cfg.quant_size, round_scale=cfg.round_scale, num_rounds=cfg.num_rounds,
                       do_cpu_sync=False, buffers=bufs)

    def step(evs=None, x=x, ti=ti, tw=tw, out=out, lg=None):
        """One dispatch + combine (preceded by gating with --gating).  evs =
        four recorded events for the per-kernel split (step start, pack begin,
        pack end, combine end), or None: then nothing is recorded between the
        kernels."""
        if args.gating:
            ep.ep_group_limited_gating(logits if lg is None else lg, 32, 4, 2, out=(ti, tw), err=gerr, check=False)
        if evs is not None:
            evs[0].record()
        pev = None if evs is None else (evs[1], evs[2])
        if args.mode == "cached":
            ep.ep_dispatch(x, quant=q, quant_size=cfg.quant_size, round_scale=cfg.round_scale,
                           num_rounds=cfg.num_rounds, buffers=bufs, events=pev, handle=bufs.handle,
                           scale_ue8m0=ue8)
        elif ll:
            ep.ep_dispatch_low_latency(x, ti, tw, M, E, R, q, quant_size=cfg.quant_size,
                                       round_scale=cfg.round_scale, workspace=bufs.workspace, buffers=ll_bufs,
                                       scale_ue8m0=ue8, events=pev)
        else:
            ep.ep_dispatch(x, ti, tw, cfg.expert_alignment, q, num_experts=E, num_ranks=R,
                           quant_size=cfg.quant_size, round_scale=cfg.round_scale, num_rounds=cfg.num_rounds,
                           do_cpu_sync=False, buffers=bufs, events=pev, scale_ue8m0=ue8)
        # y: the experts' outputs, produced on the device (random bf16, or the
        # received codes themselves with --combine-quant)
        ep.ep_combine(y, bufs.handle, tw, out=out, y_scales=y_scales, quant_size=cfg.quant_size)
        if evs is not None:
            evs[3].record()
        return out

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    time.sleep(0.5)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    bufs.handle.check()
    if args.gating:
        assert int(gerr.item()) == 0
    counts = bufs.handle.num_recv_tokens_per_expert.cpu().numpy()

    # ------------------------------------------------- headline timed region
    # K steps back to back with nothing recorded between the kernels, so the
    # programmatic launch overlap of neighbouring kernels is the caller's
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        step()
    stop.record()
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.time()
    sampler.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world, dev)

    # --------------------------------------------- per-kernel split (separate)
    # events around each kernel of every step of a separate loop; an event
    # between two kernels stops their launch overlap, so this loop runs a
    # little slower than the headline one and is used for the split only
    n_split = max(3, min(args.steps, 50))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_split)]
    for row in ev:               # create the events before handing them to the library
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for i in range(n_split):
        step(ev[i])
    torch.cuda.synchronize()
    route_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(n_split))
    pack_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(n_split))
    combine_ms = statistics.mean(ev[i][2].elapsed_time(ev[i][3]) for i in range(n_split))
    split_step_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][3]) for i in range(n_split))

    # ------------------------------------------------------------ end to end
    e2e_steps = max(3, min(args.steps, 20))
    hx = torch.from_numpy(wl.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    hti = torch.from_numpy(wl.topk_idx).pin_memory()
    htw = torch.from_numpy(wl.topk_weights).pin_memory()
    hlg = logits.cpu().pin_memory() if args.gating else None
    hout = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()

    # two device input / output sets: step i's host->device copies run on one
    # stream, its dispatch + combine on the compute stream, its device->host
    # copy on a third, so copies of neighbouring steps overlap (PCIe is full
    # duplex); every step still moves its own inputs in and its result out
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dx = [torch.empty_like(x) for _ in range(2)]
    dti = [torch.empty_like(ti) for _ in range(2)]
    dtw = [torch.empty_like(tw) for _ in range(2)]
    dlg = [torch.empty_like(logits) for _ in range(2)] if args.gating else [None, None]
    dout = [torch.empty_like(out) for _ in range(2)]
    hout2 = [hout, torch.empty_like(hout).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    for e_ in ev_done + ev_free:
        e_.record(comp)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(ev_done[b])              # step i-2 has finished reading set b
        with torch.cuda.stream(s_in):
            dx[b].copy_(hx, non_blocking=True)
            if args.gating:                  # the routing is computed on the device from the logits
                dlg[b].copy_(hlg, non_blocking=True)
            else:
                dti[b].copy_(hti, non_blocking=True)
                dtw[b].copy_(htw, non_blocking=True)
            ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_free[b])              # step i-2's result has left dout[b]
        step(None, dx[b], dti[b], dtw[b], dout[b], dlg[b])
        ev_done[b].record(comp)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            hout2[b].copy_(dout[b], non_blocking=True)
            ev_free[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    comp.wait_event(ev_free[(e2e_steps - 1) % 2])
    comp.wait_event(ev_free[e2e_steps % 2])
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    assert torch.equal(hout2[(e2e_steps - 1) % 2].view(torch.int16), out.cpu().view(torch.int16))
    h2d = hx.numel() * 2 + (hlg.numel() * 4 if args.gating else hti.numel() * 8 + htw.numel() * 4)
    d2h = hout.numel() * 2

    ab = algorithmic_bytes(cfg, counts, T, ue8, args.combine_quant, ll)
    if args.mode == "cached":
        ab["route"] = 0
    ab["gating"] = T * E * 4 + T * K * 12 if args.gating else 0     # logits read, ids and weights written
    ms_per_step = elapsed_ms / args.steps
    step_bytes = ab["gating"] + ab["route"] + ab["pack"] + ab["combine"]
    value = job_tokens_per_s(world, T, ms_per_step)
    gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    pack_gbs = ab["pack"] / (pack_ms * 1e-3) / 1e9
    combine_gbs = ab["combine"] / (combine_ms * 1e-3) / 1e9
    if pack_ms >= combine_ms:
        dom, dom_bytes, dom_gbs, dom_ms = "k_pack", ab["pack"] / cfg.num_rounds, pack_gbs, pack_ms / cfg.num_rounds
    else:
        dom, dom_bytes, dom_gbs, dom_ms = ("k_combine", ab["combine"] / cfg.num_rounds, combine_gbs,
                                           combine_ms / cfg.num_rounds)
    clocks = sampler.summary(t_wall0, t_wall1)
    default_launch = (args.mode == "full" and not args.quant and not args.ue8m0 and not args.combine_quant
                      and not args.tokens and not args.gating)
    # routing (1 cooperative kernel) unless cached, pack x rounds, combine x rounds
    launches_per_step = (0 if args.mode == "cached" else 1) + 2 * cfg.num_rounds + (1 if args.gating else 0)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if q is None else f"bf16->{q}",
        "data": "synthetic (seeded numpy PCG64; no dataset, no weights)",
        "config": config_dict(args, cfg, world),
        "hbm": {"achieved_gbs": round(gbs, 1), "algorithmic_bytes_per_step": step_bytes,
                "frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4), "frac_of_measured": round(gbs / peak, 4),
                "measured_peak_gbs": peak, "rows": ab["rows"], "rows_aligned": ab["rows_aligned"],
                "bytes": {"gating": ab["gating"], "route": ab["route"], "pack": ab["pack"],
                          "combine": ab["combine"]}},
        "kernels": {"route_ms": round(route_ms, 5), "pack_ms": round(pack_ms, 5), "pack_gbs": round(pack_gbs, 1),
                    "combine_ms": round(combine_ms, 5), "combine_gbs": round(combine_gbs, 1),
                    "split_steps": n_split, "split_step_ms": round(split_step_ms, 5),
                    "note": "per-kernel CUDA events from a separate loop after the timed one; route_ms is "
                            "the memset + routing kernel up to the pack's start"},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak, "unit": "GB/s",
                     "peak_kind": peak_kind, "frac": round(dom_gbs / peak, 4),
                     "frac_of_8tbs": round(dom_gbs / NOMINAL_HBM_GBS, 4),
                     "step_frac_of_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
                     "algorithmic_bytes_per_launch": int(dom_bytes), "launch_ms": round(dom_ms, 5),
                     # the capture holds the workload's default launch only
                     "traffic": traffic_for(dom, args.workload) if default_launch else None},
        "e2e": {"value": round(job_tokens_per_s(world, T, e2e_ms / e2e_steps), 1), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": round(e2e_ms / e2e_steps, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, wl, step_bytes / T, budget_s=args.cpu_seconds,
                                              logits=logits.cpu().numpy() if args.gating else None)
    if rank == 0:
        print(json.dumps(result), flush=True)
    barrier(world)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------ oracle (CPU)

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSampler:
    """Runs the oracle, as it stands, on token samples of a workload: one
    sample = a smaller problem of the same shape (the same number of tokens
    from every source rank, their routing and rows), through slot assignment,
    dispatch rows and combine.  Rows are mapped into a pool of 8192 rows so
    that memory stays bounded; each token's arithmetic is unchanged."""

    POOL = 8192

    def __init__(self, cfg, wl, seed=0, logits=None):
        from combine_topk_idx_rank_b200.workloads import make_y
        self.cfg, self.wl = cfg, wl
        self.logits = logits            # router logits: the routing comes from group-limited gating
        self.ypool = make_y(self.POOL, cfg.hidden, 7)
        self.rng = np.random.default_rng(seed)

    def tokens(self, per_rank):
        cfg = self.cfg
        tpr = cfg.num_tokens // cfg.num_ranks
        per_rank = max(1, min(tpr, per_rank))
        picks = [r * tpr + np.sort(self.rng.choice(tpr, size=per_rank, replace=False))
                 for r in range(cfg.num_ranks)]
        return np.concatenate(picks).astype(np.int64)

    def run(self, tok):
        """Seconds the oracle takes for the sample `tok`."""
        import oracle
        cfg, wl = self.cfg, self.wl
        idx, w, x = wl.topk_idx[tok], wl.topk_weights[tok], wl.x[tok]
        lg = None if self.logits is None else self.logits[tok]
        t0 = time.perf_counter()
        if lg is not None:
            idx, w = oracle.group_limited_gating(lg, 32, 4, 2)
        s = oracle.slots(idx, w, cfg.num_experts, cfg.num_ranks, cfg.expert_alignment)
        dst = s["dst_buffer_slot_idx"]
        pdst = np.where(dst >= 0, dst % self.POOL, -1).astype(np.int32)
        oracle.dispatch_rows(x, pdst, cfg.quant, cfg.quant_size, cfg.round_scale, num_rows=self.POOL)
        oracle.combine_rows(self.ypool, pdst, w)
        return time.perf_counter() - t0

    def calibrate(self):
        """Seconds per token, from a sample of 8 tokens per rank."""
        tok = self.tokens(8)
        self.run(tok)
        return self.run(tok) / tok.size


def cpu_baseline(cfg, wl, bytes_per_token, budget_s=12.0, logits=None):
    """The oracle timed on this host's cores: the single-threaded build on one
    core, then the OpenMP build of the same source on every core in
    sched_getaffinity, each on measured token samples (no projection)."""
    import oracle
    smp = OracleSampler(cfg, wl, logits=logits)
    res = {}
    for label, n in (("one_core", 1), ("all_cores", host_cores())):
        used = oracle.use_threads(n)
        per_tok = smp.calibrate()
        per_rank = int(max(1, (budget_s / 2 / 3) / per_tok / cfg.num_ranks))
        secs, toks = 0.0, 0
        for _ in range(3):
            tok = smp.tokens(per_rank)
            secs += smp.run(tok)
            toks += tok.size
        res[label] = {"value": round(toks / secs, 2), "cores": used, "tokens": toks, "seconds": round(secs, 2),
                      "gbs": round(toks / secs * bytes_per_token / 1e9, 4)}
    oracle.use_threads(1)
    allc, one = res["all_cores"], res["one_core"]
    return {"value": allc["value"], "unit": UNIT, "cores": allc["cores"], "kind": "oracle",
            "gbs": allc["gbs"], "one_core": one,
            "sample": f"3 samples of {allc['tokens'] // 3} tokens (the same number from each of the "
                      f"{cfg.num_ranks} ranks, with their routing) through the oracle's slot assignment, "
                      f"dispatch rows and combine; all cores ({allc['cores']} threads, OpenMP build of the "
                      f"same source) {allc['seconds']} s; one core {one['value']} tokens/s over "
                      f"{one['tokens']} tokens ({one['seconds']} s); measured, not projected"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:       # under torchrun only rank 0 times the oracle
        return
    import oracle
    cfg = workload_config(args)
    wl = make_workload(cfg, seed=args.seed)
    T = cfg.num_tokens
    cores = host_cores()
    used = oracle.use_threads(cores)
    logits = make_router_logits(T, cfg.num_experts, args.seed) if getattr(args, "gating", False) else None
    smp = OracleSampler(cfg, wl, seed=args.seed, logits=logits)
    per_tok = smp.calibrate()
    n_steps = args.steps + args.warmup
    per_rank = int(max(1, (args.ref_seconds / n_steps) / per_tok / cfg.num_ranks))
    times, toks = [], []
    for i in range(n_steps):
        tok = smp.tokens(per_rank)
        dt = smp.run(tok)
        if i >= args.warmup:
            times.append(dt)
            toks.append(tok.size)
    oracle.use_threads(1)
    value = sum(toks) / sum(times)
    ms_per_step = 1e3 * sum(times) / len(times)
    per_step_tokens = toks[0]
    sample = (f"each step: the oracle (OpenMP build, {used} threads) on {per_step_tokens} tokens "
              f"({per_step_tokens // cfg.num_ranks} from each of the {cfg.num_ranks} ranks, with their routing): "
              f"slot assignment, dispatch rows and combine (rows mapped into an {OracleSampler.POOL}-row pool); "
              f"value = measured tokens / measured seconds")
    res = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.quant == "none" else f"bf16->{cfg.quant}",
           "data": "synthetic (seeded numpy PCG64; no dataset, no weights)", "impl": "reference",
           "config": config_dict(args, cfg, world),
           "tokens_per_step": per_step_tokens,
           "projected_full_workload_ms": round(1e3 * T / value, 1),
           "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": used, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


# ------------------------------------------------------------- launcher

def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(n: int, argv, timeout_s: float = 3600.0) -> int:
    """Starts n copies of this script, one per GPU, with the environment
    torchrun gives (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR 127.0.0.1,
    MASTER_PORT); rank 0's output is this process's output.  Returns the
    first non-zero exit code, else 0."""
    port = free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__), *argv], env=env,
                                      stdout=None if r == 0 else subprocess.DEVNULL))
    rc = 0
    deadline = time.time() + timeout_s
    for p in procs:
        try:
            code = p.wait(timeout=max(1.0, deadline - time.time()))
        except subprocess.TimeoutExpired:
            for q in procs:
                if q.poll() is None:
                    q.kill()
            code = 124
        if code and not rc:
            rc = code
    return rc


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="prefill", choices=list(CONFIGS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--tokens", type=int, default=0, help="scale the workload to this many tokens")
    p.add_argument("--mode", default="full", choices=["full", "cached", "ll"],
                   help="cached: dispatch re-packing with a handle (routing computed once); "
                        "ll: low-latency fixed-capacity layout")
    p.add_argument("--quant", default=None, choices=["none", "fp8", "int8", "mxfp4"],
                   help="override the workload's dispatch quantisation")
    p.add_argument("--ue8m0", action="store_true", help="power-of-two scales stored as UE8M0 bytes")
    p.add_argument("--combine-quant", action="store_true",
                   help="combine reads the FP8 / int8 received rows (identity experts) instead of bf16 y")
    p.add_argument("--gating", action="store_true",
                   help="each step starts from router logits: group-limited gating, then dispatch and combine")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the cpu_baseline samples")
    p.add_argument("--ref-seconds", type=float, default=60.0, help="budget of the --impl reference run")
    p.add_argument("--no-cpu-baseline", action="store_true")
    argv = sys.argv[1:] if argv is None else list(argv)
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU, as torchrun would start them
        raise SystemExit(launch_ranks(args.gpus, argv))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
