"""Seeded synthetic inputs for MoE expert-parallel dispatch / combine.

This module only draws random inputs; it holds none of the dispatch / combine
arithmetic, so both the CPU oracle and the CUDA path can be fed from it.

The five workloads mirror the shapes the DeepEP pages discuss:

* ``tiny``     -- a small smoke case (256 tokens, hidden 512, 16 experts over
                  8 ranks, top-2, bf16).
* ``decode``   -- DeepSeek-V3 decode shape: 16 ranks x 128 tokens, hidden 7168,
                  256 experts, top-8 uniform, FP8 e4m3 group-128 dispatch.
* ``prefill``  -- DeepSeek-V3 prefill shape: 8 ranks x 4096 tokens, hidden 7168,
                  256 experts, top-8 with Zipf(1.2) expert popularity,
                  expert_alignment 128, bf16 dispatch and combine.
* ``qwen3``    -- Qwen3-30B-A3B EP16 shape (the model of the EFA frameworks
                  page): 16 ranks x 512 tokens, hidden 2048, 128 experts, top-8
                  uniform, 10% of top-k entries masked to -1, FP8 group-128
                  dispatch with power-of-two (ue8m0) scales.
* ``longseq``  -- the Ascend "ant moving home" long-sequence case: 65536 tokens
                  over 8 ranks in 8 rounds, hidden 7168, x ~ N(0, 2), Zipf(1.0)
                  routing, int8 per-token dispatch.

Recipe (every draw from one ``numpy.random.default_rng(seed)``, PCG64, in this
order): the expert permutation (Zipf workloads only), the routing keys
(T x E uniforms), the gate logits (T x K standard normals), the mask uniforms
(masked workloads only), then x (T x H normals, fp32, rounded to bf16
round-to-nearest-even).  Top-k selection is Gumbel-top-k: expert e gets key
log p_e + Gumbel noise and the K largest keys are taken in descending order,
which samples K distinct experts without replacement from p.  Uniform routing
has p_e = 1/E; Zipf(s) has p_e proportional to 1 / (pi(e) + 1)^s for a seeded
permutation pi.  topk_weights are the fp32 softmax of the K gate logits;
masked entries get topk_idx = -1 and weight 0 after the softmax.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = ["WorkloadConfig", "CONFIGS", "Workload", "make_workload", "make_y", "make_router_logits",
           "bf16_bits_from_f32", "bf16_bits_to_f32"]


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    num_tokens: int          # T, total over all logical ranks
    hidden: int              # H
    num_ranks: int           # R
    num_experts: int         # E
    num_topk: int            # K
    expert_alignment: int    # A
    quant: str               # "none" | "fp8" | "int8"
    quant_size: int          # 128 (group) or hidden (per token); ignored for "none"
    round_scale: bool        # power-of-two (ue8m0) scales
    routing: str             # "uniform" | "zipf"
    zipf_s: float = 0.0
    mask_frac: float = 0.0
    x_sigma: float = 1.0
    num_rounds: int = 1

    def scaled(self, num_tokens: Optional[int] = None, hidden: Optional[int] = None,
               **kw) -> "WorkloadConfig":
        """A copy with a smaller token count / hidden size (for fast tests)."""
        d = dataclasses.asdict(self)
        if num_tokens is not None:
            d["num_tokens"] = num_tokens
        if hidden is not None:
            d["hidden"] = hidden
            if self.quant_size == self.hidden:
                d["quant_size"] = hidden
        d.update(kw)
        return WorkloadConfig(**d)


CONFIGS: Dict[str, WorkloadConfig] = {
    "tiny": WorkloadConfig("tiny", 256, 512, 8, 16, 2, 1, "none", 128, False, "uniform"),
    "decode": WorkloadConfig("decode", 2048, 7168, 16, 256, 8, 1, "fp8", 128, False, "uniform"),
    "prefill": WorkloadConfig("prefill", 32768, 7168, 8, 256, 8, 128, "none", 128, False,
                              "zipf", zipf_s=1.2),
    "qwen3": WorkloadConfig("qwen3", 8192, 2048, 16, 128, 8, 1, "fp8", 128, True, "uniform",
                            mask_frac=0.1),
    "longseq": WorkloadConfig("longseq", 65536, 7168, 8, 256, 8, 1, "int8", 7168, False,
                              "zipf", zipf_s=1.0, x_sigma=2.0, num_rounds=8),
}


@dataclasses.dataclass
class Workload:
    cfg: WorkloadConfig
    seed: int
    x: np.ndarray              # uint16 [T, H], bf16 bit patterns
    topk_idx: np.ndarray       # int64 [T, K], -1 = masked
    topk_weights: np.ndarray   # float32 [T, K]


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (inputs are finite)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _topk_desc(keys: np.ndarray, k: int) -> np.ndarray:
    part = np.argpartition(-keys, k - 1, axis=1)[:, :k]
    sel = np.take_along_axis(keys, part, axis=1)
    order = np.argsort(-sel, axis=1, kind="stable")
    return np.take_along_axis(part, order, axis=1)


def make_workload(cfg: WorkloadConfig, seed: int = 0, with_x: bool = True) -> Workload:
    T, H, E, K = cfg.num_tokens, cfg.hidden, cfg.num_experts, cfg.num_topk
    rng = np.random.default_rng(seed)
    if cfg.routing == "zipf":
        perm = rng.permutation(E)
        logp = -cfg.zipf_s * np.log(perm.astype(np.float64) + 1.0)
    elif cfg.routing == "uniform":
        logp = np.zeros(E, dtype=np.float64)
    else:
        raise ValueError(cfg.routing)
    u = rng.random((T, E))
    keys = logp[None, :] - np.log(-np.log(np.clip(u, 1e-300, None)))
    topk_idx = _topk_desc(keys, K).astype(np.int64)
    del keys, u
    logits = rng.standard_normal((T, K), dtype=np.float32)
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    topk_weights = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    if cfg.mask_frac > 0:
        m = rng.random((T, K)) < cfg.mask_frac
        topk_idx[m] = -1
        topk_weights[m] = 0.0
    if with_x:
        xf = rng.standard_normal((T, H), dtype=np.float32)
        if cfg.x_sigma != 1.0:
            xf *= np.float32(cfg.x_sigma)
        x = bf16_bits_from_f32(xf)
        del xf
    else:
        x = np.zeros((0, H), dtype=np.uint16)
    return Workload(cfg, seed, x, np.ascontiguousarray(topk_idx),
                    np.ascontiguousarray(topk_weights))


def make_y(rows: int, hidden: int, seed: int, device: str = "cpu"):
    """Expert outputs y ~ N(0, 1) in bf16, [rows, hidden].

    On "cpu" returns numpy uint16 bit patterns drawn with PCG64; on a CUDA
    device returns a torch bf16 tensor drawn with torch's seeded generator
    (large sizes are generated in place on the device).
    """
    if device == "cpu":
        rng = np.random.default_rng(seed + 0x5EED)
        return bf16_bits_from_f32(rng.standard_normal((rows, hidden), dtype=np.float32))
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed + 0x5EED)
    return torch.randn((rows, hidden), generator=g, device=device, dtype=torch.bfloat16)


def make_router_logits(tokens: int, experts: int, seed: int) -> np.ndarray:
    """Router logits fp32 [tokens, experts] ~ N(0, 1) from PCG64 (seed + 0x6A7E),
    the input of the group-limited gating generator."""
    rng = np.random.default_rng(seed + 0x6A7E)
    return rng.standard_normal((tokens, experts), dtype=np.float32)
