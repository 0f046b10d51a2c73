"""The seeded input generators produce the workloads' stated structure."""
import numpy as np
import pytest

from combine_topk_idx_rank_b200.workloads import CONFIGS, bf16_bits_to_f32, make_workload


@pytest.mark.parametrize("name", list(CONFIGS))
def test_shapes_and_distinct_experts(name):
    cfg = CONFIGS[name]
    T = min(cfg.num_tokens, 2048)
    wl = make_workload(cfg.scaled(num_tokens=T, hidden=256 if cfg.quant_size != cfg.hidden else None),
                       seed=0)
    assert wl.topk_idx.shape == (T, cfg.num_topk) and wl.topk_idx.dtype == np.int64
    assert wl.topk_weights.dtype == np.float32 and wl.x.dtype == np.uint16
    valid = wl.topk_idx >= 0
    assert np.all(wl.topk_idx[valid] < cfg.num_experts)
    for row in wl.topk_idx:
        v = row[row >= 0]
        assert np.unique(v).size == v.size
    assert np.all(wl.topk_weights[~valid] == 0)
    assert np.all(wl.topk_weights.sum(1) <= 1 + 1e-5)
    if cfg.mask_frac == 0:
        assert valid.all()
        assert np.allclose(wl.topk_weights.sum(1), 1, atol=1e-5)
    xf = bf16_bits_to_f32(wl.x)
    assert abs(xf.std() - cfg.x_sigma) < 0.05 * cfg.x_sigma


def test_mask_fraction():
    wl = make_workload(CONFIGS["qwen3"], seed=0, with_x=False)
    frac = (wl.topk_idx < 0).mean()
    n = wl.topk_idx.size
    assert abs(frac - 0.1) < 4 * np.sqrt(0.09 / n)


def test_zipf_popularity_is_skewed_and_uniform_is_flat():
    wl = make_workload(CONFIGS["prefill"], seed=0, with_x=False)
    cnt = np.bincount(wl.topk_idx.ravel(), minlength=256)
    srt = np.sort(cnt)[::-1]
    assert srt[0] > 20 * srt[-1]                     # heavy head, thin tail
    assert srt[0] <= 32768                           # at most one row per token
    wu = make_workload(CONFIGS["decode"], seed=0, with_x=False)
    cu = np.bincount(wu.topk_idx.ravel(), minlength=256)
    mean = cu.mean()
    assert np.all(np.abs(cu - mean) < 6 * np.sqrt(mean))


def test_deterministic_per_seed():
    cfg = CONFIGS["tiny"]
    a, b, c = make_workload(cfg, 0), make_workload(cfg, 0), make_workload(cfg, 1)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.topk_idx, b.topk_idx)
    assert not np.array_equal(a.topk_idx, c.topk_idx)
