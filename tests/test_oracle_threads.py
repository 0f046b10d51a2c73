"""The oracle's OpenMP build (same source, token loops split across threads)
gives the single-threaded build's results byte for byte, for every row
function: bf16 / FP8 / int8 / MXFP4 dispatch rows, and the bf16 and quantised
combines with a shared expert."""
import numpy as np
import pytest

import oracle
from combine_topk_idx_rank_b200.workloads import CONFIGS, make_workload, make_y


@pytest.fixture
def threaded():
    yield
    oracle.use_threads(1)


@pytest.mark.parametrize("name", ["tiny", "decode", "qwen3", "longseq"])
def test_threaded_rows_equal_single_threaded(name, threaded):
    cfg = CONFIGS[name].scaled(num_tokens=CONFIGS[name].num_ranks * CONFIGS[name].num_rounds * 8,
                               hidden=512 if CONFIGS[name].hidden > 512 else None)
    wl = make_workload(cfg, seed=3)
    s = oracle.slots(wl.topk_idx, wl.topk_weights, cfg.num_experts, cfg.num_ranks, cfg.expert_alignment)
    dst, n = s["dst_buffer_slot_idx"], s["num_recv_rows"]
    y = make_y(n, cfg.hidden, 5)
    shared = make_y(cfg.num_tokens, cfg.hidden, 6)

    def run():
        rx, rs = oracle.dispatch_rows(wl.x, dst, cfg.quant, cfg.quant_size, cfg.round_scale, num_rows=n)
        mx = oracle.dispatch_rows_mx(wl.x, dst, "mxfp4", 32, num_rows=n)
        out = oracle.combine_rows(y, dst, wl.topk_weights)
        q = "int8" if cfg.quant == "int8" else "fp8"
        cx, cs = oracle.dispatch_rows(wl.x, dst, q, 128, False, num_rows=n)
        outq = oracle.combine_rows_q(cx, cs, q, 128, dst, wl.topk_weights, shared=shared)
        return [rx, rs, mx[0], mx[1], out, cx, cs, outq]

    one = run()
    assert oracle.use_threads(4) >= 1 and oracle.threads() == 4
    many = run()
    for a, b in zip(one, many):
        if a is None:
            assert b is None
        else:
            assert np.array_equal(np.ascontiguousarray(a).view(np.uint8), np.ascontiguousarray(b).view(np.uint8))


def test_threaded_build_reports_errors(threaded):
    oracle.use_threads(4)
    dst = np.array([[0, 5]], np.int32)
    with pytest.raises(oracle.OracleError) as e:
        oracle.dispatch_rows(np.zeros((1, 16), np.uint16), dst, num_rows=3)
    assert e.value.status == oracle.CAPACITY
