"""Host-side logic of bench.py that needs no GPU: step-time percentiles, the
prefill line's algorithmic work per kernel, the CUDA-core peak it is held to."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from compressed_sparse_attention_compressor_b200 import workloads as Wk  # noqa: E402


def test_step_stats_percentiles():
    st = bench.step_stats([5.0] * 9 + [50.0])
    assert st["median_ms"] == 5.0 and st["p10_ms"] == 5.0 and 5.0 < st["p90_ms"] <= 50.0
    assert bench.step_stats([]) is None
    v = np.arange(1, 101, dtype=float)
    st = bench.step_stats(v)
    assert abs(st["median_ms"] - 50.5) < 1e-9 and st["p10_ms"] < st["median_ms"] < st["p90_ms"]


def test_prefill_work_matches_the_published_flop_counts():
    # 4,096 queries after 131,072 cached tokens (m = 4): 32,768 .. 33,791
    # visible entries each; 2 x 64 heads x 128 dims flops per entry and query
    wl = Wk.WORKLOADS["prefill"]
    pos = np.arange(wl.context, wl.context + wl.chunk)
    n_vis = (pos + 1) // wl.m
    sum_vis = float(n_vis.sum())
    sum_keys = float(np.minimum(n_vis, wl.topk).sum() + np.minimum(pos + 1, wl.window).sum())
    f_idx, k_idx = bench.prefill_kernel_work("index_score_simt_kernel", wl, sum_vis, sum_keys)
    f_att, k_att = bench.prefill_kernel_work("attn_simt_kernel", wl, sum_vis, sum_keys)
    assert k_idx == "alu" and abs(f_idx / 1e12 - 2.2334) < 1e-3
    assert k_att == "alu" and abs(f_att / 1e12 - 0.3436) < 1e-3  # 4,096 x 640 keys x 64 x 512 x 4
    assert bench.prefill_kernel_work("attn_tc_split_kernel", wl, sum_vis, sum_keys)[1] == "tensor"
    assert bench.prefill_kernel_work("topk_row_kernel", wl, sum_vis, sum_keys) == (4.0 * sum_vis, "hbm")
    assert bench.prefill_kernel_work("something_else", wl, sum_vis, sum_keys) == (None, None)


def test_alu_peak_is_lanes_times_clock():
    # 148 SMs x 128 fp32 lanes x 2 flops (FMA) at the recorded maximum clock
    peak = bench.alu_peak_tflops(148)
    assert 60.0 < peak < 80.0
    assert abs(bench.alu_peak_tflops(74) * 2 - peak) < 1e-9
