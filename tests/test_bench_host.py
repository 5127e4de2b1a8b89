"""Host arithmetic of bench.py (CPU): the algorithmic bytes and flops the
roofline divides by, checked against counts written out independently."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import mla_workloads as W  # noqa: E402


def _inp(lens, s_q, h_q, h_kv, causal):
    return dict(cache_seqlens=np.asarray(lens, dtype=np.int32), s_q=s_q, h_q=h_q, h_kv=h_kv,
                batch=len(lens), causal=causal)


def _visible_pairs(lens, s_q, causal):
    # (query token, cached token) pairs, counted one by one from the mask rule:
    # query i sees token j iff j <= L - s_q + i (causal) or j < L
    n = 0
    for L in lens:
        for i in range(s_q):
            for j in range(L):
                n += (j <= L - s_q + i) if causal else 1
    return n


def test_work_counts_non_causal():
    wc = bench.work_counts(_inp([37, 130], 1, 16, 1, False))
    assert wc["kv_bytes"] == 167 * 576 * 2
    assert wc["tokens"] == 167
    assert wc["flops"] == 2 * (576 + 512) * 16 * 167
    assert wc["bytes"] == wc["kv_bytes"] + 2 * 1 * 16 * (576 * 2 + 512 * 2 + 4)


def test_work_counts_causal_and_grouped_heads():
    lens, s_q, h_q, h_kv = [1, 5, 64, 0, 3], 3, 32, 2
    wc = bench.work_counts(_inp(lens, s_q, h_q, h_kv, True))
    assert wc["flops"] == 2 * (576 + 512) * h_q * _visible_pairs(lens, s_q, True)
    assert wc["kv_bytes"] == sum(lens) * h_kv * 576 * 2   # each KV head's rows read once


def test_uniform_workload_roofline_figures():
    # batch 64 x 4096 tokens, 128 heads: 302.0 MB of KV, 319.8 MB in all, 73.0 GF
    inp = W.make_inputs(W.WORKLOADS["uniform"])
    wc = bench.work_counts(inp)
    assert wc["kv_bytes"] == 64 * 4096 * 1152
    assert wc["bytes"] == 64 * 4096 * 1152 + 64 * 128 * (1152 + 1024 + 4)
    assert round(wc["flops"] / 1e9, 1) == 73.0
    t, bound = bench.roofline_time(wc, {"hbm_gbs": 6551.4, "bf16_tflops": 1636.8, "bf16_tflops_sustained": 1388.9})
    assert bound == "hbm" and abs(t * 1e6 - 48.82) < 0.01


def test_roofline_picks_the_slower_unit():
    wc = dict(bytes=1e9, flops=1e15)
    t, bound = bench.roofline_time(wc, {"hbm_gbs": 1000.0, "bf16_tflops": 1000.0, "bf16_tflops_sustained": 500.0})
    assert bound == "tensor" and abs(t - 1.0) < 1e-12
    t, bound = bench.roofline_time(wc, {"hbm_gbs": 0.5, "bf16_tflops": 1000.0, "bf16_tflops_sustained": 500.0})
    assert bound == "hbm" and abs(t - 2.0) < 1e-12
