"""The benchmark's algorithmic work per step (the numerators of every roofline fraction it reports)
against figures fixed independently of its code: the FLOP counts and FP8 weight bytes of the workloads,
worked out from their sizes (T, H, E, I, k) as products, and the 4-bit format's half-byte levels. A wrong
factor (a dropped 2 for multiply-add, I in place of 2I, weights counted per slot instead of per touched
expert) fails one of them."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS  # noqa: E402

# (workload, router GFLOP, up GFLOP, down GFLOP, FP8 weight bytes of all E experts without scales; four
# significant figures), every expert keeping T k / E rows (decode: 1024 slots over all 256 experts, 4 each)
FIXED = [
    ("page", 2.147, 274.9, 137.4, 1.611e9),
    ("prefill", 30.06, 3848.3, 1924.1, 11.27e9),
    ("decode", 0.470, 60.13, 30.06, 11.27e9),
]


@pytest.mark.parametrize("name,router,up,down,wbytes", FIXED)
def test_work_matches_the_sizes(name, router, up, down, wbytes):
    cfg = CONFIGS[name]
    kept = np.full(cfg.E, cfg.T * cfg.k // cfg.E, np.int64)
    work, Rk, touched = bench.algorithmic_work(cfg, kept)
    assert Rk == cfg.T * cfg.k and touched == cfg.E
    assert work["router"]["flops"] / 1e9 == pytest.approx(router, rel=1e-3)
    assert work["gemm_up"]["flops"] / 1e9 == pytest.approx(up, rel=5e-4)
    assert work["gemm_down"]["flops"] / 1e9 == pytest.approx(down, rel=5e-4)
    H, I = cfg.H, cfg.I
    # the weights dominate the GEMMs' bytes; the rest is the activations in and out, whose sizes are
    # exact: up reads x codes + 1x128 scales and writes h codes + scales, down reads h and writes bf16 o
    act_up = Rk * (H + 4 * H // 128) + Rk * (I + 4 * I // 128)
    act_down = Rk * (I + 4 * I // 128) + Rk * H * 2
    w_up = work["gemm_up"]["bytes"] - act_up
    w_down = work["gemm_down"]["bytes"] - act_down
    scales = 4 * cfg.E * ((2 * I // 128) * (H // 128) + (H // 128) * (I // 128))
    assert w_up + w_down - scales == pytest.approx(wbytes, rel=2e-3)
    assert w_up == 2 * (w_down - 4 * cfg.E * (H // 128) * (I // 128)) + 4 * cfg.E * (2 * I // 128) * (H // 128)


def test_only_touched_experts_stream_their_weights():
    cfg = CONFIGS["decode"]
    kept = np.zeros(cfg.E, np.int64)
    kept[:3] = [5, 0, 7]                       # two experts touched
    work, Rk, touched = bench.algorithmic_work(cfg, kept)
    assert (Rk, touched) == (12, 2)
    per_expert = 3 * cfg.H * cfg.I                                           # W1, W3, W2 codes
    per_scales = 4 * (2 * (cfg.I // 128) * (cfg.H // 128) + (cfg.H // 128) * (cfg.I // 128))
    act = 12 * (cfg.H + 4 * cfg.H // 128) + 2 * 12 * (cfg.I + 4 * cfg.I // 128) + 12 * cfg.H * 2
    assert work["gemm_up"]["bytes"] + work["gemm_down"]["bytes"] == 2 * (per_expert + per_scales) + act


def test_four_bit_weights_halve_the_codes():
    fp8, w4 = CONFIGS["decode"], CONFIGS["decode_w4"]
    kept = np.full(fp8.E, 4, np.int64)
    a, _, _ = bench.algorithmic_work(fp8, kept)
    b, _, _ = bench.algorithmic_work(w4, kept)
    H, I, E = fp8.H, fp8.I, fp8.E
    codes = lambda w: w["gemm_up"]["bytes"] + w["gemm_down"]["bytes"]
    # codes: half a byte per weight instead of one; scales: one fp32 per row per 128 k instead of one per
    # 128 x 128 block
    fp8_scales = 4 * E * (2 * (I // 128) * (H // 128) + (H // 128) * (I // 128))
    w4_scales = 4 * E * (2 * I * (H // 128) + H * (I // 128))
    assert codes(a) - codes(b) == 3 * E * H * I // 2 + fp8_scales - w4_scales
    assert a["gemm_up"]["flops"] == b["gemm_up"]["flops"]


def test_hash_routing_has_no_router_flops():
    cfg = CONFIGS["decode_hash"]
    kept = np.zeros(cfg.E, np.int64)
    kept[:128] = 1
    work, _, _ = bench.algorithmic_work(cfg, kept)
    assert work["router"]["flops"] == 0.0
    assert work["router"]["bytes"] == cfg.T * 4 + cfg.T * cfg.k * 8
