"""Diagnostic of the fixed fp32 logit order (test infrastructure, oracle side only).

The pages fix no summation order for the router's logits; the build fixes one fp32 order so that expert
selection is reproducible bit for bit. This script measures what that choice costs against exact
arithmetic: for each workload's router inputs it counts the tokens whose top-k set differs between the
oracle's canonical fp32 logits (orc_router_logits) and fp64 logits (x and W_g exact in fp64, one fp64
matrix product, bias added in fp64), and the tokens whose fp64 top-k margin (k-th minus (k+1)-th
logit) is below a bound on the fp32 rounding error of the canonical order.

    python oracle/router_fp64_diagnostic.py [workload ...]

Inputs are drawn by the workloads' recipe on the host (make_router_inputs).
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402


def topk_sets(logits: np.ndarray, k: int) -> np.ndarray:
    # k largest per row, ties to the lower index (stable sort of the negated values)
    return np.sort(np.argsort(-logits, axis=1, kind="stable")[:, :k], axis=1)


def diagnose(cfg, x_bits: np.ndarray, Wg: np.ndarray, bias: np.ndarray) -> dict:
    l32 = oracle.router_logits(x_bits, Wg, bias)
    x64 = oracle.bf16_bits_to_f32(x_bits).astype(np.float64)
    l64 = x64 @ Wg.astype(np.float64).T + bias.astype(np.float64)
    k = cfg.k
    differ = np.any(topk_sets(l32, k) != topk_sets(l64, k), axis=1)
    # fp32 error bound of one canonical logit: each chain of H/32 multiply-adds and the 5-level tree,
    # about (H/32 + 5) roundings of magnitude sum_h |x_h w_h| * 2^-24
    absdot = np.abs(x64) @ np.abs(Wg.astype(np.float64)).T
    bound = (x64.shape[1] / 32 + 6) * 2.0 ** -24 * absdot
    s64 = np.sort(l64, axis=1)[:, ::-1]
    margin = s64[:, k - 1] - s64[:, k] if k < l64.shape[1] else np.full(l64.shape[0], np.inf)
    kth = np.argsort(-l64, axis=1, kind="stable")
    b_pair = np.maximum(bound[np.arange(len(bound)), kth[:, k - 1]],
                        bound[np.arange(len(bound)), kth[:, min(k, l64.shape[1] - 1)]])
    near = margin <= 2 * b_pair
    return {"T": int(x_bits.shape[0]), "differ": int(differ.sum()), "near_ties": int(near.sum()),
            "differ_frac": float(differ.mean()), "near_frac": float(near.mean()),
            "differ_within_near": bool(np.all(near[differ]))}


def main(names):
    from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, make_router_inputs
    for name in names:
        cfg = CONFIGS[name]
        if cfg.routing == "hash":
            continue
        x, Wg, bias = make_router_inputs(cfg)
        d = diagnose(cfg, x.view(__import__("torch").int16).numpy().view(np.uint16), Wg.numpy(), bias.numpy())
        print(f"{name:8s} T={d['T']:6d} top-k differs fp32 vs fp64: {d['differ']:5d} ({d['differ_frac']:.2e}); "
              f"margin below 2x the fp32 error bound: {d['near_ties']:5d} ({d['near_frac']:.2e}); "
              f"every difference is a near tie: {d['differ_within_near']}", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["tiny", "page", "prefill", "decode", "skewed"])
