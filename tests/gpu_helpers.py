"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.build import build
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, MoeInputs, interleave_w13, interleave_w13_w4, make_inputs

# Tolerances on bf16 outputs (the layer's stated bar): max_i |y_i - r_i| / max(|r_i|, rms(r))
# and sum |y - r| / sum |r|. The denominator floor rms(r) keeps the element-wise ratio finite
# near zero.
MAX_REL = 2e-2
MEAN_REL = 2e-3
W_RTOL = 1e-6        # router weights: fp64 on both sides, rounded to fp32


def bits_to_f64(bits) -> np.ndarray:
    if isinstance(bits, torch.Tensor):
        bits = bits.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    return oracle.bf16_bits_to_f32(bits).astype(np.float64)


def rel_errors(y, r):
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    rms = np.sqrt(np.mean(r * r)) if r.size else 0.0
    den = np.maximum(np.abs(r), rms)
    diff = np.abs(y - r)
    max_rel = float(np.max(diff / np.where(den > 0, den, 1.0))) if r.size else 0.0
    mean_rel = float(diff.sum() / max(np.abs(r).sum(), 1e-300)) if r.size else 0.0
    return max_rel, mean_rel


def assert_close_bf16(y_gpu_bits, y_ref_bits, what="y"):
    y, r = bits_to_f64(y_gpu_bits), bits_to_f64(y_ref_bits)
    max_rel, mean_rel = rel_errors(y, r)
    assert max_rel <= MAX_REL and mean_rel <= MEAN_REL, f"{what}: max_rel {max_rel:.3e} mean_rel {mean_rel:.3e}"
    return max_rel, mean_rel


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class LazyExperts:
    """Expert-indexed view of a (possibly device-resident) weight tensor that
    copies one expert to host memory when the oracle asks for it."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].detach().cpu().numpy()


def oracle_inputs(inp: MoeInputs) -> dict:
    return dict(x=to_np(inp.x), Wg=to_np(inp.Wg), bias=to_np(inp.bias), token_ids=to_np(inp.token_ids),
                W1q=LazyExperts(inp.W1q), S1=LazyExperts(inp.S1), W3q=LazyExperts(inp.W3q),
                S3=LazyExperts(inp.S3), W2q=LazyExperts(inp.W2q), S2=LazyExperts(inp.S2))


def ensure_lib():
    build()
    return api.lib()


def gpu_inputs(cfg: MoeConfig, T=None, on_device: bool = False) -> MoeInputs:
    """Small workloads are drawn on the host and copied; full-size ones are drawn
    directly on the device (same generator module, device RNG)."""
    if on_device:
        return make_inputs(cfg, device="cuda", T=T)
    return make_inputs(cfg, device="cpu", T=T).to("cuda")


def gpu_forward(cfg: MoeConfig, inp: MoeInputs) -> dict:
    c = api.Config.from_moe(cfg)
    dev = inp.x.device
    W13, S13 = (interleave_w13_w4 if cfg.weights == "w4" else interleave_w13)(inp.W1q, inp.S1, inp.W3q, inp.S3)
    T, k, H, E = cfg.T, cfg.k, cfg.H, cfg.E
    out = dict(
        y=torch.empty(T, H, dtype=torch.bfloat16, device=dev),
        topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
        topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
        counts=torch.empty(E, dtype=torch.int32, device=dev),
        slot_row=torch.empty(T * k, dtype=torch.int32, device=dev))
    ws = torch.empty(api.moe_workspace_size(c, True), dtype=torch.uint8, device=dev)
    api.moe_forward(c, inp.x, inp.Wg, inp.bias, inp.token_ids, W13, S13, inp.W2q, inp.S2, out["y"],
                    out["topk_idx"], out["topk_w"], out["counts"], out["slot_row"], ws)
    torch.cuda.synchronize()
    st = api.moe_get_device_status()
    assert st == api.MOE_OK, api.STATUS_NAMES.get(st)
    return out


def tile_covering_tokens(layout: str, slot_row: np.ndarray, k: int, seed: int = 0):
    """Tokens whose kept rows touch every tile the grouped GEMMs schedule.

    Contiguous layout: a tile is a 128-row M tile of the padded, expert-contiguous rows (every
    group starts on a multiple of 128, so a tile belongs to one expert; its N tiles are all
    covered by comparing whole rows). Masked layout: a tile is a 32-token slice of an expert's
    block (the swap-AB kernel's N tile). `slot_row` is the oracle's own slot -> row map. Tiles
    are visited in a seeded random order; for an uncovered tile one of its rows is picked,
    preferring the 32-row quadrant i % 4 (i = the tile's visit index) so that every promotion
    warp's lane quadrant is exercised, and among those the token that reaches the most uncovered
    tiles; every tile the token reaches is then marked.
    Returns (sorted tokens, number of tiles, number covered)."""
    slot_row = np.asarray(slot_row, np.int64)
    T = slot_row.size // k
    span = 128 if layout == "contiguous" else 32
    kept = np.nonzero(slot_row >= 0)[0]
    rows = slot_row[kept]
    tiles = rows // span
    by_tile = {}
    for r, s_, tl in zip(rows, kept, tiles):
        by_tile.setdefault(int(tl), []).append((int(r), int(s_ // k)))
    rng = np.random.default_rng(seed)
    order = rng.permutation(np.array(sorted(by_tile), dtype=np.int64))
    per_token = slot_row.reshape(T, k)
    covered, chosen = set(), []
    for i, tl in enumerate(order):
        tl = int(tl)
        if tl in covered:
            continue
        cand = by_tile[tl]
        quad = [c for c in cand if (c[0] % span) // 32 == i % 4] if span == 128 else []
        pool = quad or cand
        # of the candidates, the token whose kept rows reach the most tiles not yet covered
        gain = [len({int(r) // span for r in per_token[c[1]] if r >= 0} - covered) for c in pool]
        t = pool[int(np.argmax(gain))][1]
        chosen.append(t)
        covered.update(int(r) // span for r in per_token[t] if r >= 0)
    return np.array(sorted(set(chosen)), dtype=np.int64), len(by_tile), len(covered & set(by_tile))
