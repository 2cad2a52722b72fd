"""Seeded synthetic inputs for the FP8 MoE expert layer.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It draws random data and lays it out; it holds none of the
layer's arithmetic (routing, permutation, GEMM, SwiGLU, combine). The setup
arithmetic here is the offline quantisation of the expert weights, to E4M3
with one fp32 scale per 128x128 block (and, as a second format, to 4-bit
levels with one scale per row per 128 k, quantize_weight_int4): the layer receives its
weights already quantised (DeepGEMM's grouped call takes FP8 operands plus
fine-grained scales; discosf.com "MegaMoE ... DeepGEMM" page, sections 3.2-3.3;
DeepSeek open-source week page, "Day 3"), so weight quantisation is not a step
of the path. It uses torch's own float8_e4m3fn cast (a library routine).

Workloads (sizes from the workload list this build is measured on):

==========  =====  ====  ===  ====  ===  ==================================
name        T      H     E    I     k    notes
==========  =====  ====  ===  ====  ===  ==================================
tiny        256    512   8    256   2    bias 0, seed 0
page        4096   4096  64   2048  2    bias U[-0.01,0.01], seed 1
prefill     8192   7168  256  2048  8    bias U[-0.01,0.01], seed 2
decode      128    7168  256  2048  8    masked layout, Mmax=128, seed 3
decode_hash 128    7168  256  2048  1    hash routing, token ids U[0,102400)
skewed      16384  4096  64   1408  2    Zipf(1.1) log-prior bias, capacity
                                         ceil(T*k/E)*5/4 (=640), seed 4
==========  =====  ====  ===  ====  ===  ==================================

Value distributions: x ~ N(0,1) drawn in fp32 and rounded to bf16;
W_g ~ N(0, 0.02) fp32; expert weights W1, W3, W2 ~ N(0, 0.02) fp32 before
quantisation. The uniform bias range [-0.01, 0.01] is the initial bias range
the MegaMoE page recommends (section 2.2). The skewed workload's bias is the
log of a Zipf(s=1.1) prior over experts, b_e = ln(p_e), p_e ~ (e+1)^-1.1.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

FP8_MAX = 448.0
BLOCK = 128


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    H: int
    E: int
    I: int
    k: int
    routing: str = "softmax"          # "softmax" | "hash"
    bias: str = "zero"                # "zero" | "uniform" | "zipf"
    layout: str = "contiguous"        # "contiguous" | "masked"
    cap_num: int = 0                  # capacity factor alpha = cap_num / cap_den; 0/0 = dropless
    cap_den: int = 0
    masked_max_m: int = 0
    seed: int = 0
    weights: str = "fp8"              # "fp8" (E4M3, 128x128 block scales) | "w4" (4-bit levels, row scales)

    def replace(self, **kw) -> "MoeConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": MoeConfig("tiny", T=256, H=512, E=8, I=256, k=2, bias="zero", seed=0),
    "page": MoeConfig("page", T=4096, H=4096, E=64, I=2048, k=2, bias="uniform", seed=1),
    "prefill": MoeConfig("prefill", T=8192, H=7168, E=256, I=2048, k=8, bias="uniform", seed=2),
    "decode": MoeConfig("decode", T=128, H=7168, E=256, I=2048, k=8, bias="uniform",
                        layout="masked", masked_max_m=128, seed=3),
    "decode_hash": MoeConfig("decode_hash", T=128, H=7168, E=256, I=2048, k=1, routing="hash",
                             layout="masked", masked_max_m=128, seed=3),
    "skewed": MoeConfig("skewed", T=16384, H=4096, E=64, I=1408, k=2, bias="zipf",
                        cap_num=5, cap_den=4, seed=4),
    # the decode workload with 4-bit expert weights (DeepSeek-V4 lecture page, 3.1)
    "decode_w4": MoeConfig("decode_w4", T=128, H=7168, E=256, I=2048, k=8, bias="uniform",
                           layout="masked", masked_max_m=128, seed=3, weights="w4"),
}


@dataclasses.dataclass
class MoeInputs:
    cfg: MoeConfig
    x: torch.Tensor            # [T, H] bf16
    Wg: torch.Tensor           # [E, H] fp32
    bias: torch.Tensor         # [E] fp32
    token_ids: torch.Tensor    # [T] int32
    W1q: torch.Tensor          # [E, I, H] uint8 (E4M3 codes), K(=H)-major; w4: [E, I, H/2] packed levels
    S1: torch.Tensor           # [E, I/128, H/128] fp32; w4: [E, H/128, I] (K-block-major row scales)
    W3q: torch.Tensor          # [E, I, H] uint8; w4: [E, I, H/2]
    S3: torch.Tensor           # [E, I/128, H/128] fp32; w4: [E, H/128, I]
    W2q: torch.Tensor          # [E, H, I] uint8, K(=I)-major; w4: [E, H, I/2]
    S2: torch.Tensor           # [E, H/128, I/128] fp32; w4: [E, I/128, H]

    def to(self, device) -> "MoeInputs":
        kw = {f.name: getattr(self, f.name) for f in dataclasses.fields(self)}
        for k_, v in kw.items():
            if isinstance(v, torch.Tensor):
                kw[k_] = v.to(device)
        return MoeInputs(**kw)


def quantize_weight_blocks(w: torch.Tensor):
    """Offline weight quantisation (setup): [N, K] fp32 -> (E4M3 codes uint8 [N, K],
    fp32 scales [N/128, K/128]); scale = block max-abs / 448 (1.0 for an all-zero
    block), codes = torch's RNE e4m3 cast of the clamped ratio."""
    N, K = w.shape
    blk = w.reshape(N // BLOCK, BLOCK, K // BLOCK, BLOCK)
    amax = blk.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    ratio = blk / scale[:, None, :, None]
    q = ratio.clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return q.reshape(N, K).view(torch.uint8), scale.contiguous()


def quantize_weight_int4(w: torch.Tensor):
    """Offline 4-bit weight quantisation (setup; DeepSeek-V4 lecture page, 3.1: per-channel blocks,
    each scaled by its max-abs, levels round((w / max|w|) * (2^3 - 1))): [N, K] fp32 ->
    (codes uint8 [N, K/2], fp32 scales [N, K/128]). A block is one row by 128 consecutive k; the level
    is rounded half to even (torch.round) from the exact ratio (float64); the stored scale is
    max-abs / 7 in fp32 (1.0 for an all-zero block), so a weight dequantises to level * scale.
    Levels are stored as a sign and a 3-bit magnitude, eight consecutive k per little-endian 32-bit
    word: level i (i = 0..3) has its magnitude in bits 4i..4i+2 and its sign in bit 8i+7, level 4+i
    its magnitude in bits 16+4i..16+4i+2 and its sign in bit 8i+3 (a pure bit layout)."""
    N, K = w.shape
    blk = w.reshape(N, K // BLOCK, BLOCK)
    amax = blk.abs().amax(dim=2)
    lev = torch.where(amax[..., None] > 0, (blk.double() * 7.0 / amax.double()[..., None]).round(),
                      torch.zeros_like(blk, dtype=torch.float64))
    lev = lev.to(torch.int64).reshape(N, K // 8, 8)
    mag, neg = lev.abs(), (lev < 0).to(torch.int64)
    word = torch.zeros(N, K // 8, dtype=torch.int64, device=w.device)
    for i in range(4):
        word |= mag[..., i] << (4 * i)
        word |= neg[..., i] << (8 * i + 7)
        word |= mag[..., 4 + i] << (16 + 4 * i)
        word |= neg[..., 4 + i] << (8 * i + 3)
    codes = torch.stack([(word >> (8 * b)) & 255 for b in range(4)], dim=-1).to(torch.uint8).reshape(N, K // 2)
    scale = torch.where(amax > 0, amax / 7.0, torch.ones_like(amax))
    return codes.contiguous(), scale.contiguous()


def _bias(cfg: MoeConfig, g: torch.Generator, device) -> torch.Tensor:
    if cfg.bias == "zero":
        return torch.zeros(cfg.E, dtype=torch.float32, device=device)
    if cfg.bias == "uniform":
        return (torch.rand(cfg.E, generator=g, device=device, dtype=torch.float32) * 0.02 - 0.01)
    if cfg.bias == "zipf":
        ranks = torch.arange(1, cfg.E + 1, dtype=torch.float64)
        p = ranks.pow(-1.1)
        p = p / p.sum()
        return p.log().to(torch.float32).to(device)
    raise ValueError(cfg.bias)


def make_inputs(cfg: MoeConfig, device="cpu", T: Optional[int] = None) -> MoeInputs:
    """Draw the workload's inputs with torch's seeded generator on `device`.

    The draw order is fixed (x, W_g, bias, token ids, then per expert W1, W3,
    W2), so a given (config, device) always yields the same arrays. `T`
    overrides the token count (smaller parity cases of the same shape)."""
    if T is not None:
        cfg = cfg.replace(T=T, masked_max_m=(T if cfg.layout == "masked" else cfg.masked_max_m))
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    Tn, H, E, I = cfg.T, cfg.H, cfg.E, cfg.I
    x = torch.randn(Tn, H, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    Wg = torch.randn(E, H, generator=g, device=dev, dtype=torch.float32) * 0.02
    bias = _bias(cfg, g, dev)
    token_ids = torch.randint(0, 102400, (Tn,), generator=g, device=dev, dtype=torch.int32)
    w4 = cfg.weights == "w4"
    cols = (lambda K: K // 2) if w4 else (lambda K: K)
    W1q = torch.empty(E, I, cols(H), dtype=torch.uint8, device=dev)
    W3q = torch.empty(E, I, cols(H), dtype=torch.uint8, device=dev)
    W2q = torch.empty(E, H, cols(I), dtype=torch.uint8, device=dev)
    if w4:
        S1 = torch.empty(E, H // BLOCK, I, dtype=torch.float32, device=dev)
        S2 = torch.empty(E, I // BLOCK, H, dtype=torch.float32, device=dev)
    else:
        S1 = torch.empty(E, I // BLOCK, H // BLOCK, dtype=torch.float32, device=dev)
        S2 = torch.empty(E, H // BLOCK, I // BLOCK, dtype=torch.float32, device=dev)
    S3 = torch.empty_like(S1)
    for e in range(E):
        for (wq, ws, shape) in ((W1q, S1, (I, H)), (W3q, S3, (I, H)), (W2q, S2, (H, I))):
            w = torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * 0.02
            if w4:
                q, s = quantize_weight_int4(w)
                s = s.t()                                   # row scales, K-block-major
            else:
                q, s = quantize_weight_blocks(w)
            wq[e].copy_(q)
            ws[e].copy_(s)
    return MoeInputs(cfg, x, Wg, bias, token_ids, W1q, S1, W3q, S3, W2q, S2)


def make_router_inputs(cfg: MoeConfig, device="cpu"):
    """x, W_g and bias exactly as make_inputs draws them on `device` (they come first in its draw
    order), without drawing the expert weights: (x [T, H] bf16, W_g [E, H] fp32, bias [E] fp32)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    x = torch.randn(cfg.T, cfg.H, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    Wg = torch.randn(cfg.E, cfg.H, generator=g, device=dev, dtype=torch.float32) * 0.02
    return x, Wg, _bias(cfg, g, dev)


def interleave_w13(W1q: torch.Tensor, S1: torch.Tensor, W3q: torch.Tensor, S3: torch.Tensor):
    """Pure layout: stack W1 and W3 into one [E, 2I, H] operand whose 128-row
    blocks alternate (W1 block j, W3 block j), with the scales [E, 2I/128, H/128]
    in the same order. A 256-row tile of this operand then holds matching gate
    (W1) and up (W3) rows for 128 intermediate columns."""
    E, I, H = W1q.shape
    nb = I // BLOCK
    w = torch.stack((W1q.reshape(E, nb, BLOCK, H), W3q.reshape(E, nb, BLOCK, H)), dim=2)
    s = torch.stack((S1, S3), dim=2)
    return w.reshape(E, 2 * I, H).contiguous(), s.reshape(E, 2 * nb, H // BLOCK).contiguous()


def interleave_w13_w4(W1q: torch.Tensor, S1: torch.Tensor, W3q: torch.Tensor, S3: torch.Tensor):
    """interleave_w13 for 4-bit weights: the packed rows [E, I, H/2] alternate in 128-row blocks (W1 block
    j, W3 block j) as for E4M3, and the K-block-major row scales [E, H/128, I] follow the same row order
    along their last axis. Pure layout."""
    E, I, Hp = W1q.shape
    nb = I // BLOCK
    w = torch.stack((W1q.reshape(E, nb, BLOCK, Hp), W3q.reshape(E, nb, BLOCK, Hp)), dim=2)
    KB = S1.shape[1]
    s = torch.stack((S1.reshape(E, KB, nb, BLOCK), S3.reshape(E, KB, nb, BLOCK)), dim=3)
    return w.reshape(E, 2 * I, Hp).contiguous(), s.reshape(E, KB, 2 * I).contiguous()


def transpose_weights(W13: torch.Tensor, S13: torch.Tensor, W2: torch.Tensor, S2: torch.Tensor):
    """The backward pass's transposed operands (pure layout): W13 [E, 2I, H] -> [E, H, 2I] with its block
    scales [E, 2I/128, H/128] -> [E, H/128, 2I/128], and W2 [E, H, I] -> [E, I, H], [E, H/128, I/128] ->
    [E, I/128, H/128]. A 128x128 block keeps its scale."""
    t = lambda a: a.transpose(1, 2).contiguous()
    return t(W13), t(S13), t(W2), t(S2)


def capacity_rows_bound(cfg: MoeConfig, pad: int = BLOCK) -> int:
    """Upper bound on the rows of the permuted activation buffer: every kept
    slot plus at most pad-1 padding rows per expert (contiguous layout), or
    E * Mmax (masked layout). Pure size arithmetic for allocating buffers."""
    if cfg.layout == "masked":
        return cfg.E * cfg.masked_max_m
    R = cfg.T * cfg.k
    return int(math.ceil((R + cfg.E * (pad - 1)) / pad) * pad)
