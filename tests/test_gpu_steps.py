"""GPU parity of each C-ABI step against the oracle on identical inputs:

* moe_route: indices bit-exact (including ties), weights to 1e-6, on every
  workload at full size;
* moe_permute (fed the oracle's routing): counts, kept, offsets, row_src,
  slot_row and the quantised rows Aq / scales As bit-exact, padding included;
* moe_grouped_gemm_fp8: both layouts x both epilogues on ragged groups
  (empty groups, 1 row, tiles plus a ragged tail, a half-width N tile);
* moe_combine (fed the oracle's expert outputs), with dropped slots;
* moe_balance_bias: tallies and biases bit-exact over a sequence of steps;
* moe_grouped_gemm_w4: the masked GEMM with 4-bit weights, both epilogues.
"""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, MoeConfig, capacity_rows_bound
from gpu_helpers import (W_RTOL, assert_close_bf16, ensure_lib, gpu_inputs, oracle_inputs, rel_errors,
                         to_np)

pytestmark = pytest.mark.gpu


def _route(cfg, inp):
    c = api.Config.from_moe(cfg)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(api.moe_workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    api.moe_route(c, inp.x, inp.Wg, inp.bias, inp.token_ids, idx, w, ws)
    torch.cuda.synchronize()
    return to_np(idx), to_np(w)


@pytest.mark.parametrize("name", ["tiny", "page", "prefill", "decode", "decode_hash", "skewed"])
def test_route_full_size(name):
    ensure_lib()
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg, on_device=name not in ("tiny",))
    idx, w = _route(cfg, inp)
    ref_idx, ref_w, _ = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), to_np(inp.token_ids))
    assert np.array_equal(idx, ref_idx)
    assert np.allclose(w, ref_w, rtol=W_RTOL, atol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-5)


def test_route_ties_and_ragged_shapes():
    # E not a multiple of the kernel's expert tile, T not a multiple of its token tile,
    # and rows of x equal to each other so whole tokens tie (identical logits per expert
    # pair from duplicated W_g rows): the lower expert index must win every tie.
    ensure_lib()
    cfg = MoeConfig("ties", T=77, H=384, E=13, I=128, k=3, bias="zero", seed=21)
    inp = gpu_inputs(cfg)
    inp.Wg[5] = inp.Wg[2]
    inp.Wg[11] = inp.Wg[2]
    inp.Wg[7] = inp.Wg[0]
    inp.x[10] = inp.x[3]
    idx, w = _route(cfg, inp)
    ref_idx, ref_w, logits = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), None)
    assert np.array_equal(idx, ref_idx)
    assert np.allclose(w, ref_w, rtol=W_RTOL, atol=0)
    assert np.any(logits[:, 2] == logits[:, 5])


@pytest.mark.parametrize("layout", ["contiguous", "masked"])
def test_route_and_permute_at_the_limits(layout):
    # the largest shapes the boundary accepts: E = 512 experts, k = 32 per token, H = 16384, with a T
    # that fills no tile; routing and the permutation (capacity drops in the contiguous case) bit-exact
    ensure_lib()
    extra = dict(cap_num=5, cap_den=4) if layout == "contiguous" else dict(layout="masked", masked_max_m=32)
    cfg = MoeConfig("limits", T=40, H=16384, E=512, I=128, k=32, bias="uniform", seed=41, **extra)
    g = torch.Generator().manual_seed(41)
    x = torch.randn(cfg.T, cfg.H, generator=g).to(torch.bfloat16)
    Wg = torch.randn(cfg.E, cfg.H, generator=g) * 0.02
    bias = torch.rand(cfg.E, generator=g) * 0.02 - 0.01
    inp = SimpleNamespace(x=x.cuda(), Wg=Wg.cuda(), bias=bias.cuda(), token_ids=None)
    idx, w = _route(cfg, inp)
    x_bits = x.view(torch.int16).numpy().view(np.uint16)
    ref_idx, ref_w, _ = oracle.route(cfg, x_bits, Wg.numpy(), bias.numpy(), None)
    assert np.array_equal(idx, ref_idx)
    assert np.allclose(w, ref_w, rtol=W_RTOL, atol=0)
    got, rows = _permute(cfg, inp, ref_idx)
    ref = oracle.permute(cfg, x_bits, ref_idx, rows)
    for key in ("counts", "kept", "offsets", "slot_row"):
        assert np.array_equal(got[key], ref[key]), key
    if layout == "masked":
        M = cfg.masked_max_m
        for e in np.nonzero(ref["kept"])[0]:
            r0, n = e * M, ref["kept"][e]
            assert np.array_equal(got["Aq"][r0:r0 + n], ref["Aq"][r0:r0 + n])
            assert np.array_equal(got["As"][e, :, :n], ref["As"][e, :, :n])
    else:
        used = ref["offsets"][-1]
        assert np.array_equal(got["row_src"][:used], ref["row_src"][:used])
        assert np.array_equal(got["Aq"][:used], ref["Aq"][:used])
        assert np.array_equal(got["As"][:, :used], ref["As"][:, :used])
        assert np.count_nonzero(ref["slot_row"] < 0) > 0          # capacity 3 of 2.5 average drops slots


def _permute(cfg, inp, topk_idx):
    c = api.Config.from_moe(cfg)
    rows = api.moe_rows_capacity(c)
    H, E = cfg.H, cfg.E
    masked = cfg.layout == "masked"
    dev = "cuda"
    Aq = torch.full((rows, H), 0xAB, dtype=torch.uint8, device=dev)       # poison: every byte must be written
    if masked:
        As = torch.full((E, H // 128, cfg.masked_max_m), -7.0, dtype=torch.float32, device=dev)
    else:
        As = torch.full((H // 128, rows), -7.0, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_src = torch.full((rows,), -99, dtype=torch.int32, device=dev)
    slot_row = torch.empty(cfg.T * topk_idx.shape[1], dtype=torch.int32, device=dev)
    ws = torch.empty(api.moe_workspace_size(c), dtype=torch.uint8, device=dev)
    api.moe_permute(c, inp.x, torch.from_numpy(topk_idx).to(dev), Aq, As, counts, kept, offsets, row_src,
                    slot_row, ws)
    torch.cuda.synchronize()
    return dict(Aq=to_np(Aq), As=to_np(As), counts=to_np(counts), kept=to_np(kept), offsets=to_np(offsets),
                row_src=to_np(row_src), slot_row=to_np(slot_row)), rows


@pytest.mark.parametrize("name,T", [("tiny", None), ("skewed", 4096), ("prefill", 512), ("decode", None),
                                    ("decode_hash", None), ("page", 1000)])
def test_permute_bit_exact(name, T):
    ensure_lib()
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg, T=T, on_device=cfg.H > 1024)
    cfg = inp.cfg
    ref_idx, _, _ = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), to_np(inp.token_ids))
    got, rows = _permute(cfg, inp, ref_idx)
    ref = oracle.permute(cfg, to_np(inp.x), ref_idx, rows)
    for key in ("counts", "kept", "offsets", "slot_row"):
        assert np.array_equal(got[key], ref[key]), key
    if cfg.layout == "masked":
        M = cfg.masked_max_m
        for e in range(cfg.E):
            r0, r1 = e * M, e * M + ref["kept"][e]
            assert np.array_equal(got["row_src"][r0:r1], ref["row_src"][r0:r1])
            assert np.array_equal(got["Aq"][r0:r1], ref["Aq"][r0:r1])
            assert np.array_equal(got["As"][e, :, :ref["kept"][e]], ref["As"][e, :, :ref["kept"][e]])
    else:
        used = ref["offsets"][-1]
        assert np.array_equal(got["row_src"][:used], ref["row_src"][:used])
        assert np.all(got["row_src"][used:] == -1)                         # rows past the last group: padding
        assert np.array_equal(got["Aq"][:used], ref["Aq"][:used])          # padding rows are 0 too
        assert np.array_equal(got["As"][:, :used], ref["As"][:, :used])    # padding scales are 1
    if cfg.cap_num:
        assert np.count_nonzero(ref["slot_row"] < 0) > 0


def test_permute_extreme_magnitudes_bit_exact():
    """x quantisation across the whole bf16 range: groups scaled from the subnormals (2^-133) to 2^124,
    either side of the 2^-60 switch between the multiply-and-correct quotients and the division, groups
    of signed zeros, a single nonzero value, and values on exact E4M3 rounding midpoints (amax = 448 * 2^k,
    so every quotient is a tie that must round to even). Codes and scales bit-exact with the oracle."""
    import types
    ensure_lib()
    base = CONFIGS["tiny"]
    T = 96
    cfg = base.replace(T=T)
    G = cfg.H // 128
    rng = np.random.default_rng(11)
    x = rng.standard_normal((T, cfg.H)).astype(np.float64)
    mags = [2.0 ** -133, 2.0 ** -124, 2.0 ** -100, 2.0 ** -70, 2.0 ** -61, 2.0 ** -60, 2.0 ** -59, 2.0 ** -20,
            1.0, 2.0 ** 50, 2.0 ** 100, 2.0 ** 124]
    for t in range(T):
        for g in range(G):
            x[t, g * 128:(g + 1) * 128] *= mags[(t * G + g) % len(mags)]
    x[0, 0:128] = 0.0
    x[1, 0:128] = -0.0
    x[2, 0:128] = 0.0
    x[2, 5] = -3.0
    mids = np.array([(1 + (m + 0.5) / 8) * 2.0 ** e for e in range(-6, 8) for m in range(8)
                     if (1 + (m + 0.5) / 8) * 2.0 ** e < 448])
    for t in range(3, T, 7):
        k = int(rng.integers(-80, 80))
        grp = rng.choice(mids, 128) * rng.choice([-1.0, 1.0], 128)
        grp[int(rng.integers(0, 128))] = 448.0
        x[t, 128:256] = grp * 2.0 ** k
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    assert torch.isfinite(xb.float()).all()
    topk = np.stack([rng.permutation(cfg.E)[:cfg.k] for _ in range(T)]).astype(np.int32)
    inp = types.SimpleNamespace(x=xb.cuda())
    got, rows = _permute(cfg, inp, topk)
    ref = oracle.permute(cfg, xb.view(torch.int16).numpy().view(np.uint16), topk, rows)
    used = ref["offsets"][-1]
    assert np.array_equal(got["slot_row"], ref["slot_row"])
    assert np.array_equal(got["Aq"][:used], ref["Aq"][:used])
    assert np.array_equal(got["As"][:, :used], ref["As"][:, :used])
    assert np.any(ref["Aq"][:used] == 0x80)                    # negative zeros survive as codes


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C                              # no NaN codes
    return c


def _gemm_case(layout, epilogue, E, N, K, groups, M_rows=None, seed=0):
    rng = np.random.default_rng(seed)
    G = K // 128
    if layout == 0:
        offs = [0]
        for g in groups:
            offs.append(offs[-1] + -(-g // 128) * 128)
        rows = offs[-1] + 256                                 # some rows past the last group
        A = _rand_codes(rng, (rows, K))
        As = rng.uniform(0.002, 0.02, (G, rows)).astype(np.float32)
        gi = np.array(offs, np.int32)
        M = rows
    else:
        M = M_rows
        A = _rand_codes(rng, (E * M, K))
        As = rng.uniform(0.002, 0.02, (E, G, M)).astype(np.float32)
        gi = np.array(groups, np.int32)
    B = _rand_codes(rng, (E, N, K))
    Bs = rng.uniform(1e-4, 1e-3, (E, N // 128, G)).astype(np.float32)
    return A, As, gi, M, B, Bs


def _gemm_gpu(layout, epilogue, E, N, K, A, As, gi, M, B, Bs):
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    rows = A.shape[0]
    if epilogue == 0:
        D = torch.zeros(rows, N, dtype=torch.bfloat16, device="cuda")
        Ds = None
    else:
        D = torch.zeros(rows, N // 2, dtype=torch.uint8, device="cuda")
        G = N // 256
        Ds = torch.zeros((G, M) if layout == 0 else (E, G, M), dtype=torch.float32, device="cuda")
    api.moe_grouped_gemm_fp8(layout, E, N, K, d(A), d(As), d(gi), M, d(B), d(Bs), epilogue, D, Ds)
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    return to_np(D), (None if Ds is None else to_np(Ds))


def _valid_rows(layout, gi, M, E):
    if layout == 0:
        return np.arange(gi[-1])
    return np.concatenate([e * M + np.arange(gi[e]) for e in range(E)]).astype(np.int64)


GEMM_CASES = [
    # layout, epilogue, E, N, K, groups, M_rows
    (0, 0, 5, 640, 384, [0, 1, 130, 255, 40], None),      # half-width last N tile (640 = 2*256 + 128)
    (0, 1, 5, 512, 384, [0, 1, 130, 255, 40], None),
    (0, 0, 3, 256, 1024, [300, 0, 129], None),
    (0, 1, 3, 768, 640, [257, 384, 0], None),             # 3 M tiles per expert, 5 K blocks
    (0, 0, 6, 384, 128, [1, 128, 129, 0, 513, 2], None),  # a single K block
    (1, 0, 4, 384, 256, [0, 5, 33, 64], 64),
    (1, 1, 4, 512, 256, [0, 5, 33, 64], 64),
    (1, 1, 3, 256, 512, [32, 1, 0], 96),
    # the largest K (128 K blocks: every weight-block scale slot in use) and the largest N (H = 16384)
    (0, 0, 2, 256, 16384, [130, 1], None),
    (0, 1, 2, 256, 16384, [130, 1], None),
    (0, 0, 2, 16384, 128, [130, 1], None),
    (1, 0, 2, 256, 16384, [5, 32], 32),
    (1, 1, 2, 256, 16384, [32, 7], 32),
    # far more tiles than the 148 persistent CTAs (contiguous: 28 M tiles x 16 N tiles = 448; masked: up to
    # 16 experts x 16 weight tiles x up to 2 token tiles), so every CTA runs several tiles and the stage,
    # scale and accumulator rings wrap across tile boundaries; the masked bf16 output in both tile widths
    # (two 128-row weight blocks per tile where N allows, one for N = 1920)
    (0, 0, 8, 4096, 256, [600, 517, 0, 640, 129, 380, 700, 255], None),
    (0, 1, 8, 4096, 256, [600, 517, 0, 640, 129, 380, 700, 255], None),
    (1, 0, 16, 4096, 256, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64),
    (1, 0, 16, 1920, 256, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64),
    (1, 1, 16, 4096, 256, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64),
]

MANY_TILES = 296          # two tiles per persistent CTA on a 148-SM part


def _tile_count(layout, epi, E, N, groups, M_rows):
    if layout == 0:
        return sum(-(-g // 128) for g in groups) * -(-N // 256)
    # masked: a weight tile is 256 rows (gate and up, or two output blocks when N allows) or 128
    return sum(-(-g // 32) for g in groups) * (N // 256 if epi == 1 or N % 256 == 0 else N // 128)


def test_gemm_cases_include_multi_tile_launches():
    # the coverage the cases above claim: both layouts and both epilogues have a launch with more tiles
    # than two per CTA, the masked bf16 output in both tile widths
    for layout in (0, 1):
        for epi in (0, 1):
            assert any(c[0] == layout and c[1] == epi and _tile_count(layout, epi, c[2], c[3], c[5], c[6])
                       > MANY_TILES for c in GEMM_CASES), (layout, epi)
    for wide in (True, False):
        assert any(c[0] == 1 and c[1] == 0 and (c[3] % 256 == 0) == wide and
                   _tile_count(1, 0, c[2], c[3], c[5], c[6]) > MANY_TILES for c in GEMM_CASES), wide


class contig_form:
    """Runs the enclosed calls with the contiguous GEMM forced to one form, then restores the default."""

    def __init__(self, form):
        self.form = form

    def __enter__(self):
        api.moe_set_contig_kernel(self.form)

    def __exit__(self, *exc):
        api.moe_set_contig_kernel(api.CONTIG_AUTO)


# contiguous cases run in both forms of the kernel (single CTAs, CTA pairs: the pair form needs N a
# multiple of 256 and otherwise runs single CTAs); masked cases have one form
GEMM_RUNS = [(c, f) for c in GEMM_CASES for f in ((1, 2) if c[0] == 0 else (0,))]


@pytest.mark.parametrize("case,form", GEMM_RUNS)
def test_grouped_gemm(case, form):
    ensure_lib()
    layout, epi, E, N, K, groups, Mr = case
    A, As, gi, M, B, Bs = _gemm_case(layout, epi, E, N, K, groups, Mr, seed=sum(groups) + N)
    with contig_form(form):
        D, Ds = _gemm_gpu(layout, epi, E, N, K, A, As, gi, M, B, Bs)
    Dr, Dsr = oracle.grouped_gemm(layout, E, N, K, A, As, gi, M, B, Bs, epi)
    rows = _valid_rows(layout, gi, M, E)
    if epi == 0:
        assert_close_bf16(D[rows], Dr[rows], "D")
        assert np.mean(D[rows] == Dr[rows]) > 0.95
    else:
        same = D[rows] == Dr[rows]
        assert same.mean() > 0.999, same.mean()
        diff = np.abs(D[rows].astype(np.int32) - Dr[rows].astype(np.int32))
        assert np.all(diff[~same] == 1)                     # at worst one E4M3 step apart
        if layout == 0:
            s, sr = Ds[:, rows], Dsr[:, rows]
        else:
            s = np.concatenate([Ds[e, :, :gi[e]] for e in range(E)], axis=1)
            sr = np.concatenate([Dsr[e, :, :gi[e]] for e in range(E)], axis=1)
        assert np.allclose(s, sr, rtol=1e-5, atol=0)


W4_CASES = [
    # E, N, K, masked_m, M_rows, epilogue, seed: empty and full blocks, ragged token tiles, the largest K
    (4, 256, 384, [0, 5, 32, 64], 64, 0, 1),
    (4, 512, 384, [7, 0, 33, 64], 64, 1, 2),
    (3, 384, 1024, [1, 31, 64], 64, 0, 3),
    (2, 256, 16384, [5, 32], 32, 0, 4),
    (2, 512, 16384, [32, 9], 32, 1, 5),
    # more tiles than two per CTA in both epilogues (16 experts x 16 weight tiles x up to 2 token
    # tiles): the converter warps' stage counter, their barrier phases and the per-tile reload of the row
    # scales carry across tiles
    (16, 4096, 1024, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64, 0, 6),
    (16, 1920, 1024, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64, 0, 8),
    (16, 4096, 1024, [64, 3, 0, 33, 64, 17, 40, 1, 64, 0, 63, 32, 9, 64, 50, 2], 64, 1, 7),
]


def test_w4_cases_include_multi_tile_launches():
    for epi in (0, 1):
        assert any(c[5] == epi and _tile_count(1, epi, c[0], c[1], c[3], c[4]) > MANY_TILES for c in W4_CASES)
    for wide in (True, False):
        assert any(c[5] == 0 and (c[1] % 256 == 0) == wide and _tile_count(1, 0, c[0], c[1], c[3], c[4]) > MANY_TILES
                   for c in W4_CASES), wide


@pytest.mark.parametrize("case", W4_CASES)
def test_grouped_gemm_w4(case):
    # 4-bit weights (levels -7..7, a scale per weight row per K block) through the masked kernel
    ensure_lib()
    from fp8_grouped_gemm_fp32_b200.inputs import quantize_weight_int4
    E, N, K, mm, M, epi, seed = case
    rng = np.random.default_rng(seed)
    A = _rand_codes(rng, (E * M, K))
    As = rng.uniform(0.002, 0.02, (E, K // 128, M)).astype(np.float32)
    q, s4 = quantize_weight_int4(torch.from_numpy(rng.standard_normal((E * N, K)).astype(np.float32) * 0.02))
    B = q.numpy().reshape(E, N, K // 2)
    Bs = np.ascontiguousarray(s4.numpy().reshape(E, N, K // 128).transpose(0, 2, 1))
    gi = np.array(mm, np.int32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    if epi == 0:
        D = torch.zeros(E * M, N, dtype=torch.bfloat16, device="cuda")
        Ds = None
    else:
        D = torch.zeros(E * M, N // 2, dtype=torch.uint8, device="cuda")
        Ds = torch.zeros(E, N // 256, M, dtype=torch.float32, device="cuda")
    api.moe_grouped_gemm_w4(1, E, N, K, d(A), d(As), d(gi), M, d(B), d(Bs), epi, D, Ds)
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    Dr, Dsr = oracle.grouped_gemm(1, E, N, K, A, As, gi, M, B, Bs, epi, w4=True)
    rows = _valid_rows(1, gi, M, E)
    Dg = to_np(D)
    if epi == 0:
        assert_close_bf16(Dg[rows], Dr[rows], "D")
        assert np.mean(Dg[rows] == Dr[rows]) > 0.95
    else:
        same = Dg[rows] == Dr[rows]
        assert same.mean() > 0.999, same.mean()
        assert np.all(np.abs(Dg[rows].astype(np.int32) - Dr[rows].astype(np.int32))[~same] == 1)
        s = np.concatenate([to_np(Ds)[e, :, :gi[e]] for e in range(E)], axis=1)
        sr = np.concatenate([Dsr[e, :, :gi[e]] for e in range(E)], axis=1)
        assert np.allclose(s, sr, rtol=1e-5, atol=0)


@pytest.mark.parametrize("layout,epi,form", [(0, 0, 1), (0, 1, 1), (0, 0, 2), (0, 1, 2), (1, 0, 0), (1, 1, 0)])
def test_grouped_gemm_writes_nothing_outside_its_groups(layout, epi, form):
    # canary-filled outputs with guard rows past the end: rows outside every group (contiguous) or at
    # and past a block's count (masked) keep the canary, as do the guard rows and their scales
    ensure_lib()
    E, N, K = 3, 512, 256
    groups, Mr = ([130, 0, 1], None) if layout == 0 else ([5, 0, 32], 64)
    A, As, gi, M, B, Bs = _gemm_case(layout, epi, E, N, K, groups, Mr, seed=77)
    rows = A.shape[0]
    guard = 64
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    if epi == 0:
        Dfull = torch.full((rows + guard, N), 0x5A5A, dtype=torch.int16, device="cuda")
        Dsfull = None
    else:
        Dfull = torch.full((rows + guard, N // 2), 0x5A, dtype=torch.uint8, device="cuda")
        G = N // 256
        Dsfull = torch.full(((G, M) if layout == 0 else (E, G, M)), -3.0, dtype=torch.float32, device="cuda")
    D = Dfull[:rows]
    with contig_form(form):
        api.moe_grouped_gemm_fp8(layout, E, N, K, d(A), d(As), d(gi), M, d(B), d(Bs), epi, D, Dsfull)
        torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    Dh = to_np(Dfull)
    canary = 0x5A5A if epi == 0 else 0x5A
    valid = np.zeros(rows + guard, bool)
    valid[_valid_rows(layout, gi, M, E)] = True
    if layout == 0:
        assert np.all(Dh[gi[-1]:] == canary)                       # past the last group, guard rows too
        if epi == 1:
            assert np.all(to_np(Dsfull)[:, gi[-1]:] == -3.0)
    else:
        assert np.all(Dh[~valid] == canary)
        if epi == 1:
            Ds = to_np(Dsfull)
            for e in range(E):
                assert np.all(Ds[e, :, gi[e]:] == -3.0)
                assert np.all(Ds[e, :, :gi[e]] > 0)


@pytest.mark.parametrize("layout,epi,w4,form", [(1, 0, False, 0), (1, 1, False, 0), (1, 0, True, 0), (1, 1, True, 0),
                                                (0, 0, False, 1), (0, 1, False, 1), (0, 0, False, 2),
                                                (0, 1, False, 2)])
def test_grouped_gemm_clamps_out_of_bound_groups(layout, epi, w4, form):
    # group sizes past the buffers (a masked count above M_rows or below 0; contiguous offsets past M_rows
    # or not a multiple of 128) are clamped on the device and reported as MOE_ERR_CAPACITY: guard rows past
    # D and past the scales keep their canary, and the groups within bounds are still exact
    ensure_lib()
    E, N, K = 3, 512, 256
    if layout == 1:
        M = 32
        gi = np.array([5, -4, 40], np.int32)                  # expert 2 claims 40 rows of a 32-row block
        good = [0]
        rows = E * M
    else:
        gi = np.array([0, 128, 128, 1024], np.int32)         # the last group runs past M_rows = 384
        M = rows = 384
        good = [0]
    rng = np.random.default_rng(5)
    A = _rand_codes(rng, (rows, K))
    G = K // 128
    As = rng.uniform(0.002, 0.02, (G, rows) if layout == 0 else (E, G, M)).astype(np.float32)
    if w4:
        from fp8_grouped_gemm_fp32_b200.inputs import quantize_weight_int4
        q, s4 = quantize_weight_int4(torch.from_numpy(rng.standard_normal((E * N, K)).astype(np.float32) * 0.02))
        B = q.numpy().reshape(E, N, K // 2)
        Bs = np.ascontiguousarray(s4.numpy().reshape(E, N, K // 128).transpose(0, 2, 1))
    else:
        B = _rand_codes(rng, (E, N, K))
        Bs = rng.uniform(1e-4, 1e-3, (E, N // 128, G)).astype(np.float32)
    guard = 64
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    width = N if epi == 0 else N // 2
    dt = torch.int16 if epi == 0 else torch.uint8
    canary = 0x5A5A if epi == 0 else 0x5A
    Dfull = torch.full((rows + guard, width), canary, dtype=dt, device="cuda")
    Gs = N // 256
    Dsfull = None
    if epi == 1:
        Dsfull = torch.full((Gs * M + guard,) if layout == 0 else (E * Gs * M + guard,), -3.0,
                            dtype=torch.float32, device="cuda")
    D = Dfull[:rows]
    fn = api.moe_grouped_gemm_w4 if w4 else api.moe_grouped_gemm_fp8
    with contig_form(form):
        fn(layout, E, N, K, d(A), d(As), d(gi), M, d(B), d(Bs), epi, D, Dsfull)
        torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_ERR_CAPACITY
    assert api.moe_get_device_status() == api.MOE_OK
    Dh = to_np(Dfull)
    assert np.all(Dh[rows:] == canary)                          # nothing past D
    if epi == 1:
        assert np.all(to_np(Dsfull)[-guard:] == -3.0)           # nothing past Ds
    # a group within bounds is unaffected: expert 0's rows match the oracle
    if layout == 1:
        gi_ok = np.array([gi[0], 0, 0], np.int32)
    else:
        gi_ok = np.array([0, 128, 128, 128], np.int32)
    Dr, _ = oracle.grouped_gemm(layout, E, N, K, A, As, gi_ok, M, B, Bs, epi, w4=w4)
    r = np.arange(gi[0]) if layout == 1 else np.arange(128)
    if epi == 0:
        assert_close_bf16(Dh[r], Dr[r], "D")
    else:
        same = Dh[r] == Dr[r]
        assert same.mean() > 0.99
        assert np.all(np.abs(Dh[r].astype(np.int32) - Dr[r].astype(np.int32))[~same] == 1)


def test_combine_with_drops():
    ensure_lib()
    cfg = MoeConfig("comb", T=300, H=384, E=4, I=128, k=3, bias="uniform", cap_num=1, cap_den=2, seed=31)
    inp = gpu_inputs(cfg)
    ref_idx, ref_w, _ = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), None)
    rows = capacity_rows_bound(cfg)
    d = oracle.dispatch(ref_idx, cfg.E, oracle.capacity(cfg.T, cfg.k, cfg.E, 1, 2), 0, 128, 0, rows)
    rng = np.random.default_rng(3)
    O = torch.randn(rows, cfg.H).to(torch.bfloat16)
    O_bits = O.view(torch.int16).numpy().view(np.uint16)
    y_ref = oracle.combine(d["slot_row"], ref_w, O_bits, cfg.T, cfg.k)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    api.moe_combine(api.Config.from_moe(cfg), O.cuda(), torch.from_numpy(d["slot_row"]).cuda(),
                    torch.from_numpy(ref_w).cuda(), y)
    torch.cuda.synchronize()
    assert np.count_nonzero(d["slot_row"] < 0) > 0
    all_dropped = np.nonzero((d["slot_row"].reshape(cfg.T, cfg.k) < 0).all(1))[0]
    assert len(all_dropped) > 0 and np.all(to_np(y)[all_dropped] == 0)
    assert_close_bf16(to_np(y), y_ref)
    assert np.mean(to_np(y) == y_ref) > 0.99


@pytest.mark.parametrize("E", [1, 3, 64, 256, 512])
def test_balance_bias_bit_exact(E):
    # several update intervals of random counts (ties with the mean included), biases of both signs and
    # sizes where the step is partly or wholly lost to fp32 rounding; tallies and biases bit-exact
    ensure_lib()
    rng = np.random.default_rng(E)
    bias = np.concatenate([rng.uniform(-0.01, 0.01, E), [1.0, -1.0, 3e5, 0.0]])[:E].astype(np.float32)
    load = np.zeros(E, np.int64)
    b_dev = torch.from_numpy(bias.copy()).cuda()
    l_dev = torch.zeros(E, dtype=torch.int64, device="cuda")
    for step in range(12):
        if step == 4:
            counts = np.full(E, 7, np.int32)                  # every expert at the mean
        elif step == 8:
            counts = np.zeros(E, np.int32)                    # an empty step
        else:
            counts = rng.integers(0, 3000, E).astype(np.int32)
        update = step % 4 == 3 or step == 4
        gamma = [1e-3, 2.0 ** -25, -5e-4][step % 3]
        oracle.balance_bias(counts, load, bias, gamma, update)
        api.moe_balance_bias(E, torch.from_numpy(counts).cuda(), l_dev, b_dev, gamma, update)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(l_dev), load), step
        assert np.array_equal(to_np(b_dev).view(np.uint32), bias.view(np.uint32)), step


def test_balance_bias_from_routed_counts():
    # the counts moe_permute reports feed the update directly, on the device
    ensure_lib()
    cfg = MoeConfig("zipf", T=2048, H=512, E=64, I=128, k=2, bias="zipf", cap_num=5, cap_den=4, seed=5)
    inp = gpu_inputs(cfg)
    c = api.Config.from_moe(cfg)
    idx, _w = _route(cfg, inp)
    rows = api.moe_rows_capacity(c)
    d = lambda *s, dt=torch.int32: torch.empty(*s, dtype=dt, device="cuda")
    counts = d(cfg.E)
    ws = torch.empty(max(api.moe_workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    api.moe_permute(c, inp.x, torch.from_numpy(idx).cuda(), d(rows, cfg.H, dt=torch.uint8), d(rows * cfg.H // 128,
                    dt=torch.float32), counts, d(cfg.E), d(cfg.E + 1), d(rows), d(cfg.T * cfg.k), ws)
    load = torch.zeros(cfg.E, dtype=torch.int64, device="cuda")
    bias = inp.bias.clone()
    api.moe_balance_bias(cfg.E, counts, load, bias, 1e-3, True)
    torch.cuda.synchronize()
    ref_load = np.zeros(cfg.E, np.int64)
    ref_bias = to_np(inp.bias).copy()
    oracle.balance_bias(np.bincount(idx.ravel(), minlength=cfg.E).astype(np.int32), ref_load, ref_bias, 1e-3, True)
    assert np.array_equal(to_np(bias).view(np.uint32), ref_bias.view(np.uint32))
    assert np.array_equal(to_np(load), ref_load)
    # the Zipf prior makes expert 0 the busiest: its bias goes down
    assert to_np(bias)[0] < to_np(inp.bias)[0]


def test_empty_batch_is_a_no_op():
    ensure_lib()
    cfg = MoeConfig("empty", T=0, H=256, E=4, I=128, k=2, seed=0)
    c = api.Config.from_moe(cfg)
    ws = torch.empty(max(api.moe_workspace_size(c, True), 256), dtype=torch.uint8, device="cuda")
    z = lambda *s, dt=torch.int32: torch.empty(*s, dtype=dt, device="cuda")
    inp = gpu_inputs(cfg.replace(T=4))
    from fp8_grouped_gemm_fp32_b200.inputs import interleave_w13
    W13, S13 = interleave_w13(inp.W1q, inp.S1, inp.W3q, inp.S3)
    # zero tokens: every buffer may be empty; pass small dummies where the ABI wants a pointer
    dummy = z(64)
    api.moe_forward(c, dummy, inp.Wg, inp.bias, None, W13, S13, inp.W2q, inp.S2, dummy, dummy, dummy,
                    z(cfg.E), dummy, ws)
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK


def test_device_timeout_is_reported_and_context_survives():
    ensure_lib()
    assert api.moe_get_device_status() == api.MOE_OK
    api.moe_selftest_wait_timeout(2000)                  # a 2 ms wait on a barrier nothing completes
    assert api.moe_get_device_status() == api.MOE_ERR_DEVICE_TIMEOUT
    assert api.moe_get_device_status() == api.MOE_OK     # read-and-clear
    test_combine_with_drops()                             # the context still works


def test_host_side_errors_on_device():
    ensure_lib()
    cfg = CONFIGS["tiny"]
    inp = gpu_inputs(cfg)
    c = api.Config.from_moe(cfg)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.MoeError) as ei:
        api.moe_route(c, inp.x, inp.Wg, inp.bias, None, idx, w, small)
    assert ei.value.status == api.MOE_ERR_WORKSPACE_TOO_SMALL
    ws = torch.empty(api.moe_workspace_size(c), dtype=torch.uint8, device="cuda")
    mis = torch.empty(cfg.T * cfg.k * 4 + 4, dtype=torch.uint8, device="cuda")[4:].view(torch.int32)
    with pytest.raises(api.MoeError) as ei:
        api.moe_route(c, inp.x, inp.Wg, inp.bias, None, mis, w, ws)
    assert ei.value.status == api.MOE_ERR_INVALID_ARG          # misaligned pointer
    with pytest.raises(api.MoeError) as ei:
        api.moe_grouped_gemm_fp8(0, 4, 200, 256, inp.x, w, idx, 128, inp.x, w, 0, idx)
    assert ei.value.status == api.MOE_ERR_UNSUPPORTED_SHAPE    # N not a multiple of 128
