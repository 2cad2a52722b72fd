"""Pins for 4-bit expert weights (DeepSeek-V4 lecture page, section 3.1): the
setup quantiser against hand-derived blocks (ties, a negative maximum, tiny
magnitudes, an all-zero block), exact round trips of level grids and the
half-step error bound; the oracle's 4-bit code decoding against two's
complement for every byte; and the oracle's grouped GEMM with 4-bit weights,
in both layouts and both epilogues, against torch float64 matmuls whose weights
are unpacked and dequantised here, independently of the oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200.inputs import quantize_weight_int4

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _sparse(tok, conv):
    out = {}
    for t in tok:
        k, v = t.split(":")
        out[int(k)] = conv(v)
    return out


def golden_cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLD, "w4.txt")):
        tok = line.split("#")[0].split()
        if not tok:
            continue
        if tok[0] == "case":
            cur = {"name": tok[1]}
            cases.append(cur)
        elif tok[0] == "w":
            cur["w"] = _sparse(tok[1:], lambda v: float.fromhex(v) if "x" in v else float(v))
        elif tok[0] == "levels":
            cur["levels"] = _sparse(tok[1:], int)
        elif tok[0] == "scale":
            cur["scale"] = float.fromhex(tok[1])
        elif tok[0] == "bytes":
            cur["bytes"] = _sparse(tok[1:], lambda v: int(v, 16))
    return cases


def _unpack(codes):
    """uint8 [..., K/2] -> int levels [..., K]: low nibble first, 4-bit two's complement."""
    c = codes.astype(np.int16)
    lo, hi = c & 15, c >> 4
    lev = np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    return np.where(lev >= 8, lev - 16, lev)


def test_quantiser_golden_blocks():
    cases = golden_cases()
    assert len(cases) == 4
    for c in cases:
        w = torch.zeros(1, 128, dtype=torch.float32)
        for k, v in c["w"].items():
            w[0, k] = v
        codes, scale = quantize_weight_int4(w)
        want_lev = np.zeros(128, np.int64)
        for k, v in c["levels"].items():
            want_lev[k] = v
        want_bytes = np.zeros(64, np.uint8)
        for k, v in c["bytes"].items():
            want_bytes[k] = v
        assert np.array_equal(codes.numpy()[0], want_bytes), c["name"]
        assert np.array_equal(_unpack(codes.numpy())[0], want_lev), c["name"]
        assert scale.numpy()[0, 0] == np.float32(c["scale"]), c["name"]


def test_every_code_decodes_as_twos_complement():
    for b in range(256):
        assert oracle.w4_decode(b, False) == ((b & 15) ^ 8) - 8
        assert oracle.w4_decode(b, True) == ((b >> 4) ^ 8) - 8


def test_level_grids_round_trip_and_error_bound():
    g = torch.Generator().manual_seed(7)
    # weights on a level grid whose block max is +-7 steps come back with exactly those levels
    lev = torch.randint(-7, 8, (64, 512), generator=g)
    lev[:, ::128] = torch.where(torch.rand(64, 4, generator=g) < 0.5, 7, -7)
    step = torch.exp2(torch.randint(-20, 5, (64, 4, 1), generator=g).double()).float()
    w = (lev.reshape(64, 4, 128) * step).reshape(64, 512)
    codes, scale = quantize_weight_int4(w)
    assert np.array_equal(_unpack(codes.numpy()), lev.numpy())
    assert torch.equal(scale, (7 * step[..., 0]) / 7.0)
    # arbitrary weights: every weight within half a step of its dequantised value
    w = torch.randn(64, 512, generator=g) * 0.02
    codes, scale = quantize_weight_int4(w)
    deq = _unpack(codes.numpy()) * np.repeat(scale.numpy().astype(np.float64), 128, axis=1)
    err = np.abs(w.numpy().astype(np.float64) - deq)
    half = np.repeat(scale.numpy().astype(np.float64), 128, axis=1) / 2
    assert np.all(err <= half * (1 + 2.0 ** -20))
    assert np.all(np.abs(_unpack(codes.numpy())) <= 7)


def _deq_w4(codes, scale):
    """Independent dequantisation: unpacked levels times the row's block scales, rounded to fp32."""
    lev = torch.from_numpy(_unpack(codes).astype(np.float32))
    sc = torch.from_numpy(np.ascontiguousarray(scale)).repeat_interleave(128, -1)
    return (lev * sc).to(torch.float64)


def _rand_e4m3(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C
    return c


def _w4_weights(rng, E, N, K):
    w = torch.from_numpy(rng.standard_normal((E * N, K)).astype(np.float32) * 0.02)
    codes, scale = quantize_weight_int4(w)
    # scales K-block-major, [E, K/128, N]
    return codes.numpy().reshape(E, N, K // 2), np.ascontiguousarray(scale.numpy().reshape(E, N, K // 128)
                                                                      .transpose(0, 2, 1))


def _a_deq(A, As_rows):
    a = torch.from_numpy(A).view(torch.float8_e4m3fn).to(torch.float32)
    return (a * torch.from_numpy(As_rows).repeat_interleave(128, 1)).to(torch.float64)


def _close_bf16(ours_bits, ref64):
    ours = oracle.bf16_bits_to_f32(ours_bits).astype(np.float64)
    ref_b = oracle.bf16_bits_to_f32(oracle.f64_to_bf16_bits(ref64)).astype(np.float64)
    assert np.all(np.abs(ours - ref_b) <= np.abs(ref_b) * 2.0 ** -7 * 1.01 + 1e-30)
    assert np.mean(ours_bits == oracle.f64_to_bf16_bits(ref64)) >= 0.999


def _quant_torch(v64):
    v = v64.to(torch.float32)
    g = v.reshape(v.shape[0], -1, 128)
    amax = g.abs().amax(-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    return (g / s[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(v.shape).numpy(), s.numpy()


@pytest.mark.parametrize("layout", [0, 1])
def test_w4_grouped_gemm_equals_dense_fp64(layout):
    rng = np.random.default_rng(5 + layout)
    E, K, N = 3, 384, 256
    if layout == 0:
        groups = [130, 0, 57]
        offs = np.concatenate([[0], np.cumsum([-(-g // 128) * 128 for g in groups])]).astype(np.int32)
        M = int(offs[-1])
        A = _rand_e4m3(rng, (M, K))
        As = rng.uniform(0.002, 0.02, (K // 128, M)).astype(np.float32)
        gi = offs
        blocks = [(e, np.arange(offs[e], offs[e + 1]), As[:, offs[e]:offs[e + 1]].T) for e in range(E)]
    else:
        M = 64
        gi = np.array([5, 0, 64], np.int32)
        A = _rand_e4m3(rng, (E * M, K))
        As = rng.uniform(0.002, 0.02, (E, K // 128, M)).astype(np.float32)
        blocks = [(e, e * M + np.arange(gi[e]), As[e][:, :gi[e]].T) for e in range(E)]
    B, Bs = _w4_weights(rng, E, N, K)
    D, _ = oracle.grouped_gemm(layout, E, N, K, A, As, gi, M, B, Bs, 0, w4=True)
    # SwiGLU epilogue: N = 2I rows alternating W1 block j, W3 block j
    Dq, Ds = oracle.grouped_gemm(layout, E, N, K, A, As, gi, M, B, Bs, 1, w4=True)
    I = N // 2
    for e, rows, as_rows in blocks:
        if len(rows) == 0:
            continue
        a = _a_deq(A[rows], np.ascontiguousarray(as_rows))
        wd = _deq_w4(B[e], Bs[e].T)
        ref = (a @ wd.T).numpy()
        _close_bf16(D[rows], ref)
        gate = torch.cat([wd[2 * j * 128:(2 * j + 1) * 128] for j in range(I // 128)])
        up = torch.cat([wd[(2 * j + 1) * 128:(2 * j + 2) * 128] for j in range(I // 128)])
        h = torch.nn.functional.silu(a @ gate.T) * (a @ up.T)
        hq, hs = _quant_torch(h)
        same = Dq[rows] == hq
        assert same.mean() > 0.999
        assert np.all(np.abs(Dq[rows].astype(np.int32) - hq.astype(np.int32))[~same] == 1)
        ds = Ds[:, rows].T if layout == 0 else Ds[e][:, :len(rows)].T
        assert np.allclose(ds, hs, rtol=1e-6, atol=0)
