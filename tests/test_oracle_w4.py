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
    """uint8 [..., K/2] -> int levels [..., K]: per little-endian 32-bit word, eight consecutive k;
    level i < 4: magnitude bits 4i..4i+2, sign bit 8i+7; level 4+i: magnitude bits 16+4i..16+4i+2,
    sign bit 8i+3."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    w = c.reshape(*c.shape[:-1], c.shape[-1] // 4, 4).astype(np.int64)
    word = w[..., 0] | (w[..., 1] << 8) | (w[..., 2] << 16) | (w[..., 3] << 24)
    lev = []
    for i in range(8):
        if i < 4:
            mag, neg = (word >> (4 * i)) & 7, (word >> (8 * i + 7)) & 1
        else:
            mag, neg = (word >> (16 + 4 * (i - 4))) & 7, (word >> (8 * (i - 4) + 3)) & 1
        lev.append(np.where(neg == 1, -mag, mag))
    return np.stack(lev, axis=-1).reshape(*c.shape[:-1], c.shape[-1] * 2)


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


def test_every_level_at_every_position_decodes():
    # a word holding one level at one of its eight places, every level -7..7 at every place, and words of
    # random levels: the oracle's decode returns exactly the levels placed
    for i in range(8):
        for L in range(-7, 8):
            word = abs(L) << (4 * i if i < 4 else 16 + 4 * (i - 4))
            if L < 0:
                word |= 1 << (8 * i + 7 if i < 4 else 8 * (i - 4) + 3)
            row = np.frombuffer(int(word).to_bytes(4, "little"), np.uint8)
            assert [oracle.w4_decode(row, k) for k in range(8)] == [L if k == i else 0 for k in range(8)], (i, L)
    rng = np.random.default_rng(3)
    lev = rng.integers(-7, 8, (16, 128))
    codes, _ = quantize_weight_int4(torch.from_numpy(lev.astype(np.float32) * 7 / np.where(
        np.abs(lev).reshape(16, 1, 128).max(-1) > 0, np.abs(lev).reshape(16, 1, 128).max(-1), 1).repeat(128, 1)))
    got = np.array([[oracle.w4_decode(codes.numpy()[r], k) for k in range(128)] for r in range(16)])
    assert np.array_equal(got, _unpack(codes.numpy()))


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


def test_w4_expert_rows_equal_fp64_expert_function():
    # E_i(x) = W2 (silu(W1 x) * W3 x) with 4-bit weights, h requantised per 1x128 group and o rounded to
    # bf16: the oracle's composition of its 4-bit grouped GEMMs against numpy fp64 matmuls over weights
    # unpacked and dequantised here (a gate/up mix-up, a scale transposed or the wrong interleave fails it)
    rng = np.random.default_rng(11)
    n, H, I = 37, 256, 384
    x = rng.standard_normal((n, H)).astype(np.float32)
    xq, xs = oracle.quant_rows(x)
    wts = {}
    for name, (N, K) in (("W1", (I, H)), ("W3", (I, H)), ("W2", (H, I))):
        q, s = quantize_weight_int4(torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32) * 0.02))
        wts[name] = (q.numpy(), np.ascontiguousarray(s.numpy().T))        # scales K-block-major [K/128, N]
    o = oracle.expert_rows_w4(xq, xs, wts["W1"][0], wts["W1"][1], wts["W3"][0], wts["W3"][1], wts["W2"][0],
                              wts["W2"][1])

    def deq_w(q, s_kb_major):
        return _unpack(q).astype(np.float64) * np.repeat(s_kb_major.T.astype(np.float64), 128, axis=1)

    def deq_rows(codes, scales):
        return oracle.e4m3_decode_array(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)

    xd = deq_rows(xq, xs).astype(np.float32).astype(np.float64)       # dequantised values are fp32
    a = xd @ deq_w(*wts["W1"]).astype(np.float32).astype(np.float64).T
    b = xd @ deq_w(*wts["W3"]).astype(np.float32).astype(np.float64).T
    h = (a / (1.0 + np.exp(-a)) * b).astype(np.float32)
    hq, hs = oracle.quant_rows(h)
    hd = deq_rows(hq, hs).astype(np.float32).astype(np.float64)
    ref = oracle.f64_to_bf16_bits(hd @ deq_w(*wts["W2"]).astype(np.float32).astype(np.float64).T)
    assert np.array_equal(o, ref)
