"""Pins for the oracle's number formats (E4M3 codec, bf16 rounding, 1x128
activation quantisation) against the format definitions, hand-derived golden
values and torch's own casts (a library run, not a retyped formula)."""
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    for line in open(os.path.join(GOLD, name)):
        line = line.split("#")[0].strip()
        if line:
            out.append(line.split())
    return out


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_golden():
    for v, code in _rows("e4m3.txt"):
        assert oracle.e4m3_encode(float(v)) == int(code, 16), v


def test_e4m3_roundtrip_every_finite_code():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(7)
    # random magnitudes over the whole range, plus every exact midpoint between neighbours
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000) * 3,
                        rng.standard_normal(5000) * 1e-3]).astype(np.float32)
    vals = np.array(sorted({oracle.e4m3_decode(c) for c in range(0x7F)}))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids])
    ours = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    for v in (448.0, 450.0, 463.9, 464.0, 479.0, 480.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE


def test_bf16_golden_and_torch():
    for v, bits in _rows("bf16.txt"):
        assert oracle.lib().orc_f64_to_bf16(float(v)) == int(bits, 16), v
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    ours = oracle.f64_to_bf16_bits(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)   # fp32-representable inputs: single rounding either way


def test_quant_rows_matches_library_cast():
    rng = np.random.default_rng(11)
    v = (rng.standard_normal((64, 512)) * np.exp(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    v[3, 128:256] = 0.0                      # an all-zero group
    q, s = oracle.quant_rows(v)
    g = v.reshape(64, 4, 128)
    amax = np.abs(g).max(-1)
    s_ref = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0))
    assert np.array_equal(s, s_ref)
    ratio = (torch.from_numpy(g) / torch.from_numpy(s_ref)[..., None])          # fp32 division
    q_ref = ratio.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(64, 512)
    assert np.array_equal(q, q_ref)
    assert s[3, 1] == 1.0 and not q[3, 128:256].any()


def test_quant_grid_values_roundtrip_exactly():
    # values already on the E4M3 grid times 2^n, with the group max equal to 448 * 2^n,
    # quantise with scale 2^n and come back exactly
    rng = np.random.default_rng(5)
    finite = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], dtype=np.float64)
    for n in (-12, -3, 0, 5):
        codes = rng.choice(finite, size=(4, 256))
        codes[:, 0] = 448.0
        codes[:, 128] = -448.0
        v = (codes * 2.0 ** n).astype(np.float32)
        q, s = oracle.quant_rows(v)
        assert np.all(s == np.float32(2.0 ** n))
        deq = oracle.e4m3_decode_array(q) * s.repeat(128, axis=1)
        assert np.array_equal(deq, v.astype(np.float64))
