"""Pins for the oracle's expert math and the whole layer:

* E = 1, k = 1 reduces the layer to one dense SwiGLU FFN (weights exactly 1);
  compared with torch float64 matmuls and torch's silu.
* Concat(E_1(T_1), ..., E_E(T_E)) (MegaMoE page, section 2.1): the grouped
  GEMM over the permuted buffer equals one dense float64 matmul per expert
  over that expert's gathered rows.
* Brute force of y = sum_{i in TopK} G(x)_i E_i(x) per token on tiny inputs,
  sharing nothing with the grouped code path (fp64 logits, per-token loops).

The torch reference below re-derives the storage points the boundary fixes
(x and h in E4M3 with 1x128 scales, o in bf16) with torch casts.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, interleave_w13, make_inputs, quantize_weight_int4


def _deq_w(q, s):
    """torch: E4M3 codes * 128x128 block scales, rounded to fp32, as float64."""
    v = torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float32)
    N, K = v.shape
    sc = torch.from_numpy(np.ascontiguousarray(s)).repeat_interleave(128, 0).repeat_interleave(128, 1)
    return (v * sc).to(torch.float64)


def _quant_torch(v32):
    """torch: 1x128 group quantisation (scale = amax/448 in fp32, RNE e4m3 cast)."""
    v = v32.reshape(v32.shape[0], -1, 128)
    amax = v.abs().amax(-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (v / s[..., None]).to(torch.float8_e4m3fn)
    deq = (q.to(torch.float32) * s[..., None]).reshape(v32.shape)
    return deq.to(torch.float64)


def _ffn_torch(x_bits, W1q, S1, W3q, S3, W2q, S2):
    x = torch.from_numpy(oracle.bf16_bits_to_f32(x_bits))
    xd = _quant_torch(x)
    a = xd @ _deq_w(W1q, S1).T
    b = xd @ _deq_w(W3q, S3).T
    h = (torch.nn.functional.silu(a) * b).to(torch.float32)
    o = _quant_torch(h) @ _deq_w(W2q, S2).T
    return o


def _close_bf16(ours_bits, ref64, frac_equal=0.999):
    ours = oracle.bf16_bits_to_f32(ours_bits).astype(np.float64)
    ref_b = oracle.bf16_bits_to_f32(oracle.f64_to_bf16_bits(ref64)).astype(np.float64)
    diff = np.abs(ours - ref_b)
    ulp = np.abs(ref_b) * 2.0 ** -7 + 1e-30
    assert np.all(diff <= ulp * 1.01)                   # at most one bf16 step apart
    assert np.mean(ours_bits == oracle.f64_to_bf16_bits(ref64)) >= frac_equal


@pytest.fixture(scope="module")
def dense_inputs():
    cfg = MoeConfig("dense", T=64, H=256, E=1, I=256, k=1, bias="uniform", seed=123)
    return cfg, oracle.moe_inputs_to_numpy(make_inputs(cfg))


def test_dense_reduction_E1_k1(dense_inputs):
    cfg, inp = dense_inputs
    out = oracle.forward(cfg, inp)
    assert np.all(out["topk_idx"] == 0) and np.all(out["topk_w"] == 1.0)
    ref = _ffn_torch(inp["x"], inp["W1q"][0], inp["S1"][0], inp["W3q"][0], inp["S3"][0],
                     inp["W2q"][0], inp["S2"][0]).numpy()
    _close_bf16(out["y"], ref)


def test_grouped_gemm_equals_per_expert_dense_gemms():
    cfg = MoeConfig("g", T=96, H=256, E=4, I=128, k=2, bias="uniform", seed=5)
    t = make_inputs(cfg)
    inp = oracle.moe_inputs_to_numpy(t)
    idx, w, _ = oracle.route(cfg, inp["x"], inp["Wg"], inp["bias"], inp["token_ids"])
    rows_cap = -(-(cfg.T * cfg.k + cfg.E * 127) // 128) * 128
    d = oracle.permute(cfg, inp["x"], idx, rows_cap)
    off = d["offsets"]
    # down-projection-shaped grouped GEMM (epilogue 0: bf16 out), B = W2 stacks, K = H here
    B = np.ascontiguousarray(inp["W1q"])          # [E, I, H] used as a plain [E, N, K] operand
    Bs = np.ascontiguousarray(inp["S1"])
    D, _ = oracle.grouped_gemm(0, cfg.E, cfg.I, cfg.H, d["Aq"], d["As"], off, rows_cap, B, Bs, 0)
    for e in range(cfg.E):
        rows = slice(off[e], off[e + 1])
        A = torch.from_numpy(d["Aq"][rows]).view(torch.float8_e4m3fn).to(torch.float32)
        sA = torch.from_numpy(d["As"][:, rows].T.copy()).repeat_interleave(128, 1)
        ref = ((A * sA).to(torch.float64) @ _deq_w(B[e], Bs[e]).T).numpy()
        _close_bf16(D[rows], ref)
    # the SwiGLU epilogue over interleaved W1|W3 equals the per-row expert function
    W13, S13 = interleave_w13(t.W1q, t.S1, t.W3q, t.S3)
    Dq, Ds = oracle.grouped_gemm(0, cfg.E, 2 * cfg.I, cfg.H, d["Aq"], d["As"], off, rows_cap,
                                 W13.numpy(), S13.numpy(), 1)
    for e in range(cfg.E):
        r0, r1 = off[e], off[e] + d["kept"][e]
        xs = np.ascontiguousarray(d["As"][:, r0:r1].T)
        hq, hs, _ = oracle.expert_rows(d["Aq"][r0:r1], xs, inp["W1q"][e], inp["S1"][e], inp["W3q"][e],
                                       inp["S3"][e], inp["W2q"][e], inp["S2"][e])
        assert np.array_equal(Dq[r0:r1], hq) and np.array_equal(Ds[:, r0:r1].T, hs)


def test_masked_grouped_gemm_equals_per_expert_dense_gemms():
    # masked layout: block e of A holds masked_m[e] rows of expert e; its scales are [E][K/128][M_rows].
    # Each block's product equals one dense float64 matmul over those rows, the SwiGLU epilogue equals the
    # per-row expert function, and rows at or past masked_m[e] stay untouched (zero here).
    cfg = MoeConfig("gm", T=80, H=256, E=4, I=128, k=2, bias="uniform", layout="masked", masked_max_m=64,
                    seed=6)
    t = make_inputs(cfg)
    inp = oracle.moe_inputs_to_numpy(t)
    idx, w, _ = oracle.route(cfg, inp["x"], inp["Wg"], inp["bias"], inp["token_ids"])
    M = cfg.masked_max_m
    d = oracle.permute(cfg, inp["x"], idx, cfg.E * M)
    mm = d["kept"]
    assert mm.min() > 0 and mm.max() < M                     # every block ragged, none full
    Aq = d["Aq"].reshape(cfg.E * M, cfg.H)
    As = d["As"].reshape(cfg.E, cfg.H // 128, M)
    B, Bs = np.ascontiguousarray(inp["W1q"]), np.ascontiguousarray(inp["S1"])
    D, _ = oracle.grouped_gemm(1, cfg.E, cfg.I, cfg.H, Aq, As, mm, M, B, Bs, 0)
    W13, S13 = interleave_w13(t.W1q, t.S1, t.W3q, t.S3)
    Dq, Ds = oracle.grouped_gemm(1, cfg.E, 2 * cfg.I, cfg.H, Aq, As, mm, M, W13.numpy(), S13.numpy(), 1)
    for e in range(cfg.E):
        r0, n = e * M, int(mm[e])
        A = torch.from_numpy(Aq[r0:r0 + n]).view(torch.float8_e4m3fn).to(torch.float32)
        sA = torch.from_numpy(As[e, :, :n].T.copy()).repeat_interleave(128, 1)
        ref = ((A * sA).to(torch.float64) @ _deq_w(B[e], Bs[e]).T).numpy()
        _close_bf16(D[r0:r0 + n], ref)
        assert not D[r0 + n:r0 + M].any() and not Dq[r0 + n:r0 + M].any() and not Ds[e, :, n:].any()
        hq, hs, _ = oracle.expert_rows(Aq[r0:r0 + n], np.ascontiguousarray(As[e, :, :n].T), inp["W1q"][e],
                                       inp["S1"][e], inp["W3q"][e], inp["S3"][e], inp["W2q"][e], inp["S2"][e])
        assert np.array_equal(Dq[r0:r0 + n], hq) and np.array_equal(Ds[e, :, :n].T, hs)


def _brute_layer(cfg, inp, tokens):
    """Per token, straight from the formulas: fp64 logits, softmax over all E, top-k
    (ties to lower index), renormalise, y = sum_i w_i * E_i(x) with each expert
    evaluated on this one token."""
    x_bits = inp["x"]
    xf = oracle.bf16_bits_to_f32(x_bits).astype(np.float64)
    out = {}
    for t in tokens:
        l = xf[t] @ inp["Wg"].astype(np.float64).T + inp["bias"].astype(np.float64)
        s = np.exp(l - l.max())
        s /= s.sum()
        order = np.argsort(-s, kind="stable")[:cfg.k]
        g = s[order] / s[order].sum()
        y = np.zeros(x_bits.shape[1])
        for gi, e in zip(g, order):
            o = _ffn_torch(x_bits[t:t + 1], inp["W1q"][e], inp["S1"][e], inp["W3q"][e], inp["S3"][e],
                           inp["W2q"][e], inp["S2"][e]).numpy()[0]
            o_bf16 = oracle.bf16_bits_to_f32(oracle.f64_to_bf16_bits(o)).astype(np.float64)
            y += gi * o_bf16
        out[t] = (order, y)
    return out


def test_brute_force_y_formula_tiny():
    cfg = MoeConfig("bf", T=8, H=256, E=8, I=128, k=2, bias="uniform", seed=9)
    inp = oracle.moe_inputs_to_numpy(make_inputs(cfg))
    res = oracle.forward(cfg, inp)
    brute = _brute_layer(cfg, inp, range(cfg.T))
    for t, (order, y) in brute.items():
        assert res["topk_idx"][t].tolist() == order.tolist()
        _close_bf16(res["y"][t:t + 1], y[None], frac_equal=0.99)


def test_sampled_forward_equals_full_forward():
    cfg = MoeConfig("s", T=200, H=256, E=8, I=128, k=2, bias="zipf", cap_num=5, cap_den=4, seed=4)
    inp = oracle.moe_inputs_to_numpy(make_inputs(cfg))
    full = oracle.forward(cfg, inp)
    toks = np.array([0, 7, 150, 199])
    part = oracle.forward(cfg, inp, tokens=toks)
    assert np.array_equal(part["y"][toks], full["y"][toks])
    assert np.array_equal(part["slot_row"], full["slot_row"])
    assert np.count_nonzero(full["slot_row"] < 0) > 0          # capacity dropped some slots


def test_all_dropped_token_gives_zero():
    cfg = MoeConfig("z", T=300, H=128, E=2, I=128, k=1, bias="zero", cap_num=1, cap_den=2, seed=1)
    inp = oracle.moe_inputs_to_numpy(make_inputs(cfg))
    out = oracle.forward(cfg, inp)
    dropped = np.nonzero(out["slot_row"] < 0)[0]
    assert len(dropped) > 0
    assert np.all(out["y"][dropped] == 0)


def test_results_do_not_depend_on_the_thread_count():
    # the oracle splits work items (rows, columns) across threads, never a sum: 1, 3 and 8 threads
    # give identical bits for the router, the grouped GEMM (both epilogues, both weight formats) and
    # the expert rows
    cfg = MoeConfig("thr", T=70, H=256, E=4, I=256, k=2, bias="uniform", seed=9)
    t = make_inputs(cfg)
    inp = oracle.moe_inputs_to_numpy(t)
    logits = [oracle.router_logits(inp["x"], inp["Wg"], inp["bias"], nthreads=n) for n in (1, 3, 8)]
    assert all(np.array_equal(logits[0].view(np.uint32), l.view(np.uint32)) for l in logits[1:])
    idx, w, _ = oracle.route(cfg, inp["x"], inp["Wg"], inp["bias"], inp["token_ids"])
    rows_cap = -(-(cfg.T * cfg.k + cfg.E * 127) // 128) * 128
    d = oracle.permute(cfg, inp["x"], idx, rows_cap)
    W13, S13 = interleave_w13(t.W1q, t.S1, t.W3q, t.S3)
    q4, s4 = quantize_weight_int4(torch.randn(cfg.E * 2 * cfg.I, cfg.H, generator=torch.Generator().manual_seed(3)))
    B4 = q4.numpy().reshape(cfg.E, 2 * cfg.I, cfg.H // 2)
    S4 = np.ascontiguousarray(s4.numpy().reshape(cfg.E, 2 * cfg.I, cfg.H // 128).transpose(0, 2, 1))
    for B, Bs, w4 in ((W13.numpy(), S13.numpy(), False), (B4, S4, True)):
        for epi in (0, 1):
            outs = [oracle.grouped_gemm(0, cfg.E, 2 * cfg.I, cfg.H, d["Aq"], d["As"], d["offsets"], rows_cap, B, Bs,
                                        epi, nthreads=n, w4=w4) for n in (1, 3, 8)]
            for D, Ds in outs[1:]:
                assert np.array_equal(D, outs[0][0])
                assert Ds is None or np.array_equal(Ds.view(np.uint32), outs[0][1].view(np.uint32))
    e, n = 0, int(d["kept"][0])
    xs = np.ascontiguousarray(d["As"][:, :n].T)
    rows = [oracle.expert_rows(d["Aq"][:n], xs, inp["W1q"][e], inp["S1"][e], inp["W3q"][e], inp["S3"][e],
                               inp["W2q"][e], inp["S2"][e], nthreads=k) for k in (1, 3, 8)]
    for r in rows[1:]:
        assert all(np.array_equal(a, b) for a, b in zip(r, rows[0]))
