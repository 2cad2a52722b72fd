"""Pins of the oracle's backward pass (TP-MoE page, 4.1 step 5), each against something other than itself:

* the router part (dw, dl, dW_g, db and the gate's share of dx) against torch float64 autograd of the
  renormalised top-k softmax over W_g x + b with the selection held fixed;
* the SwiGLU derivative against torch float64 autograd of silu(a) * b;
* the 128 x 128 block quantisation of the weight-gradient operands against torch's E4M3 cast;
* the whole backward against torch float64 autograd of the unquantised layer (dequantised weights, no
  FP8 steps in between): within the FP8 quantisation error, which a transposed operand, a dropped term
  or a wrong sign would exceed by far.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, make_inputs


def _inputs(cfg, seed=0):
    inp = make_inputs(cfg)
    d = oracle.moe_inputs_to_numpy(inp)
    g = torch.Generator().manual_seed(seed)
    dy = (torch.randn(cfg.T, cfg.H, generator=g) * 0.1).to(torch.bfloat16)
    return inp, d, dy.view(torch.int16).numpy().view(np.uint16)


CFG = MoeConfig("bwd", T=96, H=256, E=4, I=256, k=2, bias="zipf", cap_num=1, cap_den=1, seed=3)
# experts of up to three 128-row tiles (several K blocks in the weight-gradient sums) and a ragged 384-wide H
CFG_TILES = MoeConfig("bwd_tiles", T=600, H=384, E=8, I=256, k=4, bias="uniform", cap_num=1, cap_den=1, seed=4)
_CFGS = {"small": CFG, "tiles": CFG_TILES}


@pytest.fixture(scope="module", params=list(_CFGS))
def bwd(request):
    cfg = _CFGS[request.param]
    inp, d, dy = _inputs(cfg)
    return cfg, inp, d, dy, oracle.backward(cfg, d, dy)


def test_router_gradients_equal_autograd(bwd):
    cfg, inp, d, dy, r = bwd
    f = r["forward"]
    idx = torch.from_numpy(f["topk_idx"].astype(np.int64))
    x = torch.from_numpy(oracle.bf16_bits_to_f32(d["x"]).astype(np.float64)).requires_grad_()
    Wg = torch.from_numpy(d["Wg"].astype(np.float64)).requires_grad_()
    b = torch.from_numpy(d["bias"].astype(np.float64)).requires_grad_()
    logits = x @ Wg.T + b
    sel = torch.gather(logits, 1, idx)
    w = torch.softmax(sel, dim=1)                  # renormalised over the selected k
    loss = (w * torch.from_numpy(r["dw"].astype(np.float64))).sum()
    loss.backward()
    assert np.allclose(w.detach().numpy(), f["topk_w"], rtol=1e-6, atol=0)
    dsel = torch.autograd.functional.vjp(lambda s: torch.softmax(s, 1), sel.detach(),
                                         torch.from_numpy(r["dw"].astype(np.float64)))[1]
    assert np.allclose(r["dl"], dsel.numpy(), rtol=1e-5, atol=1e-9)
    assert np.allclose(r["dWg"], Wg.grad.numpy(), rtol=1e-5, atol=1e-8)
    assert np.allclose(r["db"], b.grad.numpy(), rtol=1e-5, atol=1e-8)
    assert np.count_nonzero(f["slot_row"] < 0) > 0            # dropped slots still move the gate


def test_swiglu_derivative_equals_autograd():
    rng = np.random.default_rng(1)
    a = torch.from_numpy(rng.standard_normal(500) * 4).requires_grad_()
    b = torch.from_numpy(rng.standard_normal(500)).requires_grad_()
    dh = torch.from_numpy(rng.standard_normal(500))
    (torch.nn.functional.silu(a) * b * dh).sum().backward()
    da, db = oracle.swiglu_backward(a.detach().numpy(), b.detach().numpy(), dh.numpy())
    assert np.allclose(da, a.grad.numpy(), rtol=1e-12, atol=1e-15)
    assert np.allclose(db, b.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_block_quantisation_equals_e4m3_cast():
    rng = np.random.default_rng(2)
    rows, C = 384, 256
    V = (rng.standard_normal((rows, C)) * np.exp(rng.uniform(-5, 5, (rows, 1)))).astype(np.float32)
    offsets = np.array([0, 128, 128, 384], np.int32)            # an empty expert, a ragged one
    kept = np.array([100, 0, 200], np.int32)
    q, s = oracle.tile_transpose_quant(V, offsets, kept, "block")
    W = np.zeros((384, C), np.float32)
    W[0:100] = V[0:100]
    W[128:328] = V[128:328]
    for m in range(3):
        blk = torch.from_numpy(np.ascontiguousarray(W[128 * m:128 * m + 128].T))
        for cb in range(2):
            part = blk[128 * cb:128 * cb + 128]
            amax = part.abs().max()
            sc = torch.where(amax > 0, amax / 448.0, torch.ones(()))
            assert np.float32(s[m, cb]) == np.float32(sc.item())
            want = (part / sc).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            got = q[m, 128 * cb:128 * cb + 128]
            nz = part.numpy() != 0
            assert np.array_equal(got[nz], want[nz])
    qr, sr = oracle.tile_transpose_quant(V, offsets, kept, "row")
    q2, s2 = oracle.quant_rows(np.ascontiguousarray(W.reshape(3, 128, C).transpose(0, 2, 1)).reshape(3 * C, 128))
    assert np.array_equal(qr.reshape(3 * C, 128), q2) and np.array_equal(sr.reshape(3 * C), s2[:, 0])


def test_whole_backward_within_fp8_error_of_unquantised_autograd(bwd):
    cfg, inp, d, dy, r = bwd
    f = r["forward"]
    T, k, E, H, I = cfg.T, cfg.k, cfg.E, cfg.H, cfg.I
    t64 = lambda a: torch.from_numpy(np.asarray(a, np.float64))

    def deq_w(q, s):
        v = oracle.e4m3_decode_array(q)
        return v * np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)

    W1 = [t64(deq_w(d["W1q"][e], d["S1"][e])).requires_grad_() for e in range(E)]
    W3 = [t64(deq_w(d["W3q"][e], d["S3"][e])).requires_grad_() for e in range(E)]
    W2 = [t64(deq_w(d["W2q"][e], d["S2"][e])).requires_grad_() for e in range(E)]
    x = t64(oracle.bf16_bits_to_f32(d["x"])).requires_grad_()
    Wg = t64(d["Wg"]).requires_grad_()
    b = t64(d["bias"]).requires_grad_()
    idx = torch.from_numpy(f["topk_idx"].astype(np.int64))
    w = torch.softmax(torch.gather(x @ Wg.T + b, 1, idx), dim=1)
    y = torch.zeros(T, H, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            if f["slot_row"][t * k + j] < 0:
                continue
            e = int(idx[t, j])
            h = torch.nn.functional.silu(W1[e] @ x[t]) * (W3[e] @ x[t])
            y[t] = y[t] + w[t, j] * (W2[e] @ h)
    (y * t64(oracle.bf16_bits_to_f32(dy))).sum().backward()

    def rel(got, want):
        got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
        return np.linalg.norm(got - want) / np.linalg.norm(want)

    bf = lambda a: oracle.bf16_bits_to_f32(a)
    if cfg is CFG_TILES:
        assert int(np.max(f["kept"])) > 256                   # some expert spans three row tiles
    # E4M3 keeps 3 mantissa bits (a rounding error of up to 1/16 of each value): the FP8 forward's y sits
    # about 4.5 % from the unquantised layer, and every backward product adds one or two more quantised
    # operands. db sums signed per-token terms that largely cancel, so its error is that of the terms.
    # 0.1 holds all of this; a dropped term, a swapped operand or a wrong sign gives errors near 1.
    tol = 0.1
    assert rel(bf(f["y"]), y.detach().numpy()) < 0.06
    assert rel(bf(r["dx"]), x.grad.numpy()) < tol
    assert rel(r["dWg"], Wg.grad.numpy()) < tol
    assert rel(r["db"], b.grad.numpy()) < tol
    for e in range(E):
        dW13 = bf(r["dW13"][e]).reshape(I // 128, 2, 128, H)
        assert rel(dW13[:, 0].reshape(I, H), W1[e].grad.numpy()) < tol, e
        assert rel(dW13[:, 1].reshape(I, H), W3[e].grad.numpy()) < tol, e
        assert rel(bf(r["dW2"][e]), W2[e].grad.numpy()) < tol, e


def test_sampled_backward_equals_the_whole_one():
    # the restricted form the full-size GPU check uses: dx of some tokens and the weight gradients of some
    # experts, each equal bit for bit to the whole backward's (same routines, same order, on fewer rows)
    cfg = CFG_TILES
    inp, d, dy = _inputs(cfg)
    full = oracle.backward(cfg, d, dy)
    f = full["forward"]
    dropped_tok = int(np.nonzero((f["slot_row"] < 0).reshape(cfg.T, cfg.k).any(axis=1))[0][0])
    tokens = [0, 7, dropped_tok, cfg.T - 1]                        # one of them has a slot dropped
    experts = [int(np.argmax(f["kept"])), 3]
    s = oracle.backward_sampled(cfg, d, dy, tokens, experts)
    for t in tokens:
        assert np.array_equal(s["dx"][t], full["dx"][t]), t
    for e in experts:
        assert np.array_equal(s["dW13"][e], full["dW13"][e]), e
        assert np.array_equal(s["dW2"][e], full["dW2"][e]), e
