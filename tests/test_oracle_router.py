"""Pins for the oracle's router: the canonical fp32 logit order (hand-built
cases whose result differs under any other pairing or without the fused
multiply-add), the fp32 error bound against an exact fp64 dot product, the
bias placement, top-k selection and tie-break, the renormalised weights, and
hash routing."""
import os

import numpy as np
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_logit_tree_pairs_lane_j_with_j_plus_16():
    # H = 128: lane j sums h = 4j .. 4j+3. Put 2^24 in lane 0 (h = 0) and 1 in lanes 8 (h = 32) and
    # 24 (h = 96). Canonical halving: (p8 + p24) = 2 meets 2^24 exactly at the w=8 level -> 2^24 + 2.
    # Any left-to-right order loses both 1s against 2^24 (ulp 2) -> 2^24.
    H = 128
    x = np.zeros((1, H), np.float32)
    W = np.zeros((1, H), np.float32)
    x[0, [0, 32, 96]] = 1.0
    W[0, 0] = 2.0 ** 24
    W[0, 32] = 1.0
    W[0, 96] = 1.0
    l = oracle.router_logits(_bf16_bits(x), W, None, nthreads=1)
    assert l[0, 0] == np.float32(2.0 ** 24 + 2)


def _cancelling_pair(H, h0, h1):
    # x[h0] * W[h0] = -(1 + 2^-7) exactly; x[h1] * W[h1] = (1 + 2^-7)(1 + 2^-23) = 1 + 2^-7 + 2^-23 + 2^-30.
    # In one fused multiply-add chain (h0 first) they cancel exactly to 2^-23 + 2^-30; rounding the second
    # product on its own (a different lane, or no fused multiply-add) loses 2^-30.
    x = np.zeros((1, H), np.float32)
    W = np.zeros((1, H), np.float32)
    x[0, h0], W[0, h0] = -1.0, 1.0 + 2.0 ** -7
    x[0, h1], W[0, h1] = 1.0 + 2.0 ** -7, 1.0 + 2.0 ** -23
    return oracle.router_logits(_bf16_bits(x), W, None, nthreads=1)[0, 0]


def test_logit_lane_partial_uses_fused_multiply_add():
    # h = 0 and h = 1 are consecutive in lane 0's chain: p = fma(x1, w1, fma(x0, w0, 0)).
    assert _cancelling_pair(128, 0, 1) == np.float32(2.0 ** -23 + 2.0 ** -30)
    assert np.float32(2.0 ** -23 + 2.0 ** -30) != np.float32(2.0 ** -23)


def test_logit_chain_takes_four_consecutive_h_per_128_block():
    # lane 0's chain continues from h = 3 (end of its first group of four) to h = 128 (start of its
    # group in the next 128-wide block): the pair still cancels inside one fused chain
    assert _cancelling_pair(256, 3, 128) == np.float32(2.0 ** -23 + 2.0 ** -30)
    # h = 4 and h = 32 belong to lanes 1 and 8: the second product is rounded before the lanes meet
    assert _cancelling_pair(128, 4, 32) == np.float32(2.0 ** -23)


def test_logits_within_fp32_bound_of_exact():
    rng = np.random.default_rng(0)
    T, H, E = 16, 4096, 64
    x = _bf16_bits(rng.standard_normal((T, H)))
    xf = oracle.bf16_bits_to_f32(x).astype(np.float64)
    W = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    b = rng.uniform(-0.01, 0.01, E).astype(np.float32)
    l = oracle.router_logits(x, W, b)
    exact = xf @ W.astype(np.float64).T + b.astype(np.float64)       # products exact in fp64
    mag = np.abs(xf) @ np.abs(W.astype(np.float64)).T + np.abs(b)
    u = 2.0 ** -24
    bound = (H // 32 + 5 + 1) * u * mag * 1.01
    assert np.all(np.abs(l - exact) <= bound)
    assert np.abs(l - exact).max() > 0       # and it is genuinely fp32, not fp64


def test_bias_is_added_last_in_fp32():
    rng = np.random.default_rng(1)
    x = _bf16_bits(rng.standard_normal((8, 256)))
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    b = rng.uniform(-1, 1, 16).astype(np.float32)
    l0 = oracle.router_logits(x, W, None)
    l1 = oracle.router_logits(x, W, b)
    assert np.array_equal(l1, (l0 + b).astype(np.float32))


def test_one_hot_token_gives_exact_weight_column():
    E, H = 8, 128
    W = (np.random.default_rng(2).standard_normal((E, H)) * 0.02).astype(np.float32)
    x = np.zeros((1, H), np.float32)
    x[0, 77] = 2.0
    l = oracle.router_logits(_bf16_bits(x), W, None)
    assert np.array_equal(l[0], (2.0 * W[:, 77]).astype(np.float32))


def test_topk_ties_go_to_lowest_index_and_output_is_descending():
    logits = np.array([[0.5, 1.0, 1.0, -2.0, 1.0, 0.5],
                       [3.0, 3.0, 3.0, 3.0, 3.0, 3.0],
                       [-1.0, -0.5, 0.25, 0.25, 9.0, -9.0]], np.float32)
    idx, w = oracle.topk_softmax(logits, 3)
    assert idx.tolist() == [[1, 2, 4], [0, 1, 2], [4, 2, 3]]
    assert np.allclose(w[1], 1 / 3, atol=1e-7)


def test_topk_matches_full_softmax_then_renormalise():
    # softmax over all E (fp64 library exp), stable argsort for the top-k, renormalise:
    # the route the router formula takes; equal to the oracle's top-k-of-logits form.
    rng = np.random.default_rng(4)
    T, E, k = 500, 64, 8
    logits = (rng.standard_normal((T, E)) * 1.3).astype(np.float32)
    idx, w = oracle.topk_softmax(logits, k)
    s = torch.softmax(torch.from_numpy(logits.astype(np.float64)), dim=-1).numpy()
    order = np.argsort(-s, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, order)
    sel = np.take_along_axis(s, order, 1)
    w_ref = sel / sel.sum(1, keepdims=True)
    assert np.allclose(w, w_ref, rtol=2e-7, atol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)


def test_topk_with_k_equal_E_is_plain_softmax():
    logits = np.random.default_rng(6).standard_normal((10, 8)).astype(np.float32)
    idx, w = oracle.topk_softmax(logits, 8)
    s = torch.softmax(torch.from_numpy(logits.astype(np.float64)), -1).numpy()
    assert np.allclose(np.take_along_axis(s, idx, 1), w, rtol=2e-7)


def test_hash_golden_and_histogram():
    rows = [l.split("#")[0].split() for l in open(os.path.join(GOLD, "hash.txt"))]
    rows = [r for r in rows if r]
    for tid, E, exp in rows:
        idx, w = oracle.route_hash(np.array([int(tid)], np.int32), int(E))
        assert idx[0, 0] == int(exp) and w[0, 0] == 1.0
    tids = np.random.default_rng(9).integers(0, 102400, 5000).astype(np.int32)
    idx, _ = oracle.route_hash(tids, 256)
    tally = np.zeros(256, np.int64)
    for t in tids.tolist():
        tally[((t * 2654435761) & 0xFFFFFFFF) % 256] += 1
    assert np.array_equal(np.bincount(idx[:, 0], minlength=256), tally)


def test_fixed_fp32_order_selects_as_exact_arithmetic_on_the_page_workload():
    # the fixed fp32 logit order (a reading: the pages give none) against fp64 logits on the page workload's
    # router inputs: no token's top-k set differs, and any token whose top-k could differ has a margin within
    # the fp32 error bound of the canonical order
    from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, make_router_inputs
    from oracle.router_fp64_diagnostic import diagnose
    cfg = CONFIGS["page"]
    x, Wg, bias = make_router_inputs(cfg)
    d = diagnose(cfg, x.view(torch.int16).numpy().view(np.uint16), Wg.numpy(), bias.numpy())
    assert d["differ"] == 0
    assert d["differ_within_near"]
    assert 0 < d["near_ties"] < 0.01 * cfg.T
