"""Pins for the oracle's auxiliary-loss-free bias balancing (MegaMoE page,
section 2.2): hand-derived cases (direction of the step, a mean that is not an
integer, the tally over the update interval, fp32 rounding of the step, signs,
degenerate tallies), and the closed loop the method exists for: repeated
updates fed by the oracle's own router must even out a skewed expert load, and
the same loop with the step's sign reversed must not."""
import os

import numpy as np
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _floats(tok):
    return np.array([float.fromhex(t) for t in tok], np.float32)


def golden_cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLD, "balance_bias.txt")):
        tok = line.split("#")[0].split()
        if not tok:
            continue
        if tok[0] == "case":
            cur = {"name": tok[1], "E": int(tok[2]), "gamma": float.fromhex(tok[3]), "steps": []}
            cases.append(cur)
        elif tok[0] == "bias0":
            cur["bias0"] = _floats(tok[1:])
        elif tok[0] == "step":
            cur["steps"].append((bool(int(tok[1])), np.array([int(t) for t in tok[2:]], np.int32)))
        elif tok[0] == "bias":
            cur["bias"] = _floats(tok[1:])
        elif tok[0] == "load":
            cur["load"] = np.array([int(t) for t in tok[1:]], np.int64)
    return cases


def test_golden_cases():
    cases = golden_cases()
    assert len(cases) == 8
    for c in cases:
        E = c["E"]
        assert c["bias0"].shape == (E,) and c["bias"].shape == (E,) and c["load"].shape == (E,), c["name"]
        bias = c["bias0"].copy()
        load = np.zeros(E, np.int64)
        for update, counts in c["steps"]:
            oracle.balance_bias(counts, load, bias, c["gamma"], update)
        # bit-exact, so that the sign of a zero counts too
        assert np.array_equal(bias.view(np.uint32), c["bias"].view(np.uint32)), (c["name"], bias, c["bias"])
        assert np.array_equal(load, c["load"]), c["name"]


def test_no_update_only_tallies():
    rng = np.random.default_rng(3)
    E = 16
    bias = rng.uniform(-0.01, 0.01, E).astype(np.float32)
    b0 = bias.copy()
    load = np.zeros(E, np.int64)
    total = np.zeros(E, np.int64)
    for _ in range(5):
        c = rng.integers(0, 1000, E).astype(np.int32)
        total += c
        oracle.balance_bias(c, load, bias, 1e-3, False)
    assert np.array_equal(bias, b0) and np.array_equal(load, total)


def test_large_tallies_compare_exactly():
    # E * load[0] = 3 * (2^40 + 1) exceeds the total 3 * 2^40 + 1 by 2, the others fall short by 1; a
    # float32 tally and mean (both 2^40 after rounding) would leave all three unchanged.
    E = 3
    big = 2 ** 40
    load = np.array([big + 1, big, big], np.int64)
    bias = np.zeros(E, np.float32)
    oracle.balance_bias(np.zeros(E, np.int32), load, bias, 0.5, True)
    assert bias.tolist() == [-0.5, 0.5, 0.5]


def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _imbalance_after(steps, gamma):
    # A Zipf(1.1) log-prior bias (the skewed workload's) sends every token to expert 0 at first; the loop
    # updates the bias after every step (interval 1) from the oracle router's own selections. Returns the
    # largest expert load over the mean load, per step.
    T, H, E, k = 512, 128, 8, 2
    g = np.random.default_rng(11)
    x = _bf16_bits(g.standard_normal((T, H)))
    Wg = (0.02 * g.standard_normal((E, H))).astype(np.float32)
    p = (np.arange(1, E + 1, dtype=np.float64)) ** -1.1
    bias = np.log(p / p.sum()).astype(np.float32)
    load = np.zeros(E, np.int64)
    ratios = []
    for _ in range(steps):
        idx, _w = oracle.topk_softmax(oracle.router_logits(x, Wg, bias, nthreads=1), k)
        counts = np.bincount(idx.ravel(), minlength=E).astype(np.int32)
        ratios.append(counts.max() / (T * k / E))
        oracle.balance_bias(counts, load, bias, gamma, True)
    return ratios


def test_balancing_evens_out_a_skewed_load():
    r = _imbalance_after(200, 0.01)
    assert r[0] == 4.0                     # expert 0 takes every token's first slot
    assert max(r[-20:]) < 1.1              # close to an even split once the biases have moved
    # the step's sign reversed: the load stays as skewed as it started
    assert min(_imbalance_after(40, -0.01)[-10:]) == 4.0
    # a step five times larger settles sooner but keeps oscillating further from the even split, the
    # trade-off the page describes
    big = _imbalance_after(200, 0.05)
    assert max(big[-20:]) > max(r[-20:]) + 0.1
