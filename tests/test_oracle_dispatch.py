"""Pins for capacity and dispatch: the worked capacity example, brute-force
ranking on small inputs, and the permutation invariants."""
import os

import numpy as np

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_capacity_golden():
    for line in open(os.path.join(GOLD, "capacity.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        T, k, E, num, den, exp = map(int, line)
        assert oracle.capacity(T, k, E, num, den) == exp
    assert oracle.capacity(2048, 2, 64, 0, 0) == -1


def _brute_dispatch(idx, E, cap, pad):
    # Python lists: per expert, the slots in token order; the first `cap` are kept.
    T, k = idx.shape
    per = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            per[idx[t, j]].append((t, j))
    kept = [len(p) if cap < 0 else min(len(p), cap) for p in per]
    off = [0]
    for e in range(E):
        off.append(off[-1] + -(-kept[e] // pad) * pad)
    slot_row = -np.ones(T * k, np.int64)
    for e in range(E):
        for r, (t, j) in enumerate(per[e][:kept[e]]):
            slot_row[t * k + j] = off[e] + r
    return [len(p) for p in per], kept, off, slot_row


def _random_routing(rng, T, E, k, skew):
    p = np.arange(1, E + 1, dtype=np.float64) ** -skew
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def test_dispatch_matches_brute_force():
    rng = np.random.default_rng(0)
    for T, E, k, cap in ((50, 8, 2, -1), (200, 16, 4, 30), (333, 8, 2, 50), (64, 64, 8, 3)):
        idx = _random_routing(rng, T, E, k, 1.1)
        rows_cap = -(-(T * k + E * 127) // 128) * 128
        d = oracle.dispatch(idx, E, cap, 0, 128, 0, rows_cap)
        counts, kept, off, slot_row = _brute_dispatch(idx, E, cap, 128)
        assert d["counts"].tolist() == counts
        assert d["kept"].tolist() == kept
        assert d["offsets"].tolist() == off
        assert np.array_equal(d["slot_row"], slot_row)


def test_dispatch_invariants_with_capacity():
    rng = np.random.default_rng(1)
    T, E, k = 2048, 64, 2
    idx = _random_routing(rng, T, E, k, 1.1)
    cap = oracle.capacity(T, k, E, 6, 5)
    assert cap == 76
    rows_cap = -(-(T * k + E * 127) // 128) * 128
    d = oracle.dispatch(idx, E, cap, 0, 128, 0, rows_cap)
    kept, off, src, sr = d["kept"], d["offsets"], d["row_src"], d["slot_row"]
    assert np.all(kept <= cap) and kept.max() == cap           # the skew does overflow
    assert kept.sum() + np.count_nonzero(sr < 0) == T * k
    assert np.all(off % 128 == 0) and np.all(np.diff(off) >= kept)
    # each kept slot appears exactly once, and row_src inverts slot_row
    kept_slots = np.nonzero(sr >= 0)[0]
    assert np.array_equal(src[sr[kept_slots]], kept_slots)
    assert np.count_nonzero(src >= 0) == kept.sum()
    for e in range(E):
        rows = src[off[e]:off[e] + kept[e]]
        assert np.all(rows >= 0) and np.all(np.diff(rows // k) > 0)     # token order
        assert np.all(idx.reshape(-1)[rows] == e)
        assert np.all(src[off[e] + kept[e]:off[e + 1]] == -1)          # padding
    # a dropped slot's expert had `cap` earlier tokens
    for s in np.nonzero(sr < 0)[0][:200]:
        t, e = s // k, idx.reshape(-1)[s]
        assert np.count_nonzero(idx[:t] == e) >= cap
    # dropless: nothing dropped
    d2 = oracle.dispatch(idx, E, -1, 0, 128, 0, rows_cap)
    assert np.all(d2["slot_row"] >= 0) and np.array_equal(d2["kept"], d2["counts"])


def test_single_token_activates_at_most_k_experts():
    # "a single token activates at most two experts" for top-2 (DeepSeek MoE page, ch.1)
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((300, 64)).astype(np.float32)
    idx, _ = oracle.topk_softmax(logits, 2)
    assert all(len(set(r)) == 2 for r in idx.tolist())


def test_masked_layout_rows_and_overflow():
    rng = np.random.default_rng(3)
    T, E, k, M = 128, 256, 8, 128
    idx = _random_routing(rng, T, E, k, 0.0)
    d = oracle.dispatch(idx, E, -1, 1, 128, M, E * M)
    assert not d["overflow"]
    assert d["offsets"].tolist() == [e * M for e in range(E + 1)]
    for e in range(E):
        rows = d["row_src"][e * M:e * M + d["kept"][e]]
        assert np.all(np.diff(rows // k) > 0) and np.all(idx.reshape(-1)[rows] == e)
    # a masked group smaller than its count overflows and keeps the first M by token order
    idx2 = np.zeros((10, 1), np.int32)
    d2 = oracle.dispatch(idx2, 2, -1, 1, 128, 4, 8)
    assert d2["overflow"] and d2["kept"].tolist() == [4, 0]
    assert d2["slot_row"].tolist() == [0, 1, 2, 3] + [-1] * 6
