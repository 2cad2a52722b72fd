"""Expert parallelism on the host: the library's exchange planner (moe_ep_plan) and the torch.distributed
transport, without a GPU.

The planner is checked against the oracle's one-process dispatch of the ranks' batches concatenated in rank
order: for every slot, kept or dropped alike, and for every kept slot the same rank within its expert (so the
same row of the expert's group); per-expert kept counts and padded group sizes identical.

The two-rank gloo test runs the planner and DistTransport (all-gather of counts, all-to-all of rows both ways)
with the oracle's arithmetic standing in for the kernels, which need a GPU: each rank's y must equal the
one-process oracle's y for its tokens, bit for bit."""
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import ep
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, interleave_w13, make_inputs
from gpu_helpers import to_np


def _local_ranks(idx, E):
    """rank of each slot (t, j) among this batch's slots of the same expert, in token order."""
    T, k = idx.shape
    seen = np.zeros(E, np.int64)
    r = np.zeros((T, k), np.int64)
    for t in range(T):
        for j in range(k):
            r[t, j] = seen[idx[t, j]]
            seen[idx[t, j]] += 1
    return r


def _routing(cfg):
    inp = make_inputs(cfg)
    idx, w, _ = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), None)
    return inp, idx, w


def _split(T, G, seed):
    # unequal batches per rank (one may be empty), in rank order
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.integers(0, T + 1, G - 1))
    return np.diff(np.concatenate([[0], cuts, [T]])).astype(int)


CASES = [
    (MoeConfig("ep_a", T=300, H=128, E=8, I=128, k=2, bias="uniform", seed=3), 2),
    (MoeConfig("ep_b", T=301, H=128, E=16, I=128, k=4, bias="zipf", cap_num=5, cap_den=4, seed=4), 4),
    (MoeConfig("ep_c", T=257, H=128, E=8, I=128, k=2, bias="zipf", cap_num=1, cap_den=1, seed=5), 2),
    (MoeConfig("ep_d", T=64, H=128, E=4, I=128, k=1, bias="uniform", seed=6), 1),
    (MoeConfig("ep_e", T=200, H=128, E=8, I=128, k=3, bias="zipf", cap_num=3, cap_den=2, seed=7), 8),
]


@pytest.mark.parametrize("chunks", [1, 2, 3])
@pytest.mark.parametrize("cfg,G", CASES)
def test_plan_matches_one_process_dispatch(cfg, G, chunks):
    inp, idx, _ = _routing(cfg)
    E, k, El = cfg.E, cfg.k, cfg.E // G
    if chunks > El:
        pytest.skip("more chunks than local experts")
    cap = oracle.capacity(cfg.T, k, E, cfg.cap_num, cfg.cap_den)
    rows_cap = -(-(cfg.T * k + E * 127) // 128) * 128
    ref = oracle.dispatch(idx, E, cap, 0, 128, 0, rows_cap)
    sizes = _split(cfg.T, G, cfg.seed)
    bounds = np.concatenate([[0], np.cumsum(sizes)])
    counts_all = np.stack([np.bincount(idx[bounds[s]:bounds[s + 1]].ravel(), minlength=E) for s in range(G)])
    plans = [ep.plan(G, r, E, cfg.T, k, cfg.cap_num, cfg.cap_den, counts_all, chunks) for r in range(G)]
    for s in range(G):
        p = plans[s]
        assert p.chunks == chunks and p.chunk_first[0] == 0 and p.chunk_first[chunks] == El
        assert p.rows_send == sum(p.send_rows[:G]) == p.send_chunk[chunks]
        for d in range(G):
            assert p.send_rows[d] == plans[d].recv_rows[s]     # what s sends to d is what d expects from s
            for c in range(chunks):                             # ... chunk by chunk
                assert p.send_rows_c[c][d] == plans[d].recv_rows_c[c][s]
        for c in range(chunks):
            assert p.send_chunk[c + 1] - p.send_chunk[c] == sum(p.chunk_send(c))
            assert p.recv_chunk[c + 1] - p.recv_chunk[c] == sum(p.chunk_recv(c))
    for d in range(G):
        p = plans[d]
        assert p.rows_recv == p.recv_start[G * El] == sum(p.recv_rows[:G])
        for l in range(El):
            e = d * El + l
            assert p.kept[l] == ref["kept"][e]
            assert p.offsets[l + 1] - p.offsets[l] == ref["offsets"][e + 1] - ref["offsets"][e]
        assert p.rows_group == p.offsets[El]
    # every slot: kept iff the one-process dispatch keeps it, at the same rank within its expert
    for s in range(G):
        loc = idx[bounds[s]:bounds[s + 1]]
        lr = _local_ranks(loc, E)
        p = plans[s]
        seen_send = set()
        for t in range(loc.shape[0]):
            for j in range(k):
                e = int(loc[t, j])
                g_slot = (bounds[s] + t) * k + j
                kept = lr[t, j] < p.kept_mine[e]
                assert kept == (ref["slot_row"][g_slot] >= 0), (s, t, j)
                if not kept:
                    continue
                srow = p.send_off[e] + lr[t, j]
                assert srow not in seen_send and srow < p.rows_send
                seen_send.add(srow)
                d, l = divmod(e, El)
                c = int(np.searchsorted(np.array(p.chunk_first[:chunks + 1]), l, side="right")) - 1
                # the send row lies in its chunk's slice, in the part for destination d
                lo = p.send_chunk[c] + sum(p.send_rows_c[c][:d])
                assert lo <= srow < lo + p.send_rows_c[c][d]
                q = plans[d]
                # receive block of (source s, local expert l): blocks run (chunk, source, expert)
                cf = q.chunk_first
                b = G * cf[c] + s * (cf[c + 1] - cf[c]) + (l - cf[c])
                grow = q.group_start[b] + lr[t, j]
                assert grow - q.offsets[l] == ref["slot_row"][g_slot] - ref["offsets"][e]
                rrow = q.recv_start[b] + lr[t, j]
                assert q.recv_chunk[c] <= rrow < q.recv_start[b + 1] <= q.recv_chunk[c + 1]
                # ... at the same place in d's chunk slice as srow in s's part of it
                assert rrow - q.recv_chunk[c] - sum(q.recv_rows_c[c][:s]) == srow - lo


def test_plan_rejects_bad_arguments():
    from fp8_grouped_gemm_fp32_b200 import api
    c = np.zeros((2, 8), np.int32)
    with pytest.raises(api.MoeError):
        ep.plan(2, 0, 8, 10, 2, 0, 0, c, chunks=5)     # more chunks than the 4 local experts
    with pytest.raises(api.MoeError):
        ep.plan(2, 0, 8, 10, 2, 0, 0, c, chunks=0)
    with pytest.raises(api.MoeError):
        ep.plan(2, 2, 8, 10, 2, 0, 0, c)              # rank outside [0, G)
    with pytest.raises(api.MoeError):
        ep.plan(3, 0, 8, 10, 2, 0, 0, np.zeros((3, 8), np.int32))   # E not a multiple of G
    c[1, 3] = -1
    with pytest.raises(api.MoeError):
        ep.plan(2, 0, 8, 10, 2, 0, 0, c)              # negative count


# ---------------------------------------------------------------- two ranks over gloo
CFG2 = MoeConfig("ep_gloo", T=160, H=256, E=8, I=256, k=2, bias="zipf", cap_num=5, cap_den=4, seed=9)
SIZES2 = [70, 90]


def _rank_main(rank, port, out, chunks):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        cfg, G = CFG2, 2
        E, k, H, El = cfg.E, cfg.k, cfg.H, cfg.E // 2
        inp = make_inputs(cfg)
        xg = to_np(inp.x)
        t0, t1 = sum(SIZES2[:rank]), sum(SIZES2[:rank + 1])
        x = xg[t0:t1]
        c_loc = cfg.replace(T=t1 - t0)
        idx, w, _ = oracle.route(c_loc, x, to_np(inp.Wg), to_np(inp.bias), None)
        tr = ep.DistTransport()
        counts_all = tr.all_gather_counts(torch.from_numpy(np.bincount(idx.ravel(), minlength=E).astype(np.int32)))
        p = ep.plan(G, rank, E, cfg.T, k, cfg.cap_num, cfg.cap_den, counts_all, chunks)
        # send rows as the dispatch kernel lays them out: codes, scales, padding to 16 bytes
        xq, xs = oracle.quant_rows(oracle.bf16_bits_to_f32(x))
        rb = ep.row_bytes(H)
        send = np.zeros((p.rows_send, rb), np.uint8)
        lr = _local_ranks(idx, E)
        base = np.array(p.send_off[:E])
        slot_row = np.full(idx.size, -1, np.int32)
        for t in range(idx.shape[0]):
            for j in range(k):
                e = int(idx[t, j])
                if lr[t, j] < p.kept_mine[e]:
                    r = base[e] + lr[t, j]
                    send[r, :H] = xq[t]
                    send[r, H:H + 4 * (H // 128)] = xs[t].view(np.uint8)
                    slot_row[t * k + j] = r
        # one all-to-all per chunk, each on its slice of the send and receive rows
        recv = np.concatenate([tr.exchange(torch.from_numpy(send[p.send_chunk[c]:p.send_chunk[c + 1]]), p.chunk_send(c),
                                           p.chunk_recv(c)).numpy() for c in range(chunks)])
        # the owner's grouped layout and its experts (the oracle's grouped GEMMs on the local weights)
        M = max(p.rows_group, 128)
        Aq = np.zeros((M, H), np.uint8)
        As = np.ones((H // 128, M), np.float32)
        group_row = np.zeros(p.rows_recv, np.int64)
        for b in range(G * El):
            for i in range(p.recv_start[b], p.recv_start[b + 1]):
                gr = p.group_start[b] + (i - p.recv_start[b])
                group_row[i] = gr
                Aq[gr] = recv[i, :H]
                As[:, gr] = recv[i, H:H + 4 * (H // 128)].view(np.float32)
        sl = slice(rank * El, (rank + 1) * El)
        W13, S13 = interleave_w13(inp.W1q[sl], inp.S1[sl], inp.W3q[sl], inp.S3[sl])
        off = np.array(p.offsets[:El + 1], np.int32)
        Hq, Hs = oracle.grouped_gemm(0, El, 2 * cfg.I, H, Aq, As, off, M, W13.numpy(), S13.numpy(), 1)
        O, _ = oracle.grouped_gemm(0, El, H, cfg.I, Hq, Hs, off, M, to_np(inp.W2q[sl]), to_np(inp.S2[sl]), 0)
        ret = O[group_row] if p.rows_recv else np.zeros((0, H), np.uint16)
        back = np.concatenate([tr.exchange(torch.from_numpy(ret[p.recv_chunk[c]:p.recv_chunk[c + 1]].view(np.int16)),
                                           p.chunk_recv(c), p.chunk_send(c)).numpy() for c in range(chunks)])
        back = back.view(np.uint16).reshape(-1, H)
        y = oracle.combine(slot_row, w, back if back.shape[0] else np.zeros((1, H), np.uint16), c_loc.T, k)
        np.save(os.path.join(out, f"y{rank}.npy"), y)
        np.save(os.path.join(out, f"slot_row{rank}.npy"), slot_row)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("chunks", [1, 3])
def test_two_ranks_over_gloo_equal_one_process(tmp_path, chunks):
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    mp.spawn(_rank_main, args=(port, str(tmp_path), chunks), nprocs=2, join=True)
    cfg = CFG2
    inp = make_inputs(cfg)
    ref = oracle.forward(cfg, oracle.moe_inputs_to_numpy(inp))
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(2)])
    assert np.array_equal(y, ref["y"])
    dropped = np.concatenate([np.load(tmp_path / f"slot_row{r}.npy") for r in range(2)]) < 0
    assert np.array_equal(dropped, ref["slot_row"] < 0)
    assert dropped.any()                                    # the capacity really drops slots
