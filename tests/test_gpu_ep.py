"""Expert parallelism on one GPU, through the C ABI.

G ranks are emulated in one process (ep.forward_local: each collective is a concatenation and split of the
ranks' buffers between their kernels; no kernel waits on another rank's), and a one-rank NCCL group runs
the torch.distributed transport (ep.forward_dist). Against the oracle on the ranks' batches concatenated in
rank order: dropped slots bit-exact, the send rows' codes and scales bit-exact with the oracle's 1x128
quantisation, y within max_rel 2e-2 / mean_rel 2e-3; and against moe_forward on the same concatenated batch
(one GPU, same kernel form): y bit for bit, since every row meets the same arithmetic. Plans of several
chunks (each chunk's rows exchanged, its experts run and their outputs returned in turn; in the NCCL case
the collectives on a stream of their own) give the same y bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import api, ep
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, interleave_w13
from gpu_helpers import assert_close_bf16, ensure_lib, gpu_forward, gpu_inputs, oracle_inputs, to_np

pytestmark = pytest.mark.gpu

CFG = MoeConfig("ep_gpu", T=600, H=512, E=16, I=256, k=4, bias="zipf", cap_num=5, cap_den=4, seed=21)


def _ranks(cfg, inp, G, sizes):
    El = cfg.E // G
    W13, S13 = interleave_w13(inp.W1q, inp.S1, inp.W3q, inp.S3)
    ranks, xs = [], []
    t0 = 0
    for r in range(G):
        sl = slice(r * El, (r + 1) * El)
        w = ep.RankWeights(W13[sl].contiguous(), S13[sl].contiguous(), inp.W2q[sl].contiguous(),
                           inp.S2[sl].contiguous())
        c = api.Config.from_moe(cfg.replace(T=int(sizes[r])))
        ranks.append(ep.EpRank(c, G, r, inp.Wg, inp.bias, w))
        xs.append(inp.x[t0:t0 + int(sizes[r])].contiguous())
        t0 += int(sizes[r])
    return ranks, xs


@pytest.mark.parametrize("G,sizes,chunks", [(1, [600], 1), (2, [250, 350], 1), (4, [100, 0, 300, 200], 1),
                                            (1, [600], 5), (2, [250, 350], 3), (4, [100, 0, 300, 200], 4)])
def test_ep_local_ranks_equal_one_gpu(G, sizes, chunks):
    ensure_lib()
    cfg = CFG
    inp = gpu_inputs(cfg)
    api.moe_set_contig_kernel(api.CONTIG_SINGLE)
    try:
        ranks, xs = _ranks(cfg, inp, G, sizes)
        ys = ep.forward_local(ranks, xs, chunks=chunks)
        torch.cuda.synchronize()
        assert api.moe_get_device_status() == api.MOE_OK
        one = gpu_forward(cfg, inp)
    finally:
        api.moe_set_contig_kernel(api.CONTIG_AUTO)
    y = torch.cat(ys)
    assert torch.equal(y, one["y"])                               # same rows, same arithmetic
    ref = oracle.forward(cfg, oracle_inputs(inp))
    assert_close_bf16(to_np(y), ref["y"])
    k = cfg.k
    dropped = np.concatenate([to_np(r.slot_row) < 0 for r in ranks])
    assert np.array_equal(dropped, ref["slot_row"] < 0) and dropped.any()
    # send rows: the oracle's codes and scales of the slot's token
    H, G128 = cfg.H, cfg.H // 128
    t0 = 0
    for r in ranks:
        send = to_np(r.send)[:r.plan.rows_send]
        sr = to_np(r.slot_row).reshape(-1, k)
        for t in range(r.cfg.T):
            for j in range(k):
                row = sr[t, j]
                if row < 0:
                    continue
                gt = t0 + t
                assert np.array_equal(send[row, :H], ref["xq"][gt])
                assert np.array_equal(send[row, H:H + 4 * G128].view(np.float32), ref["xs"][gt])
        t0 += r.cfg.T


@pytest.mark.parametrize("chunks", [1, 4])
def test_ep_forward_dist_one_rank_nccl(chunks):
    # the torch.distributed transport on a one-rank NCCL group: all-gather and both all-to-alls really run
    import torch.distributed as dist
    ensure_lib()
    cfg = CFG.replace(T=300)
    inp = gpu_inputs(cfg)
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        api.moe_set_contig_kernel(api.CONTIG_SINGLE)
        ranks, xs = _ranks(cfg, inp, 1, [cfg.T])
        y = ep.forward_dist(ranks[0], xs[0], ep.DistTransport(), cfg.T, chunks=chunks)
        torch.cuda.synchronize()
        one = gpu_forward(cfg, inp)
    finally:
        api.moe_set_contig_kernel(api.CONTIG_AUTO)
        dist.destroy_process_group()
    assert api.moe_get_device_status() == api.MOE_OK
    assert torch.equal(y, one["y"])
