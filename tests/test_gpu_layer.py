"""GPU parity of the whole layer (moe_forward through the C ABI) against the
oracle: routing indices, per-expert counts and the slot -> row map (which
fixes the permutation and the dropped set) bit-exact; router weights to 1e-6;
the bf16 output within max_rel 2e-2 / mean_rel 2e-3.

Small cases run the oracle on every token; full-size workloads (in the launch
configuration the benchmark times) run the oracle's routing and dispatch on
every token and its expert math on a set of tokens that reaches every tile the
grouped GEMMs schedule."""
import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, MoeConfig, interleave_w13
from gpu_helpers import (W_RTOL, assert_close_bf16, ensure_lib, gpu_forward, gpu_inputs, oracle_inputs,
                         tile_covering_tokens, to_np)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": (CONFIGS["tiny"], None),
    "page_shape_T96": (CONFIGS["page"], 96),
    "skewed_small": (MoeConfig("skewed_small", T=700, H=256, E=8, I=384, k=2, bias="zipf", cap_num=5,
                               cap_den=4, seed=11), None),
    "masked_small": (MoeConfig("masked_small", T=64, H=384, E=16, I=256, k=4, bias="uniform",
                               layout="masked", masked_max_m=64, seed=12), None),
    "hash_small": (MoeConfig("hash_small", T=96, H=256, E=16, I=128, k=1, routing="hash",
                             layout="masked", masked_max_m=96, seed=13), None),
    "one_expert": (MoeConfig("one_expert", T=200, H=256, E=1, I=256, k=1, bias="zero", seed=14), None),
    "w4_masked": (MoeConfig("w4_masked", T=80, H=384, E=16, I=256, k=4, bias="uniform", layout="masked",
                            masked_max_m=64, seed=15, weights="w4"), None),
    # the most experts and the largest k the boundary takes, through both GEMMs: 512 groups of a few rows
    # (contiguous: 512 padded 128-row groups; masked: 512 blocks of 32 rows, E4M3 and 4-bit weights)
    "limits_contig": (MoeConfig("limits_contig", T=64, H=256, E=512, I=128, k=32, bias="uniform", seed=16), None),
    "limits_masked": (MoeConfig("limits_masked", T=64, H=256, E=512, I=128, k=32, bias="uniform", layout="masked",
                                masked_max_m=32, seed=17), None),
    "limits_w4": (MoeConfig("limits_w4", T=64, H=256, E=512, I=128, k=32, bias="uniform", layout="masked",
                            masked_max_m=32, seed=18, weights="w4"), None),
}


def _check_layer(cfg, inp, ref, out, tokens):
    k = ref["topk_idx"].shape[1]
    assert np.array_equal(to_np(out["topk_idx"]), ref["topk_idx"])
    w_gpu = to_np(out["topk_w"])
    assert np.allclose(w_gpu, ref["topk_w"], rtol=W_RTOL, atol=0)
    assert np.array_equal(to_np(out["counts"]), ref["counts"])
    assert np.array_equal(to_np(out["slot_row"]), ref["slot_row"])
    y = to_np(out["y"])
    return assert_close_bf16(y[tokens], ref["y"][tokens])


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small(name):
    ensure_lib()
    cfg, T = SMALL[name]
    inp = gpu_inputs(cfg, T=T)
    cfg = inp.cfg
    ref = oracle.forward(cfg, oracle_inputs(inp))
    out = gpu_forward(cfg, inp)
    _check_layer(cfg, inp, ref, out, np.arange(cfg.T))


@pytest.mark.parametrize("name,form", [("page", api.CONTIG_AUTO), ("page", api.CONTIG_PAIR),
                                       ("prefill", api.CONTIG_AUTO), ("prefill", api.CONTIG_PAIR),
                                       ("decode", api.CONTIG_AUTO),
                                       ("decode_hash", api.CONTIG_AUTO), ("skewed", api.CONTIG_AUTO),
                                       ("decode_w4", api.CONTIG_AUTO)])
def test_layer_full_size_tile_covering(name, form):
    # Every workload at full size, in the launch configuration the benchmark times: routing, counts and the
    # slot -> row map (permutation and dropped set) on every token, and y on a set of tokens whose kept rows
    # reach every tile the two grouped GEMMs schedule (each 128-row M tile of the contiguous layout, each
    # 32-token slice of an expert's block in the masked layout), chosen from the oracle's own dispatch.
    # The default kernel choice runs on every workload; the page workload also runs with CTA pairs forced,
    # where most experts fill one or two 128-row tiles, so many pair tiles are lone (one CTA of the pair
    # idle), and prefill with CTA pairs forced, where most experts fill two or three.
    ensure_lib()
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg, on_device=True)
    api.moe_set_contig_kernel(form)
    try:
        out = gpu_forward(cfg, inp)
    finally:
        api.moe_set_contig_kernel(api.CONTIG_AUTO)
    o_in = oracle_inputs(inp)
    idx, _w, _l = oracle.route(cfg, o_in["x"], o_in["Wg"], o_in["bias"], o_in["token_ids"])
    k = idx.shape[1]
    c = api.Config.from_moe(cfg)
    rows_cap = api.moe_rows_capacity(c)
    cap = oracle.capacity(cfg.T, k, cfg.E, cfg.cap_num, cfg.cap_den)
    d = oracle.dispatch(idx, cfg.E, cap, 1 if cfg.layout == "masked" else 0, 128, cfg.masked_max_m, rows_cap)
    toks, n_tiles, n_cov = tile_covering_tokens(cfg.layout, d["slot_row"], k, seed=cfg.seed)
    assert n_cov == n_tiles and n_tiles > 0                      # the coverage this test claims
    if cfg.layout == "contiguous":
        assert n_tiles == d["offsets"][-1] // 128               # = every M tile the kernels schedule
    else:
        assert n_tiles == int(np.sum(-(-d["kept"] // 32)))
    ref = oracle.forward(cfg, o_in, tokens=toks)
    assert np.array_equal(ref["slot_row"], d["slot_row"])
    _check_layer(cfg, inp, ref, out, toks)
    if cfg.cap_num:
        assert np.count_nonzero(ref["slot_row"] < 0) > 0        # the capacity really drops slots


@pytest.mark.parametrize("name", ["tiny", "masked_small"])
def test_forward_replays_from_a_cuda_graph(name):
    # moe_forward allocates nothing, synchronises nothing and reads no device state on the host, so a
    # stream capture records the whole layer; replayed on new tokens written into the captured input
    # buffer, it gives bit for bit what a direct call on those tokens gives
    ensure_lib()
    cfg, T = SMALL[name]
    inp = gpu_inputs(cfg, T=T)
    cfg = inp.cfg
    c = api.Config.from_moe(cfg)
    W13, S13 = interleave_w13(inp.W1q, inp.S1, inp.W3q, inp.S3)
    dev = inp.x.device
    out = dict(y=torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev),
               topk_idx=torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev),
               counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
               slot_row=torch.empty(cfg.T * cfg.k, dtype=torch.int32, device=dev))
    ws = torch.empty(api.moe_workspace_size(c, True), dtype=torch.uint8, device=dev)

    def call(stream):
        api.moe_forward(c, inp.x, inp.Wg, inp.bias, inp.token_ids, W13, S13, inp.W2q, inp.S2, out["y"],
                        out["topk_idx"], out["topk_w"], out["counts"], out["slot_row"], ws, stream)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        call(side)
    torch.cuda.synchronize()

    inp.x.copy_(gpu_inputs(cfg.replace(seed=cfg.seed + 100), T=cfg.T).x)   # new tokens, same buffer
    call(None)
    torch.cuda.synchronize()
    direct = {k: v.clone() for k, v in out.items()}
    for v in out.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    for k in out:
        assert torch.equal(out[k], direct[k]), k
    ref = oracle.forward(cfg, oracle_inputs(inp))
    _check_layer(cfg, inp, ref, out, np.arange(cfg.T))
    del graph
