"""GPU parity of the layer's backward pass (moe_backward through the C ABI) against the oracle's backward:
dx and the weight gradients dW13, dW2 (bf16) within max_rel 2e-2 / mean_rel 2e-3, the gate's dW_g and db
(fp32) within 1e-3 of the largest entry. The cases drop slots at capacity (their gate gradients still
count), leave an expert empty or nearly so, and give experts several 128-row tiles, so the weight-gradient
GEMM runs several K blocks per expert. The backward after moe_forward_train (the gate and up values saved
by the forward) equals the one after moe_forward (recomputed) bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, MoeConfig, interleave_w13, make_inputs, transpose_weights
from gpu_helpers import assert_close_bf16, ensure_lib, gpu_inputs, oracle_inputs, to_np

pytestmark = pytest.mark.gpu

CASES = {
    "small": MoeConfig("bwd_small", T=96, H=256, E=4, I=256, k=2, bias="zipf", cap_num=1, cap_den=1, seed=3),
    "tiles": MoeConfig("bwd_tiles", T=600, H=384, E=8, I=256, k=4, bias="uniform", cap_num=1, cap_den=1, seed=4),
}


def _rel_fp32(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-30))


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    ensure_lib()
    cfg = CASES[name]
    inp = make_inputs(cfg).to("cuda")
    g = torch.Generator().manual_seed(7)
    dy = (torch.randn(cfg.T, cfg.H, generator=g) * 0.1).to(torch.bfloat16).cuda()
    c = api.Config.from_moe(cfg)
    dev = "cuda"
    T, k, H, E, I = cfg.T, cfg.k, cfg.H, cfg.E, cfg.I
    W13, S13 = interleave_w13(inp.W1q, inp.S1, inp.W3q, inp.S3)
    W13T, S13T, W2T, S2T = transpose_weights(W13, S13, inp.W2q, inp.S2)

    def run(train):
        y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        w = torch.empty(T, k, dtype=torch.float32, device=dev)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        slot_row = torch.empty(T * k, dtype=torch.int32, device=dev)
        # workspaces hold stale bytes, as reused memory does: nothing may depend on their contents
        fws = torch.full((api.moe_workspace_size(c, 2 if train else 1),), 0x5a, dtype=torch.uint8, device=dev)
        fwd = api.moe_forward_train if train else api.moe_forward
        fwd(c, inp.x, inp.Wg, inp.bias, inp.token_ids, W13, S13, inp.W2q, inp.S2, y, idx, w, counts, slot_row, fws)
        out = dict(slot_row=slot_row, dx=torch.empty(T, H, dtype=torch.bfloat16, device=dev),
                   dWg=torch.empty(E, H, dtype=torch.float32, device=dev), db=torch.empty(E, dtype=torch.float32, device=dev),
                   dW13=torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=dev),
                   dW2=torch.empty(E, H, I, dtype=torch.bfloat16, device=dev))
        bws = torch.full((api.moe_backward_workspace_size(c),), 0x5a, dtype=torch.uint8, device=dev)
        api.moe_backward(c, inp.x, inp.Wg, W13, S13, W13T, S13T, W2T, S2T, idx, w, slot_row, fws, dy, out["dx"],
                         out["dWg"], out["db"], out["dW13"], out["dW2"], bws, fwd_train=train)
        return out

    out = run(False)
    trained = run(True)
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    for key in out:
        assert torch.equal(out[key], trained[key]), key
    dx, dWg, db, dW13, dW2, slot_row = (out[key] for key in ("dx", "dWg", "db", "dW13", "dW2", "slot_row"))
    ref = oracle.backward(cfg, oracle.moe_inputs_to_numpy(inp), to_np(dy))
    f = ref["forward"]
    assert np.array_equal(to_np(slot_row), f["slot_row"])
    assert np.count_nonzero(f["slot_row"] < 0) > 0                    # the capacity drops slots
    assert_close_bf16(to_np(dx), ref["dx"], "dx")
    assert _rel_fp32(to_np(dWg), ref["dWg"]) < 1e-3
    assert _rel_fp32(to_np(db), ref["db"]) < 1e-3
    assert_close_bf16(to_np(dW13).reshape(E, -1), ref["dW13"].reshape(E, -1), "dW13")
    assert_close_bf16(to_np(dW2).reshape(E, -1), ref["dW2"].reshape(E, -1), "dW2")
    if name == "tiles":
        assert int(np.max(f["kept"])) > 256                           # some expert spans three row tiles


def test_backward_full_size_sampled():
    # the prefill workload at full size, as the benchmark runs it (moe_forward_train, then moe_backward
    # reading the kept gate and up values): one token's dx row and one expert's whole weight gradients against
    # the oracle's backward restricted to those outputs (a few minutes of CPU: each of the token's eight
    # slots runs the oracle's GEMMs with a whole expert's weights)
    ensure_lib()
    cfg = CONFIGS["prefill"]
    inp = gpu_inputs(cfg, on_device=True)
    c = api.Config.from_moe(cfg)
    dev = "cuda"
    T, k, H, E, I = cfg.T, cfg.k, cfg.H, cfg.E, cfg.I
    g = torch.Generator(device=dev).manual_seed(17)
    dy = (torch.randn(T, H, generator=g, device=dev) * 0.1).to(torch.bfloat16)
    W13, S13 = interleave_w13(inp.W1q, inp.S1, inp.W3q, inp.S3)
    W13T, S13T, W2T, S2T = transpose_weights(W13, S13, inp.W2q, inp.S2)
    z = lambda *shape, dt: torch.empty(*shape, dtype=dt, device=dev)
    y, idx, w = z(T, H, dt=torch.bfloat16), z(T, k, dt=torch.int32), z(T, k, dt=torch.float32)
    counts, slot_row = z(E, dt=torch.int32), z(T * k, dt=torch.int32)
    fws = z(api.moe_workspace_size(c, 2), dt=torch.uint8)
    api.moe_forward_train(c, inp.x, inp.Wg, inp.bias, inp.token_ids, W13, S13, inp.W2q, inp.S2, y, idx, w, counts,
                          slot_row, fws)
    dx, dWg, db = z(T, H, dt=torch.bfloat16), z(E, H, dt=torch.float32), z(E, dt=torch.float32)
    dW13, dW2 = z(E, 2 * I, H, dt=torch.bfloat16), z(E, H, I, dt=torch.bfloat16)
    bws = z(api.moe_backward_workspace_size(c), dt=torch.uint8)
    api.moe_backward(c, inp.x, inp.Wg, W13, S13, W13T, S13T, W2T, S2T, idx, w, slot_row, fws, dy, dx, dWg, db, dW13,
                     dW2, bws, fwd_train=True)
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    del W13T, S13T, W2T, S2T, bws
    oin = oracle_inputs(inp)
    # the sampled outputs are chosen from the oracle's own routing: the expert with the most rows, and the
    # first token routed to it
    idx_o, _, _ = oracle.route(cfg, oin["x"], oin["Wg"], oin["bias"], oin["token_ids"])
    counts_o = np.bincount(idx_o.reshape(-1), minlength=E)
    assert np.array_equal(to_np(counts), counts_o)
    e = int(np.argmax(counts_o))
    assert -(-int(counts_o[e]) // 128) >= 3                            # three or more 128-row tiles
    t = int(np.nonzero((idx_o == e).any(axis=1))[0][0])
    ref = oracle.backward_sampled(cfg, oin, to_np(dy), [t], [e])
    assert np.array_equal(to_np(slot_row), ref["slot_row"])
    assert_close_bf16(to_np(dx[t]), ref["dx"][t], f"dx[{t}]")
    assert_close_bf16(to_np(dW13[e]), ref["dW13"][e], f"dW13[{e}]")
    assert_close_bf16(to_np(dW2[e]), ref["dW2"][e], f"dW2[{e}]")
