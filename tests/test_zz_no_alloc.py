"""moe_permute_noalloc, the permutation entry point for callers that may not
allocate device memory (graph capture, fixed-budget servers, plugin hosts
whose memory belongs to another allocator): it must give exactly what
moe_permute gives with a caller workspace, call after call, although every
call reuses the same fixed scratch array inside the library.

This file is collected last on purpose, so a run that stops at the first
failure has run every other test before it. It passes alone in a fresh
process as well as after the rest of the suite."""
import numpy as np
import pytest
import torch

from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS, MoeConfig, make_inputs

pytestmark = pytest.mark.gpu


def _route(cfg, inp):
    c = api.Config.from_moe(cfg)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(api.moe_workspace_size(c), 16), dtype=torch.uint8, device="cuda")
    api.moe_route(c, inp.x, inp.Wg, inp.bias, inp.token_ids, idx, w, ws)
    return idx


def _outputs(cfg, fill):
    c = api.Config.from_moe(cfg)
    rows = api.moe_rows_capacity(c)
    H, E, dev = cfg.H, cfg.E, "cuda"
    return dict(
        Aq=torch.full((rows, H), fill, dtype=torch.uint8, device=dev),
        As=torch.full((rows * (H // 128),), float(fill), dtype=torch.float32, device=dev),
        counts=torch.full((E,), fill, dtype=torch.int32, device=dev),
        kept=torch.full((E,), fill, dtype=torch.int32, device=dev),
        offsets=torch.full((E + 1,), fill, dtype=torch.int32, device=dev),
        row_src=torch.full((rows,), fill, dtype=torch.int32, device=dev),
        slot_row=torch.full((cfg.T * cfg.k,), fill, dtype=torch.int32, device=dev))


def _compare(cfg, a, b):
    for key in ("counts", "kept", "offsets", "slot_row"):
        assert torch.equal(a[key], b[key]), key
    kept = a["kept"].cpu().numpy()
    offsets = a["offsets"].cpu().numpy()
    G = cfg.H // 128
    if cfg.layout == "masked":
        M = cfg.masked_max_m
        As_a = a["As"].view(cfg.E, G, M)
        As_b = b["As"].view(cfg.E, G, M)
        for e in range(cfg.E):
            r0, r1 = e * M, e * M + int(kept[e])
            assert torch.equal(a["row_src"][r0:r1], b["row_src"][r0:r1])
            assert torch.equal(a["Aq"][r0:r1], b["Aq"][r0:r1])
            assert torch.equal(As_a[e, :, :kept[e]], As_b[e, :, :kept[e]])
    else:
        used = int(offsets[-1])
        rows = a["row_src"].numel()
        assert torch.equal(a["row_src"][:used], b["row_src"][:used])
        assert torch.equal(a["Aq"][:used], b["Aq"][:used])
        assert torch.equal(a["As"].view(G, rows)[:, :used], b["As"].view(G, rows)[:, :used])


def _run_both(cfg):
    inp = make_inputs(cfg, device="cuda")
    idx = _route(cfg, inp)
    c = api.Config.from_moe(cfg)
    ref = _outputs(cfg, 0x5A)
    ws = torch.empty(api.moe_workspace_size(c), dtype=torch.uint8, device="cuda")
    api.moe_permute(c, inp.x, idx, ref["Aq"], ref["As"], ref["counts"], ref["kept"], ref["offsets"],
                    ref["row_src"], ref["slot_row"], ws)
    got = _outputs(cfg, 0x33)          # different poison, so unwritten entries cannot match by accident
    api.moe_permute_noalloc(c, inp.x, idx, got["Aq"], got["As"], got["counts"], got["kept"], got["offsets"],
                            got["row_src"], got["slot_row"])
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK
    _compare(cfg, got, ref)


def test_noalloc_permute_matches_workspace_permute_twice_in_a_row():
    api.lib()
    # first call: capacity drops on a skewed contiguous workload
    _run_both(CONFIGS["skewed"].replace(T=3000))
    # second call, reusing the same scratch array: a larger masked workload
    _run_both(CONFIGS["decode"])
    # and once more with the first shape, after the array held the other call's counts
    _run_both(CONFIGS["skewed"].replace(T=3000))


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    api.lib()
    cfg = MoeConfig("too_big", T=40000, H=256, E=512, I=128, k=2, seed=0)   # 8 * 1250 * 512 bytes > 2 MiB
    c = api.Config.from_moe(cfg)
    d = torch.empty(64, dtype=torch.int32, device="cuda")
    with pytest.raises(api.MoeError) as ei:
        api.moe_permute_noalloc(c, d, d, d, d, d, d, d, d, d)
    assert ei.value.status == api.MOE_ERR_UNSUPPORTED_SHAPE
