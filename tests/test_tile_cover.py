"""Host test of the token selection that the full-size GPU parity tests use: the chosen tokens' kept
rows reach every tile the grouped GEMMs schedule (contiguous 128-row M tiles; masked 32-token slices),
on the oracle's own routing and dispatch."""
import numpy as np
import pytest

import oracle
from fp8_grouped_gemm_fp32_b200.inputs import MoeConfig, capacity_rows_bound, make_inputs
from gpu_helpers import tile_covering_tokens, to_np


@pytest.mark.parametrize("cfg", [
    MoeConfig("c", T=2048, H=256, E=16, I=128, k=4, bias="uniform", seed=1),
    MoeConfig("cap", T=3000, H=256, E=8, I=128, k=2, bias="zipf", cap_num=5, cap_den=4, seed=2),
    MoeConfig("m", T=256, H=256, E=32, I=128, k=4, bias="uniform", layout="masked", masked_max_m=96, seed=3),
])
def test_selected_tokens_cover_every_tile(cfg):
    inp = make_inputs(cfg)
    idx, _, _ = oracle.route(cfg, to_np(inp.x), to_np(inp.Wg), to_np(inp.bias), None)
    layout = 1 if cfg.layout == "masked" else 0
    cap = oracle.capacity(cfg.T, cfg.k, cfg.E, cfg.cap_num, cfg.cap_den)
    d = oracle.dispatch(idx, cfg.E, cap, layout, 128, cfg.masked_max_m, capacity_rows_bound(cfg))
    toks, n_tiles, n_cov = tile_covering_tokens(cfg.layout, d["slot_row"], cfg.k, seed=cfg.seed)
    assert n_cov == n_tiles
    span = 32 if layout else 128
    sr = d["slot_row"].reshape(cfg.T, cfg.k)
    reached = {int(r) // span for t in toks for r in sr[t] if r >= 0}
    all_tiles = {int(r) // span for r in d["slot_row"] if r >= 0}
    assert reached == all_tiles
    if layout == 0:
        assert len(all_tiles) == d["offsets"][-1] // 128
        # every lane quadrant of the tiles is exercised somewhere
        quads = {(int(r) % 128) // 32 for t in toks for r in sr[t] if r >= 0}
        assert quads == {0, 1, 2, 3}
    else:
        assert len(all_tiles) == int(np.sum(-(-d["kept"] // 32)))
    assert len(toks) < cfg.T                                   # a sample, not every token
