"""Host checks of the seeded input module: the same configuration draws the same
arrays; the W1/W3 interleave is a pure re-layout (gate block j, then up block
j); the E4M3 weight quantiser keeps every block within one E4M3 step of the
fp32 weights; the row bound of the permuted buffers matches the C ABI's."""
import torch

from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.build import build
from fp8_grouped_gemm_fp32_b200.inputs import (CONFIGS, MoeConfig, capacity_rows_bound, interleave_w13,
                                               make_inputs, quantize_weight_blocks)


def test_same_config_draws_the_same_arrays():
    cfg = MoeConfig("det", T=48, H=256, E=3, I=128, k=2, bias="uniform", seed=17)
    a, b = make_inputs(cfg), make_inputs(cfg)
    for name in ("x", "Wg", "bias", "token_ids", "W1q", "S1", "W3q", "S3", "W2q", "S2"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    c = make_inputs(cfg.replace(seed=18))
    assert not torch.equal(a.x, c.x)


def test_interleave_is_a_pure_relayout():
    cfg = MoeConfig("il", T=8, H=256, E=2, I=384, k=1, seed=3)
    t = make_inputs(cfg)
    W13, S13 = interleave_w13(t.W1q, t.S1, t.W3q, t.S3)
    assert W13.shape == (2, 768, 256) and S13.shape == (2, 6, 2)
    for j in range(3):
        assert torch.equal(W13[:, 256 * j:256 * j + 128], t.W1q[:, 128 * j:128 * (j + 1)])
        assert torch.equal(W13[:, 256 * j + 128:256 * (j + 1)], t.W3q[:, 128 * j:128 * (j + 1)])
        assert torch.equal(S13[:, 2 * j], t.S1[:, j]) and torch.equal(S13[:, 2 * j + 1], t.S3[:, j])


def test_e4m3_weight_blocks_within_one_step():
    g = torch.Generator().manual_seed(5)
    w = torch.randn(256, 384, generator=g) * 0.02
    w[:128, :128] = 0.0                                        # an all-zero block: scale 1, codes 0
    q, s = quantize_weight_blocks(w)
    deq = q.view(torch.float8_e4m3fn).float() * s.repeat_interleave(128, 0).repeat_interleave(128, 1)
    assert torch.all(q[:128, :128] == 0) and s[0, 0] == 1.0
    blk_max = w.abs().reshape(2, 128, 3, 128).amax(dim=(1, 3))
    assert torch.allclose(s[blk_max > 0], blk_max[blk_max > 0] / 448.0, rtol=0, atol=0)
    # E4M3 has 3 mantissa bits: relative error at most 2^-4 in the normal range, absolute below that
    tol = torch.maximum(w.abs() * 2.0 ** -4, s.repeat_interleave(128, 0).repeat_interleave(128, 1) * 2.0 ** -9)
    assert torch.all((deq - w).abs() <= tol * 1.0001)


def test_row_bound_matches_the_abi():
    build()                                                   # the library's host-side size query
    for name in ("tiny", "page", "prefill", "decode", "decode_hash", "skewed"):
        cfg = CONFIGS[name]
        assert capacity_rows_bound(cfg) == api.moe_rows_capacity(api.Config.from_moe(cfg)), name
