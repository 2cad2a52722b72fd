"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports every
entry point include/moe_fp8.h declares, and rejects bad configurations on the
host before touching a device. Also checks that the product path and the
oracle share no code."""
import ctypes
import os
import re

import pytest

from fp8_grouped_gemm_fp32_b200 import api
from fp8_grouped_gemm_fp32_b200.build import build
from fp8_grouped_gemm_fp32_b200.inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_fp8.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    build()
    return api.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(api.EXPORTS)


def declared_arity():
    """name -> number of parameters of each prototype in the header (MOE_EP_ROW_BYTES-style macros aside)."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(L):
    # every ctypes prototype of the binding takes exactly the header's parameters
    arity = declared_arity()
    assert set(arity) == set(api.EXPORTS)
    for name, n in arity.items():
        assert len(getattr(L, name).argtypes) == n, name


def test_status_strings(L):
    for code in range(8):
        assert api.status_string(code)
    assert "sm_100" in api.status_string(api.MOE_ERR_UNSUPPORTED_DEVICE)


def test_rows_and_workspace_sizes(L):
    c = api.Config.from_moe(CONFIGS["prefill"])
    assert api.moe_rows_capacity(c) == -(-(8192 * 8 + 256 * 127) // 128) * 128
    assert api.moe_rows_capacity(api.Config.from_moe(CONFIGS["decode"])) == 256 * 128
    assert api.moe_workspace_size(c, True) > api.moe_workspace_size(c, False) > 0


@pytest.mark.parametrize("field,value,code", [
    ("H", 100, api.MOE_ERR_UNSUPPORTED_SHAPE), ("I", 200, api.MOE_ERR_UNSUPPORTED_SHAPE),
    ("E", 513, api.MOE_ERR_UNSUPPORTED_SHAPE), ("k", 9, api.MOE_ERR_INVALID_ARG),
    ("k", 0, api.MOE_ERR_INVALID_ARG), ("T", -1, api.MOE_ERR_INVALID_ARG),
    ("routing", 5, api.MOE_ERR_INVALID_ARG), ("cap_num", 3, api.MOE_ERR_INVALID_ARG),
    ("layout", 2, api.MOE_ERR_INVALID_ARG), ("H", 16512, api.MOE_ERR_UNSUPPORTED_SHAPE)])
def test_bad_config_rejected_before_any_device_work(L, field, value, code):
    c = api.Config.from_moe(CONFIGS["tiny"])
    setattr(c, field, value)
    assert api.moe_workspace_size(c) == 0
    st = L.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, 0, None)
    assert st == code


@pytest.mark.parametrize("layout,N,K,M_rows,epi,code", [
    (0, 200, 256, 128, 0, api.MOE_ERR_UNSUPPORTED_SHAPE),      # N not a multiple of 128
    (0, 384, 256, 128, 1, api.MOE_ERR_UNSUPPORTED_SHAPE),      # SwiGLU needs N a multiple of 256
    (0, 256, 16512, 128, 0, api.MOE_ERR_UNSUPPORTED_SHAPE),    # K above 16384
    (0, 256, 256, 130, 0, api.MOE_ERR_INVALID_ARG),            # contiguous M_rows not a multiple of 4
    (1, 256, 256, 48, 0, api.MOE_ERR_INVALID_ARG),             # masked M_rows not a multiple of 32
    (2, 256, 256, 128, 0, api.MOE_ERR_INVALID_ARG),            # unknown layout
])
def test_bad_gemm_shape_rejected_before_any_device_work(L, layout, N, K, M_rows, epi, code):
    p = ctypes.c_void_p(4096)                  # aligned, never dereferenced: the call returns first
    st = L.moe_grouped_gemm_fp8(layout, 4, N, K, p, p, p, M_rows, p, p, epi, p, p, None)
    assert st == code


def test_hash_routing_needs_k1_and_masked_needs_rows(L):
    c = api.Config.from_moe(CONFIGS["decode_hash"])
    c.k = 2
    assert api.moe_workspace_size(c) == 0
    c = api.Config.from_moe(CONFIGS["decode"])
    c.masked_max_m = 100                       # not a multiple of 32
    assert api.moe_workspace_size(c) == 0


@pytest.mark.parametrize("layout,N,K,M_rows,epi,code", [
    (0, 256, 256, 128, 0, api.MOE_ERR_UNSUPPORTED_SHAPE),      # 4-bit weights: masked layout only
    (1, 200, 256, 32, 0, api.MOE_ERR_UNSUPPORTED_SHAPE),
    (1, 384, 256, 32, 1, api.MOE_ERR_UNSUPPORTED_SHAPE),
    (1, 256, 16512, 32, 0, api.MOE_ERR_UNSUPPORTED_SHAPE),
    (1, 256, 256, 48, 0, api.MOE_ERR_INVALID_ARG),
    (1, 256, 256, 32, 2, api.MOE_ERR_INVALID_ARG)])
def test_bad_w4_gemm_shape_rejected_before_any_device_work(L, layout, N, K, M_rows, epi, code):
    p = ctypes.c_void_p(4096)
    assert L.moe_grouped_gemm_w4(layout, 4, N, K, p, p, p, M_rows, p, p, epi, p, p, None) == code


@pytest.mark.parametrize("E,gamma,ptr,code", [
    (0, 1e-3, 4096, api.MOE_ERR_INVALID_ARG), (513, 1e-3, 4096, api.MOE_ERR_UNSUPPORTED_SHAPE),
    (8, float("nan"), 4096, api.MOE_ERR_INVALID_ARG), (8, float("inf"), 4096, api.MOE_ERR_INVALID_ARG),
    (8, 1e-3, 4100, api.MOE_ERR_INVALID_ARG), (8, 1e-3, 0, api.MOE_ERR_INVALID_ARG)])
def test_bad_balance_arguments_rejected_before_any_device_work(L, E, gamma, ptr, code):
    p = ctypes.c_void_p(ptr)                   # never dereferenced: the call returns first
    assert L.moe_balance_bias(E, p, p, p, gamma, 1, None) == code


def test_product_and_oracle_share_no_code():
    pkg = os.path.join(ROOT, "fp8_grouped_gemm_fp32_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "moe_oracle" not in src, f
    osrc = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    assert not re.search(r"^\s*(import|from)\s+fp8_grouped_gemm_fp32_b200\b", osrc, re.M)
    assert "moe_fp8.h" not in open(os.path.join(ROOT, "oracle", "moe_oracle.c")).read()


def test_ep_plan_struct_layout_matches_the_header(tmp_path):
    """The binding's moe_ep_plan_t (ctypes) has the C compiler's size and field offsets: the planner writes
    the whole struct into it and the kernels read a byte copy of it."""
    import ctypes
    import shutil
    import subprocess
    from fp8_grouped_gemm_fp32_b200 import ep
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in ep.EpPlan._fields_]
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include "moe_fp8.h"\nint main(void) {\n'
                   '  printf("%zu\\n", sizeof(moe_ep_plan_t));\n' +
                   "".join(f'  printf("%zu\\n", offsetof(moe_ep_plan_t, {f}));\n' for f in fields) + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    assert got[0] == ctypes.sizeof(ep.EpPlan)
    assert got[1:] == [getattr(ep.EpPlan, f).offset for f in fields]


def test_training_workspace_only_for_what_the_training_forward_takes(L):
    prefill = api.Config.from_moe(CONFIGS["prefill"])
    rows = api.moe_rows_capacity(prefill)
    # the training forward keeps the gate and up values: 2 I bf16 values, 4 I bytes, per row
    assert api.moe_workspace_size(prefill, 2) >= api.moe_workspace_size(prefill, 1) + 4 * 2048 * rows
    for name in ("decode", "decode_hash", "decode_w4"):                # masked, hash, 4-bit: no backward
        assert api.moe_workspace_size(api.Config.from_moe(CONFIGS[name]), 2) == 0, name
        assert api.moe_workspace_size(api.Config.from_moe(CONFIGS[name]), 1) > 0, name
    assert L.moe_workspace_size(ctypes.byref(prefill), 3) == 0
    assert L.moe_workspace_size(ctypes.byref(prefill), -1) == 0


@pytest.mark.parametrize("name", ["decode", "decode_hash", "decode_w4"])
def test_training_calls_reject_what_the_backward_does_not_take(L, name):
    # returned before the device is queried: no GPU needed, no pointer read
    c = api.Config.from_moe(CONFIGS[name])
    p = None
    st = L.moe_forward_train(ctypes.byref(c), *([p] * 14), 0, None)
    assert st == api.MOE_ERR_UNSUPPORTED_SHAPE
    assert api.moe_backward_workspace_size(c) == 0
    st = L.moe_backward(ctypes.byref(c), *([p] * 12), 1, *([p] * 7), 0, None)
    assert st == api.MOE_ERR_UNSUPPORTED_SHAPE


def test_backward_rejects_experts_beyond_its_k_limit(L):
    # an expert's rows are the K of its weight-gradient GEMMs, at most 16384; without a capacity every
    # token may reach one expert
    c = api.Config.from_moe(CONFIGS["prefill"])
    c.T = 16512
    assert api.moe_workspace_size(c, 2) > 0                             # a valid forward configuration
    assert api.moe_backward_workspace_size(c) == 0
    st = L.moe_backward(ctypes.byref(c), *([None] * 12), 1, *([None] * 7), 0, None)
    assert st == api.MOE_ERR_UNSUPPORTED_SHAPE
    # a capacity bounds every expert's rows (ceil(T k / E) = 516 here), so the shape passes; the call then
    # stops at the device query (no GPU: a CUDA error, or a device other than sm_100) or at the null pointers
    c.cap_num, c.cap_den = 1, 1
    assert api.moe_backward_workspace_size(c) > 0
    st = L.moe_backward(ctypes.byref(c), *([None] * 12), 1, *([None] * 7), 0, None)
    assert st in (api.MOE_ERR_CUDA, api.MOE_ERR_UNSUPPORTED_DEVICE, api.MOE_ERR_INVALID_ARG)
