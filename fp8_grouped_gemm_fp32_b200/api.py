"""Thin ctypes binding of include/moe_fp8.h with the same entry-point names.

Argument marshalling only: every step runs in libmoe_fp8.so's kernels. Tensors
are torch CUDA tensors (torch provides device memory and streams); their data
pointers are passed straight through. A missing library raises at import of
the first call; there is no fallback path."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build import LIB

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_UNSUPPORTED_DEVICE = 3
MOE_ERR_WORKSPACE_TOO_SMALL = 4
MOE_ERR_CAPACITY = 5
MOE_ERR_CUDA = 6
MOE_ERR_DEVICE_TIMEOUT = 7
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
                3: "MOE_ERR_UNSUPPORTED_DEVICE", 4: "MOE_ERR_WORKSPACE_TOO_SMALL", 5: "MOE_ERR_CAPACITY",
                6: "MOE_ERR_CUDA", 7: "MOE_ERR_DEVICE_TIMEOUT"}
ROUTE_SOFTMAX_TOPK, ROUTE_HASH = 0, 1
LAYOUT_CONTIGUOUS, LAYOUT_MASKED = 0, 1
EPI_BF16, EPI_SWIGLU_FP8 = 0, 1
CONTIG_AUTO, CONTIG_SINGLE, CONTIG_PAIR = 0, 1, 2
WEIGHTS_FP8, WEIGHTS_W4 = 0, 1
EXPORTS = ("moe_rows_capacity", "moe_workspace_size", "moe_route", "moe_permute", "moe_grouped_gemm_fp8",
           "moe_combine", "moe_forward", "moe_forward_train", "moe_get_device_status", "moe_selftest_wait_timeout", "moe_status_string",
           "moe_permute_noalloc", "moe_balance_bias", "moe_grouped_gemm_w4", "moe_set_contig_kernel",
           "moe_ep_plan", "moe_ep_plan_chunked", "moe_ep_workspace_size", "moe_ep_count", "moe_ep_dispatch",
           "moe_ep_receive", "moe_ep_receive_chunk", "moe_ep_return", "moe_backward_workspace_size", "moe_backward")


class MoeError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "H", "E", "I", "k", "routing", "cap_num", "cap_den",
                                            "layout", "masked_max_m", "weights")]

    @classmethod
    def from_moe(cls, cfg) -> "Config":
        """From an inputs.MoeConfig."""
        return cls(cfg.T, cfg.H, cfg.E, cfg.I, cfg.k,
                   ROUTE_HASH if cfg.routing == "hash" else ROUTE_SOFTMAX_TOPK,
                   cfg.cap_num, cfg.cap_den,
                   LAYOUT_MASKED if cfg.layout == "masked" else LAYOUT_CONTIGUOUS,
                   cfg.masked_max_m, WEIGHTS_W4 if getattr(cfg, "weights", "fp8") == "w4" else WEIGHTS_FP8)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"native library {LIB} is missing: run fp8_grouped_gemm_fp32_b200.build.build()")
        L = ctypes.CDLL(LIB)
        P, I, SZ, CP = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.POINTER(Config)
        L.moe_rows_capacity.argtypes = [CP]
        L.moe_rows_capacity.restype = SZ
        L.moe_workspace_size.argtypes = [CP, I]
        L.moe_workspace_size.restype = SZ
        L.moe_route.argtypes = [CP, P, P, P, P, P, P, P, SZ, P]
        L.moe_permute.argtypes = [CP, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_permute_noalloc.argtypes = [CP, P, P, P, P, P, P, P, P, P, P]
        L.moe_grouped_gemm_fp8.argtypes = [I, I, I, I, P, P, P, I, P, P, I, P, P, P]
        L.moe_grouped_gemm_w4.argtypes = [I, I, I, I, P, P, P, I, P, P, I, P, P, P]
        L.moe_combine.argtypes = [CP, P, P, P, P, P]
        L.moe_forward.argtypes = [CP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_forward_train.argtypes = [CP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_balance_bias.argtypes = [I, P, P, P, ctypes.c_float, I, P]
        L.moe_get_device_status.argtypes = [P]
        L.moe_selftest_wait_timeout.argtypes = [I, P]
        L.moe_set_contig_kernel.argtypes = [I]
        L.moe_ep_plan.argtypes = [I, I, I, ctypes.c_int64, I, I, I, P, P]
        L.moe_ep_plan_chunked.argtypes = [I, I, I, ctypes.c_int64, I, I, I, P, I, P]
        L.moe_ep_workspace_size.argtypes = [CP]
        L.moe_ep_workspace_size.restype = SZ
        L.moe_ep_count.argtypes = [CP, P, P, P, SZ, P]
        L.moe_ep_dispatch.argtypes = [CP, P, P, P, P, P, P, SZ, P]
        L.moe_ep_receive.argtypes = [I, P, I, P, P, P, I, P, P, P]
        L.moe_ep_receive_chunk.argtypes = [I, P, I, P, P, P, I, P, P, P]
        L.moe_ep_return.argtypes = [I, I, P, P, P, P]
        L.moe_backward_workspace_size.argtypes = [CP]
        L.moe_backward_workspace_size.restype = SZ
        L.moe_backward.argtypes = [CP] + [P] * 12 + [I] + [P] * 7 + [SZ, P]
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = ctypes.c_char_p
        for f in EXPORTS:
            if f not in ("moe_rows_capacity", "moe_workspace_size", "moe_status_string", "moe_ep_workspace_size",
                         "moe_backward_workspace_size"):
                getattr(L, f).restype = I
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return ctypes.c_void_p(int(t))
    if t.numel() and not t.is_cuda:
        raise ValueError("moe_fp8 entry points take CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("moe_fp8 entry points take contiguous tensors")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() else None


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st: int, call: str):
    if st != MOE_OK:
        raise MoeError(st, call)


def status_string(st: int) -> str:
    return lib().moe_status_string(st).decode()


def moe_rows_capacity(cfg: Config) -> int:
    return int(lib().moe_rows_capacity(ctypes.byref(cfg)))


def moe_workspace_size(cfg: Config, for_forward: int = 0) -> int:
    """Scratch bytes: 0 route / permute, 1 moe_forward, 2 moe_forward_train."""
    return int(lib().moe_workspace_size(ctypes.byref(cfg), int(for_forward)))


def moe_route(cfg, x, Wg, bias, token_ids, topk_idx, topk_w, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(token_ids), _p(topk_idx), _p(topk_w),
                           _p(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)),
           "moe_route")


def moe_permute(cfg, x, topk_idx, Aq, As, counts, kept, offsets, row_src, slot_row, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(Aq), _p(As), _p(counts), _p(kept),
                             _p(offsets), _p(row_src), _p(slot_row), _p(ws), ws.numel() * ws.element_size(),
                             _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, x, topk_idx, Aq, As, counts, kept, offsets, row_src, slot_row, stream=None):
    """moe_permute without a workspace: for callers that may not allocate device memory.
    Uses the library's fixed device scratch; calls that overlap on the GPU race."""
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(Aq), _p(As), _p(counts), _p(kept),
                                     _p(offsets), _p(row_src), _p(slot_row), _stream(stream)), "moe_permute_noalloc")


def moe_grouped_gemm_fp8(layout, E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds=None, stream=None):
    _check(lib().moe_grouped_gemm_fp8(layout, E, N, K, _p(A), _p(As), _p(group_info), M_rows, _p(B), _p(Bs),
                                      epilogue, _p(D), _p(Ds), _stream(stream)), "moe_grouped_gemm_fp8")


def moe_grouped_gemm_w4(layout, E, N, K, A, As, group_info, M_rows, B, Bs, epilogue, D, Ds=None, stream=None):
    """moe_grouped_gemm_fp8 with 4-bit weights: B [E, N, K/2] packed levels, Bs [E, K/128, N] row scales."""
    _check(lib().moe_grouped_gemm_w4(layout, E, N, K, _p(A), _p(As), _p(group_info), M_rows, _p(B), _p(Bs),
                                     epilogue, _p(D), _p(Ds), _stream(stream)), "moe_grouped_gemm_w4")


def moe_combine(cfg, O, slot_row, topk_w, y, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _p(O), _p(slot_row), _p(topk_w), _p(y), _stream(stream)),
           "moe_combine")


def moe_forward(cfg, x, Wg, bias, token_ids, W13, S13, W2, S2, y, topk_idx, topk_w, counts, slot_row, ws,
                stream=None):
    _check(lib().moe_forward(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(token_ids), _p(W13), _p(S13), _p(W2),
                             _p(S2), _p(y), _p(topk_idx), _p(topk_w), _p(counts), _p(slot_row), _p(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "moe_forward")


def moe_forward_train(cfg, x, Wg, bias, token_ids, W13, S13, W2, S2, y, topk_idx, topk_w, counts, slot_row, ws,
                      stream=None):
    """moe_forward that also keeps the gate and up values in ws (moe_workspace_size(cfg, 2) bytes) for
    moe_backward(..., fwd_train=True)."""
    _check(lib().moe_forward_train(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(token_ids), _p(W13), _p(S13),
                                   _p(W2), _p(S2), _p(y), _p(topk_idx), _p(topk_w), _p(counts), _p(slot_row), _p(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "moe_forward_train")


def moe_balance_bias(E, counts, load, bias, gamma, update, stream=None):
    """Auxiliary-loss-free bias step: load (int64) += counts; if update, bias (fp32) moves by -gamma / +gamma
    for experts above / below the mean tally, and load is cleared."""
    _check(lib().moe_balance_bias(E, _p(counts), _p(load), _p(bias), float(gamma), int(bool(update)),
                                  _stream(stream)), "moe_balance_bias")


def moe_get_device_status(stream=None) -> int:
    return int(lib().moe_get_device_status(_stream(stream)))


def moe_selftest_wait_timeout(limit_us: int, stream=None):
    _check(lib().moe_selftest_wait_timeout(limit_us, _stream(stream)), "moe_selftest_wait_timeout")


def moe_set_contig_kernel(form: int):
    """Form of the contiguous-layout grouped GEMM for later calls: CONTIG_AUTO, CONTIG_SINGLE or CONTIG_PAIR."""
    _check(lib().moe_set_contig_kernel(int(form)), "moe_set_contig_kernel")


# ---------------------------------------------------------------- expert parallelism (see ep.py)
def _nbytes(t):
    return t.numel() * t.element_size() if t is not None else 0


def moe_ep_workspace_size(cfg: Config) -> int:
    return int(lib().moe_ep_workspace_size(ctypes.byref(cfg)))


def moe_ep_count(cfg, topk_idx, counts, ws, stream=None):
    _check(lib().moe_ep_count(ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(ws), _nbytes(ws), _stream(stream)),
           "moe_ep_count")


def moe_ep_dispatch(cfg, x, topk_idx, plan_dev, send, slot_row, ws, stream=None):
    _check(lib().moe_ep_dispatch(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(plan_dev), _p(send), _p(slot_row), _p(ws),
                                 _nbytes(ws), _stream(stream)), "moe_ep_dispatch")


def moe_ep_receive(H, plan_dev, rows_recv, recv, Aq, As, M_rows, offsets, group_row, stream=None):
    _check(lib().moe_ep_receive(H, _p(plan_dev), rows_recv, _p(recv) if rows_recv else None, _p(Aq), _p(As), M_rows,
                                _p(offsets), _p(group_row), _stream(stream)), "moe_ep_receive")


def moe_ep_receive_chunk(H, plan_dev, chunk, recv, Aq, As, M_rows, offsets, group_row, stream=None):
    _check(lib().moe_ep_receive_chunk(H, _p(plan_dev), chunk, _p(recv), _p(Aq), _p(As), M_rows, _p(offsets),
                                      _p(group_row), _stream(stream)), "moe_ep_receive_chunk")


def moe_ep_return(H, rows_recv, O, group_row, ret, stream=None):
    _check(lib().moe_ep_return(H, rows_recv, _p(O), _p(group_row), _p(ret), _stream(stream)), "moe_ep_return")


# ---------------------------------------------------------------- backward pass
def moe_backward_workspace_size(cfg: Config) -> int:
    return int(lib().moe_backward_workspace_size(ctypes.byref(cfg)))


def moe_backward(cfg, x, Wg, W13, S13, W13T, S13T, W2T, S2T, topk_idx, topk_w, slot_row, fwd_ws, dy, dx, dWg, db,
                 dW13, dW2, ws, stream=None, fwd_train: bool = False):
    """fwd_train: fwd_ws comes from moe_forward_train (the gate and up values are read, not recomputed)."""
    _check(lib().moe_backward(ctypes.byref(cfg), _p(x), _p(Wg), _p(W13), _p(S13), _p(W13T), _p(S13T), _p(W2T),
                              _p(S2T), _p(topk_idx), _p(topk_w), _p(slot_row), _p(fwd_ws), int(bool(fwd_train)),
                              _p(dy), _p(dx), _p(dWg), _p(db), _p(dW13), _p(dW2), _p(ws), _nbytes(ws),
                              _stream(stream)), "moe_backward")
