"""CPU oracle for the FP8 MoE expert layer -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product library (fp8_grouped_gemm_fp32_b200) never does,
and the two share no code: this package wraps the plain C in moe_oracle.c
(see moe_oracle.h for the page citations and the readings it follows) and
composes its steps with numpy.

Parity pins for every function here are in tests/test_oracle_*.py. One part
is "parity unpinned" beyond invariants and special cases: the end-to-end
values of y for general inputs (the pages print no worked numeric example).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GROUP = 128


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            return any(line.startswith("flags") and " fma " in line + " " for line in f)
    except OSError:
        return False


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (no contraction, no fast-math)."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + ".tmp"
        # -mfma only selects the hardware instruction for fmaf (same correctly rounded result)
        fma = ["-mfma"] if _cpu_has_fma() else []
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math", *fma,
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _declare(_lib)
    return _lib


_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64


def _declare(L):
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_f32.restype = ctypes.c_float
    L.orc_f64_to_bf16.argtypes = [ctypes.c_double]
    L.orc_f64_to_bf16.restype = ctypes.c_uint16
    L.orc_router_logits.argtypes = [_i, _i, _i, _p, _p, _p, _p, _i]
    L.orc_topk_softmax.argtypes = [_i, _i, _i, _p, _p, _p]
    L.orc_route_hash.argtypes = [_i, _i, _p, _p, _p]
    L.orc_capacity.argtypes = [_i, _i, _i, _i, _i]
    L.orc_capacity.restype = _i64
    L.orc_dispatch.argtypes = [_i, _i, _i, _p, _i64, _i, _i, _i, _i64, _p, _p, _p, _p, _p]
    L.orc_dispatch.restype = _i
    L.orc_quant_rows.argtypes = [_i64, _i, _p, _p, _p]
    L.orc_expert_rows.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i]
    L.orc_grouped_gemm.argtypes = [_i, _i, _i, _i, _p, _p, _p, _i, _p, _p, _i, _p, _p, _i]
    L.orc_combine.argtypes = [_i, _i, _i, _p, _p, _p, _p]
    L.orc_balance_bias.argtypes = [_i, _p, _p, _p, ctypes.c_float, _i]
    L.orc_grouped_gemm_w4.argtypes = [_i, _i, _i, _i, _p, _p, _p, _i, _p, _p, _i, _p, _p, _i]
    L.orc_w4_decode.argtypes = [_p, _i]
    L.orc_w4_decode.restype = _i
    L.orc_quant_group.argtypes = [_i64, _p, _p, _p]


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# ---------------------------------------------------------------- scalars
def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(v)


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(v, dtype=np.float32).ravel()
    return np.array([L.orc_e4m3_encode(float(x)) for x in flat], dtype=np.uint8).reshape(np.shape(v))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    L = lib()
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([L.orc_f64_to_bf16(float(x)) for x in flat], dtype=np.uint16).reshape(np.shape(v))


# ---------------------------------------------------------------- steps
def router_logits(x_bf16_bits: np.ndarray, Wg: np.ndarray, bias: Optional[np.ndarray],
                  nthreads: Optional[int] = None) -> np.ndarray:
    x = _c(x_bf16_bits, np.uint16)
    Wg = _c(Wg, np.float32)
    T, H = x.shape
    E = Wg.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), dtype=np.float32)
    lib().orc_router_logits(T, H, E, _ptr(x), _ptr(Wg), _ptr(b), _ptr(out), nthreads or default_threads())
    return out


def topk_softmax(logits: np.ndarray, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    lib().orc_topk_softmax(T, E, k, _ptr(logits), _ptr(idx), _ptr(w))
    return idx, w


def route_hash(token_ids: np.ndarray, E: int):
    tid = _c(token_ids, np.int32)
    T = tid.shape[0]
    idx = np.empty((T, 1), dtype=np.int32)
    w = np.empty((T, 1), dtype=np.float32)
    lib().orc_route_hash(T, E, _ptr(tid), _ptr(idx), _ptr(w))
    return idx, w


def capacity(T: int, k: int, E: int, cap_num: int, cap_den: int) -> int:
    return int(lib().orc_capacity(T, k, E, cap_num, cap_den))


def dispatch(topk_idx: np.ndarray, E: int, cap: int, layout: int, pad: int, masked_max_m: int,
             rows_cap: int):
    idx = _c(topk_idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    kept = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    row_src = np.empty(rows_cap, dtype=np.int32)
    slot_row = np.empty(T * k, dtype=np.int32)
    overflow = lib().orc_dispatch(T, k, E, _ptr(idx), cap, layout, pad, masked_max_m, rows_cap,
                                  _ptr(counts), _ptr(kept), _ptr(offsets), _ptr(row_src), _ptr(slot_row))
    return dict(counts=counts, kept=kept, offsets=offsets, row_src=row_src, slot_row=slot_row,
                overflow=bool(overflow))


def quant_rows(v: np.ndarray):
    v = _c(v, np.float32)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.uint8)
    s = np.empty((rows, K // GROUP), dtype=np.float32)
    lib().orc_quant_rows(rows, K, _ptr(v), _ptr(q), _ptr(s))
    return q, s


def expert_rows(xq, xs, W1q, S1, W3q, S3, W2q, S2, nthreads: Optional[int] = None):
    xq = _c(xq, np.uint8)
    xs = _c(xs, np.float32)
    n, H = xq.shape
    I = W1q.shape[0]
    args = [_c(a, t) for a, t in ((W1q, np.uint8), (S1, np.float32), (W3q, np.uint8), (S3, np.float32),
                                  (W2q, np.uint8), (S2, np.float32))]
    hq = np.empty((n, I), dtype=np.uint8)
    hs = np.empty((n, I // GROUP), dtype=np.float32)
    o = np.empty((n, H), dtype=np.uint16)
    lib().orc_expert_rows(n, H, I, _ptr(xq), _ptr(xs), *[_ptr(a) for a in args],
                          _ptr(hq), _ptr(hs), _ptr(o), nthreads or default_threads())
    return hq, hs, o


def w4_decode(row: np.ndarray, k: int) -> int:
    """The 4-bit weight level of element k of a packed row (DeepSeek-V4 lecture page, 3.1): sign and 3-bit
    magnitude, eight consecutive k per little-endian 32-bit word (moe_oracle.c, orc_w4_decode)."""
    r = _c(row, np.uint8)
    return int(lib().orc_w4_decode(_ptr(r), int(k)))


def grouped_gemm(layout: int, E: int, N: int, K: int, A, As, group_info, M_rows: int, B, Bs,
                 epilogue: int, nthreads: Optional[int] = None, w4: bool = False):
    """Oracle of moe_grouped_gemm_fp8. Rows outside every group are left 0. With w4, B holds
    4-bit weight codes [E, N, K/2] and Bs one scale per weight row per 128-wide K block,
    K-block-major [E, K/128, N] (DeepSeek-V4 lecture page, 3.1)."""
    A = _c(A, np.uint8)
    As = _c(As, np.float32)
    gi = _c(group_info, np.int32)
    B = _c(B, np.uint8)
    Bs = _c(Bs, np.float32)
    rows = A.shape[0] if layout == 0 else E * M_rows
    if epilogue == 0:
        D = np.zeros((rows, N), dtype=np.uint16)
        Ds = None
    else:
        D = np.zeros((rows, N // 2), dtype=np.uint8)
        G = N // 2 // GROUP
        Ds = np.zeros((G, M_rows) if layout == 0 else (E, G, M_rows), dtype=np.float32)
    fn = lib().orc_grouped_gemm_w4 if w4 else lib().orc_grouped_gemm
    fn(layout, E, N, K, _ptr(A), _ptr(As), _ptr(gi), M_rows, _ptr(B), _ptr(Bs), epilogue, _ptr(D), _ptr(Ds),
       nthreads or default_threads())
    return D, Ds


def combine(slot_row: np.ndarray, topk_w: np.ndarray, O: np.ndarray, T: int, k: int) -> np.ndarray:
    sr = _c(slot_row, np.int32)
    w = _c(topk_w, np.float32)
    O = _c(O, np.uint16)
    H = O.shape[1]
    y = np.empty((T, H), dtype=np.uint16)
    lib().orc_combine(T, k, H, _ptr(sr), _ptr(w), _ptr(O), _ptr(y))
    return y


# ---------------------------------------------------------------- pipeline
def balance_bias(counts: np.ndarray, load: np.ndarray, bias: np.ndarray, gamma: float, update: bool):
    """Auxiliary-loss-free bias balancing (MegaMoE page, 2.2), one step, in place:
    load (int64) += counts; on an update step the bias (fp32) of every expert whose
    load is above the mean drops by gamma, below it rises by gamma, and load is cleared."""
    assert load.dtype == np.int64 and bias.dtype == np.float32
    assert load.flags["C_CONTIGUOUS"] and bias.flags["C_CONTIGUOUS"]
    c = _c(counts, np.int32)
    E = c.shape[0]
    assert load.shape == (E,) and bias.shape == (E,)
    lib().orc_balance_bias(E, _ptr(c), _ptr(load), _ptr(bias), float(gamma), int(bool(update)))


def route(cfg, x_bits, Wg, bias, token_ids, nthreads=None):
    """Routing step of the layer: (topk_idx [T,k], topk_w [T,k], logits or None)."""
    if cfg.routing == "hash":
        idx, w = route_hash(token_ids, cfg.E)
        return idx, w, None
    logits = router_logits(x_bits, Wg, bias, nthreads)
    idx, w = topk_softmax(logits, cfg.k)
    return idx, w, logits


def permute(cfg, x_bits, topk_idx, rows_cap: int, pad: int = GROUP):
    """Dispatch + activation quantisation in the boundary's layout:
    Aq [rows_cap, H] (masked: [E*Mmax, H]) and As K-block-major [H/128][ld]
    (masked: [E][H/128][Mmax]); padding rows hold code 0 and scale 1.0."""
    T, H = x_bits.shape
    layout = 1 if cfg.layout == "masked" else 0
    cap = capacity(T, topk_idx.shape[1], cfg.E, cfg.cap_num, cfg.cap_den)
    d = dispatch(topk_idx, cfg.E, cap, layout, pad, cfg.masked_max_m, rows_cap)
    xq, xs = quant_rows(bf16_bits_to_f32(x_bits))
    k = topk_idx.shape[1]
    G = H // GROUP
    Aq = np.zeros((rows_cap, H), dtype=np.uint8)
    src = d["row_src"]
    valid = src >= 0
    tok = np.where(valid, src // k, 0)
    Aq[valid] = xq[tok[valid]]
    if layout == 0:
        As = np.ones((G, rows_cap), dtype=np.float32)
        As[:, valid] = xs[tok[valid]].T
    else:
        M = cfg.masked_max_m
        As = np.ones((cfg.E, G, M), dtype=np.float32)
        rows = np.nonzero(valid)[0]
        As[rows // M, :, rows % M] = xs[tok[rows]]
    d.update(cap=cap, Aq=Aq, As=As, xq=xq, xs=xs)
    return d


def expert_rows_w4(xq, xs, W1q, S1, W3q, S3, W2q, S2, nthreads: Optional[int] = None):
    """The expert function with 4-bit weights (DeepSeek-V4 lecture page, 3.1) for n rows: the 4-bit grouped
    GEMM (orc_grouped_gemm_w4) with W1/W3 rows alternating in 128-row blocks and the SwiGLU + 1x128
    requantisation epilogue, then with W2 and the bf16 epilogue, one expert in the masked layout.
    W1q, W3q [I, H/2] and W2q [H, I/2] packed levels; S1, S3 [H/128, I] and S2 [I/128, H] row scales
    (K-block-major). Returns o bf16 bits [n, H]."""
    xq = _c(xq, np.uint8)
    n, H = xq.shape
    I = W1q.shape[0]
    M = max(32, -(-n // 32) * 32)
    A = np.zeros((M, H), np.uint8)
    A[:n] = xq
    As = np.ones((1, H // GROUP, M), np.float32)
    As[0, :, :n] = np.asarray(xs, np.float32).T
    nb = I // GROUP
    W13 = np.stack((np.asarray(W1q).reshape(nb, GROUP, -1), np.asarray(W3q).reshape(nb, GROUP, -1)),
                   axis=1).reshape(2 * I, -1)
    S13 = np.stack((np.asarray(S1).reshape(H // GROUP, nb, GROUP), np.asarray(S3).reshape(H // GROUP, nb, GROUP)),
                   axis=2).reshape(H // GROUP, 2 * I)
    gi = np.array([n], np.int32)
    hq, hs = grouped_gemm(1, 1, 2 * I, H, A, As, gi, M, W13[None], S13[None], 1, nthreads, w4=True)
    o, _ = grouped_gemm(1, 1, H, I, hq, hs, gi, M, np.asarray(W2q)[None], np.asarray(S2)[None], 0, nthreads,
                        w4=True)
    return o[:n]


def expert_outputs_for_rows(inp, rows_by_expert, xq, xs, nthreads=None, w4: bool = False):
    """{expert: (token list)} -> {expert: o bf16 [n, H]} through orc_expert_rows (E4M3 weights) or the
    4-bit grouped GEMMs (w4)."""
    out = {}
    fn = expert_rows_w4 if w4 else (lambda *a: expert_rows(*a)[2])
    for e, toks in rows_by_expert.items():
        toks = np.asarray(toks, dtype=np.int64)
        out[e] = fn(xq[toks], xs[toks], inp["W1q"][e], inp["S1"][e], inp["W3q"][e], inp["S3"][e],
                    inp["W2q"][e], inp["S2"][e], nthreads)
    return out


def forward(cfg, inp: dict, tokens: Optional[np.ndarray] = None, rows_cap: Optional[int] = None,
            nthreads=None):
    """The whole layer. `inp` holds numpy arrays: x (bf16 bits [T,H]), Wg, bias,
    token_ids, W1q, S1, W3q, S3, W2q, S2 (natural, non-interleaved layout).
    With `tokens`, y is evaluated only for those tokens (routing, capacity and
    permutation still run over all T, since ranks are global); rows of y for
    other tokens are left 0. Returns a dict of every intermediate."""
    T = inp["x"].shape[0]
    idx, w, logits = route(cfg, inp["x"], inp["Wg"], inp["bias"], inp["token_ids"], nthreads)
    k = idx.shape[1]
    if rows_cap is None:
        rows_cap = (cfg.E * cfg.masked_max_m if cfg.layout == "masked"
                    else -(-(T * k + cfg.E * (GROUP - 1)) // GROUP) * GROUP)
    d = permute(cfg, inp["x"], idx, rows_cap)
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    by_e = {}
    for t in sel:
        for j in range(k):
            if d["slot_row"][t * k + j] >= 0:
                by_e.setdefault(int(idx[t, j]), []).append(int(t))
    outs = expert_outputs_for_rows(inp, by_e, d["xq"], d["xs"], nthreads, w4=getattr(cfg, "weights", "fp8") == "w4")
    H = inp["x"].shape[1]
    O = np.zeros((rows_cap, H), dtype=np.uint16)
    for e, toks in by_e.items():
        for n, t in enumerate(toks):
            j = int(np.nonzero(idx[t] == e)[0][0])
            O[d["slot_row"][t * k + j]] = outs[e][n]
    y_all = combine(d["slot_row"], w, O, T, k)
    y = np.zeros_like(y_all)
    y[sel] = y_all[sel]
    d.update(topk_idx=idx, topk_w=w, logits=logits, O=O, y=y, tokens=sel)
    return d


def moe_inputs_to_numpy(inp) -> dict:
    """torch MoeInputs -> numpy dict (bit-preserving views; host copies)."""
    import torch
    return dict(
        x=inp.x.detach().cpu().view(torch.int16).numpy().view(np.uint16),
        Wg=inp.Wg.detach().cpu().numpy(), bias=inp.bias.detach().cpu().numpy(),
        token_ids=inp.token_ids.detach().cpu().numpy(),
        W1q=inp.W1q.detach().cpu().numpy(), S1=inp.S1.detach().cpu().numpy(),
        W3q=inp.W3q.detach().cpu().numpy(), S3=inp.S3.detach().cpu().numpy(),
        W2q=inp.W2q.detach().cpu().numpy(), S2=inp.S2.detach().cpu().numpy())


# ---------------------------------------------------------------- backward pass
# The layer's backward (TP-MoE page, 4.1 step 5: gradients go back along the dispatch path and the gate
# network is updated too). The pages fix no precision for it; the readings this oracle follows:
#  * the quantisation steps of the forward pass count as the identity (their gradient passes straight
#    through), and top-k selection, capacity and routing are held fixed;
#  * every operand of a backward grouped GEMM is FP8 with fp32 scales, like the forward's: a gradient
#    operand in 1x128 groups along the contraction, the other operand of a weight-gradient GEMM in
#    128x128 blocks (the forward's weight granularity); sums in fp64; GEMM outputs bf16 (RNE);
#  * intermediates stored between steps: dO = w * dy in fp32, then FP8; dh, a, b and g in bf16.
def quant_group(v: np.ndarray):
    """One scale for all of v: (codes like v's shape, scale)."""
    v = _c(v, np.float32)
    q = np.empty(v.shape, dtype=np.uint8)
    s = np.empty(1, dtype=np.float32)
    lib().orc_quant_group(v.size, _ptr(v), _ptr(q), _ptr(s))
    return q, float(s[0])


def tile_transpose_quant(V: np.ndarray, offsets: np.ndarray, kept: np.ndarray, mode: str):
    """The weight-gradient operand of one activation-like matrix V [rows, C] (fp32) in the contiguous
    grouped layout (expert e's rows at offsets[e] .. offsets[e] + kept[e]; other rows count as 0): for
    every 128-row tile m of that layout, the transposed block V[128 m : 128 m + 128]^T [C, 128]
    quantised. mode "row": each of the C rows of 128 values one 1x128 group (scales [tiles, C]);
    mode "block": each 128 x 128 block one scale (scales [tiles, C / 128]). Returns codes
    [tiles, C, 128], scales."""
    tiles = int(offsets[-1]) // GROUP
    C = V.shape[1]
    W = np.zeros((tiles * GROUP, C), np.float32)
    for e in range(len(kept)):
        a, n = int(offsets[e]), int(kept[e])
        W[a:a + n] = V[a:a + n]
    Tt = np.ascontiguousarray(W.reshape(tiles, GROUP, C).transpose(0, 2, 1))
    if mode == "row":
        q, s = quant_rows(Tt.reshape(tiles * C, GROUP))
        return q.reshape(tiles, C, GROUP), s.reshape(tiles, C)
    q = np.empty((tiles, C, GROUP), np.uint8)
    s = np.empty((tiles, C // GROUP), np.float32)
    for m in range(tiles):
        for cb in range(C // GROUP):
            q[m, cb * GROUP:(cb + 1) * GROUP], s[m, cb] = quant_group(Tt[m, cb * GROUP:(cb + 1) * GROUP])
    return q, s


def _deq_tiles(q, s):
    """codes [tiles, C, 128] with scales [tiles, C] or [tiles, C/128] -> fp32 values."""
    v = e4m3_decode_array(q).astype(np.float32)
    if s.shape[1] == q.shape[1]:
        return (v * s[:, :, None]).astype(np.float32)
    return (v * np.repeat(s, GROUP, axis=1)[:, :, None]).astype(np.float32)


def swiglu_backward(a: np.ndarray, b: np.ndarray, dh: np.ndarray):
    """h = silu(a) * b: (da, db) in fp64 from a, b, dh (any float arrays)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    dh = np.asarray(dh, np.float64)
    sg = 1.0 / (1.0 + np.exp(-a))
    return dh * b * sg * (1.0 + a * (1.0 - sg)), dh * a * sg


def router_backward(w: np.ndarray, dw: np.ndarray):
    """w_j = exp(l_j - m) / sum_{top-k} exp(l_i - m): dl_j = w_j (dw_j - sum_i w_i dw_i), fp64."""
    w = np.asarray(w, np.float64)
    dw = np.asarray(dw, np.float64)
    return w * (dw - np.sum(w * dw, axis=1, keepdims=True))


def backward(cfg, inp: dict, dy_bits: np.ndarray, nthreads=None):
    """The layer's backward for a gradient dy [T, H] (bf16 bits) of its output. `inp` as for forward.
    Returns dx [T, H] (bf16 bits), dWg [E, H] and db [E] (fp32), dW13 [E, 2I, H] (bf16 bits; rows in
    the W1/W3 128-row block alternation of the forward's up operand) and dW2 [E, H, I] (bf16 bits),
    with the intermediates."""
    f = forward(cfg, inp, nthreads=nthreads)
    idx, w, slot_row = f["topk_idx"], f["topk_w"], f["slot_row"]
    offsets, kept, row_src = f["offsets"], f["kept"], f["row_src"]
    T, k = idx.shape
    H = inp["x"].shape[1]
    E = cfg.E
    I = inp["W1q"][0].shape[0]
    G = H // GROUP
    rows_cap = row_src.shape[0]
    x32 = bf16_bits_to_f32(inp["x"])
    dy = bf16_bits_to_f32(dy_bits)
    # per-row data of the forward in its contiguous layout: x codes/scales, h codes/scales, o
    Aq = f["Aq"]
    As = f["As"]                                   # [G][rows_cap]
    hq = np.zeros((rows_cap, I), np.uint8)
    hs = np.ones((rows_cap, I // GROUP), np.float32)
    O = np.zeros((rows_cap, H), np.uint16)
    for e in range(E):
        a0, n = int(offsets[e]), int(kept[e])
        if n == 0:
            continue
        toks = row_src[a0:a0 + n] // k
        q_, s_, o_ = expert_rows(f["xq"][toks], f["xs"][toks], inp["W1q"][e], inp["S1"][e], inp["W3q"][e],
                                 inp["S3"][e], inp["W2q"][e], inp["S2"][e], nthreads)
        hq[a0:a0 + n], hs[a0:a0 + n], O[a0:a0 + n] = q_, s_, o_
    # router: dw, dl, the gate's gradients and the gate's share of dx
    Of = bf16_bits_to_f32(O).astype(np.float64)
    dw = np.zeros((T, k), np.float64)
    for s in range(T * k):
        if slot_row[s] >= 0:
            dw[s // k, s % k] = np.dot(dy[s // k].astype(np.float64), Of[slot_row[s]])
    dw = dw.astype(np.float32)
    dl = router_backward(w, dw).astype(np.float32)
    dWg = np.zeros((E, H), np.float64)
    db = np.zeros(E, np.float64)
    Wg = np.asarray(inp["Wg"], np.float64)
    dx_router = np.zeros((T, H), np.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            dWg[e] += float(dl[t, j]) * x32[t].astype(np.float64)
            db[e] += float(dl[t, j])
            dx_router[t] += float(dl[t, j]) * Wg[e]
    # dO = w * dy (fp32) on kept rows, 1x128 FP8 along H
    dO = np.zeros((rows_cap, H), np.float32)
    for s in range(T * k):
        r = slot_row[s]
        if r >= 0:
            dO[r] = np.float32(w[s // k, s % k]) * dy[s // k]
    dOq, dOs = quant_rows(dO)
    # transposed weights (layout only): W2^T [E, I, H] with S2^T, W13^T [E, H, 2I] with S13^T
    W13 = np.stack([np.stack((np.asarray(inp["W1q"][e]).reshape(I // GROUP, GROUP, H),
                              np.asarray(inp["W3q"][e]).reshape(I // GROUP, GROUP, H)), axis=1).reshape(2 * I, H)
                    for e in range(E)])
    S13 = np.stack([np.stack((np.asarray(inp["S1"][e]), np.asarray(inp["S3"][e])), axis=1).reshape(2 * I // GROUP, G)
                    for e in range(E)])
    W2 = np.stack([np.asarray(inp["W2q"][e]) for e in range(E)])
    S2 = np.stack([np.asarray(inp["S2"][e]) for e in range(E)])
    W2T, S2T = np.ascontiguousarray(W2.transpose(0, 2, 1)), np.ascontiguousarray(S2.transpose(0, 2, 1))
    W13T, S13T = np.ascontiguousarray(W13.transpose(0, 2, 1)), np.ascontiguousarray(S13.transpose(0, 2, 1))
    # dh = dO W2 (bf16), a|b recomputed (bf16), g = SwiGLU backward (bf16), dx rows = g W13 (bf16)
    dh, _ = grouped_gemm(0, E, I, H, dOq, np.ascontiguousarray(dOs.T), offsets, rows_cap, W2T, S2T, 0, nthreads)
    ab, _ = grouped_gemm(0, E, 2 * I, H, Aq, As, offsets, rows_cap, W13, S13, 0, nthreads)
    abf = bf16_bits_to_f32(ab).reshape(rows_cap, I // GROUP, 2, GROUP)
    dhf = bf16_bits_to_f32(dh).reshape(rows_cap, I // GROUP, GROUP)
    da, dbb = swiglu_backward(abf[:, :, 0], abf[:, :, 1], dhf)
    g = f64_to_bf16_bits(np.stack((da, dbb), axis=2).reshape(rows_cap, 2 * I))
    valid = row_src >= 0
    g[~valid] = 0
    gf = bf16_bits_to_f32(g)
    gq, gs = quant_rows(gf)
    dxr, _ = grouped_gemm(0, E, H, 2 * I, gq, np.ascontiguousarray(gs.T), offsets, rows_cap, W13T, S13T, 0, nthreads)
    dxrf = bf16_bits_to_f32(dxr).astype(np.float64)
    dx64 = dx_router.copy()
    for s in range(T * k):
        if slot_row[s] >= 0:
            dx64[s // k] += dxrf[slot_row[s]]
    dx = f64_to_bf16_bits(dx64)
    # weight gradients over each expert's 128-row tiles
    hf = (e4m3_decode_array(hq).astype(np.float32) * np.repeat(hs, GROUP, axis=1)).astype(np.float32)
    xf = (e4m3_decode_array(Aq).astype(np.float32) * np.repeat(np.ascontiguousarray(As.T), GROUP, axis=1)
          ).astype(np.float32)
    A2 = _deq_tiles(*tile_transpose_quant(dO, offsets, kept, "row"))        # [tiles, H, 128]
    B2 = _deq_tiles(*tile_transpose_quant(hf, offsets, kept, "block"))      # [tiles, I, 128]
    A13 = _deq_tiles(*tile_transpose_quant(gf, offsets, kept, "row"))       # [tiles, 2I, 128]
    B13 = _deq_tiles(*tile_transpose_quant(xf, offsets, kept, "block"))     # [tiles, H, 128]
    dW2 = np.zeros((E, H, I), np.uint16)
    dW13 = np.zeros((E, 2 * I, H), np.uint16)
    for e in range(E):
        m0, m1 = int(offsets[e]) // GROUP, int(offsets[e + 1]) // GROUP
        acc2 = np.zeros((H, I), np.float64)
        acc13 = np.zeros((2 * I, H), np.float64)
        for m in range(m0, m1):
            acc2 += A2[m].astype(np.float64) @ B2[m].astype(np.float64).T
            acc13 += A13[m].astype(np.float64) @ B13[m].astype(np.float64).T
        dW2[e] = f64_to_bf16_bits(acc2)
        dW13[e] = f64_to_bf16_bits(acc13)
    return dict(dx=dx, dWg=dWg.astype(np.float32), db=db.astype(np.float32), dW13=dW13, dW2=dW2, dw=dw, dl=dl,
                dOq=dOq, dOs=dOs, dh=dh, ab=ab, g=g, gq=gq, gs=gs, dx_rows=dxr, forward=f)



def _w13_of(inp, e, I, H):
    """Expert e's up operand as the backward uses it: W13 [2I, H] (W1 and W3 128-row blocks alternating)
    and S13 [2I/128, H/128]."""
    W13 = np.stack((np.asarray(inp["W1q"][e]).reshape(I // GROUP, GROUP, H),
                    np.asarray(inp["W3q"][e]).reshape(I // GROUP, GROUP, H)), axis=1).reshape(2 * I, H)
    S13 = np.stack((np.asarray(inp["S1"][e]), np.asarray(inp["S3"][e])), axis=1).reshape(2 * I // GROUP, H // GROUP)
    return np.ascontiguousarray(W13), np.ascontiguousarray(S13)


def backward_sampled(cfg, inp: dict, dy_bits: np.ndarray, tokens, experts, nthreads=None):
    """`backward` restricted to what some outputs need, for checks at sizes the whole oracle cannot reach:
    dx of `tokens` and dW13[e], dW2[e] of `experts`. Routing, capacity and the permutation still run over
    all T (ranks are global); every other step runs on the rows involved only, through the same routines
    in the same order (each row's GEMMs are independent of the others', an expert's weight gradients sum
    over its own tiles), so the results equal `backward`'s at those entries. Returns dx {token: bf16 row},
    dW13 {e: [2I, H] bf16}, dW2 {e: [H, I] bf16}."""
    x32 = bf16_bits_to_f32(inp["x"])
    dy = bf16_bits_to_f32(dy_bits)
    T, H = inp["x"].shape
    E = cfg.E
    I = np.asarray(inp["W1q"][0]).shape[0]
    idx, w, _ = route(cfg, inp["x"], inp["Wg"], inp["bias"], inp["token_ids"], nthreads)
    k = idx.shape[1]
    rows_cap = -(-(T * k + E * (GROUP - 1)) // GROUP) * GROUP
    cap = capacity(T, k, E, cfg.cap_num, cfg.cap_den)
    d = dispatch(idx, E, cap, 0, GROUP, 0, rows_cap)
    slot_row, offsets, kept, row_src = d["slot_row"], d["offsets"], d["kept"], d["row_src"]
    xq, xs = quant_rows(x32)
    Wg = np.asarray(inp["Wg"], np.float64)

    def rows_chain(e, rows):
        """Expert e on some of its rows (grouped-layout indices): the forward's h and o, then dO, dh, a | b,
        g and the dx rows, as `backward` computes them row by row."""
        rows = np.asarray(rows, np.int64)
        n = rows.size
        slots = row_src[rows]
        toks = slots // k
        hq, hs, o = expert_rows(xq[toks], xs[toks], inp["W1q"][e], inp["S1"][e], inp["W3q"][e], inp["S3"][e],
                                inp["W2q"][e], inp["S2"][e], nthreads)
        dO = np.float32(w[toks, slots % k])[:, None] * dy[toks]
        dOq, dOs = quant_rows(dO.astype(np.float32))
        gi = np.array([0, n], np.int32)
        W13, S13 = _w13_of(inp, e, I, H)
        W2 = np.asarray(inp["W2q"][e])
        S2 = np.asarray(inp["S2"][e])
        W2T, S2T = np.ascontiguousarray(W2.T)[None], np.ascontiguousarray(S2.T)[None]
        W13T, S13T = np.ascontiguousarray(W13.T)[None], np.ascontiguousarray(S13.T)[None]
        dh, _ = grouped_gemm(0, 1, I, H, dOq, np.ascontiguousarray(dOs.T), gi, n, W2T, S2T, 0, nthreads)
        ab, _ = grouped_gemm(0, 1, 2 * I, H, xq[toks], np.ascontiguousarray(xs[toks].T), gi, n, W13[None],
                             S13[None], 0, nthreads)
        abf = bf16_bits_to_f32(ab).reshape(n, I // GROUP, 2, GROUP)
        dhf = bf16_bits_to_f32(dh).reshape(n, I // GROUP, GROUP)
        da, dbb = swiglu_backward(abf[:, :, 0], abf[:, :, 1], dhf)
        gf = bf16_bits_to_f32(f64_to_bf16_bits(np.stack((da, dbb), axis=2).reshape(n, 2 * I)))
        gq, gs = quant_rows(gf)
        dxr, _ = grouped_gemm(0, 1, H, 2 * I, gq, np.ascontiguousarray(gs.T), gi, n, W13T, S13T, 0, nthreads)
        hf = (e4m3_decode_array(hq).astype(np.float32) * np.repeat(hs, GROUP, axis=1)).astype(np.float32)
        xf = (e4m3_decode_array(xq[toks]).astype(np.float32) * np.repeat(xs[toks], GROUP, axis=1)).astype(np.float32)
        return dict(o=o, dO=dO.astype(np.float32), h=hf, g=gf, x=xf, dxr=dxr)

    dx = {}
    for t in np.asarray(tokens, np.int64):
        t = int(t)
        dw = np.zeros((1, k), np.float64)
        dxr_rows = {}
        for j in range(k):
            r = int(slot_row[t * k + j])
            if r < 0:
                continue
            c = rows_chain(int(idx[t, j]), [r])
            dw[0, j] = np.dot(dy[t].astype(np.float64), bf16_bits_to_f32(c["o"][0]).astype(np.float64))
            dxr_rows[j] = bf16_bits_to_f32(c["dxr"][0]).astype(np.float64)
        dl = router_backward(w[t:t + 1], dw.astype(np.float32)).astype(np.float32)
        acc = np.zeros(H, np.float64)
        for j in range(k):
            acc += float(dl[0, j]) * Wg[int(idx[t, j])]
        for j in range(k):
            if j in dxr_rows:
                acc += dxr_rows[j]
        dx[t] = f64_to_bf16_bits(acc)
    dW13, dW2 = {}, {}
    for e in experts:
        e = int(e)
        a0, n = int(offsets[e]), int(kept[e])
        pad = int(offsets[e + 1]) - a0
        if n == 0:
            dW13[e] = np.zeros((2 * I, H), np.uint16)
            dW2[e] = np.zeros((H, I), np.uint16)
            continue
        c = rows_chain(e, np.arange(a0, a0 + n))
        off1, kept1 = np.array([0, pad], np.int32), np.array([n], np.int32)

        def padded(v):
            out = np.zeros((pad, v.shape[1]), np.float32)
            out[:n] = v
            return out
        A2 = _deq_tiles(*tile_transpose_quant(padded(c["dO"]), off1, kept1, "row"))
        B2 = _deq_tiles(*tile_transpose_quant(padded(c["h"]), off1, kept1, "block"))
        A13 = _deq_tiles(*tile_transpose_quant(padded(c["g"]), off1, kept1, "row"))
        B13 = _deq_tiles(*tile_transpose_quant(padded(c["x"]), off1, kept1, "block"))
        acc2 = np.zeros((H, I), np.float64)
        acc13 = np.zeros((2 * I, H), np.float64)
        for m in range(pad // GROUP):
            acc2 += A2[m].astype(np.float64) @ B2[m].astype(np.float64).T
            acc13 += A13[m].astype(np.float64) @ B13[m].astype(np.float64).T
        dW2[e] = f64_to_bf16_bits(acc2)
        dW13[e] = f64_to_bf16_bits(acc13)
    return dict(dx=dx, dW13=dW13, dW2=dW2, slot_row=slot_row, offsets=offsets, kept=kept)
