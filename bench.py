"""Benchmark of the FP8 MoE expert layer on B200: tokens/s of moe_forward,
grouped-GEMM TFLOPS and the dominant kernel's roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config prefill] [--impl ours|reference]

A step is one moe_forward (route -> permute -> up GEMM + SwiGLU/requant ->
down GEMM -> combine) over one batch of synthetic tokens with inputs resident
in HBM. With N > 1 (one process per GPU under torch.distributed) every rank runs
an independent replica of the layer on its own batch: the layer has no
cross-GPU exchange on one GPU's path, so there is no data-path collective and
scaling is weak. Rank 0 prints one JSON line.

`--impl reference` times the CPU oracle (the plain C implementation the
parity tests check against) on the host cores, on bounded samples of the same
workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from fp8_grouped_gemm_fp32_b200.inputs import (CONFIGS, MoeConfig, interleave_w13, interleave_w13_w4,  # noqa: E402
                                                make_inputs)

METRIC = "MoE layer tokens/s; grouped FP8 GEMM TFLOPS and % of B200 roofline"
FP8_PER_BF16 = 2.0          # nominal dense FP8 : BF16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # CUDA-core fp32 peak at the max SM clock
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def describe(cfg: MoeConfig) -> str:
    s = (f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} I={cfg.I} "
         f"{'hash k=1' if cfg.routing == 'hash' else f'top-{cfg.k} softmax'} {cfg.layout} layout")
    if cfg.weights == "w4":
        s += " 4-bit weights (row scales)"
    if cfg.cap_num:
        s += f" capacity ceil(T*k/E)*{cfg.cap_num}/{cfg.cap_den}"
    return s + f" bias={cfg.bias} seed={cfg.seed}"


KERNEL_SOURCES = {"gemm_up": "grouped_gemm.cu", "gemm_down": "grouped_gemm.cu", "router": "router.cu",
                  "permute": "permute.cu", "combine": "combine.cu"}


def source_hash(step: str) -> str:
    import hashlib
    path = os.path.join(ROOT, "fp8_grouped_gemm_fp32_b200", "csrc", KERNEL_SOURCES[step])
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(step: str, workload: str):
    """DRAM bytes per launch (read + write) of a step's kernel from profiles/dram_traffic.txt,
    a summary of one ncu capture; only valid while the kernel's source is unchanged."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = source_hash(step)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == step and parts[1] == workload:
                return float(parts[3]) if parts[2] == want else None
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def measure_fp8_peak(dev, n: int = 8192, reps: int = 10) -> dict:
    """Dense FP8 (E4M3 x E4M3 -> bf16, per-tensor scales) throughput of the library GEMM on this GPU:
    torch._scaled_mm (cuBLASLt) on n x n x n, best of `reps` launches timed with CUDA events. A second
    denominator for the grouped GEMM's tensor roofline, beside 2 x the measured bf16 peak."""
    try:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return {"tflops": 2.0 * n ** 3 / (best / 1e3) / 1e12, "ms": best,
                "how": f"torch._scaled_mm E4M3 {n}^3 -> bf16, per-tensor scales, best of {reps}"}
    except Exception as e:  # pragma: no cover - library without FP8 GEMM support
        return {"tflops": None, "error": str(e)[:200]}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls NVML (SM clock, max clock, throttle reasons) on a thread while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0}
        mhz = [s for s, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = sorted({n for b, n in self.REASONS.items() if bits & b})
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": float(self.max_mhz), "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ algorithmic work
def algorithmic_work(cfg: MoeConfig, kept: np.ndarray):
    """Minimum bytes each step must move and the FLOPs it must do (unpadded rows)."""
    T, H, E, I, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.k
    Rk = int(kept.sum())
    touched = int(np.count_nonzero(kept))
    G = lambda n: n // 128
    if cfg.weights == "w4":       # packed levels (half a byte each) and one fp32 scale per row per K block
        w13 = touched * (2 * I * H // 2 + 4 * 2 * I * G(H))
        w2 = touched * (H * I // 2 + 4 * H * G(I))
    else:
        w13 = touched * (2 * I * H + 4 * G(2 * I) * G(H))
        w2 = touched * (H * I + 4 * G(H) * G(I))
    work = {
        "router": dict(bytes=(T * H * 2 + E * H * 4 + T * k * 8) if cfg.routing != "hash" else T * 4 + T * k * 8,
                       flops=2.0 * T * E * H if cfg.routing != "hash" else 0.0),
        "permute": dict(bytes=T * H * 2 + Rk * (H + 4 * G(H)) + 12 * T * k, flops=0.0),
        "gemm_up": dict(bytes=w13 + Rk * (H + 4 * G(H)) + Rk * (I + 4 * G(I)), flops=2.0 * Rk * 2 * I * H),
        "gemm_down": dict(bytes=w2 + Rk * (I + 4 * G(I)) + Rk * H * 2, flops=2.0 * Rk * H * I),
        "combine": dict(bytes=Rk * H * 2 + T * H * 2 + T * k * 8, flops=0.0),
    }
    return work, Rk, touched


# ------------------------------------------------------------------ our arm
class Layer:
    """Device buffers + the C-ABI calls of one replica of the layer."""

    def __init__(self, cfg: MoeConfig, dev, seed_offset: int = 0):
        from fp8_grouped_gemm_fp32_b200 import api
        self.api = api
        self.cfg = cfg
        self.inp = make_inputs(cfg.replace(seed=cfg.seed + seed_offset), device=dev)
        inter = interleave_w13_w4 if cfg.weights == "w4" else interleave_w13
        self.W13, self.S13 = inter(self.inp.W1q, self.inp.S1, self.inp.W3q, self.inp.S3)
        self.c = api.Config.from_moe(cfg)
        T, k, H, E, I = cfg.T, cfg.k, cfg.H, cfg.E, cfg.I
        z = lambda *s, dt: torch.empty(*s, dtype=dt, device=dev)
        self.y = z(T, H, dt=torch.bfloat16)
        self.topk_idx = z(T, k, dt=torch.int32)
        self.topk_w = z(T, k, dt=torch.float32)
        self.counts = z(E, dt=torch.int32)
        self.slot_row = z(T * k, dt=torch.int32)
        self.ws = z(api.moe_workspace_size(self.c, True), dt=torch.uint8)
        # step-wise buffers (per-kernel breakdown)
        rows = api.moe_rows_capacity(self.c)
        self.rows = rows
        masked = cfg.layout == "masked"
        self.M_rows = cfg.masked_max_m if masked else rows
        self.Aq = z(rows, H, dt=torch.uint8)
        self.As = z(rows * (H // 128), dt=torch.float32)
        self.Hq = z(rows, I, dt=torch.uint8)
        self.Hs = z(rows * (I // 128), dt=torch.float32)
        self.O = z(rows, H, dt=torch.bfloat16)
        self.kept = z(E, dt=torch.int32)
        self.offsets = z(E + 1, dt=torch.int32)
        self.row_src = z(rows, dt=torch.int32)
        self.step_ws = z(api.moe_workspace_size(self.c, False), dt=torch.uint8)
        # router (logits + top-k, or hash) + permute (count, scan, map, quantise) + 2 GEMMs + combine
        self.launches_per_step = (1 if cfg.routing == "hash" else 2) + 4 + 2 + 1

    def forward(self, x=None, stream=None):
        a = self.api
        i = self.inp
        a.moe_forward(self.c, i.x if x is None else x, i.Wg, i.bias, i.token_ids, self.W13, self.S13, i.W2q, i.S2,
                      self.y, self.topk_idx, self.topk_w, self.counts, self.slot_row, self.ws, stream)

    def steps(self, ev):
        """The same five steps as separate C-ABI calls, with an event after each."""
        a, i, cfg = self.api, self.inp, self.cfg
        masked = cfg.layout == "masked"
        group = self.kept if masked else self.offsets
        ev[0].record()
        a.moe_route(self.c, i.x, i.Wg, i.bias, i.token_ids, self.topk_idx, self.topk_w, self.step_ws)
        ev[1].record()
        a.moe_permute(self.c, i.x, self.topk_idx, self.Aq, self.As, self.counts, self.kept, self.offsets,
                      self.row_src, self.slot_row, self.step_ws)
        ev[2].record()
        gemm = a.moe_grouped_gemm_w4 if cfg.weights == "w4" else a.moe_grouped_gemm_fp8
        gemm(int(masked), cfg.E, 2 * cfg.I, cfg.H, self.Aq, self.As, group, self.M_rows, self.W13, self.S13,
             a.EPI_SWIGLU_FP8, self.Hq, self.Hs)
        ev[3].record()
        gemm(int(masked), cfg.E, cfg.H, cfg.I, self.Hq, self.Hs, group, self.M_rows, i.W2q, i.S2, a.EPI_BF16, self.O)
        ev[4].record()
        a.moe_combine(self.c, self.O, self.slot_row, self.topk_w, self.y)
        ev[5].record()


def time_backward(layer, cfg, steps):
    """The layer's backward (moe_backward) after one forward, timed over `steps` calls with CUDA events:
    the training side of the layer, reported beside the forward. Contiguous layout, E4M3 weights, softmax
    routing only."""
    if cfg.layout != "contiguous" or cfg.weights != "fp8" or cfg.routing != "softmax":
        return None
    from fp8_grouped_gemm_fp32_b200.inputs import transpose_weights
    api, i = layer.api, layer.inp
    dev = layer.y.device
    W13T, S13T, W2T, S2T = transpose_weights(layer.W13, layer.S13, i.W2q, i.S2)
    g = torch.Generator(device=dev).manual_seed(17)
    dy = (torch.randn(cfg.T, cfg.H, generator=g, device=dev) * 0.1).to(torch.bfloat16)
    z = lambda *s_, dt: torch.empty(*s_, dtype=dt, device=dev)
    dx, dWg, db = z(cfg.T, cfg.H, dt=torch.bfloat16), z(cfg.E, cfg.H, dt=torch.float32), z(cfg.E, dt=torch.float32)
    dW13, dW2 = z(cfg.E, 2 * cfg.I, cfg.H, dt=torch.bfloat16), z(cfg.E, cfg.H, cfg.I, dt=torch.bfloat16)
    bws = z(api.moe_backward_workspace_size(layer.c), dt=torch.uint8)
    # the training forward keeps the gate and up values, so the backward reads them instead of recomputing
    tws = z(api.moe_workspace_size(layer.c, 2), dt=torch.uint8)

    def fwd_train():
        api.moe_forward_train(layer.c, i.x, i.Wg, i.bias, i.token_ids, layer.W13, layer.S13, i.W2q, i.S2, layer.y,
                              layer.topk_idx, layer.topk_w, layer.counts, layer.slot_row, tws)

    def call():
        api.moe_backward(layer.c, i.x, i.Wg, layer.W13, layer.S13, W13T, S13T, W2T, S2T, layer.topk_idx, layer.topk_w,
                         layer.slot_row, tws, dy, dx, dWg, db, dW13, dW2, bws, fwd_train=True)

    def timed(fn, n):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    fwd_ms = timed(fwd_train, steps)           # leaves the last training forward's state in tws
    torch.cuda.nvtx.range_push("backward")     # lets a profiler select this leg's launches (ncu --nvtx)
    ms = timed(call, steps)
    torch.cuda.nvtx.range_pop()
    assert api.moe_get_device_status() == api.MOE_OK
    Rk = int(layer.kept.sum().item()) if hasattr(layer.kept, "sum") else 0
    # FP8 tensor work: dh (H x I), dx rows (H x 2I), dW2 (H x I), dW13 (2I x H), each 2 FLOP per
    # multiply-add over the kept rows (a | b comes from the training forward)
    flops = 2.0 * Rk * cfg.H * cfg.I * (1 + 2 + 1 + 2)
    del bws, dW13, dW2, tws
    return {"ms": ms, "tokens_per_s": cfg.T / (ms / 1e3), "calls": steps, "gemm_tflops_lower_bound": flops / (ms / 1e3) / 1e12,
            "forward_train_ms": fwd_ms,
            "what": "moe_backward: dx, dW_g, db, dW13, dW2 of one step (four FP8 grouped GEMMs, two of them "
                    "K-grouped weight gradients) after moe_forward_train, which keeps the gate and up values "
                    "(forward_train_ms: that forward's own time)"}


def run_e2e(layer, cfg, steps, world):
    dev = layer.inp.x.device
    hash_routing = cfg.routing == "hash"
    x_host = [layer.inp.x.cpu().pin_memory() for _ in range(2)]
    tid_host = [layer.inp.token_ids.cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(layer.inp.x) for _ in range(2)]
    tid_dev = [torch.empty_like(layer.inp.token_ids) for _ in range(2)]
    y_dev = [torch.empty_like(layer.y) for _ in range(2)]
    up, comp, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    uploaded = [ev(), ev()]       # x_dev[b] holds this step's tokens
    computed = [ev(), ev()]       # y_dev[b] holds this step's output, x_dev[b] may be overwritten
    downloaded = [ev(), ev()]     # y_dev[b] has been read back, it may be overwritten
    for b in range(2):
        downloaded[b].record(down)
        computed[b].record(comp)

    def step(i):
        b = i & 1
        with torch.cuda.stream(up):
            up.wait_event(computed[b])
            x_dev[b].copy_(x_host[b], non_blocking=True)
            if hash_routing:
                tid_dev[b].copy_(tid_host[b], non_blocking=True)
            uploaded[b].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(uploaded[b])
            comp.wait_event(downloaded[b])
            i_ = layer.inp
            layer.api.moe_forward(layer.c, x_dev[b], i_.Wg, i_.bias, tid_dev[b] if hash_routing else i_.token_ids,
                                  layer.W13, layer.S13, i_.W2q, i_.S2, y_dev[b], layer.topk_idx, layer.topk_w,
                                  layer.counts, layer.slot_row, layer.ws, comp)
            computed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            downloaded[b].record(down)

    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(up)
    for i in range(steps):
        step(i)
    end.record(down)          # the last download is the last work of the region
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / steps, world)
    h2d = x_host[0].numel() * 2 + (tid_host[0].numel() * 4 if hash_routing else 0)
    d2h = y_host[0].numel() * 2
    return ms, h2d, d2h


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif n_gpus > 1:
        raise SystemExit("--gpus N > 1 runs under torch.distributed.run (one process per GPU)")
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (a device time: the job is as slow as its slowest rank)."""
    if world == 1:
        return v
    on_gpu = torch.distributed.get_backend() == "nccl"
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def routing_stats(counts, kept) -> dict:
    """Per-expert slot counts of the last step (the router's choice) and the slots the capacity dropped."""
    counts = np.asarray(counts, dtype=np.int64)
    kept = np.asarray(kept, dtype=np.int64)
    return {"count_min": int(counts.min()), "count_max": int(counts.max()), "count_mean": float(counts.mean()),
            "max_over_mean": float(counts.max() / max(counts.mean(), 1e-9)),
            "dropped_slots": int(counts.sum() - kept.sum())}


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time per step."""
    return world * tokens_per_rank / (ms_max / 1e3)


class _HostExperts:
    """Expert-indexed host view of a device weight tensor (one expert copied per access)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].cpu().numpy()


def _oracle_view(inp):
    """numpy view of a MoeInputs for the oracle; weights stay put until an expert is used."""
    return dict(x=inp.x.cpu().view(torch.int16).numpy().view(np.uint16), Wg=inp.Wg.cpu().numpy(),
                bias=inp.bias.cpu().numpy(), token_ids=inp.token_ids.cpu().numpy(),
                W1q=_HostExperts(inp.W1q), S1=_HostExperts(inp.S1), W3q=_HostExperts(inp.W3q),
                S3=_HostExperts(inp.S3), W2q=_HostExperts(inp.W2q), S2=_HostExperts(inp.S2))


def _oracle_step(cfg, view, n, threads):
    """One oracle pass over the first n tokens of the workload as one batch; returns seconds."""
    import oracle
    sub = dict(view)
    sub["x"] = view["x"][:n]
    sub["token_ids"] = view["token_ids"][:n]
    c = cfg.replace(T=n, masked_max_m=(-(-n // 32) * 32 if cfg.layout == "masked" else cfg.masked_max_m))
    t0 = time.perf_counter()
    oracle.forward(c, sub, nthreads=threads)
    return time.perf_counter() - t0


def cpu_baseline(cfg: MoeConfig, inp, target_s: float = 12.0):
    """The oracle, as it stands, on a bounded sample of the workload's tokens."""
    import oracle
    threads = oracle.default_threads()
    view = _oracle_view(inp)
    n = 2
    dt = _oracle_step(cfg, view, n, threads)
    n = int(max(1, min(cfg.T, math.floor(n * target_s / max(dt, 1e-3)))))
    dt = _oracle_step(cfg, view, n, threads)
    return {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n} tokens of the {cfg.name} workload as one batch (routing, permutation, "
                      f"expert math in fp64 split over {threads} threads, combine), {dt:.1f} s"}


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = CONFIGS[args.config]
    if args.experts:
        cfg = cfg.replace(E=args.experts)
    if args.tokens:
        cfg = cfg.replace(T=args.tokens, masked_max_m=(-(-args.tokens // 32) * 32 if cfg.layout == "masked"
                                                       else cfg.masked_max_m))
    from fp8_grouped_gemm_fp32_b200 import api
    api.lib()                                      # fails loudly if the native library is missing
    api.moe_set_contig_kernel({"auto": api.CONTIG_AUTO, "single": api.CONTIG_SINGLE,
                               "pair": api.CONTIG_PAIR}[args.contig])
    layer = Layer(cfg, dev, seed_offset=rank)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        layer.forward()
    torch.cuda.synchronize()
    assert api.moe_get_device_status() == api.MOE_OK

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        start.record()
        for _ in range(args.steps):
            layer.forward()
        end.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = start.elapsed_time(end) / args.steps
    ms_max = max_over_ranks(ms, world)
    st = api.moe_get_device_status()
    assert st == api.MOE_OK, api.STATUS_NAMES.get(st)
    value = job_tokens_per_s(cfg.T, world, ms_max)

    # End to end through the public call with host buffers: every step copies its tokens (x, and the
    # token ids for hash routing) from pinned host memory to the device, runs moe_forward and copies y
    # back to pinned host memory. Two buffer sets and three streams let step i+1's upload and step
    # i-1's download overlap step i's kernels; the timed region covers all K steps' copies and kernels.
    e2e_ms, h2d, d2h = run_e2e(layer, cfg, args.steps, world)

    # per-kernel breakdown through the step-wise calls (same kernels, one event between each)
    names = ["router", "permute", "gemm_up", "gemm_down", "combine"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for _ in range(2):
        layer.steps([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    torch.cuda.synchronize()
    for i in range(args.steps):
        layer.steps(evs[i])
    torch.cuda.synchronize()
    per = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
           for j, n in enumerate(names)}
    kept = layer.kept.cpu().numpy()
    work, Rk, touched = algorithmic_work(cfg, kept)

    # training side, outside the forward step: the auxiliary-loss-free bias update fed by this step's
    # counts, one launch per training step with an update every 100th (the page's interval). The 100
    # launches are replayed from a CUDA graph so that the device time, not the host's per-call cost, is
    # measured.
    bal_load = torch.zeros(cfg.E, dtype=torch.int64, device=layer.counts.device)
    bal_bias = layer.inp.bias.clone()
    side = torch.cuda.Stream(layer.counts.device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            api.moe_balance_bias(cfg.E, layer.counts, bal_load, bal_bias, 1e-3, False, side)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gs = torch.cuda.current_stream()
        for i in range(100):
            api.moe_balance_bias(cfg.E, layer.counts, bal_load, bal_bias, 1e-3, i == 99, gs)
    graph.replay()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record()
    for _ in range(2):
        graph.replay()
    b1.record()
    torch.cuda.synchronize()
    del graph
    balance = {"us_per_call": 1e3 * b0.elapsed_time(b1) / 200, "calls": 200, "timing": "CUDA graph replay",
               "bytes_per_call": 28 * cfg.E, "bound": "launch latency (one block, 28 B per expert)"}

    backward = None
    if args.backward:
        try:
            backward = time_backward(layer, cfg, max(3, min(args.steps, 20)))
        except Exception as exc:     # the forward line stands on its own; report the failure in its key
            backward = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    # The per-kernel events time each GEMM as a burst of a few milliseconds, so the tensor roofline takes
    # the burst figure: FP8 = 2 x the measured bf16 cuBLAS burst rate (the nominal B200 FP8:BF16 ratio).
    fp8_burst = FP8_PER_BF16 * float(peaks["bf16_tflops"])
    fp8_sus = FP8_PER_BF16 * float(peaks["bf16_tflops_sustained"])
    if backward and "gemm_tflops_lower_bound" in backward:
        # the backward's FP8 GEMM work against the burst FP8 rate (its elementwise steps count as time only)
        backward["frac_fp8_burst_lower_bound"] = backward["gemm_tflops_lower_bound"] / fp8_burst
    fp8_lib = measure_fp8_peak(dev)
    dom = max(per, key=per.get)
    w = work[dom]
    t_s = per[dom] / 1e3
    t_tensor = w["flops"] / (fp8_burst * 1e12) if dom.startswith("gemm") else 0.0
    t_alu = w["flops"] / (FP32_FMA_TFLOPS * 1e12) if dom == "router" else 0.0
    t_hbm = w["bytes"] / (hbm * 1e9)
    if dom.startswith("gemm") and t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": w["flops"] / t_s / 1e12, "peak": fp8_burst, "unit": "TFLOP/s"}
        src = f"{peak_src}: FP8 = 2 x burst bf16 cuBLAS (nominal FP8:BF16 ratio)"
        roof["frac_nominal_4500"] = roof["achieved"] / 4500.0
        if fp8_lib.get("tflops"):
            roof["frac_fp8_scaled_mm"] = roof["achieved"] / fp8_lib["tflops"]
    elif dom == "router" and t_alu >= t_hbm:
        # the router's fp32 multiply-adds run on the CUDA cores in a fixed order, not on the tensor cores
        roof = {"bound": "alu", "achieved": w["flops"] / t_s / 1e12, "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s"}
        src = "derived: 148 SMs x 128 fp32 lanes x 2 FLOP per FMA x 1965 MHz (max SM clock)"
    else:
        roof = {"bound": "hbm", "achieved": w["bytes"] / t_s / 1e9, "peak": hbm, "unit": "GB/s"}
        src = f"{peak_src}: HBM copy"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["kernel_ms"] = per[dom]
    roof["algorithmic_flops"] = w["flops"]
    # the captures cover the named workloads at their own sizes; a reduced case (--experts, --tokens) has none
    roof["traffic"] = None if (args.experts or args.tokens) else measured_traffic(dom, cfg.name)
    roof["algorithmic_bytes"] = w["bytes"]
    roof["peak_source"] = src
    gemm_ms = per["gemm_up"] + per["gemm_down"]
    gemm_flops = work["gemm_up"]["flops"] + work["gemm_down"]["flops"]
    gemm_tflops = gemm_flops / (gemm_ms / 1e3) / 1e12

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "data": "synthetic",
        "dtype": ("4-bit weight levels (as e4m3) x fp8e4m3 activations, fp32 accumulate" if cfg.weights == "w4"
                  else "fp8e4m3 (fp32 accumulate)"),
        "config": {"workload": describe(cfg), "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "contig_gemm": args.contig,
                   "l2": "no flush: the FP8 weights streamed every step (%.2f GB) exceed the 126 MB L2"
                         % ((work["gemm_up"]["bytes"] + work["gemm_down"]["bytes"]) / 1e9)},
        "roofline": roof,
        "gemm": {"tflops": gemm_tflops, "frac_fp8_burst": gemm_tflops / fp8_burst,
                 "frac_fp8_sustained": gemm_tflops / fp8_sus, "frac_fp8_nominal_4500": gemm_tflops / 4500.0,
                 "frac_fp8_scaled_mm": (gemm_tflops / fp8_lib["tflops"]) if fp8_lib.get("tflops") else None,
                 "ms": gemm_ms, "rows_kept": Rk, "experts_touched": touched,
                 "up_tflops": work["gemm_up"]["flops"] / (per["gemm_up"] / 1e3) / 1e12,
                 "down_tflops": work["gemm_down"]["flops"] / (per["gemm_down"] / 1e3) / 1e12},
        "fp8_peak_library": fp8_lib,
        "kernels_ms": per,
        "routing": routing_stats(layer.counts.cpu().numpy(), kept),
        "balance_bias": balance,
        "backward": backward,
        "e2e": {"value": job_tokens_per_s(cfg.T, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": layer.launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, layer.inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    cfg = CONFIGS[args.config]
    threads = oracle.default_threads()
    # The seeded workload is drawn exactly as the GPU arm draws it (same device generator, full T), so
    # both arms see the same tokens and weights; each step takes the first n tokens. Without a GPU the
    # draw is made on the host at a reduced T (its weights then differ from the GPU arm's).
    if torch.cuda.is_available():
        view = _oracle_view(make_inputs(cfg, device="cuda"))
    else:
        view = _oracle_view(make_inputs(cfg, device="cpu", T=min(cfg.T, 512)))
    budget = 150.0 / max(1, args.steps + args.warmup)        # whole run within a few minutes
    dt = _oracle_step(cfg, view, 2, threads)
    t_avail = view["x"].shape[0]
    n = int(max(1, min(512, t_avail, math.floor(2 * min(budget, 10.0) / max(dt, 1e-3)))))
    for _ in range(args.warmup):
        _oracle_step(cfg, view, n, threads)
    times = [_oracle_step(cfg, view, n, threads) for _ in range(args.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = n / (ms / 1e3)
    sample = f"first {n} tokens of the {cfg.name} workload per step as one batch, {threads} threads"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp64 (oracle)", "data": "synthetic",
            "config": {"workload": describe(cfg), "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle", "cores": threads,
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="prefill", choices=sorted(CONFIGS),
                    help="workload (default: prefill, the largest that fits one GPU)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the layer's backward pass (contiguous FP8 workloads)")
    ap.add_argument("--contig", default="auto", choices=["auto", "single", "pair"],
                    help="form of the contiguous grouped GEMM (default: chosen by shape)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the workload's expert count (reduced cases for profiling captures)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (reduced cases for profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
