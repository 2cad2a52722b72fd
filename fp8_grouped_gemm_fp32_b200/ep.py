"""Expert-parallel MoE layer across GPUs: one process per GPU, experts split evenly.

Rank r holds experts [r E/G, (r+1) E/G) and routes its own tokens; all-to-all
carries each kept slot's FP8 row (codes and 1x128 scales) to the rank of its
expert and the expert's bf16 output back (TP-MoE page, sections 3.3 and 4.1
step 3; MegaMoE page, 3.4: dispatch and combine; TP-MoE page, 6.2: an FP8
payload). Every step that touches the data runs in the C library's kernels
(include/moe_fp8.h, "expert parallelism"); this module only sequences them
around the collectives and makes the one host round trip the collectives need
(the row counts each rank sends and receives).

The result on every rank equals one GPU's layer on the ranks' batches
concatenated in rank order, bit for bit in routing, capacity drop and row
placement (the plan ranks slots in that global token order).

With a plan of C chunks the local experts of every rank fall into C
consecutive groups and each buffer is ordered chunk first, so a chunk's rows
travel in an all-to-all of their own while an earlier chunk's experts run
(MegaMoE page, 2.3: the chunked overlap of exchange and compute); the result is
the same bit for bit.

Two transports carry the collectives:
  DistTransport   torch.distributed (NCCL between GPUs; gloo works for the
                  host-side exchange);
  LocalTransport  the G ranks of one process on one device, for tests: each
                  collective is a plain concatenation and split of the ranks'
                  buffers, done between the ranks' kernels (no kernel of one
                  rank waits on another's).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import api

MAX_RANKS = 64
MAX_E = 512
MAX_CHUNKS = 8


class EpPlan(ctypes.Structure):
    """moe_ep_plan_t (include/moe_fp8.h)."""
    _fields_ = [("G", ctypes.c_int32), ("rank", ctypes.c_int32), ("E", ctypes.c_int32), ("E_local", ctypes.c_int32),
                ("cap", ctypes.c_int32), ("rows_send", ctypes.c_int32), ("rows_recv", ctypes.c_int32),
                ("rows_group", ctypes.c_int32),
                ("kept_mine", ctypes.c_int32 * MAX_E), ("send_rows", ctypes.c_int32 * MAX_RANKS),
                ("recv_rows", ctypes.c_int32 * MAX_RANKS), ("recv_start", ctypes.c_int32 * (MAX_E + 1)),
                ("group_start", ctypes.c_int32 * MAX_E), ("offsets", ctypes.c_int32 * (MAX_E + 1)),
                ("kept", ctypes.c_int32 * MAX_E), ("chunks", ctypes.c_int32),
                ("chunk_first", ctypes.c_int32 * (MAX_CHUNKS + 1)), ("send_off", ctypes.c_int32 * MAX_E),
                ("send_chunk", ctypes.c_int32 * (MAX_CHUNKS + 1)), ("recv_chunk", ctypes.c_int32 * (MAX_CHUNKS + 1)),
                ("send_rows_c", (ctypes.c_int32 * MAX_RANKS) * MAX_CHUNKS),
                ("recv_rows_c", (ctypes.c_int32 * MAX_RANKS) * MAX_CHUNKS)]

    def chunk_send(self, c: int) -> List[int]:
        return list(self.send_rows_c[c][:self.G])

    def chunk_recv(self, c: int) -> List[int]:
        return list(self.recv_rows_c[c][:self.G])


def row_bytes(H: int) -> int:
    """MOE_EP_ROW_BYTES(H): codes, scales, padded to 16 bytes."""
    return (H + 4 * (H // 128) + 15) // 16 * 16


def plan(G: int, rank: int, E: int, T_total: int, k: int, cap_num: int, cap_den: int,
         counts_all: np.ndarray, chunks: int = 1) -> EpPlan:
    """The host planner of the library (moe_ep_plan_chunked) on every rank's counts [G, E]."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    assert c.shape == (G, E)
    p = EpPlan()
    api._check(api.lib().moe_ep_plan_chunked(G, rank, E, ctypes.c_int64(T_total), k, cap_num, cap_den,
                                             c.ctypes.data_as(ctypes.c_void_p), chunks, ctypes.byref(p)),
               "moe_ep_plan_chunked")
    return p


def plan_to_device(p: EpPlan, device) -> torch.Tensor:
    """One copy of the plan's bytes to the device (the kernels read it there)."""
    host = torch.frombuffer(bytearray(bytes(p)), dtype=torch.uint8)
    return host.to(device)


# ---------------------------------------------------------------- transports
class DistTransport:
    """Collectives of torch.distributed on the default (or given) process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather_counts(self, counts: torch.Tensor) -> np.ndarray:
        """[E] int32 per rank -> [G, E] on every rank (host copy: the one round trip of a step)."""
        parts = [torch.empty_like(counts) for _ in range(self.G)]
        self.dist.all_gather(parts, counts, group=self.group)
        return torch.stack(parts).cpu().numpy()

    def exchange(self, send: torch.Tensor, send_rows: List[int], recv_rows: List[int]) -> torch.Tensor:
        """All-to-all of rows: send_rows[d] rows of `send` to rank d, recv_rows[s] rows from rank s, in
        rank order. Rows travel as bytes."""
        width = send.shape[1] * send.element_size() if send.dim() == 2 else 0
        out = torch.empty(sum(recv_rows), width, dtype=torch.uint8, device=send.device)
        self.exchange_into(out, send, send_rows, recv_rows)
        return out.view(send.dtype).reshape(sum(recv_rows), send.shape[1])

    def exchange_into(self, out: torch.Tensor, send: torch.Tensor, send_rows: List[int], recv_rows: List[int],
                      async_op: bool = False):
        """The same into rows of `out` (same row width as `send`); returns the collective's work when
        async_op."""
        width = send.shape[1] * send.element_size()
        return self.dist.all_to_all_single(out.view(torch.uint8).reshape(-1, width),
                                           send.contiguous().view(torch.uint8).reshape(-1, width), list(recv_rows),
                                           list(send_rows), group=self.group, async_op=async_op)

    def run_chunks(self, rs: "EpRank", recv: torch.Tensor, back: torch.Tensor):
        """The chunks of one step: each chunk's rows go out, its experts run, their outputs come back. On
        CUDA the collectives run on a stream of their own: every chunk's dispatch is queued at once, and
        each chunk's experts start as soon as its rows have arrived, while later chunks travel."""
        p = rs.plan
        C = p.chunks
        sl = lambda t, a, c: t[a[c]:a[c + 1]]
        if not recv.is_cuda:
            for c in range(C):
                self.exchange_into(sl(recv, p.recv_chunk, c), sl(rs.send, p.send_chunk, c), p.chunk_send(c),
                                   p.chunk_recv(c))
                rs.experts_chunk(recv, c)
                self.exchange_into(sl(back, p.send_chunk, c), sl(rs.ret, p.recv_chunk, c), p.chunk_recv(c),
                                   p.chunk_send(c))
            return
        comp = torch.cuda.current_stream()
        if getattr(self, "comm", None) is None:
            self.comm = torch.cuda.Stream(device=recv.device)
        ready = torch.cuda.Event()
        ready.record(comp)
        arrived = []
        with torch.cuda.stream(self.comm):
            self.comm.wait_event(ready)
            for c in range(C):
                arrived.append(self.exchange_into(sl(recv, p.recv_chunk, c), sl(rs.send, p.send_chunk, c),
                                                  p.chunk_send(c), p.chunk_recv(c), async_op=True))
        returned = []
        for c in range(C):
            arrived[c].wait()                 # the compute stream waits for this chunk's rows
            rs.experts_chunk(recv, c)
            done = torch.cuda.Event()
            done.record(comp)
            with torch.cuda.stream(self.comm):
                self.comm.wait_event(done)
                returned.append(self.exchange_into(sl(back, p.send_chunk, c), sl(rs.ret, p.recv_chunk, c),
                                                   p.chunk_recv(c), p.chunk_send(c), async_op=True))
        for w in returned:
            w.wait()


# ---------------------------------------------------------------- one rank's steps
@dataclass
class RankWeights:
    """The experts one rank holds (local index l = global expert r*E/G + l)."""
    W13: torch.Tensor      # [E_local, 2I, H] u8, W1/W3 128-row blocks interleaved
    S13: torch.Tensor      # [E_local, 2I/128, H/128] fp32
    W2: torch.Tensor       # [E_local, H, I] u8
    S2: torch.Tensor       # [E_local, H/128, I/128] fp32


class EpRank:
    """One rank of the expert-parallel layer. `cfg` is the layer's configuration with T = this rank's
    tokens and E = all experts; capacity (cap_num/cap_den) applies to the global T."""

    def __init__(self, cfg: api.Config, G: int, rank: int, Wg: torch.Tensor, bias: Optional[torch.Tensor],
                 weights: RankWeights):
        assert cfg.E % G == 0
        self.cfg, self.G, self.rank = cfg, G, rank
        self.Wg, self.bias, self.w = Wg, bias, weights
        self.El = cfg.E // G
        self.dev = Wg.device

    # -- before the count exchange
    def route_and_count(self, x: torch.Tensor, token_ids: Optional[torch.Tensor] = None, stream=None):
        c, dev = self.cfg, self.dev
        self.x, self.T = x, c.T
        self.topk_idx = torch.empty(c.T, c.k, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(c.T, c.k, dtype=torch.float32, device=dev)
        ws = torch.empty(max(api.moe_workspace_size(c), 16), dtype=torch.uint8, device=dev)
        api.moe_route(c, x, self.Wg, self.bias, token_ids, self.topk_idx, self.topk_w, ws, stream)
        self.counts = torch.empty(c.E, dtype=torch.int32, device=dev)
        self.ep_ws = torch.empty(max(api.moe_ep_workspace_size(c), 16), dtype=torch.uint8, device=dev)
        api.moe_ep_count(c, self.topk_idx, self.counts, self.ep_ws, stream)
        return self.counts

    # -- after it
    def dispatch(self, counts_all: np.ndarray, T_total: int, stream=None, chunks: int = 1):
        c = self.cfg
        self.plan = plan(self.G, self.rank, c.E, T_total, c.k, c.cap_num, c.cap_den, counts_all, chunks)
        self.plan_dev = plan_to_device(self.plan, self.dev)
        self.send = torch.empty(max(self.plan.rows_send, 1), row_bytes(c.H), dtype=torch.uint8, device=self.dev)
        self.slot_row = torch.empty(c.T * c.k, dtype=torch.int32, device=self.dev)
        api.moe_ep_dispatch(c, self.x, self.topk_idx, self.plan_dev, self.send, self.slot_row, self.ep_ws, stream)
        return self.send[:self.plan.rows_send], list(self.plan.send_rows[:self.G]), list(self.plan.recv_rows[:self.G])

    def alloc_experts(self):
        """The grouped layout and output buffers of this step's plan."""
        c, p, dev = self.cfg, self.plan, self.dev
        self.M = M = max(p.rows_group, 128)
        self.Aq = torch.empty(M, c.H, dtype=torch.uint8, device=dev)
        self.As = torch.empty(c.H // 128, M, dtype=torch.float32, device=dev)
        self.Hq = torch.empty(M, c.I, dtype=torch.uint8, device=dev)
        self.Hs = torch.empty(c.I // 128, M, dtype=torch.float32, device=dev)
        self.O = torch.empty(M, c.H, dtype=torch.bfloat16, device=dev)
        self.group_row = torch.empty(max(p.rows_recv, 1), dtype=torch.int32, device=dev)
        self.ret = torch.empty(max(p.rows_recv, 1), c.H, dtype=torch.bfloat16, device=dev)
        # offsets of each chunk's experts, 16-byte aligned rows
        self.offsets_c = torch.empty(p.chunks, (self.El + 1 + 3) // 4 * 4, dtype=torch.int32, device=dev)

    def experts_chunk(self, recv: torch.Tensor, ch: int, stream=None):
        """Chunk ch of the received rows (recv: the whole receive buffer) -> grouped layout -> the chunk's
        experts (two grouped GEMMs on its rows) -> their output rows, in receive order, into self.ret."""
        c, p = self.cfg, self.plan
        e0, e1 = p.chunk_first[ch], p.chunk_first[ch + 1]
        r0, r1 = p.recv_chunk[ch], p.recv_chunk[ch + 1]
        off = self.offsets_c[ch]
        api.moe_ep_receive_chunk(c.H, self.plan_dev, ch, recv, self.Aq, self.As, self.M, off, self.group_row, stream)
        g0, g1 = p.offsets[e0], p.offsets[e1]
        if g1 > g0:
            # the chunk's rows of the grouped layout: row offsets into each buffer, the scales' row stride M
            A, As = self.Aq.data_ptr() + g0 * c.H, self.As.data_ptr() + 4 * g0
            Hq, Hs = self.Hq.data_ptr() + g0 * c.I, self.Hs.data_ptr() + 4 * g0
            O = self.O.data_ptr() + 2 * g0 * c.H
            api.moe_grouped_gemm_fp8(api.LAYOUT_CONTIGUOUS, e1 - e0, 2 * c.I, c.H, A, As, off, self.M,
                                     self.w.W13[e0:e1], self.w.S13[e0:e1], api.EPI_SWIGLU_FP8, Hq, Hs, stream)
            api.moe_grouped_gemm_fp8(api.LAYOUT_CONTIGUOUS, e1 - e0, c.H, c.I, Hq, Hs, off, self.M, self.w.W2[e0:e1],
                                     self.w.S2[e0:e1], api.EPI_BF16, O, None, stream)
        if r1 > r0:
            api.moe_ep_return(c.H, r1 - r0, self.O, self.group_row[r0:], self.ret[r0:], stream)

    def experts(self, recv: torch.Tensor, stream=None) -> torch.Tensor:
        """Received rows -> grouped layout -> the local experts (two grouped GEMMs) -> rows to return, every
        chunk of the plan in turn."""
        self.alloc_experts()
        recv = recv if recv.shape[0] > 0 else torch.zeros(1, row_bytes(self.cfg.H), dtype=torch.uint8,
                                                           device=self.dev)
        for ch in range(self.plan.chunks):
            self.experts_chunk(recv, ch, stream)
        return self.ret[:self.plan.rows_recv]

    def combine(self, back: torch.Tensor, stream=None) -> torch.Tensor:
        """y of this rank's tokens from the returned rows (the send order: slot_row indexes them)."""
        c = self.cfg
        y = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=self.dev)
        O = back if back.shape[0] > 0 else torch.zeros(1, c.H, dtype=torch.bfloat16, device=self.dev)
        api.moe_combine(c, O, self.slot_row, self.topk_w, y, stream)
        return y


def forward_dist(rank_state: EpRank, x: torch.Tensor, transport: DistTransport, T_total: int,
                 token_ids: Optional[torch.Tensor] = None, chunks: int = 1) -> torch.Tensor:
    """One step of the layer on this rank, collectives through torch.distributed; with chunks > 1 the
    exchange of each chunk overlaps the experts of the chunks before it."""
    counts = rank_state.route_and_count(x, token_ids)
    counts_all = transport.all_gather_counts(counts)
    send, send_rows, recv_rows = rank_state.dispatch(counts_all, T_total, chunks=chunks)
    if chunks == 1:
        recv = transport.exchange(send, send_rows, recv_rows)
        ret = rank_state.experts(recv)
        back = transport.exchange(ret, recv_rows, send_rows)
        return rank_state.combine(back)
    p, c = rank_state.plan, rank_state.cfg
    rank_state.alloc_experts()
    recv = torch.empty(max(p.rows_recv, 1), row_bytes(c.H), dtype=torch.uint8, device=rank_state.dev)
    back = torch.empty(max(p.rows_send, 1), c.H, dtype=torch.bfloat16, device=rank_state.dev)
    transport.run_chunks(rank_state, recv, back)
    return rank_state.combine(back[:p.rows_send])


class LocalTransport:
    """All G ranks in this process: collectives as concatenation and split of the ranks' buffers."""

    def __init__(self, G: int):
        self.G = G

    def all_gather_counts(self, counts: List[torch.Tensor]) -> np.ndarray:
        return torch.stack(counts).cpu().numpy()

    def exchange(self, sends: List[torch.Tensor], send_rows: List[List[int]]) -> List[torch.Tensor]:
        """sends[s] holds send_rows[s][d] rows for each d in order; rank d receives from s = 0..G-1."""
        pieces = [list(torch.split(sends[s], send_rows[s])) for s in range(self.G)]
        return [torch.cat([pieces[s][d] for s in range(self.G)]) for d in range(self.G)]


def forward_local(ranks: List[EpRank], xs: List[torch.Tensor],
                  token_ids: Optional[List[torch.Tensor]] = None, chunks: int = 1) -> List[torch.Tensor]:
    """One step of the layer for G ranks held by one process (tests on one GPU): chunk by chunk, the
    chunk's rows are exchanged, every rank runs the chunk's experts, and their outputs are exchanged back."""
    G = len(ranks)
    tr = LocalTransport(G)
    T_total = sum(int(x.shape[0]) for x in xs)
    counts = [r.route_and_count(x, None if token_ids is None else token_ids[i]) for i, (r, x) in
              enumerate(zip(ranks, xs))]
    counts_all = tr.all_gather_counts(counts)
    for r in ranks:
        r.dispatch(counts_all, T_total, chunks=chunks)
        r.alloc_experts()
    H, dev = ranks[0].cfg.H, ranks[0].dev
    recvs = [torch.empty(max(r.plan.rows_recv, 1), row_bytes(H), dtype=torch.uint8, device=dev) for r in ranks]
    backs = [torch.empty(max(r.plan.rows_send, 1), H, dtype=torch.bfloat16, device=dev) for r in ranks]
    for ch in range(chunks):
        sends = [r.send[r.plan.send_chunk[ch]:r.plan.send_chunk[ch + 1]] for r in ranks]
        got = tr.exchange(sends, [r.plan.chunk_send(ch) for r in ranks])
        for d, r in enumerate(ranks):
            recvs[d][r.plan.recv_chunk[ch]:r.plan.recv_chunk[ch + 1]] = got[d]
            r.experts_chunk(recvs[d], ch)
        rets = [r.ret[r.plan.recv_chunk[ch]:r.plan.recv_chunk[ch + 1]] for r in ranks]
        back = tr.exchange(rets, [r.plan.chunk_recv(ch) for r in ranks])
        for s_, r in enumerate(ranks):
            backs[s_][r.plan.send_chunk[ch]:r.plan.send_chunk[ch + 1]] = back[s_]
    return [r.combine(b[:r.plan.rows_send]) for r, b in zip(ranks, backs)]
