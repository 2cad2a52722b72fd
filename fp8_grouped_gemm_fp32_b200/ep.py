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


class EpPlan(ctypes.Structure):
    """moe_ep_plan_t (include/moe_fp8.h)."""
    _fields_ = [("G", ctypes.c_int32), ("rank", ctypes.c_int32), ("E", ctypes.c_int32), ("E_local", ctypes.c_int32),
                ("cap", ctypes.c_int32), ("rows_send", ctypes.c_int32), ("rows_recv", ctypes.c_int32),
                ("rows_group", ctypes.c_int32),
                ("kept_mine", ctypes.c_int32 * MAX_E), ("send_rows", ctypes.c_int32 * MAX_RANKS),
                ("recv_rows", ctypes.c_int32 * MAX_RANKS), ("recv_start", ctypes.c_int32 * (MAX_E + 1)),
                ("group_start", ctypes.c_int32 * MAX_E), ("offsets", ctypes.c_int32 * (MAX_E + 1)),
                ("kept", ctypes.c_int32 * MAX_E)]


def row_bytes(H: int) -> int:
    """MOE_EP_ROW_BYTES(H): codes, scales, padded to 16 bytes."""
    return (H + 4 * (H // 128) + 15) // 16 * 16


def plan(G: int, rank: int, E: int, T_total: int, k: int, cap_num: int, cap_den: int,
         counts_all: np.ndarray) -> EpPlan:
    """The host planner of the library (moe_ep_plan) on every rank's counts [G, E]."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    assert c.shape == (G, E)
    p = EpPlan()
    api._check(api.lib().moe_ep_plan(G, rank, E, ctypes.c_int64(T_total), k, cap_num, cap_den,
                                     c.ctypes.data_as(ctypes.c_void_p), ctypes.byref(p)), "moe_ep_plan")
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
        self.dist.all_to_all_single(out, send.contiguous().view(torch.uint8).reshape(-1, width), list(recv_rows),
                                    list(send_rows), group=self.group)
        return out.view(send.dtype).reshape(sum(recv_rows), -1)


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
    def dispatch(self, counts_all: np.ndarray, T_total: int, stream=None):
        c = self.cfg
        self.plan = plan(self.G, self.rank, c.E, T_total, c.k, c.cap_num, c.cap_den, counts_all)
        self.plan_dev = plan_to_device(self.plan, self.dev)
        self.send = torch.empty(max(self.plan.rows_send, 1), row_bytes(c.H), dtype=torch.uint8, device=self.dev)
        self.slot_row = torch.empty(c.T * c.k, dtype=torch.int32, device=self.dev)
        api.moe_ep_dispatch(c, self.x, self.topk_idx, self.plan_dev, self.send, self.slot_row, self.ep_ws, stream)
        return self.send[:self.plan.rows_send], list(self.plan.send_rows[:self.G]), list(self.plan.recv_rows[:self.G])

    def experts(self, recv: torch.Tensor, stream=None) -> torch.Tensor:
        """Received rows -> grouped layout -> the local experts (two grouped GEMMs) -> rows to return."""
        c, p, dev = self.cfg, self.plan, self.dev
        M = max(p.rows_group, 128)
        Aq = torch.empty(M, c.H, dtype=torch.uint8, device=dev)
        As = torch.empty(c.H // 128, M, dtype=torch.float32, device=dev)
        offsets = torch.empty(self.El + 1, dtype=torch.int32, device=dev)
        group_row = torch.empty(max(p.rows_recv, 1), dtype=torch.int32, device=dev)
        api.moe_ep_receive(c.H, self.plan_dev, p.rows_recv, recv, Aq, As, M, offsets, group_row, stream)
        Hq = torch.empty(M, c.I, dtype=torch.uint8, device=dev)
        Hs = torch.empty(c.I // 128, M, dtype=torch.float32, device=dev)
        O = torch.empty(M, c.H, dtype=torch.bfloat16, device=dev)
        if p.rows_group > 0:
            api.moe_grouped_gemm_fp8(api.LAYOUT_CONTIGUOUS, self.El, 2 * c.I, c.H, Aq, As, offsets, M, self.w.W13,
                                     self.w.S13, api.EPI_SWIGLU_FP8, Hq, Hs, stream)
            api.moe_grouped_gemm_fp8(api.LAYOUT_CONTIGUOUS, self.El, c.H, c.I, Hq, Hs, offsets, M, self.w.W2,
                                     self.w.S2, api.EPI_BF16, O, None, stream)
        ret = torch.empty(max(p.rows_recv, 1), c.H, dtype=torch.bfloat16, device=dev)
        api.moe_ep_return(c.H, p.rows_recv, O, group_row, ret, stream)
        return ret[:p.rows_recv]

    def combine(self, back: torch.Tensor, stream=None) -> torch.Tensor:
        """y of this rank's tokens from the returned rows (the send order: slot_row indexes them)."""
        c = self.cfg
        y = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=self.dev)
        O = back if back.shape[0] > 0 else torch.zeros(1, c.H, dtype=torch.bfloat16, device=self.dev)
        api.moe_combine(c, O, self.slot_row, self.topk_w, y, stream)
        return y


def forward_dist(rank_state: EpRank, x: torch.Tensor, transport: DistTransport, T_total: int,
                 token_ids: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One step of the layer on this rank, collectives through torch.distributed."""
    counts = rank_state.route_and_count(x, token_ids)
    counts_all = transport.all_gather_counts(counts)
    send, send_rows, recv_rows = rank_state.dispatch(counts_all, T_total)
    recv = transport.exchange(send, send_rows, recv_rows)
    ret = rank_state.experts(recv)
    back = transport.exchange(ret, recv_rows, send_rows)
    return rank_state.combine(back)


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
                  token_ids: Optional[List[torch.Tensor]] = None) -> List[torch.Tensor]:
    """One step of the layer for G ranks held by one process (tests on one GPU)."""
    G = len(ranks)
    tr = LocalTransport(G)
    T_total = sum(int(x.shape[0]) for x in xs)
    counts = [r.route_and_count(x, None if token_ids is None else token_ids[i]) for i, (r, x) in
              enumerate(zip(ranks, xs))]
    counts_all = tr.all_gather_counts(counts)
    disp = [r.dispatch(counts_all, T_total) for r in ranks]
    recvs = tr.exchange([d[0] for d in disp], [d[1] for d in disp])
    rets = [r.experts(recv) for r, recv in zip(ranks, recvs)]
    backs = tr.exchange(rets, [d[2] for d in disp])
    return [r.combine(b) for r, b in zip(ranks, backs)]
