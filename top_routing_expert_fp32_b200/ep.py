"""Expert parallelism for the MoE FFN layer: the E experts partitioned over the ranks of a
process group, each kept record's token row sent to the rank that holds its expert and the
expert output sent back (Grok-1 book 5.6, expert parallel vs tensor parallel: every device holds
whole experts and tokens travel by all-to-all; MoE series 4.1: a dispatch and a combine
exchange, 2 * N * k * d_model * s bytes per layer).

Every rank routes and dispatches its own tokens over all E experts with the single-GPU
kernels. Capacity, when set, is per rank: each rank's batch is one group, the reading under
which an expert-parallel layer gives every rank the result of the single-device layer on its
own tokens. Experts are owned in contiguous blocks (expert_ranges), so the expert-contiguous
rows X_perm of a rank are already ordered by destination rank. Then:

  1. the per-expert kept counts are exchanged (all_to_all_single of E_max int32 per peer);
  2. the kept rows go to their experts' ranks (all_to_all_single, rows as 32-bit words);
  3. the receiving rank reorders them expert-major (moe_gather_rows), runs the grouped FFN of
     its own experts, and reorders the outputs back to source-major (moe_gather_rows);
  4. a second all_to_all_single returns the outputs, which land where the source rank's own
     expert GEMMs would have written them, so the combine is the single-GPU combine.

The split sizes of all_to_all_single are host integers: each layer reads the exchanged counts
back once (one device-to-host copy of the count matrix). The compute of steps 1-4 is supplied
by a LocalCompute object: CudaCompute runs this library's kernels; the collectives are
torch.distributed (NCCL between GPUs)."""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist


def expert_ranges(E: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous expert blocks [e0, e1) per rank; the first E % world ranks own one more."""
    if E <= 0 or world <= 0:
        raise ValueError("E and world must be positive")
    base, extra = divmod(E, world)
    starts = [r * base + min(r, extra) for r in range(world + 1)]
    return [(starts[r], starts[r + 1]) for r in range(world)]


@dataclass
class ExchangePlan:
    """Host-side bookkeeping of one layer's exchange, seen from one rank."""
    send_rows: List[int]          # rows sent to each rank (kept records of its experts)
    recv_rows: List[int]          # rows received from each rank
    recv_counts: np.ndarray       # [world, E_local] rows of each local expert from each source
    local_offsets: np.ndarray     # [E_local + 1] expert-major segments of the received rows
    to_expert_major: np.ndarray   # [R_recv] int32: expert-major row j = received row [j]
    to_source_major: np.ndarray   # [R_recv] int32: received row i = expert-major row [i]


def plan_exchange(offsets: np.ndarray, recv_counts: np.ndarray,
                  ranges: List[Tuple[int, int]]) -> ExchangePlan:
    """offsets: this rank's dispatch offsets [E+1]; recv_counts: [world, E_local] counts of
    this rank's experts sent by each source rank. The received buffer is source-major and,
    inside a source's block, expert-major (the source's X_perm order)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    recv_counts = np.asarray(recv_counts, dtype=np.int64)
    world = len(ranges)
    if recv_counts.ndim != 2 or recv_counts.shape[0] != world:
        raise ValueError("recv_counts must be [world, E_local]")
    send_rows = [int(offsets[e1] - offsets[e0]) for (e0, e1) in ranges]
    recv_rows = [int(v) for v in recv_counts.sum(axis=1)]
    el = recv_counts.shape[1]
    src_base = np.concatenate([[0], np.cumsum(recv_rows)])[:-1]
    within = np.concatenate([np.zeros((world, 1), np.int64), np.cumsum(recv_counts, axis=1)],
                            axis=1)[:, :el]
    per_expert = recv_counts.sum(axis=0)
    local_offsets = np.concatenate([[0], np.cumsum(per_expert)]).astype(np.int32)
    pieces = [np.arange(src_base[s] + within[s, e], src_base[s] + within[s, e] + recv_counts[s, e],
                        dtype=np.int64)
              for e in range(el) for s in range(world)]
    total = int(sum(recv_rows))
    to_em = (np.concatenate(pieces) if pieces else np.zeros((0,), np.int64)).astype(np.int32)
    if to_em.shape[0] != total:
        raise ValueError("inconsistent exchange counts")
    to_sm = np.empty_like(to_em)
    to_sm[to_em] = np.arange(total, dtype=np.int32)
    return ExchangePlan(send_rows, recv_rows, recv_counts, local_offsets, to_em, to_sm)


def a2a_bytes(num_tokens: int, model_dim: int, top_k: int, bytes_per_elem: int) -> int:
    """Dispatch plus combine volume of one layer when no record is dropped (MoE series 4.1)."""
    if min(num_tokens, model_dim, top_k, bytes_per_elem) < 0:
        raise ValueError("inputs must be non-negative")
    return 2 * num_tokens * top_k * model_dim * bytes_per_elem


def _words(t: torch.Tensor) -> torch.Tensor:
    """Rows of t as 32-bit words (the exchange moves bytes; gloo has no 16-bit types)."""
    t = t.contiguous()
    if (t.shape[-1] * t.element_size()) % 4 != 0:
        raise ValueError("row size must be a multiple of 4 bytes")
    return t.view(torch.int32)


def _exchange_rows(x: torch.Tensor, send_rows: List[int], recv_rows: List[int],
                   group) -> torch.Tensor:
    out = torch.empty((sum(recv_rows),) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(_words(out), _words(x[: sum(send_rows)]), recv_rows, send_rows,
                           group=group)
    return out


def _exchange_counts(counts: torch.Tensor, ranges, rank: int, group) -> np.ndarray:
    """counts: this rank's kept rows per expert [E] (int32, on the exchange device). Returns
    [world, E_local] counts of this rank's experts from every source (host)."""
    world = len(ranges)
    el_max = max(e1 - e0 for e0, e1 in ranges)
    send = torch.zeros((world, el_max), dtype=torch.int32, device=counts.device)
    for d, (e0, e1) in enumerate(ranges):
        send[d, : e1 - e0] = counts[e0:e1]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(-1), send.view(-1), group=group)
    e0, e1 = ranges[rank]
    return recv.cpu().numpy()[:, : e1 - e0]


class LocalCompute:
    """The per-rank compute of an expert-parallel layer (see CudaCompute)."""

    def route_dispatch(self, X) -> dict:
        """Route X over all E experts and dispatch it: dict with at least "offsets" ([E+1]
        int32 tensor on the exchange device) and "X_perm" (expert-contiguous kept rows)."""
        raise NotImplementedError

    def expert_ffn(self, X_loc: torch.Tensor, local_offsets: np.ndarray,
                   expert_range: Tuple[int, int]) -> torch.Tensor:
        raise NotImplementedError

    def gather_rows(self, src: torch.Tensor, index: np.ndarray) -> torch.Tensor:
        raise NotImplementedError

    def combine(self, Y_perm: torch.Tensor, routed: dict) -> torch.Tensor:
        raise NotImplementedError


def forward(compute: LocalCompute, X, E: int, group=None) -> Tuple[torch.Tensor, dict]:
    """One expert-parallel layer on this rank's tokens X. Returns (out, info) with info =
    dict(plan, sent_bytes, received_bytes) (the rows this rank put into both exchanges, its
    own included)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ranges = expert_ranges(E, world)
    routed = compute.route_dispatch(X)
    offsets = routed["offsets"]
    counts = (offsets[1:] - offsets[:-1]).to(torch.int32)
    recv_counts = _exchange_counts(counts, ranges, rank, group)
    plan = plan_exchange(offsets.cpu().numpy(), recv_counts, ranges)
    X_recv = _exchange_rows(routed["X_perm"], plan.send_rows, plan.recv_rows, group)
    X_loc = compute.gather_rows(X_recv, plan.to_expert_major)
    Y_loc = compute.expert_ffn(X_loc, plan.local_offsets, ranges[rank])
    Y_recv = compute.gather_rows(Y_loc, plan.to_source_major)
    Y_back = _exchange_rows(Y_recv, plan.recv_rows, plan.send_rows, group)
    out = compute.combine(Y_back, routed)
    row_in = X_recv[0].numel() * X_recv.element_size() if X_recv.shape[0] else 0
    row_out = Y_back[0].numel() * Y_back.element_size() if Y_back.shape[0] else 0
    info = dict(plan=plan,
                sent_bytes=sum(plan.send_rows) * row_in + sum(plan.recv_rows) * row_out,
                received_bytes=sum(plan.recv_rows) * row_in + sum(plan.send_rows) * row_out)
    return out, info


class CudaCompute(LocalCompute):
    """LocalCompute on this library's kernels (C ABI): the router and dispatch of the rank's
    tokens over all E experts, the grouped gated FFN of the rank's own experts (weights
    W1, W2 [E_local, D, F], W3 [E_local, F, D] of experts [e0, e1)), the row reorders
    (moe_gather_rows) and the gate-weighted combine."""

    def __init__(self, cfg, W_r, bias, W1_local, W2_local, W3_local, device="cuda"):
        from . import abi
        self.abi = abi
        self.cfg = cfg
        self.W_r, self.bias = W_r, bias
        self.W1, self.W2, self.W3 = W1_local, W2_local, W3_local
        self.device = torch.device(device)
        self.p = abi.problem(cfg)
        self.ws = abi.workspace(self.p, self.device)
        self._rows = 0          # received rows the local-layer buffers below are sized for
        self._ws_loc = None
        self._H = None

    def route_dispatch(self, X) -> dict:
        a, cfg, dev = self.abi, self.cfg, self.device
        N, k, E, D = cfg.N, cfg.k, cfg.E, cfg.D
        r = dict(idx=torch.empty((N, k), dtype=torch.int32, device=dev),
                 gate=torch.empty((N, k), dtype=torch.float32, device=dev),
                 load=torch.empty((E,), dtype=torch.int32, device=dev),
                 offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
                 pos=torch.empty((N, k), dtype=torch.int32, device=dev),
                 dropped=torch.empty((N, k), dtype=torch.uint8, device=dev),
                 row_token=torch.empty((N * k,), dtype=torch.int32, device=dev),
                 X_perm=torch.empty((N * k, D), dtype=X.dtype, device=dev))
        a.route(self.p, X, self.W_r, self.bias, None, r["idx"], r["gate"], None, self.ws)
        a.dispatch(self.p, X, r["idx"], r["load"], r["offsets"], r["pos"], r["dropped"],
                   r["row_token"], r["X_perm"], self.ws)
        return r

    def expert_ffn(self, X_loc, local_offsets, expert_range):
        a = self.abi
        e0, e1 = expert_range
        R = X_loc.shape[0]
        Y = torch.empty((R, self.cfg.D), dtype=X_loc.dtype, device=self.device)
        if R == 0 or e1 == e0:
            return Y
        # The local experts as a layer of their own: R rows, one slot each, E_local experts. Its
        # workspace and H are kept and regrown only when more rows arrive than ever before.
        p = a.problem(self.cfg.with_(N=R, k=1, E=e1 - e0, capacity_factor=0.0, min_capacity=0))
        if R > self._rows:
            self._ws_loc = a.workspace(p, self.device)
            self._H = torch.empty((R, self.cfg.F), dtype=X_loc.dtype, device=self.device)
            self._rows = R
        off = torch.from_numpy(np.ascontiguousarray(local_offsets, dtype=np.int32)).to(self.device)
        a.expert_up(p, X_loc, off, self.W1, self.W2, self._H, self._ws_loc)
        a.expert_down(p, self._H, off, self.W3, Y, self._ws_loc)
        return Y

    def gather_rows(self, src, index):
        dst = torch.empty((index.shape[0],) + tuple(src.shape[1:]), dtype=src.dtype,
                          device=self.device)
        if index.shape[0]:
            idx = torch.from_numpy(np.ascontiguousarray(index, dtype=np.int32)).to(self.device)
            self.abi.gather_rows(src, idx, dst, self.ws)
        return dst

    def combine(self, Y_perm, r):
        cfg = self.cfg
        out = torch.empty((cfg.N, cfg.D), dtype=Y_perm.dtype, device=self.device)
        Y = Y_perm
        if Y.shape[0] == 0:  # every record dropped: the combine reads no row
            Y = torch.zeros((1, cfg.D), dtype=Y_perm.dtype, device=self.device)
        self.abi.combine(self.p, Y, r["idx"], r["gate"], r["offsets"], r["pos"], r["dropped"],
                         out)
        return out

    def device_error(self) -> int:
        """First nonzero device error code of the rank's workspaces (0 if none); clears them."""
        codes = [self.abi.device_error(self.ws)]
        if self._ws_loc is not None:
            codes.append(self.abi.device_error(self._ws_loc))
        return next((c for c in codes if c != 0), 0)
