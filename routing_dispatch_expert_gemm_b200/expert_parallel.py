"""Expert parallelism: experts sharded over ranks, token rows exchanged by two all-to-alls
around each rank's local grouped GEMMs.

Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 3, When the
experts live on different GPUs (each GPU holds a subset of the experts; a token's rows go
to the GPU that owns its expert and the results come back, an all-to-all each way);
"Mixture-of-Experts: routing and capacity", Communication (the dispatch and combine
all-to-alls are the communication cost of expert parallelism).

Layout.  With W ranks and E experts (E divisible by W), rank r owns experts
[r E/W, (r+1) E/W).  Every rank routes and packs its own tokens for all E experts
(``moe_route``, ``moe_dispatch``): the packed rows are expert-major, so the rows bound for
rank q's experts are one contiguous range of the sender's packed buffer.

Exchange.  ``plan_exchange`` sends, in one all-to-all of E integers per rank, how many rows
each sender has for each of the receiver's experts.  ``exchange_rows`` sends the row ranges
in one all-to-all into the receiver's own memory (source-major there) and reorders them
expert-major, so that the local grouped GEMM reads a segment table of E/W experts from local
memory: a remote row crosses the link once, and no tensor-memory-access load, multicast or
library kernel ever reads another GPU's memory.  ``return_rows`` undoes both steps, leaving
each expert output row at its place in the sender's packed order, where the local combine
runs unchanged (slot order, fp32, as on one GPU).

Only ``torch.distributed`` collectives carry the rows, so the same code runs on gloo CPU
ranks and on NCCL GPU ranks; rows travel as raw bytes, whatever their dtype.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class ExchangePlan:
    """Row counts of one rank's side of the exchange.

    send_counts[q, e]  rows this rank sends for rank q's local expert e
    recv_counts[s, e]  rows this rank receives from rank s for its local expert e
    send_rows[q], recv_rows[s]  their sums per peer
    local_offsets[e]   start of local expert e's segment in the expert-major local rows
                       (length E/W + 1)
    perm[j]            index, in the source-major received buffer, of local row j
    """
    world: int
    rank: int
    E: int
    send_counts: torch.Tensor
    recv_counts: torch.Tensor
    send_rows: list
    recv_rows: list
    local_offsets: torch.Tensor
    perm: torch.Tensor

    @property
    def E_local(self) -> int:
        return self.E // self.world

    @property
    def rows_sent(self) -> int:
        return int(sum(self.send_rows))

    @property
    def rows_received(self) -> int:
        return int(sum(self.recv_rows))


def experts_of(rank: int, world: int, E: int) -> range:
    """The experts rank `rank` owns: a contiguous block of E / world."""
    if E % world != 0:
        raise ValueError(f"E={E} experts do not divide over {world} ranks")
    n = E // world
    return range(rank * n, (rank + 1) * n)


def _world_rank(group):
    return dist.get_world_size(group), dist.get_rank(group)


def _comm_device(group, like: torch.Tensor) -> torch.device:
    """NCCL moves device tensors; gloo moves host tensors."""
    return like.device if dist.get_backend(group) == "nccl" else torch.device("cpu")


def plan_exchange(counts: torch.Tensor, group=None) -> ExchangePlan:
    """The exchange plan from this rank's rows per expert (``counts``, length E: the
    segment sizes of its expert-major packed buffer).  One all-to-all of E integers; the
    row sizes are then known on the host of every rank (the rows' all-to-all needs them)."""
    W, r = _world_rank(group)
    E = int(counts.numel())
    El = len(experts_of(r, W, E))
    dev = _comm_device(group, counts)
    send = counts.to(device=dev, dtype=torch.int64).reshape(W, El).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(-1), send.view(-1), group=group)
    send_c, recv_c = send.cpu(), recv.cpu()
    # received buffer: source-major, then expert-major within a source; local rows: expert-
    # major, then source-major within an expert (so rank 0's rows of an expert come first)
    src_start = torch.cumsum(recv_c.reshape(-1), 0) - recv_c.reshape(-1)          # (s, e)
    seg_len = recv_c.t().reshape(-1)                                             # (e, s)
    tgt_start = torch.cumsum(seg_len, 0) - seg_len                               # (e, s)
    src_of_seg = src_start.reshape(W, El).t().reshape(-1)                        # (e, s)
    total = int(seg_len.sum())
    perm = (torch.repeat_interleave(src_of_seg - tgt_start, seg_len) +
            torch.arange(total, dtype=torch.int64))
    per_expert = recv_c.sum(0)
    local_offsets = torch.zeros(El + 1, dtype=torch.int64)
    local_offsets[1:] = torch.cumsum(per_expert, 0)
    return ExchangePlan(W, r, E, send_c, recv_c, send_c.sum(1).tolist(),
                        recv_c.sum(1).tolist(), local_offsets, perm)


def _all_to_all_rows(rows: torch.Tensor, out_rows: int, out_splits, in_splits, group):
    """All-to-all of whole rows as raw bytes (any dtype), on the backend's device."""
    dev = _comm_device(group, rows)
    width = rows.shape[1] * rows.element_size()
    src = rows.contiguous().view(torch.uint8).reshape(rows.shape[0], width).to(dev)
    dst = torch.empty((out_rows, width), dtype=torch.uint8, device=dev)
    dist.all_to_all_single(dst, src, output_split_sizes=list(out_splits),
                           input_split_sizes=list(in_splits), group=group)
    return dst.to(rows.device).view(rows.dtype).reshape(out_rows, rows.shape[1])


def exchange_rows(x_packed: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """Dispatch: the sender's routed rows (the first ``plan.rows_sent`` rows of its expert-
    major packed buffer) to their experts' owners; returns this rank's received rows,
    expert-major over its local experts (segments ``plan.local_offsets``)."""
    recv = _all_to_all_rows(x_packed[:plan.rows_sent], plan.rows_received, plan.recv_rows,
                            plan.send_rows, group)
    return recv.index_select(0, plan.perm.to(recv.device))


def return_rows(y_local: torch.Tensor, plan: ExchangePlan, group=None) -> torch.Tensor:
    """Combine's exchange: the expert outputs of the received rows back to their senders;
    returns this rank's ``plan.rows_sent`` rows in its own packed order."""
    y = y_local[:plan.rows_received]
    back = torch.empty_like(y)
    back.index_copy_(0, plan.perm.to(y.device), y)
    return _all_to_all_rows(back, plan.rows_sent, plan.send_rows, plan.recv_rows, group)


def ep_forward(cfg, x, w_router, logit_bias, w_gate_local, w_up_local, w_down_local,
               group=None):
    """One MoE layer on this rank's tokens with the experts sharded over the group's ranks:
    moe_route and moe_dispatch over all E experts, the exchange, moe_expert_ffn over the
    E/W local experts (w_*_local hold only those, [E/W, ...]), the return exchange, then
    moe_combine.  Ragged layout (drop or dropless), no shared expert.  Returns y [T, d]."""
    from . import native as N
    ragged = cfg.layout == N.LAYOUTS["ragged"] and cfg.overflow == N.OVERFLOWS["drop"]
    if cfg.has_shared or not ragged:
        raise ValueError("ep_forward: ragged layout, drop or dropless, no shared expert")
    W, r = _world_rank(group)
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    El = len(experts_of(r, W, E))
    dev = x.device
    ws = N.workspace(cfg, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    N.moe_route(cfg, x, w_router, logit_bias, ids, gates, ws)
    rmax = N.moe_max_rows(cfg)
    x_packed = torch.empty((rmax, d), dtype=x.dtype, device=dev)
    row_token = torch.empty(rmax, dtype=torch.int32, device=dev)
    route_row = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(N.offsets_len(cfg), dtype=torch.int32, device=dev)
    demand = torch.empty(E, dtype=torch.int32, device=dev)
    N.moe_dispatch(cfg, x, ids, None, x_packed, row_token, route_row, offsets, demand, ws)
    plan = plan_exchange((offsets[1:E + 1] - offsets[:E]).to(torch.int64), group)
    x_local = exchange_rows(x_packed, plan, group)
    # the local experts' grouped GEMMs: one row per received route (k = 1)
    n = max(plan.rows_received, 1)
    lcfg = type(cfg).from_buffer_copy(cfg)
    lcfg.T, lcfg.E, lcfg.k, lcfg.capacity = n, El, 1, -1
    lcfg.add_residual, lcfg.stats, lcfg.fuse = 0, 0, 0
    loff = torch.empty(El + 2, dtype=torch.int32, device=dev)
    loff[:El + 1] = plan.local_offsets.to(dev)
    loff[El + 1] = int(plan.local_offsets[-1])
    xl = torch.zeros((n, d), dtype=x.dtype, device=dev)
    xl[:plan.rows_received] = x_local
    h = torch.empty((n, cfg.d_ff), dtype=x.dtype, device=dev)
    y_local = torch.empty((n, d), dtype=x.dtype, device=dev)
    N.moe_expert_ffn(lcfg, None, xl, loff, w_gate_local, w_up_local, w_down_local, None, None,
                     None, h, y_local, N.workspace(lcfg, device=dev))
    y_packed = torch.empty((rmax, d), dtype=x.dtype, device=dev)
    y_packed[:plan.rows_sent] = return_rows(y_local, plan, group)
    y = torch.empty_like(x)
    N.moe_combine(cfg, y_packed, route_row, gates, offsets, x if cfg.add_residual else None, y)
    return y
