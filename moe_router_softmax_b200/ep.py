"""Expert parallelism across GPUs: one process per GPU, all-to-all exchanges
over a torch.distributed process group (NCCL over NVLink on B200s).

Rank d of N holds the local experts [d*El, (d+1)*El) of a layer (El = E/N).  It
is the multi-GPU form of the pages' remote-expert runtime (Winery-Strata
src/core/remote_experts.cpp: a secondary GPU owns a claimed subset of the
experts; RemoteExperts::begin groups the routes by expert and stages the rows
routed to it, RemoteExperts::finish copies the compact result rows back to
their routes).  One layer call on every rank:

  begin   route the rank's own tokens over all E experts and group the routes
          by expert (moe_route_topk, moe_permute); because experts are owned
          in contiguous blocks, the routes for rank d are one contiguous range
          of the sorted order.  Pack the routed tokens' rows in that order
          (moe_gather_rows).
  plan    exchange the per-expert counts (El per rank pair), read them on the
          host once, and turn them into the row splits (moe_ep_splits).
  ---     all-to-all of the packed bf16 rows to their owners.
  serve   label the received rows with their local expert (moe_ep_recv_ids),
          group them (moe_permute with k = 1), run the grouped FFN on this
          rank's experts, and put the fp32 result rows back in arrival order
          (moe_gather_rows).
  ---     the reverse all-to-all: the rows land in the sender's sorted order,
          exactly where a one-GPU moe_grouped_ffn would have written them.
  finish  weighted combine (moe_combine).

Every step on the data path runs in the library's kernels or in the
collective; this module only sequences them and allocates the buffers.  The
phases are separate methods so that several ranks can also be driven in
lockstep from one process.
"""
from __future__ import annotations

from dataclasses import dataclass
from types import SimpleNamespace

import torch
import torch.distributed as dist

from . import (MoeLayer, moe_combine, moe_ep_recv_ids, moe_ep_splits, moe_gather_rows, moe_grouped_ffn,
               moe_permute, moe_route_topk)

# The calls a layer step makes.  Tests on machines without a GPU pass a
# namespace of host implementations with the same signatures to check the
# exchange logic across processes; the library itself never substitutes them.
KERNELS = SimpleNamespace(moe_route_topk=moe_route_topk, moe_permute=moe_permute, moe_gather_rows=moe_gather_rows,
                          moe_ep_recv_ids=moe_ep_recv_ids, moe_ep_splits=moe_ep_splits,
                          moe_grouped_ffn=moe_grouped_ffn, moe_combine=moe_combine)


class TorchExchange:
    """All-to-all over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits=None, in_splits=None) -> torch.Tensor:
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        return out


@dataclass
class EpStep:
    """The buffers of one layer call on one rank."""
    T: int
    k: int
    ids: torch.Tensor            # int32 [T, k]
    w: torch.Tensor              # fp32 [T, k]
    counts: torch.Tensor         # int32 [E], routes per expert
    offsets: torch.Tensor        # int32 [E + 1]
    sorted_route: torch.Tensor   # int32 [T*k]
    route_pos: torch.Tensor      # int32 [T*k]
    xs: torch.Tensor             # bf16 [T*k, H], packed rows in sorted order
    recv_counts: torch.Tensor | None = None   # int32 [N, El], from every source
    send_rows: list | None = None             # rows to each rank
    recv_rows: list | None = None             # rows from each rank
    xr: torch.Tensor | None = None            # bf16 [n_recv, H], received rows
    rows_out: torch.Tensor | None = None      # fp32 [n_recv, H], results in arrival order
    rows_back: torch.Tensor | None = None     # fp32 [T*k, H], results in sorted order


class ExpertParallelLayer:
    """One MoE layer split by expert over `world` ranks; this object is rank
    `rank` and holds `local_layer`, the blobs of its El = E / world experts
    (local expert e is global expert rank*El + e)."""

    def __init__(self, local_layer: MoeLayer, E: int, rank: int, world: int, exchange=None, ops=None):
        if world < 1 or E % world:
            raise ValueError(f"E={E} must be a multiple of the number of ranks ({world})")
        if not 0 <= rank < world:
            raise ValueError(f"rank {rank} outside [0, {world})")
        self.El = E // world
        if local_layer.E != self.El:
            raise ValueError(f"the local layer holds {local_layer.E} experts, expected E/world = {self.El}")
        self.layer, self.E, self.rank, self.world = local_layer, E, rank, world
        self.H = local_layer.H
        self.exchange = exchange
        self.ops = KERNELS if ops is None else ops

    # -------------------------------------------------------------- phases
    def begin(self, logits: torch.Tensor, x: torch.Tensor, k: int) -> EpStep:
        o = self.ops
        T = x.shape[0]
        ids, w = o.moe_route_topk(logits, k)
        counts, offsets, sorted_route, route_pos = o.moe_permute(ids, self.E)
        xs = o.moe_gather_rows(x, sorted_route, k)
        return EpStep(T, k, ids, w, counts, offsets, sorted_route, route_pos, xs)

    def plan(self, st: EpStep) -> None:
        """Row splits from this rank's counts and st.recv_counts (one device->host read)."""
        host = torch.cat([st.counts.reshape(-1), st.recv_counts.reshape(-1)]).cpu().numpy()
        send, recv = self.ops.moe_ep_splits(host[:self.E], host[self.E:].reshape(self.world, self.El))
        st.send_rows = [int(v) for v in send]
        st.recv_rows = [int(v) for v in recv]

    def serve(self, st: EpStep, hits: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's experts over the received rows st.xr; hits (uint32 [El],
        optional) accumulates the local experts' hit counts."""
        o = self.ops
        n = sum(st.recv_rows)
        if n == 0:
            st.rows_out = torch.empty((0, self.H), dtype=torch.float32, device=st.xs.device)
            return st.rows_out
        eid = o.moe_ep_recv_ids(st.recv_counts, n)
        counts, offsets, sorted_route, route_pos = o.moe_permute(eid.view(n, 1), self.El, hits=hits)
        rows = o.moe_grouped_ffn(self.layer, st.xr, 1, counts, offsets, sorted_route)
        st.rows_out = o.moe_gather_rows(rows, route_pos, 1)
        return st.rows_out

    def finish(self, st: EpStep) -> torch.Tensor:
        return self.ops.moe_combine(st.rows_back, st.route_pos, st.w)

    # ---------------------------------------------------------- one call
    def forward(self, logits: torch.Tensor, x: torch.Tensor, k: int, hits: torch.Tensor | None = None) -> torch.Tensor:
        """y [T, H] bf16 for this rank's tokens; every rank must call it together."""
        if self.exchange is None:
            raise RuntimeError("forward needs an exchange (TorchExchange); drive the phases directly otherwise")
        ex, dev = self.exchange, x.device
        st = self.begin(logits, x, k)
        st.recv_counts = torch.empty((self.world, self.El), dtype=torch.int32, device=dev)
        ex.all_to_all(st.recv_counts.view(-1), st.counts.reshape(-1))
        self.plan(st)
        n_send, n_recv = sum(st.send_rows), sum(st.recv_rows)
        st.xr = torch.empty((n_recv, self.H), dtype=st.xs.dtype, device=dev)
        ex.all_to_all(st.xr, st.xs[:n_send], st.recv_rows, st.send_rows)
        self.serve(st, hits)
        st.rows_back = torch.empty((max(st.T * k, 1), self.H), dtype=st.rows_out.dtype, device=dev)
        ex.all_to_all(st.rows_back[:n_send], st.rows_out, st.send_rows, st.recv_rows)
        return self.finish(st)


def local_layer_of(layer: MoeLayer, rank: int, world: int) -> MoeLayer:
    """The rank's share of a layer whose E blobs are all in `layer.home`: a view of
    its El consecutive blobs (no copy).  A rank that should hold only its own
    experts builds them directly instead: make_layer(fmt, w13[d*El:(d+1)*El],
    w2[d*El:(d+1)*El])."""
    El = layer.E // world
    eb = layer.expert_bytes
    home = layer.home[rank * El * eb:(rank + 1) * El * eb]
    return MoeLayer(layer.fmt, El, layer.H, layer.I, home, expert_bytes=eb)
