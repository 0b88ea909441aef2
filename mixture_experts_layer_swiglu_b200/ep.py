"""Expert-parallel MoE layer: the routed experts split over the ranks of a
process group, the rows exchanged with NCCL (or any torch.distributed
backend) send/receive.

Each rank routes, permutes and combines its own tokens with the library's
kernels.  The rows of expert e go to the rank that owns e (contiguous ranges
of expert ids: ``moe_ep_expert_range``), which computes them with the grouped
GEMM over the blocks it received, laid out expert-major with the source rank
inside (``moe_ep_plan``); the results come back block by block to the rows
they came from, so the combine is the single-rank one.  Between two ranks the
blocks are sent and received in increasing expert order, so the transfers
match one to one whatever the backend.

Only the exchange is done here (torch.distributed point-to-point calls);
every step of the layer is a call into libmoe.so.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _abi as abi
from .layer import StageBuffers, out_dtype


@dataclass
class ExchangePlan:
    """Where every block of rows goes, for one rank (host integers)."""
    G: int
    E: int
    rank: int
    lo: int                       # first owned expert
    hi: int                       # one past the last
    counts: torch.Tensor          # [G, E] int32: rows of rank q for expert e
    recv_offsets: torch.Tensor    # [n_own, G]: block (owned expert i, source q) in the receive buffer
    recv_counts: torch.Tensor     # [n_own, G]
    local_offsets: torch.Tensor   # [n_own + 1]: group offsets of the owned experts
    total: int                    # rows received

    @property
    def n_own(self) -> int:
        return self.hi - self.lo


def gather_counts(expert_offsets: torch.Tensor, n_ffn: int, group=None) -> torch.Tensor:
    """Every rank's per-expert row counts, [G, n_ffn] int32 on the host (one
    all-gather of the count vectors; the only synchronising step)."""
    counts = (expert_offsets[1:n_ffn + 1] - expert_offsets[:n_ffn]).to(torch.int32).contiguous()
    G = dist.get_world_size(group)
    out = torch.empty((G * n_ffn,), dtype=torch.int32, device=counts.device)
    dist.all_gather_into_tensor(out, counts, group=group)
    return out.view(G, n_ffn).cpu()


def make_plan(counts: torch.Tensor, rank: int) -> ExchangePlan:
    G, E = counts.shape
    lo, hi = abi.moe_ep_expert_range(G, E, rank)
    ro, rc, loc, total = abi.moe_ep_plan(counts, rank)
    return ExchangePlan(G, E, rank, lo, hi, counts, ro, rc, loc, total)


def _run(ops) -> None:
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


def _peer(group, r: int) -> int:
    return r if group is None else dist.get_global_rank(group, r)


def dispatch(x_sorted: torch.Tensor, offsets_host: torch.Tensor, plan: ExchangePlan, group=None,
             out: torch.Tensor | None = None) -> torch.Tensor:
    """Rows of this rank's x_sorted -> the owners' receive buffers.  Returns
    this rank's receive buffer [max(total, 1), d] (rows of its owned experts,
    expert-major, source rank inside)."""
    d = x_sorted.shape[1]
    if out is None:
        out = torch.empty((max(plan.total, 1), d), dtype=x_sorted.dtype, device=x_sorted.device)
    me, G, E = plan.rank, plan.G, plan.E
    ops = []
    for e in range(E):                                  # sends, increasing expert order
        c = int(plan.counts[me, e])
        if c == 0:
            continue
        o = int(offsets_host[e])
        owner = abi.moe_ep_owner(G, E, e)
        if owner == me:
            i = e - plan.lo
            r0 = int(plan.recv_offsets[i, me])
            out[r0:r0 + c].copy_(x_sorted[o:o + c])
        else:
            ops.append(dist.P2POp(dist.isend, x_sorted[o:o + c], _peer(group, owner), group, tag=e))
    for i in range(plan.n_own):                         # receives, increasing expert order per source
        for q in range(G):
            c = int(plan.recv_counts[i, q])
            if q == me or c == 0:
                continue
            r0 = int(plan.recv_offsets[i, q])
            ops.append(dist.P2POp(dist.irecv, out[r0:r0 + c], _peer(group, q), group, tag=plan.lo + i))
    _run(ops)
    return out


def combine_return(recv_y: torch.Tensor, y_sorted: torch.Tensor, offsets_host: torch.Tensor, plan: ExchangePlan,
                   group=None) -> torch.Tensor:
    """The owners' results -> the rows of y_sorted the inputs came from (the
    inverse of dispatch)."""
    me, G, E = plan.rank, plan.G, plan.E
    ops = []
    for i in range(plan.n_own):                         # sends back, increasing expert order per source
        for q in range(G):
            c = int(plan.recv_counts[i, q])
            if c == 0:
                continue
            r0 = int(plan.recv_offsets[i, q])
            if q == me:
                o = int(offsets_host[plan.lo + i])
                y_sorted[o:o + c].copy_(recv_y[r0:r0 + c])
            else:
                ops.append(dist.P2POp(dist.isend, recv_y[r0:r0 + c], _peer(group, q), group, tag=plan.lo + i))
    for e in range(E):                                  # receives, increasing expert order
        c = int(plan.counts[me, e])
        owner = abi.moe_ep_owner(G, E, e)
        if c == 0 or owner == me:
            continue
        o = int(offsets_host[e])
        ops.append(dist.P2POp(dist.irecv, y_sorted[o:o + c], _peer(group, owner), group, tag=e))
    _run(ops)
    return y_sorted


class ExpertParallelMoELayer:
    """A SwiGLU MoE layer whose routed experts are split over a process group.

    ``weights`` holds the router (all rows, replicated), the MoE++ tensors if
    any, and the gate/up/down weights of THIS rank's experts only
    ([n_own, ...], experts lo..hi-1 of moe_ep_expert_range).  ``desc`` is the
    whole layer's descriptor for this rank's token batch (n_ffn = all routed
    experts).  Shared experts are not supported here.
    """

    def __init__(self, desc: abi.MoELayerDesc, weights: dict, group=None):
        if desc.kind != abi.MOE_EXPERT_SWIGLU or desc.n_shared:
            raise ValueError("expert parallelism: SwiGLU kind without shared experts")
        self.desc, self.weights, self.group = desc, weights, group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.lo, self.hi = abi.moe_ep_expert_range(self.G, desc.n_ffn, self.rank)
        self.ws = abi.weights_struct(weights)
        self.plan = None

    def _local_desc(self, rows: int) -> abi.MoELayerDesc:
        """Descriptor of the grouped step over the received rows: the owned
        experts as groups, a row capacity of at least `rows`."""
        d = self.desc
        return abi.MoELayerDesc(T=max(rows, 1), d_model=d.d_model, top_k=1, dtype=d.dtype, kind=d.kind,
                                n_ffn=self.hi - self.lo, hidden=d.hidden, n_shared=0, hidden_shared=0,
                                n_zero=0, n_copy=0, n_const=0, pk_rows=0, pk_cols=0, pk_topk_half=0,
                                d_query=0, out_f32=0)

    def forward(self, x: torch.Tensor, prev_logits=None) -> torch.Tensor:
        """The layer for this rank's tokens x [T, d] (on torch's current stream,
        which torch.distributed orders the exchanges against)."""
        d = self.desc
        dev = x.device
        b = StageBuffers(d, device=dev)
        cm = b.const_mix if d.n_const > 0 else None
        abi.moe_route(d, self.ws, x, prev_logits, None, b.idx, b.gate, cm, b.workspace)
        abi.moe_permute(d, b.idx, x, b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace)
        counts = gather_counts(b.offsets, d.n_ffn, self.group)
        self.plan = plan = make_plan(counts, self.rank)
        offsets_host = b.offsets.cpu()
        recv_x = dispatch(b.x_sorted, offsets_host, plan, self.group)
        recv_y = torch.empty((max(plan.total, 1), d.d_model), dtype=torch.float32, device=dev)
        if plan.n_own > 0 and plan.total > 0:
            ld = self._local_desc(plan.total)
            ws_local = torch.empty((abi.moe_workspace_size(ld),), dtype=torch.uint8, device=dev)
            loc = plan.local_offsets.to(dev)
            abi.moe_grouped_ffn_phase(ld, self.ws, 1, recv_x, loc, recv_y, ws_local)
            abi.moe_grouped_ffn_phase(ld, self.ws, 2, recv_x, loc, recv_y, ws_local)
        combine_return(recv_y, b.y_sorted, offsets_host, plan, self.group)
        y = torch.empty((d.T, d.d_model), dtype=out_dtype(d), device=dev)
        abi.moe_combine(d, self.ws, b.y_sorted, b.offsets, b.row_of, b.idx, b.gate, cm, x, y)
        return y

    __call__ = forward


def local_expert_weights(weights: dict, lo: int, hi: int) -> dict:
    """A rank's share of a full weight dict: the router and MoE++ tensors as
    they are, the routed experts' gate/up/down weights lo..hi-1."""
    w = dict(weights)
    for k in ("w_gate", "w_up", "w_down"):
        if weights.get(k) is not None:
            w[k] = weights[k][lo:hi].contiguous() if hi > lo else None
    return w


__all__ = ["ExchangePlan", "ExpertParallelMoELayer", "combine_return", "dispatch", "gather_counts",
           "local_expert_weights", "make_plan"]
