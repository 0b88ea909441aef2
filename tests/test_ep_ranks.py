"""Expert parallelism on CPU: two gloo ranks (no GPU).

The routed experts are split over the ranks (contiguous id ranges); each rank
permutes its own tokens, sends each expert's block of rows to the expert's
owner, the owner computes them, and the results come back to the rows they
came from.  With a per-row expert function evaluated the same way on every
rank, the layer split over two ranks must equal the layer computed by one
rank alone bit for bit; every received block must hold exactly the rows its
source rank grouped for that expert.  The permutation is the oracle's
(expert, token) order; the exchange plan and ownership are the library's host
functions (moe_ep_*), the exchange is ep.dispatch / ep.combine_return.
"""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
D = 8


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_batch(rank: int, E: int, k: int, T: int, skip_expert: int | None):
    """A rank's tokens and routing: distinct experts per token (never
    `skip_expert` on rank 1, so that expert has no rows there)."""
    g = torch.Generator().manual_seed(100 + rank)
    x = torch.randn((T, D), generator=g, dtype=torch.float64)
    allowed = [e for e in range(E) if not (rank == 1 and e == skip_expert)]
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        perm = torch.randperm(len(allowed), generator=g)[:k].tolist()
        idx[t] = [allowed[p] for p in perm]
    gate = torch.rand((T, k), generator=g, dtype=torch.float64)
    return x, idx, gate / gate.sum(dim=1, keepdim=True)


def _expert_weights(E: int):
    g = torch.Generator().manual_seed(7)
    return torch.randn((E, D, D), generator=g, dtype=torch.float64) / D ** 0.5


def _expert_rows(rows: torch.Tensor, expert_of_row, W: torch.Tensor) -> torch.Tensor:
    """Stand-in expert: tanh(W_e x) per row, evaluated one row at a time so
    the bits do not depend on how many rows are computed together."""
    out = torch.empty_like(rows)
    for r in range(rows.shape[0]):
        out[r] = torch.tanh(torch.mv(W[int(expert_of_row[r])], rows[r]))
    return out


def _combine(y_sorted, row_of, gate):
    T, k = row_of.shape
    y = torch.zeros((T, D), dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            y[t] += gate[t, j] * y_sorted[int(row_of[t, j])]
    return y


def _worker(rank: int, world: int, port: int, E: int, k: int, out):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from mixture_experts_layer_swiglu_b200 import _abi, ep
        T = 37 + 11 * rank
        skip = E - 2 if E > 2 else None
        x, idx, gate = _rank_batch(rank, E, k, T, skip)
        counts, offsets, row_of, token_of, _ = oracle.group_tasks(idx, E, E)
        x_sorted = x[torch.from_numpy(token_of).long()]
        off_t = torch.from_numpy(offsets.astype(np.int32))
        counts_all = ep.gather_counts(off_t, E)
        plan = ep.make_plan(counts_all, rank)
        recv_x = ep.dispatch(x_sorted, off_t, plan)

        # every received block holds the rows its source grouped for that expert
        blocks_ok = True
        for i in range(plan.n_own):
            e = plan.lo + i
            for q in range(world):
                xq, iq, _ = _rank_batch(q, E, k, 37 + 11 * q, skip)
                _, oq, _, tq, _ = oracle.group_tasks(iq, E, E)
                c = int(plan.recv_counts[i, q])
                r0 = int(plan.recv_offsets[i, q])
                want = xq[torch.from_numpy(tq[oq[e]:oq[e + 1]]).long()]
                blocks_ok &= c == oq[e + 1] - oq[e] and torch.equal(recv_x[r0:r0 + c], want)
            blocks_ok &= int(plan.local_offsets[i]) == int(plan.recv_offsets[i, 0])

        W = _expert_weights(E)
        local_expert = np.repeat(np.arange(plan.lo, plan.hi), np.diff(plan.local_offsets.numpy()))
        recv_y = _expert_rows(recv_x[:plan.total], local_expert, W) if plan.total else recv_x[:0].clone()
        y_sorted = torch.full((int(offsets[E]), D), float("nan"), dtype=torch.float64)
        ep.combine_return(recv_y, y_sorted, off_t, plan)
        y_ep = _combine(y_sorted, row_of, gate)

        # the same tokens on one rank with every expert local
        expert_of_row = np.repeat(np.arange(E), counts)
        y_one = _combine(_expert_rows(x_sorted, expert_of_row, W), row_of, gate)
        owners = [_abi.moe_ep_owner(world, E, e) for e in range(E)]
        out.put((rank, bool(blocks_ok), bool(torch.equal(y_ep, y_one)), plan.lo, plan.hi, plan.total,
                 int(counts_all.sum()), owners))
    except Exception as exc:   # noqa: BLE001 -- reported to the parent
        out.put((rank, repr(exc)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("E,k", [(5, 2), (1, 1), (8, 3)])
def test_expert_parallel_layer_equals_one_rank_bit_for_bit(E, k):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, E, k, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        item = q.get(timeout=180)
        assert len(item) > 2, f"rank {item[0]} failed: {item[1]}"
        res[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lo_hi = [(res[r][2], res[r][3]) for r in (0, 1)]
    assert lo_hi == [(0, E // 2), (E // 2, E)]          # contiguous id ranges, rank 0 first
    assert res[0][6] == res[1][6] == [0 if e < E // 2 else 1 for e in range(E)]
    for r in (0, 1):
        blocks_ok, equal, _, _, total, all_rows, _ = res[r]
        assert blocks_ok, f"rank {r}: a received block differs from its source rows"
        assert equal, f"rank {r}: the expert-parallel layer differs from the one-rank layer"
    # every routed row is received by exactly one owner
    assert res[0][4] + res[1][4] == res[0][5] == (37 + 48) * k


def test_plan_host_functions():
    sys.path.insert(0, str(ROOT))
    from mixture_experts_layer_swiglu_b200 import _abi
    assert [_abi.moe_ep_expert_range(3, 8, r) for r in range(3)] == [(0, 2), (2, 5), (5, 8)]
    assert [_abi.moe_ep_owner(3, 8, e) for e in range(8)] == [0, 0, 1, 1, 1, 2, 2, 2]
    assert [_abi.moe_ep_owner(4, 2, e) for e in range(2)] == [1, 3]   # E < G: ranks 0 and 2 own nothing
    assert _abi.moe_ep_expert_range(4, 2, 0) == (0, 0)
    c = torch.tensor([[1, 2, 3, 4, 5, 6, 7, 8], [10, 20, 30, 40, 50, 60, 70, 80], [0, 0, 1, 0, 0, 0, 0, 9]],
                     dtype=torch.int32)
    ro, rc, loc, total = _abi.moe_ep_plan(c, 1)              # rank 1 owns experts 2, 3, 4
    assert rc.tolist() == [[3, 30, 1], [4, 40, 0], [5, 50, 0]]
    assert ro.tolist() == [[0, 3, 33], [34, 38, 78], [78, 83, 133]]
    assert loc.tolist() == [0, 34, 78, 133] and total == 133
    with pytest.raises(_abi.MoEError):
        _abi.moe_ep_plan(torch.tensor([[1, -1]], dtype=torch.int32), 0)
