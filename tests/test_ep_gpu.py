"""The expert-parallel layer on one GPU through NCCL (a group of one rank).

With one rank every expert is local, so the exchange reduces to local copies,
and the layer must equal the two-pass path (moe_route, moe_permute,
moe_grouped_ffn, moe_combine) bit for bit: the same permutation, the same
grouped GEMMs over the received rows (the owned experts as groups), the same
combine.  Several ranks need several GPUs; their exchange logic is
covered by the gloo tests (test_ep_ranks.py).
"""

from __future__ import annotations

import datetime
import socket

import pytest
import torch
import torch.distributed as dist

from moe_workloads import get_config, make_inputs, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_swiglu_b200 as moe
    from mixture_experts_layer_swiglu_b200 import ep
    from parity import to_device


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("name,T", [("mixtral", 600), ("moepp", 700)])
def test_expert_parallel_one_rank_equals_two_pass_layer(nccl_group, name, T):
    base = get_config(name)
    cfg = scaled(base, T=T, d=2048 if name == "mixtral" else 256, hidden=512 if name == "mixtral" else 256)
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    stages = moe.StageBuffers(desc)
    moe.run_stages(desc, inp, inp["x"], stages, prev_logits=inp.get("z_prev"))
    y_ref = stages.y
    lo, hi = moe.moe_ep_expert_range(1, cfg.n_ffn, 0)
    assert (lo, hi) == (0, cfg.n_ffn)
    layer = ep.ExpertParallelMoELayer(desc, ep.local_expert_weights(inp, lo, hi))
    y = layer.forward(inp["x"], prev_logits=inp.get("z_prev"))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    assert layer.plan.total == int(layer.plan.counts.sum())
    assert torch.equal(y, y_ref)
