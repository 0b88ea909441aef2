"""The fused expert step (moe_fused_ffn_combine) through the C ABI vs the
fp64 oracle, element by element: the gate/up GEMM on x_sorted (or, `gather`,
on token rows it gathers from x with its own loads), the gate-weighted
combine done by the down GEMM's epilogue into an fp32 accumulator (no
y_sorted), then the zero-computation terms and one rounding.  Routing and the permutation are checked as for the
two-pass path; the bf16 output must be the round-to-nearest-even of the fp32
result.  (moe_layer_forward keeps the two-pass step, measured faster.)
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from moe_workloads import get_config, make_inputs, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_swiglu_b200 as moe  # noqa: E402
    from parity import check_swiglu_layer, run_gpu_fused, to_device  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status():
    if torch.cuda.is_available():
        moe.moe_get_device_status(reset=True)
    yield


def _sample(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n, T), replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s), dtype=np.int32)


@pytest.mark.parametrize("gather", [False, True])
@pytest.mark.parametrize("T,d,H,E", [(333, 256, 384, 4), (600, 2048, 512, 2), (1100, 2048, 1024, 4),
                                     (513, 512, 256, 2)])
def test_fused_mixtral_shaped_ragged(T, d, H, E, gather):
    cfg = scaled(get_config("mixtral"), T=T, d=d, hidden=H, n_ffn=E)
    rep = check_swiglu_layer(cfg, make_inputs(cfg), fused=True, gather=gather)
    assert rep["R"] == T * 2


@pytest.mark.parametrize("gather", [False, True])
@pytest.mark.parametrize("T", [1, 2, 127, 129])
def test_fused_token_counts_across_tile_edges(T, gather):
    cfg = scaled(get_config("mixtral"), T=T, d=256, hidden=384, n_ffn=4)
    check_swiglu_layer(cfg, make_inputs(cfg), fused=True, gather=gather)


def test_fused_moepp_zero_copy_const_and_tokens_without_ffn_slots():
    """Zero-computation slots are added after the accumulator; tokens whose
    slots are all zero-computation experts never have an accumulator row
    written and must not read one."""
    cfg = scaled(get_config("moepp"), T=300, hidden=640)
    inp = make_inputs(cfg)
    rep = check_swiglu_layer(cfg, inp, fused=True)
    assert rep["R"] < 300 * 2
    check_swiglu_layer(cfg, inp, fused=True, gather=True)
    idx = rep["idx_oracle"]
    assert ((idx >= cfg.n_ffn).all(axis=1)).any(), "the case should hold a token with no FFN slot"


def test_fused_nearly_empty_group_top1():
    cfg = scaled(get_config("mixtral"), T=1100, d=2048, hidden=1024, n_ffn=2, top_k=1)
    inp = make_inputs(cfg)
    inp["router_bias"] = torch.tensor([3.5, 0.0])
    rep = check_swiglu_layer(cfg, inp, fused=True)
    assert rep["R"] == 1100


def test_fused_all_tokens_one_expert():
    cfg = scaled(get_config("mixtral"), T=300, d=256, hidden=256, n_ffn=6, top_k=1)
    inp = make_inputs(cfg)
    inp["router_bias"] = torch.tensor([0, 0, 0, 50.0, 0, 0])
    rep = check_swiglu_layer(cfg, inp, fused=True)
    assert rep["R"] == 300


@pytest.mark.parametrize("name,T,changes", [("mixtral", 600, {"d": 2048, "hidden": 512, "n_ffn": 4}),
                                            ("moepp", 700, {"hidden": 640})])
def test_fused_step_in_one_call_equals_phase_by_phase(name, T, changes):
    """Phase 0 (the three phases in one call) equals phases 1, 2, 3 called one
    by one, bit for bit; the two-pass layer (moe_layer_forward) agrees within
    the bar (another summation order; both are checked against the oracle)."""
    cfg = scaled(get_config(name), T=T, **changes)
    inp = to_device(make_inputs(cfg))
    r = run_gpu_fused(cfg, inp)
    b = r["bufs"]
    desc16 = moe.desc_from(cfg)
    y0 = torch.empty_like(r["y16"])
    cm = b.const_mix if desc16.n_const > 0 else None
    moe.moe_fused_ffn_combine(desc16, inp, 0, inp["x"], b.x_sorted, b.idx, b.gate, cm, b.offsets, b.row_of,
                              b.token_of, y0, b.fused_workspace)
    layer = moe.MoELayer(desc16, inp)
    y2 = layer.forward(inp["x"], prev_logits=inp.get("z_prev"))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    assert torch.equal(y0, r["y16"])
    rms = float(y2.float().pow(2).mean().sqrt())
    assert float((y2.float() - y0.float()).abs().max()) <= 2e-2 * rms


def test_fused_step_refuses_layers_it_does_not_cover():
    cfg = scaled(get_config("longtail"), T=64)          # shared experts, k = 6
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    assert moe.moe_fused_workspace_size(desc) == -1
    b = moe.StageBuffers(desc)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_fused_ffn_combine(desc, inp, 0, inp["x"], b.x_sorted, b.idx, b.gate, None, b.offsets, b.row_of,
                                  b.token_of, b.y, b.workspace)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_fused_mixtral_full_size_sampled():
    cfg = get_config("mixtral")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 12), fused=True)
    print(f"\nmixtral fused: fp32 result err/rms {rep['rel_err']:.3e}, bf16 output {rep['rel_err_out']:.3e}")


def test_fused_moepp_full_size_sampled():
    cfg = get_config("moepp")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 24), fused=True)
    print(f"\nmoepp fused: fp32 result err/rms {rep['rel_err']:.3e}, bf16 output {rep['rel_err_out']:.3e}")
