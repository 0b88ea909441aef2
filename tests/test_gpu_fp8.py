"""FP8 experts through the C ABI vs the fp64 oracle ("PCoMoE" summary,
"Improvements", 3: FP8 for the expert computation, BF16 for the gating).

The expert weights are e4m3 codes with fp32 row scales, read exactly by the
oracle; the activations are quantized per row with power-of-two scales, which
the oracle models step by step (the codes and scales of the permuted x rows
must match it bit for bit), so the layer output meets the same bar as the
bf16 layer: max |y - y_oracle| <= 2e-2 rms(y_oracle) on the fp32 result, the
bf16 output its round-to-nearest-even.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from moe_workloads import get_config, make_inputs, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_swiglu_b200 as moe  # noqa: E402
    from parity import check_swiglu_layer, to_device  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status():
    if torch.cuda.is_available():
        moe.moe_get_device_status(reset=True)
    yield


def _sample(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n, T), replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s), dtype=np.int32)


@pytest.mark.parametrize("name,T,changes", [
    ("mixtral_fp8", 333, {"d": 256, "hidden": 384, "n_ffn": 4}),     # ragged groups, one K box of 256
    ("mixtral_fp8", 600, {"d": 2048, "hidden": 512, "n_ffn": 2}),
    ("mixtral_fp8", 129, {"d": 512, "hidden": 256, "n_ffn": 4}),
    ("longtail_fp8", 200, {}),                                       # shared experts, k = 6
    ("moepp_fp8", 300, {"hidden": 640}),                             # zero-computation slots, residual
])
def test_fp8_layer_small(name, T, changes):
    cfg = scaled(get_config(name), T=T, **changes)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    print(f"\n{name} T={T}: fp32 result err/rms {rep['rel_err']:.3e}, bf16 output {rep['rel_err_out']:.3e}")


def test_fp8_layer_forward_equals_stages():
    cfg = scaled(get_config("longtail_fp8"), T=150)
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    stages = moe.StageBuffers(desc)
    moe.run_stages(desc, inp, inp["x"], stages)
    y = moe.MoELayer(desc, inp).forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(y, stages.y)
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK


def test_fp8_mixtral_full_size_sampled():
    cfg = get_config("mixtral_fp8")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 12))
    print(f"\nmixtral_fp8: fp32 result err/rms {rep['rel_err']:.3e}, bf16 output {rep['rel_err_out']:.3e}")


def test_fp8_moepp_full_size_sampled():
    cfg = get_config("moepp_fp8")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 16))
    print(f"\nmoepp_fp8: fp32 result err/rms {rep['rel_err']:.3e}")
