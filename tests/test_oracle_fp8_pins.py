"""Pins for the oracle's FP8 expert path (CPU only).

"PCoMoE" summary, "Improvements", 3 (Mixed Precision Execution): the expert
computation in FP8 (E4M3), the gating in BF16.  The oracle's e4m3 decoding
and rounding are checked against torch's float8_e4m3fn conversion (a library
routine) on every code and on a dense sweep of values with all the ties; the
power-of-two row scale against its closed form; and the whole FP8 expert on
hand-worked cases with one hidden unit, where every quantization step can be
followed by hand (a dropped scale or a skipped rounding changes the result).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from moe_workloads import MoEConfig

F8 = torch.float8_e4m3fn


def test_e4m3_decode_every_code_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(F8).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert nan.sum() == 2 and (np.isnan(got) == nan).all()             # 0x7f and 0xff
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6 and oracle.e4m3_decode(0x38) == 1.0


def test_e4m3_round_matches_torch_on_values_and_ties():
    grid = np.unique(np.abs(torch.arange(256, dtype=torch.int32).to(torch.uint8).view(F8).to(torch.float64)
                            .numpy()))
    grid = grid[np.isfinite(grid)]
    mids = (grid[1:] + grid[:-1]) / 2                                  # every tie
    rng = np.random.default_rng(0)
    rand = rng.uniform(0, 448, 20000)
    small = rng.uniform(0, 2.0 ** -5, 5000)
    vals = np.concatenate([grid, mids, rand, small, np.nextafter(mids, 0), np.nextafter(mids, 1000)])
    vals = np.concatenate([vals, -vals])
    ref = torch.from_numpy(vals).to(torch.float32).to(F8).to(torch.float64).numpy()
    # torch rounds through float32; every value here is exact in float32 except
    # the nextafter neighbours of the ties, whose float32 rounding is the tie itself
    exact32 = torch.from_numpy(vals).to(torch.float32).to(torch.float64).numpy() == vals
    got = np.array([oracle.e4m3_round(v) for v in vals])
    np.testing.assert_array_equal(got[exact32], ref[exact32])
    assert oracle.e4m3_round(1.0625) == 1.0          # tie between 1 and 1.125 -> even mantissa
    assert oracle.e4m3_round(1.1875) == 1.25         # tie between 1.125 and 1.25 -> even
    assert oracle.e4m3_round(2.0 ** -10) == 0.0      # tie between 0 and the smallest subnormal
    assert oracle.e4m3_round(3 * 2.0 ** -10) == 2 * 2.0 ** -9
    assert oracle.e4m3_round(460.0) == 448.0 and oracle.e4m3_round(-1e9) == -448.0


@pytest.mark.parametrize("amax,s", [(448.0, 1.0), (448.0001, 2.0), (447.9, 1.0), (224.0, 0.5), (224.01, 1.0),
                                    (60.0, 0.25), (1.0, 2.0 ** -8), (1e-30, 2.0 ** -108), (0.0, 1.0)])
def test_pow2_scale_closed_form(amax, s):
    assert oracle.pow2_scale(amax) == s
    if amax > 0:
        assert 448.0 * s >= amax > 448.0 * s / 2


def test_quantize_rows_bounds_and_exact_rows():
    g = torch.Generator().manual_seed(3)
    x = torch.randn((5, 64), generator=g).to(torch.bfloat16)
    q, sc = oracle.quantize_rows(x)
    xd = x.double().numpy()
    for r in range(5):
        assert np.abs(q[r]).max() <= 448.0
        assert sc[r] == oracle.pow2_scale(np.abs(xd[r]).max())
        # each element within half an e4m3 spacing (relative 2^-4 for normals)
        err = np.abs(q[r] * sc[r] - xd[r])
        assert (err <= np.maximum(2.0 ** -4 * np.abs(xd[r]), 2.0 ** -10 * sc[r]) * (1 + 1e-12)).all()
    # a row already on the grid of its scale comes back exactly
    row = torch.tensor([[448.0, -240.0, 3.25, 0.0, 2.0 ** -9]]) * 2.0 ** -5
    q, sc = oracle.quantize_rows(row)
    assert sc[0] == 2.0 ** -5
    np.testing.assert_array_equal(q[0] * sc[0], row.double().numpy()[0])


def _one_unit_layer(gate_w: float, up_w: float, down_code_val: float, s_down: float, x_val: float = 1.0):
    """A layer of one FFN expert with hidden width 1 and d = 1, top-1:
    g = x * gate_w, u = x * up_w, y = s_down * code * h8 * s_h."""
    cfg = MoEConfig(name="fp8pin", T=1, d=1, top_k=1, dtype="f32", n_ffn=1, hidden=1)
    enc = lambda v: torch.tensor([[[v]]], dtype=torch.float32).to(F8).view(torch.uint8)  # noqa: E731
    inp = {"x": torch.tensor([[x_val]], dtype=torch.float32), "w_router": torch.zeros((1, 1)),
           "w_gate8": enc(1.0), "s_gate": torch.tensor([[gate_w]]), "w_up8": enc(1.0), "s_up": torch.tensor([[up_w]]),
           "w_down8": enc(down_code_val), "s_down": torch.tensor([[s_down]])}
    y, idx, gate, _ = oracle.fp8_moe_tokens(cfg, inp, np.arange(1))
    assert idx[0, 0] == 0 and gate[0, 0] == 1.0
    return y[0, 0]


def test_fp8_expert_hand_worked_exact_case():
    # x = 1 -> scale 2^-8, x8 = 256 (on the grid); g = 2^-8 * 30 * 256 = 30 (silu(30) = 30 to bf16),
    # u = 2; h = 60 -> scale 1/4 (448/4 = 112 >= 60 > 56), h8 = 240 (a multiple of 16 in [128, 256));
    # y = (1/4) * s_down * code * 240 = 60 * 1.5 * 0.5
    y = _one_unit_layer(30.0, 2.0, 1.5, 0.5)
    assert y == 60.0 * 1.5 * 0.5


def test_fp8_expert_hand_worked_rounding_of_h():
    # u = 2.1 -> h = 63 (bf16 63 exactly) -> h / (1/4) = 252, which e4m3 (spacing 16
    # in [128, 256)) rounds to 256 -> y = (1/4) * 256 * code * s_down = 64 * 1.5 * 0.5
    y = _one_unit_layer(30.0, 2.1, 1.5, 0.5)
    silu30 = 30.0 / (1.0 + math.exp(-30.0))
    assert abs(silu30 * 2.1 - 63.0) < 1e-9
    assert y == 64.0 * 1.5 * 0.5


def test_fp8_expert_hand_worked_bf16_rounding_of_h():
    # u = 2.01 -> h = 60.3 -> bf16 (spacing 0.25 in [32, 64)) = 60.25 -> / (1/4) = 241 -> e4m3 240
    y = _one_unit_layer(30.0, 2.01, 1.0, 1.0)
    assert y == 60.0


def _fp8_rand_inputs(cfg: MoEConfig, seed: int):
    """Random bf16 layer and its FP8 experts: weight rows quantized with an
    fp32 row scale amax / 448 (the dequantized weights are code * scale)."""
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g)  # noqa: E731
    d, H, E = cfg.d, cfg.hidden, cfg.n_ffn
    inp = {"x": r(cfg.T, d).to(torch.bfloat16), "w_router": (r(cfg.n_routed, d) * 0.7).to(torch.bfloat16)}
    for name, shape, fan in (("gate", (E, H, d), d), ("up", (E, H, d), d), ("down", (E, d, H), H)):
        w = r(*shape) * fan ** -0.5
        s = w.abs().amax(dim=-1, keepdim=True) / 448.0
        code = (w / s).to(F8)
        inp[f"w_{name}8"], inp[f"s_{name}"] = code.view(torch.uint8), s
        inp[f"w_{name}"] = (code.to(torch.float32) * s)              # the dequantized weights (fp32)
    return inp


def test_fp8_layer_is_the_dequantized_layer_up_to_activation_quantization():
    """The FP8 layer differs from the layer on its dequantized weights only by
    the e4m3 rounding of x and h: a relative error at the 2^-4 scale of a
    3-bit mantissa (here 1%-8% of rms), never O(1) (a lost scale or a
    transposed operand would be)."""
    cfg = MoEConfig(name="fp8pin", T=12, d=64, top_k=2, dtype="f32", n_ffn=4, hidden=48)
    inp = _fp8_rand_inputs(cfg, 5)
    y8, idx8, _, _ = oracle.fp8_moe_tokens(cfg, inp, np.arange(cfg.T))
    exact = {k_: v for k_, v in inp.items() if not k_.endswith("8") and not k_.startswith("s_")}
    exact["x"] = inp["x"].float()
    exact["w_router"] = inp["w_router"].float()
    y, idx, _, _ = oracle.moe_tokens(cfg, exact, np.arange(cfg.T))
    assert (idx8 == idx).all()                           # the gating does not see the FP8 experts
    rel = np.sqrt(((y8 - y) ** 2).mean() / (y ** 2).mean())
    assert 0.005 < rel < 0.08, rel
