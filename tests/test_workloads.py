"""The seeded workload generator: determinism, shapes, distributions (CPU)."""

import numpy as np
import torch

import oracle
from moe_workloads import CONFIGS, get_config, make_activations, make_weights, scaled
from moe_workloads.gen import load_router_bias, zipf_targets


def test_deterministic_and_independent_of_T():
    cfg = get_config("tiny_f32")
    a = make_weights(cfg)
    b = make_weights(scaled(cfg, T=7))
    for k in a:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k
    x1 = make_activations(cfg)["x"]
    x2 = make_activations(cfg)["x"]
    assert torch.equal(x1, x2) and x1.shape == (64, 128) and x1.dtype == torch.float32


def test_distributions_tiny():
    cfg = get_config("tiny_f32")
    w = make_weights(cfg)
    x = make_activations(cfg)["x"]
    assert abs(x.std().item() - 128 ** -0.5) < 0.05 * 128 ** -0.5
    assert abs(w["w_gate"].std().item() - 128 ** -0.5) < 0.02 * 128 ** -0.5
    assert abs(w["w_down"].std().item() - 256 ** -0.5) < 0.02 * 256 ** -0.5
    assert w["w_gate"].shape == (8, 256, 128) and w["w_down"].shape == (8, 128, 256)


def test_bf16_cast_is_round_to_nearest():
    cfg = scaled(get_config("longtail"), T=4)
    x = make_activations(cfg)["x"]
    assert x.dtype == torch.bfloat16 and x.shape == (4, 2048)


def test_router_bias_files():
    lt = load_router_bias(get_config("longtail"))
    mp = load_router_bias(get_config("moepp"))
    assert lt.shape == (64,) and mp.shape == (20,)
    assert (mp[:16] == 0).all() and (mp[16:] == mp[16]).all() and mp[16] > 0
    t = zipf_targets(get_config("longtail"))
    assert abs(sum(t) - 2048 * 6) < 1e-6 and max(t) <= 2048 + 1e-9
    assert all(t[i] >= t[i + 1] - 1e-9 for i in range(63))


def test_longtail_bias_realises_zipf_load():
    """Reported property of the stored bias: the realised per-expert load is
    within 8 tokens of the Zipf(1.2) targets (the fit gave 5.2)."""
    cfg = get_config("longtail")
    x = make_activations(cfg)["x"]
    w = make_weights(cfg)
    z = oracle.router_logits(x, w["w_router"], w["router_bias"])
    idx, _, _ = oracle.topk(z, cfg.top_k)
    c = np.bincount(idx.reshape(-1), minlength=64)
    assert np.abs(c - np.array(zipf_targets(cfg))).max() < 8


def test_all_configs_have_consistent_sizes():
    for name, cfg in CONFIGS.items():
        assert cfg.T > 0 and cfg.d > 0
        if cfg.kind == "atomic":
            assert cfg.d_query % 2 == 0 and cfg.top_k <= cfg.pk_topk_half ** 2
        else:
            assert cfg.top_k <= cfg.n_routed
