"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, a special case that reduces to a textbook computation, or a brute-force
evaluation written differently (dense over all experts, masked by the gates,
with torch fp64 matmuls).  Together they are chosen so that a dropped term, a
wrong sign, a swapped operand or a wrong tie rule fails at least one of them.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from moe_workloads import MoEConfig

F64 = torch.float64


def _cfg(**kw) -> MoEConfig:
    base = dict(name="pin", T=8, d=12, top_k=2, dtype="f32", n_ffn=4, hidden=10)
    base.update(kw)
    return MoEConfig(**base)


def _rand_inputs(cfg: MoEConfig, seed: int, dtype=torch.float32, bias=False, zprev=False):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g).to(dtype)  # noqa: E731
    d, H, E = cfg.d, cfg.hidden, cfg.n_ffn
    inp = {"x": r(cfg.T, d), "w_router": r(cfg.n_routed, d) * 0.7,
           "w_gate": r(E, H, d) * d ** -0.5, "w_up": r(E, H, d) * d ** -0.5,
           "w_down": r(E, d, H) * H ** -0.5}
    if cfg.n_shared:
        S, Hs = cfg.n_shared, cfg.hidden_shared
        inp.update(ws_gate=r(S, Hs, d) * d ** -0.5, ws_up=r(S, Hs, d) * d ** -0.5,
                   ws_down=r(S, d, Hs) * Hs ** -0.5)
    if cfg.n_const:
        inp.update(w_const_mix=r(cfg.n_const, 2, d) * d ** -0.5, const_vec=r(cfg.n_const, d))
    if bias:
        inp["router_bias"] = torch.randn(cfg.n_routed, generator=g).float()
    if zprev:
        inp["z_prev"] = torch.randn(cfg.T, cfg.n_routed, generator=g).float()
    for k_, v in list(inp.items()):
        if k_ not in ("router_bias", "z_prev"):
            inp[k_] = v.to(dtype).contiguous()
    return inp


def _rank_desc(z: np.ndarray) -> np.ndarray:
    """Indices by descending value, equal values by ascending index."""
    return np.lexsort((np.arange(z.shape[-1]), -z))


def _dense_reference(cfg: MoEConfig, inp: dict) -> np.ndarray:
    """Every expert evaluated on every token, mixed by a gate vector that is
    zero outside the top-k: g_e = p_e / sum_{e' in top-k} p_e', p = softmax(z)."""
    x = inp["x"].to(F64)
    z = x @ inp["w_router"].to(F64).T
    if inp.get("router_bias") is not None:
        z = z + inp["router_bias"].to(F64)
    if inp.get("z_prev") is not None:
        z = z + inp["z_prev"].to(F64)
    p = torch.softmax(z, dim=1)
    T, E_r = z.shape
    mask = torch.zeros_like(p)
    for t in range(T):
        for e in _rank_desc(z[t].numpy())[: cfg.top_k]:
            mask[t, int(e)] = 1.0
    g = p * mask
    g = g / g.sum(dim=1, keepdim=True)
    outs = []
    for e in range(cfg.n_ffn):
        h = torch.nn.functional.silu(x @ inp["w_gate"][e].to(F64).T) * (x @ inp["w_up"][e].to(F64).T)
        outs.append(h @ inp["w_down"][e].to(F64).T)
    outs += [torch.zeros_like(x)] * cfg.n_zero + [x] * cfg.n_copy
    for c in range(cfg.n_const):
        a = torch.softmax(x @ inp["w_const_mix"][c].to(F64).T, dim=1)
        outs.append(a[:, :1] * x + a[:, 1:] * inp["const_vec"][c].to(F64))
    y = sum(g[:, e:e + 1] * outs[e] for e in range(E_r))
    for s in range(cfg.n_shared):
        h = torch.nn.functional.silu(x @ inp["ws_gate"][s].to(F64).T) * (x @ inp["ws_up"][s].to(F64).T)
        y = y + h @ inp["ws_down"][s].to(F64).T
    return y.numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("variant", ["plain", "shared", "moepp", "bias"])
def test_oracle_equals_dense_masked_bruteforce(dtype, variant):
    kw = {}
    if variant == "shared":
        kw = dict(n_shared=2, hidden_shared=6, top_k=3, n_ffn=6)
    if variant == "moepp":
        kw = dict(n_zero=1, n_copy=1, n_const=2, gating_residual=True)
    cfg = _cfg(**kw)
    inp = _rand_inputs(cfg, seed=11, dtype=dtype, bias=(variant == "bias"),
                       zprev=(variant == "moepp"))
    y, idx, gate, _ = oracle.moe_tokens(cfg, inp, np.arange(cfg.T))
    ref = _dense_reference(cfg, inp)
    assert np.abs(y - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    if variant == "moepp":   # the routing does reach the zero-computation experts
        assert (idx >= cfg.n_ffn).any()


def test_single_expert_top1_is_dense_swiglu():
    cfg = _cfg(n_ffn=1, top_k=1, T=5, d=7, hidden=9)
    inp = _rand_inputs(cfg, seed=3)
    y, idx, gate, _ = oracle.moe_tokens(cfg, inp, np.arange(cfg.T))
    assert (idx == 0).all() and (gate == 1.0).all()
    x = inp["x"].to(F64)
    a = x @ inp["w_gate"][0].to(F64).T
    ref = ((a * torch.sigmoid(a)) * (x @ inp["w_up"][0].to(F64).T)) @ inp["w_down"][0].to(F64).T
    np.testing.assert_allclose(y, ref.numpy(), rtol=0, atol=1e-13)


def _scalar_layer(wg, wu, wd, x=1.0):
    """d = H = 1, one expert: y = wd * silu(wg x) * (wu x)."""
    cfg = _cfg(T=1, d=1, hidden=1, n_ffn=1, top_k=1)
    t = lambda v: torch.tensor(v, dtype=torch.float32)  # noqa: E731
    inp = {"x": t([[x]]), "w_router": t([[1.0]]), "w_gate": t([[[wg]]]),
           "w_up": t([[[wu]]]), "w_down": t([[[wd]]])}
    return oracle.moe_tokens(cfg, inp, [0])[0][0, 0]


def test_silu_closed_forms():
    # silu(ln 3) = ln3 / (1 + 1/3) = 0.75 ln 3;  y = 0.5 * silu * 2
    a = float(np.float32(math.log(3.0)))
    assert abs(_scalar_layer(a, 2.0, 0.5) - 0.75 * math.log(3.0)) < 1e-6
    # silu(0) = 0 whatever the up projection
    assert _scalar_layer(0.0, 5.0, 3.0) == 0.0
    # silu(a) -> a for large a, -> 0 for large -a (sign of the exponent)
    assert abs(_scalar_layer(40.0, 1.0, 1.0) - 40.0) < 1e-12
    assert abs(_scalar_layer(-40.0, 1.0, 1.0)) < 1e-15
    # the up projection multiplies (not adds): wu = 0 gives 0
    assert _scalar_layer(3.0, 0.0, 1.0) == 0.0
    # the down projection scales linearly and keeps its sign
    assert abs(_scalar_layer(3.0, 1.0, -2.0) + 2.0 * _scalar_layer(3.0, 1.0, 1.0)) < 1e-15


def test_gates_closed_form_k_equals_E():
    # logits ln1, ln2, ln4 -> softmax (1, 2, 4)/7; order by descending logit
    z = np.log(np.array([[1.0, 2.0, 4.0]]))
    idx, gate, margin = oracle.topk(z, 3)
    assert idx.tolist() == [[2, 1, 0]]
    np.testing.assert_allclose(gate[0], [4 / 7, 2 / 7, 1 / 7], rtol=0, atol=1e-15)
    assert margin[0] == np.inf


def test_gates_renormalised_over_selected():
    # top-2 of (ln1, ln2, ln4, ln8): selected 8 and 4 -> 8/12, 4/12
    z = np.log(np.array([[1.0, 2.0, 4.0, 8.0]]))
    idx, gate, margin = oracle.topk(z, 2)
    assert idx.tolist() == [[3, 2]]
    np.testing.assert_allclose(gate[0], [2 / 3, 1 / 3], atol=1e-15)
    np.testing.assert_allclose(margin[0], math.log(2.0), atol=1e-15)


def test_topk_ties_go_to_lower_index():
    z = np.array([[1.0, 3.0, 3.0, 2.0, 3.0], [0.5, 0.5, 0.5, 0.5, 0.5]])
    idx, gate, margin = oracle.topk(z, 2)
    assert idx.tolist() == [[1, 2], [0, 1]]
    assert margin.tolist() == [0.0, 0.0]
    idx3, _, _ = oracle.topk(z, 3)
    assert idx3.tolist() == [[1, 2, 4], [0, 1, 2]]


def test_topk_matches_bruteforce_random():
    rng = np.random.default_rng(5)
    z = rng.integers(-3, 4, size=(200, 9)).astype(np.float64)  # many ties
    for k in (1, 2, 4, 9):
        idx, gate, margin = oracle.topk(z, k)
        for t in range(z.shape[0]):
            assert idx[t].tolist() == _rank_desc(z[t])[:k].tolist()
        np.testing.assert_allclose(gate.sum(1), 1.0, atol=1e-12)
        assert (np.diff(gate, axis=1) <= 1e-15).all()


def test_group_tasks_bruteforce():
    rng = np.random.default_rng(1)
    T, k, n_ffn, n_ids = 300, 3, 7, 10
    idx = np.stack([rng.choice(n_ids, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, row_of, token_of, slot_of = oracle.group_tasks(idx, n_ffn, n_ids)
    expect = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k) if idx[t, j] < n_ffn)
    assert [(int(idx[t, j]), t, j) for t, j in zip(token_of, slot_of)] == expect
    assert counts.sum() == len(expect) == offsets[-1]
    assert (np.diff(offsets) == counts).all() and offsets[0] == 0
    for p, (e, t, j) in enumerate(expect):
        assert row_of[t, j] == p and offsets[e] <= p < offsets[e + 1]
    # every token appears exactly k times counting the non-grouped (-1) slots
    assert ((row_of >= 0).sum(1) + (row_of < 0).sum(1) == k).all()
    assert ((row_of < 0) == (idx >= n_ffn)).all()
    with pytest.raises(ValueError):
        oracle.group_tasks(np.array([[0, n_ids]], np.int32), n_ffn, n_ids)


def _forced(cfg: MoEConfig, inp: dict, target: int):
    inp = dict(inp)
    b = torch.zeros(cfg.n_routed)
    b[target] = 1e6
    inp["router_bias"] = b
    return oracle.moe_tokens(cfg, inp, np.arange(cfg.T))


def test_moepp_zero_copy_const_special_cases():
    cfg = _cfg(n_zero=1, n_copy=1, n_const=2, top_k=1)
    inp = _rand_inputs(cfg, seed=2)
    zero_id, copy_id, const0 = cfg.n_ffn, cfg.n_ffn + 1, cfg.n_ffn + 2
    y, idx, gate, _ = _forced(cfg, inp, zero_id)
    assert (idx == zero_id).all() and (y == 0.0).all()
    y, idx, gate, _ = _forced(cfg, inp, copy_id)
    assert (gate == 1.0).all()
    np.testing.assert_array_equal(y, inp["x"].double().numpy())
    inp0 = dict(inp)
    inp0["w_const_mix"] = torch.zeros_like(inp["w_const_mix"])
    for c in range(2):
        y, idx, _, _ = _forced(cfg, inp0, const0 + c)
        ref = 0.5 * inp["x"].double().numpy() + 0.5 * inp["const_vec"][c].double().numpy()
        np.testing.assert_allclose(y, ref, atol=1e-15)
    # a mix weight that puts all mass on v: y = v for every token
    inp1 = dict(inp)
    wc = torch.zeros_like(inp["w_const_mix"])
    inp1["x"] = torch.ones_like(inp["x"])
    wc[0, 1, :] = 100.0
    inp1["w_const_mix"] = wc
    y, _, _, _ = _forced(cfg, inp1, const0)
    np.testing.assert_allclose(y, np.broadcast_to(inp["const_vec"][0].double().numpy(), y.shape),
                               atol=1e-12)


def test_zero_expert_gate_dilutes_ffn():
    # top-2 forced onto (FFN 0, zero expert) with equal logits -> y = 0.5 * E_0(x)
    cfg = _cfg(n_zero=1, top_k=2, n_ffn=2)
    inp = _rand_inputs(cfg, seed=4)
    inp["w_router"] = torch.zeros_like(inp["w_router"])
    inp["router_bias"] = torch.tensor([5.0, -5.0, 5.0])
    y, idx, gate, _ = oracle.moe_tokens(cfg, inp, np.arange(cfg.T))
    assert (idx == np.array([0, 2])).all() and np.allclose(gate, 0.5, atol=0)
    cfg1 = _cfg(n_ffn=1, top_k=1)
    inp1 = {k_: v[:1] if k_ in ("w_gate", "w_up", "w_down", "w_router") else v
            for k_, v in inp.items() if k_ != "router_bias"}
    y1 = oracle.moe_tokens(cfg1, inp1, np.arange(cfg.T))[0]
    np.testing.assert_allclose(y, 0.5 * y1, atol=1e-15)


def test_gating_residual_and_bias_add_to_logits():
    cfg = _cfg(T=6, n_ffn=5)
    inp = _rand_inputs(cfg, seed=9, bias=True, zprev=True)
    z = oracle.router_logits(inp["x"], inp["w_router"], inp["router_bias"], inp["z_prev"])
    z0 = oracle.router_logits(inp["x"], inp["w_router"])
    np.testing.assert_allclose(z - z0, inp["router_bias"].double().numpy()[None]
                               + inp["z_prev"].double().numpy(), atol=1e-12)
    ref = (inp["x"].double() @ inp["w_router"].double().T).numpy()
    np.testing.assert_allclose(z0, ref, atol=1e-12)


def test_idx_override_recomputes_gates_from_logits():
    cfg = _cfg(T=4, n_ffn=5, top_k=2)
    inp = _rand_inputs(cfg, seed=8)
    y, idx, gate, _ = oracle.moe_tokens(cfg, inp, np.arange(4))
    y2, idx2, gate2, _ = oracle.moe_tokens(cfg, inp, np.arange(4), idx_in=idx)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_allclose(gate, gate2, atol=0)
    np.testing.assert_allclose(y, y2, atol=0)
    flipped = idx[:, ::-1].copy()
    y3, idx3, gate3, _ = oracle.moe_tokens(cfg, inp, np.arange(4), idx_in=flipped)
    np.testing.assert_allclose(y3, y, atol=1e-14)   # order of the slots does not matter


# ---------------------------------------------------------- atomic experts

PHI1 = 0.8413447460685429   # standard normal CDF at 1 (textbook table value)


def test_gelu_closed_forms():
    d = 4
    x = torch.tensor([[1.0, 0.0, 0.0, 0.0]])
    u = torch.zeros(3, d)
    v = torch.zeros(3, d)
    u[0, 0], u[1, 0], u[2, 0] = 1.0, 0.0, -30.0      # u.x = 1, 0, -30
    v[:, 1] = torch.tensor([2.0, 5.0, 7.0])
    for e, expect in ((0, 2.0 * PHI1), (1, 0.0), (2, 0.0)):
        y = oracle.atomic_tokens(x, u, v, [0], np.array([[e]]), np.array([[1.0]]))
        assert abs(y[0, 1] - expect) < 1e-12 and abs(y[0, 0]) == 0.0
    # GELU(a) -> a for large a; the gate scales the contribution
    u[0, 0] = 30.0
    y = oracle.atomic_tokens(x, u, v, [0], np.array([[0, 1]]), np.array([[0.25, 0.75]]))
    assert abs(y[0, 1] - 0.25 * 30.0 * 2.0) < 1e-9


def _pk_inputs(seed, T=6, d=16, dq=8, rows=16, cols=16, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(T, d, generator=g).to(dtype), torch.randn(dq, d, generator=g).to(dtype),
            torch.randn(rows, dq // 2, generator=g).to(dtype),
            torch.randn(cols, dq // 2, generator=g).to(dtype))


def test_pk_scores_are_products_with_each_half():
    x, wq, kr, kc = _pk_inputs(1)
    sr, sc, q = oracle.pk_scores(x, wq, kr, kc, want_q=True)
    q_ref = x.double() @ wq.double().T
    np.testing.assert_allclose(q, q_ref.numpy(), atol=1e-12)
    np.testing.assert_allclose(sr, (q_ref[:, :4] @ kr.double().T).numpy(), atol=1e-12)
    np.testing.assert_allclose(sc, (q_ref[:, 4:] @ kc.double().T).numpy(), atol=1e-12)


def test_pk_select_equals_bruteforce_when_halves_keep_K():
    # with kh >= K the K best grid cells all lie among the kh x kh candidates
    x, wq, kr, kc = _pk_inputs(2)
    sr, sc = oracle.pk_scores(x, wq, kr, kc)
    K = 8
    idx, gate, mg = oracle.pk_select(sr, sc, kh=8, K=K)
    for t in range(x.shape[0]):
        full = (sr[t][:, None] + sc[t][None, :]).reshape(-1)   # id = r*cols + c
        best = _rank_desc(full)[:K]
        assert idx[t].tolist() == best.tolist()
        p = np.exp(full[best] - full[best].max())
        np.testing.assert_allclose(gate[t], p / p.sum(), atol=1e-14)


def test_pk_select_reduces_to_1d_topk_with_flat_columns():
    rng = np.random.default_rng(3)
    sr = rng.standard_normal((5, 16))
    sc = np.zeros((5, 16))            # all column sub-keys score the same
    idx, gate, mg = oracle.pk_select(sr, sc, kh=4, K=4)
    for t in range(5):
        r = int(_rank_desc(sr[t])[0])
        assert idx[t].tolist() == [r * 16 + c for c in range(4)]  # ties -> lower id
        np.testing.assert_allclose(gate[t], 0.25, atol=1e-15)
    idx, gate, mg = oracle.pk_select(sr, sc, kh=4, K=8)
    for t in range(5):
        r0, r1 = _rank_desc(sr[t])[:2]
        assert idx[t].tolist() == [int(r0) * 16 + c for c in range(4)] + [int(r1) * 16 + c for c in range(4)]


def test_pk_candidates_can_miss_global_topk():
    # the method is an approximation: with kh < K a grid cell outside the
    # kh x kh candidates can beat a selected one; the oracle must follow the
    # method, not the brute force.
    sr = np.array([[10.0, 9.0, 0.0, -50.0]])
    sc = np.array([[10.0, 9.0, 8.9, -50.0]])
    idx, _, _ = oracle.pk_select(sr, sc, kh=2, K=4)
    assert sorted(idx[0].tolist()) == sorted([0 * 4 + 0, 0 * 4 + 1, 1 * 4 + 0, 1 * 4 + 1])
    # brute force would take (0, 2) = 18.9 over (1, 1) = 18.0
    assert 0 * 4 + 2 not in idx[0].tolist()


def test_atomic_layer_dense_masked_bruteforce():
    x, wq, kr, kc = _pk_inputs(4, T=5, d=16, dq=8, rows=8, cols=8)
    g = torch.Generator().manual_seed(7)
    u = torch.randn(64, 16, generator=g) * 0.25
    v = torch.randn(64, 16, generator=g) * 0.25
    sr, sc = oracle.pk_scores(x, wq, kr, kc)
    idx, gate, _ = oracle.pk_select(sr, sc, kh=6, K=5)
    y = oracle.atomic_tokens(x, u, v, np.arange(5), idx, gate)
    # dense: every atomic expert on every token, masked by the gate vector
    a = x.double() @ u.double().T                                # [T, N]
    act = 0.5 * a * (1.0 + torch.special.erf(a / math.sqrt(2.0)))
    G = np.zeros((5, 64))
    for t in range(5):
        G[t, idx[t]] = gate[t]
    ref = (torch.from_numpy(G) * act) @ v.double()
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-13)
    np.testing.assert_allclose(gate.sum(1), 1.0, atol=1e-14)


def test_atomic_layer_top1_is_one_expert_with_gate_one():
    """K = 1: the best pair of the product grid is (best row, best column), so
    the product-key choice equals brute force over all N experts for any kept
    half size, the gate is exactly 1, and y_t = GELU(u_e . x_t) v_e (worked
    here with math.erf, element by element)."""
    rows = cols = 8
    x, wq, kr, kc = _pk_inputs(9, T=6, d=16, dq=8, rows=rows, cols=cols)
    g = torch.Generator().manual_seed(13)
    u = torch.randn(rows * cols, 16, generator=g) * 0.25
    v = torch.randn(rows * cols, 16, generator=g) * 0.25
    sr, sc = oracle.pk_scores(x, wq, kr, kc)
    for kh in (1, 3, 8):
        idx, gate, _ = oracle.pk_select(sr, sc, kh=kh, K=1)
        full = sr[:, :, None] + sc[:, None, :]                    # [T, rows, cols]
        assert idx[:, 0].tolist() == [int(np.argmax(f.reshape(-1))) for f in full]
        assert (gate == 1.0).all()
    y = oracle.atomic_tokens(x, u, v, np.arange(6), idx, gate)
    xd, ud, vd = x.double().numpy(), u.double().numpy(), v.double().numpy()
    for t in range(6):
        e = int(idx[t, 0])
        a = float(sum(ud[e, i] * xd[t, i] for i in range(16)))
        act = 0.5 * a * (1.0 + math.erf(a / math.sqrt(2.0)))
        np.testing.assert_allclose(y[t], act * vd[e], rtol=0, atol=1e-13)


def test_full_omnimoe_layer_is_atomic_plus_shared_swiglu():
    """The full OmniMoE layer (shared dense branch beside the atomic experts)
    minus the atomic-only layer equals the shared SwiGLU branch, computed two
    other ways: by the SwiGLU-kind layer whose one routed expert has a zero
    down projection, and densely with torch."""
    x, wq, kr, kc = _pk_inputs(5, T=5, d=16, dq=8, rows=8, cols=8)
    g = torch.Generator().manual_seed(11)
    u = torch.randn(64, 16, generator=g) * 0.25
    v = torch.randn(64, 16, generator=g) * 0.25
    Hs = 24
    sh = {"ws_gate": torch.randn(1, Hs, 16, generator=g) * 0.25, "ws_up": torch.randn(1, Hs, 16, generator=g) * 0.25,
          "ws_down": torch.randn(1, 16, Hs, generator=g) * 0.2}
    sr, sc = oracle.pk_scores(x, wq, kr, kc)
    idx, gate, _ = oracle.pk_select(sr, sc, kh=6, K=5)
    y_full = oracle.atomic_tokens(x, u, v, np.arange(5), idx, gate, shared=sh)
    y_atom = oracle.atomic_tokens(x, u, v, np.arange(5), idx, gate)
    cfg = _cfg(T=5, d=16, top_k=1, n_ffn=1, hidden=4, n_shared=1, hidden_shared=Hs)
    inp = {"x": x, "w_router": torch.ones(1, 16), "w_gate": torch.randn(1, 4, 16, generator=g),
           "w_up": torch.randn(1, 4, 16, generator=g), "w_down": torch.zeros(1, 16, 4), **sh}
    y_sh = oracle.moe_tokens(cfg, inp, np.arange(5))[0]
    np.testing.assert_allclose(y_full - y_atom, y_sh, rtol=0, atol=1e-13)
    xd = x.double()
    a = xd @ sh["ws_gate"][0].double().T
    dense = ((a * torch.sigmoid(a)) * (xd @ sh["ws_up"][0].double().T)) @ sh["ws_down"][0].double().T
    np.testing.assert_allclose(y_full - y_atom, dense.numpy(), rtol=0, atol=1e-13)
    assert np.abs(dense.numpy()).max() > 0.05          # the branch is not negligible here


# ----------------------------------------------------------- constant-expert mix
#
# "MoE++" summary, Approach: a constant expert mixes the token with a
# trainable vector, y = a1 x + a2 v, with (a1, a2) a 2-way softmax of W_c x.
# The GPU's const_mix output is checked against orc_const_mix, so that routine
# is pinned here by itself (the layer's own constant-expert arithmetic is a
# separate code path, pinned by test_moepp_zero_copy_const_special_cases).

def _logistic(u: float) -> float:
    """a1 of a 2-way softmax (l0, l1) = 1 / (1 + e^(l1 - l0)) for u = l0 - l1."""
    return 1.0 / (1.0 + math.exp(-u))


def test_const_mix_zero_weights_give_halves():
    x = torch.randn(5, 8, generator=torch.Generator().manual_seed(0))
    a = oracle.const_mix(x, torch.zeros(3, 2, 8))
    assert a.shape == (5, 3, 2)
    assert (a == 0.5).all()


def test_const_mix_one_dim_hand_computed():
    # d = 1: l0 = w0 x, l1 = w1 x, so a1 = logistic((w0 - w1) x) and a2 = 1 - a1
    x = torch.tensor([[1.0], [2.0], [-4.0]])
    wc = torch.tensor([[[0.5], [-0.25]]])            # one constant expert
    a = oracle.const_mix(x, wc)
    for t, xv in enumerate((1.0, 2.0, -4.0)):
        a1 = _logistic(0.75 * xv)
        assert abs(a[t, 0, 0] - a1) < 1e-15
        assert abs(a[t, 0, 1] - (1.0 - a1)) < 1e-15
    # x = 1: 1 / (1 + e^-0.75), to the digits printed by any table of e^x
    assert abs(a[0, 0, 0] - 0.679178699175393) < 1e-14


def test_const_mix_dominant_row_and_slot_swap():
    x = torch.ones(2, 4)
    wc = torch.zeros(1, 2, 4)
    wc[0, 1, :] = 25.0                                # l1 = 100, l0 = 0
    a = oracle.const_mix(x, wc)
    assert a[0, 0, 0] < 1e-40 and a[0, 0, 1] == 1.0
    a_sw = oracle.const_mix(x, wc.flip(1).contiguous())   # rows swapped -> slots swapped
    assert a_sw[0, 0, 0] == 1.0 and a_sw[0, 0, 1] < 1e-40
    # a mild case: the swap maps (a1, a2) to (a2, a1) exactly
    g = torch.Generator().manual_seed(1)
    x = torch.randn(6, 4, generator=g)
    wc = torch.randn(1, 2, 4, generator=g)
    a, a_sw = oracle.const_mix(x, wc), oracle.const_mix(x, wc.flip(1).contiguous())
    np.testing.assert_allclose(a_sw[:, :, ::-1], a, atol=1e-15)


def test_const_mix_experts_use_their_own_row_pairs():
    # expert c reads rows (2c, 2c + 1) of the flattened [n_const * 2, d] weights:
    # distinct pairs per expert, each checked by hand (d = 1, x = 1)
    x = torch.ones(1, 1)
    wc = torch.tensor([[[1.0], [0.0]],               # expert 0: l = (1, 0)
                       [[0.0], [2.0]],               # expert 1: l = (0, 2)
                       [[3.0], [3.0]]])              # expert 2: l = (3, 3)
    a = oracle.const_mix(x, wc)
    assert abs(a[0, 0, 0] - _logistic(1.0)) < 1e-15
    assert abs(a[0, 1, 0] - _logistic(-2.0)) < 1e-15
    assert a[0, 2, 0] == 0.5 and a[0, 2, 1] == 0.5


def test_const_mix_matches_layer_forced_to_constant_expert():
    # with v = 0 the layer forced onto constant expert c outputs a1 * x, so
    # y / x recovers a1: the layer's constant-expert code and orc_const_mix
    # agree (two separate code paths of the oracle)
    cfg = _cfg(n_zero=1, n_copy=1, n_const=2, top_k=1)
    inp = _rand_inputs(cfg, seed=12)
    inp["const_vec"] = torch.zeros_like(inp["const_vec"])
    a = oracle.const_mix(inp["x"], inp["w_const_mix"])
    xd = inp["x"].double().numpy()
    for c in range(2):
        y, idx, gate, _ = _forced(cfg, inp, cfg.n_ffn + cfg.n_zero + cfg.n_copy + c)
        assert (gate == 1.0).all()
        np.testing.assert_allclose(y, a[:, c, 0:1] * xd, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------ product-key margins
#
# "OmniMoE" technical summary, 2.2 Cartesian Product Router.  pk_select's
# margins set which mis-routed tokens the GPU parity check forgives: [0] the
# kh-th minus the (kh+1)-th row sub-score, [1] the same for the columns, [2]
# the K-th minus the (K+1)-th candidate sum; +inf where nothing is left out.

def test_pk_margins_hand_built():
    sr = np.array([[5.0, 1.0, 3.0, 2.0]])      # rows by score: 0 (5), 2 (3) | 3 (2), 1 (1)
    sc = np.array([[0.5, 4.0, 0.25, 3.5]])     # cols by score: 1 (4), 3 (3.5) | 0 (0.5), 2
    idx, gate, mg = oracle.pk_select(sr, sc, kh=2, K=3)
    # candidates (0,1) 9, (0,3) 8.5, (2,1) 7, (2,3) 6.5 -> the best 3
    assert idx[0].tolist() == [0 * 4 + 1, 0 * 4 + 3, 2 * 4 + 1]
    assert mg[0, 0] == 3.0 - 2.0                # kh-th row minus (kh+1)-th
    assert mg[0, 1] == 3.5 - 0.5                # kh-th column minus (kh+1)-th
    assert mg[0, 2] == 7.0 - 6.5                # K-th candidate minus (K+1)-th, not 8.5 - 7
    p = np.exp(np.array([9.0, 8.5, 7.0]) - 9.0)
    np.testing.assert_allclose(gate[0], p / p.sum(), atol=1e-15)


def test_pk_margins_infinite_when_nothing_left_out():
    sr = np.array([[2.0, -1.0, 0.5, 4.0]])
    sc = np.array([[1.0, 3.0, -2.0, 0.0]])
    _, _, mg = oracle.pk_select(sr, sc, kh=4, K=16)   # every row, column and candidate kept
    assert np.isinf(mg[0]).all() and (mg[0] > 0).all()
    _, _, mg = oracle.pk_select(sr, sc, kh=4, K=15)   # halves complete, one candidate out
    assert np.isinf(mg[0, :2]).all()
    assert mg[0, 2] == (0.5 - 2.0) - (-1.0 - 2.0)     # 15th best sum minus the 16th (the worst)


def test_pk_margins_zero_on_ties():
    sr = np.array([[1.0, 1.0, 0.0]])               # rows 0 and 1 tie at the kh = 1 boundary
    sc = np.array([[2.0, 0.0, 2.0]])               # columns 0 and 2 tie likewise
    idx, _, mg = oracle.pk_select(sr, sc, kh=1, K=1)
    assert idx[0].tolist() == [0]                  # ties go to the lower sub-index
    assert mg[0, 0] == 0.0 and mg[0, 1] == 0.0


def test_pk_margins_match_sorted_scores_random():
    rng = np.random.default_rng(11)
    sr, sc = rng.standard_normal((7, 12)), rng.standard_normal((7, 10))
    kh, K = 3, 5
    idx, _, mg = oracle.pk_select(sr, sc, kh=kh, K=K)
    for t in range(7):
        r_sorted, c_sorted = np.sort(sr[t])[::-1], np.sort(sc[t])[::-1]
        assert mg[t, 0] == r_sorted[kh - 1] - r_sorted[kh]
        assert mg[t, 1] == c_sorted[kh - 1] - c_sorted[kh]
        cand = np.sort((r_sorted[:kh][:, None] + c_sorted[:kh][None, :]).reshape(-1))[::-1]
        assert mg[t, 2] == cand[K - 1] - cand[K]
        assert mg[t].min() > 0
