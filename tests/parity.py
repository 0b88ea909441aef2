"""Parity checks of the CUDA path (through the C ABI) against the fp64 oracle.

Bars (floating point): max|y_gpu - y_oracle| <= 2e-2 * rms(y_oracle) for bf16
layers and <= 1e-4 * rms(y_oracle) for fp32 layers, applied to the layer's
fp32 result (the combine's accumulator); the bf16 output of a bf16 layer must
equal its round-to-nearest-even bit for bit.  (Rounding the exact result to
bf16 alone costs up to 2^-8 |y|: 1.5% of rms on the Mixtral-shaped case and
3.3% on the atomic layer, whose outputs reach 12 rms.)  Integer results
(routing indices, group offsets, the permutation) must match exactly.

Routing is checked in two stages:
  A. the oracle's selection code run on the GPU's own logits / sub-key scores
     must reproduce the GPU's indices exactly (same values, same decisions);
  B. against the oracle's fp64 logits: every GPU logit must lie within the
     a-priori fp32 error bound (gamma_n * sum |x_i w_i| for an n-term fp32
     dot product, gamma_n = n u / (1 - n u), u = 2^-24, plus the rounding of
     the bias / residual additions), and a token may differ only if its k-th
     vs (k+1)-th margin is below max(1e-6, twice the measured error of its
     logits), and may list the same experts in another order only if two of
     its selected logits are that close.  Such tokens are counted (and those
     below 1e-6 separately);
     their outputs are compared with the oracle evaluated on the GPU's
     routing (both routings are consistent with the arithmetic).
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import mixture_experts_layer_swiglu_b200 as moe

U32 = 2.0 ** -24
TOL = {"bf16": 2e-2, "f32": 1e-4}


def gamma(n: int) -> float:
    return n * U32 / (1 - n * U32)


def to_device(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device).contiguous() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_gpu(cfg, inp_dev: dict, T: int | None = None) -> dict:
    """All four stages through the C ABI with an fp32 output (the combine's
    fp32 result before its final rounding), then the combine again with the
    layer's own output dtype: that output must be exactly the round-to-
    nearest-even of the fp32 one."""
    desc = moe.desc_from(cfg, T, out_f32=True)
    bufs = moe.StageBuffers(desc)
    moe.run_stages(desc, inp_dev, inp_dev["x"], bufs, prev_logits=inp_dev.get("z_prev"))
    out = {"desc": desc, "bufs": bufs}
    if cfg.dtype == "bf16":
        d16 = moe.desc_from(cfg, T, out_f32=False)
        y16 = torch.empty(bufs.y.shape, dtype=torch.bfloat16, device=bufs.y.device)
        cm = bufs.const_mix if d16.n_const > 0 else None
        moe.moe_combine(d16, inp_dev, bufs.y_sorted, bufs.offsets, bufs.row_of, bufs.idx, bufs.gate, cm,
                        inp_dev["x"], y16)
        torch.cuda.synchronize()
        assert torch.equal(y16, bufs.y.to(torch.bfloat16)), "bf16 output != RNE(fp32 output)"
        out["y16"] = y16
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(reset=True)
    assert status == moe.MOE_OK, moe.status_string(status)
    return out


def run_gpu_fused(cfg, inp_dev: dict, T: int | None = None, gather: bool = False) -> dict:
    """Route, permute, then the fused expert step phase by phase (gate/up
    GEMM reading x_sorted -- or, with `gather`, gathering the token rows from
    x by its own loads, no x_sorted made -- combine in the down GEMM's
    epilogue, the zero-computation terms and the rounding last) with an fp32
    output; then phase 3 again with the layer's bf16 output, which must be
    exactly the round-to-nearest-even of the fp32 one."""
    desc = moe.desc_from(cfg, T, out_f32=True)
    b = moe.StageBuffers(desc)
    assert b.fused_workspace is not None, "the fused expert step does not apply to this layer"
    x = inp_dev["x"]
    cm = b.const_mix if desc.n_const > 0 else None
    moe.moe_route(desc, inp_dev, x, inp_dev.get("z_prev"), b.logits, b.idx, b.gate, cm, b.workspace)
    xs = None if gather else b.x_sorted
    moe.moe_permute(desc, b.idx, x, b.offsets, b.row_of, b.token_of, xs, b.workspace)
    for phase in (1, 2, 3):
        moe.moe_fused_ffn_combine(desc, inp_dev, phase, x, xs, b.idx, b.gate, cm, b.offsets, b.row_of, b.token_of,
                                  b.y, b.fused_workspace)
    d16 = moe.desc_from(cfg, T, out_f32=False)
    y16 = torch.empty(b.y.shape, dtype=torch.bfloat16, device=b.y.device)
    moe.moe_fused_ffn_combine(d16, inp_dev, 3, x, xs, b.idx, b.gate, cm, b.offsets, b.row_of, b.token_of, y16,
                              b.fused_workspace)
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(reset=True)
    assert status == moe.MOE_OK, moe.status_string(status)
    assert torch.equal(y16, b.y.to(torch.bfloat16)), "bf16 output != RNE(fp32 output)"
    return {"desc": desc, "bufs": b, "y16": y16}


def logit_error_bound(cfg, inp: dict, z_abs_max: np.ndarray) -> np.ndarray:
    """Per-token bound of |z_gpu - z_exact| for the SwiGLU router (fp32)."""
    x = inp["x"].double().abs()
    w = inp["w_router"].double().abs()
    S = (x @ w.T).numpy()                                  # sum |x_i w_i| per (t, e)
    e = gamma(cfg.d) * S.max(axis=1) + 3 * U32 * z_abs_max
    return 2.0 * e


def check_swiglu_routing(cfg, inp: dict, gpu_logits: np.ndarray, gpu_idx: np.ndarray,
                         gpu_gate: np.ndarray) -> dict:
    # stage A: oracle selection on the GPU's logits
    idx_a, gate_a, _ = oracle.topk(gpu_logits.astype(np.float64), cfg.top_k)
    np.testing.assert_array_equal(gpu_idx, idx_a, err_msg="stage A: top-k on GPU logits")
    assert np.abs(gpu_gate - gate_a).max() <= 2e-6, "gates vs softmax of the GPU logits"
    # stage B: against fp64 logits
    z = oracle.router_logits(inp["x"], inp["w_router"], inp.get("router_bias"), inp.get("z_prev"))
    idx_b, gate_b, margin = oracle.topk(z, cfg.top_k)
    err_z = np.abs(gpu_logits - z).max(axis=1)
    bound = logit_error_bound(cfg, inp, np.abs(z).max(axis=1))
    assert (err_z <= bound / 2).all(), "GPU logits outside the fp32 error bound"
    vals = np.take_along_axis(z, idx_b.astype(np.int64), axis=1)
    return _stage_b(gpu_idx, idx_b, margin, vals, 2.0 * err_z) | {"z": z, "idx_oracle": idx_b}


def _stage_b(gpu_idx, idx_ref, margin, vals_ref, err2) -> dict:
    """Routing of every token against the fp64 routing.  A token may select a
    different set only if its boundary margin (k-th vs (k+1)-th) is below
    twice the measured error of the values compared (or 1e-6); it may list the
    same set in a different order only if two of its selected values (fp64,
    in the oracle's order `vals_ref`) are that close.  Both orders are then
    consistent with the arithmetic.  Counts are returned for the report."""
    tol = np.maximum(1e-6, err2)
    same_set = (np.sort(gpu_idx, axis=1) == np.sort(idx_ref, axis=1)).all(axis=1)
    same_order = (gpu_idx == idx_ref).all(axis=1)
    set_mis = np.where(~same_set)[0]
    ord_mis = np.where(same_set & ~same_order)[0]
    gap = np.abs(np.diff(vals_ref, axis=1)).min(axis=1) if vals_ref.shape[1] > 1 else np.full(len(margin), np.inf)
    bad_set = [t for t in set_mis if not margin[t] < tol[t]]
    bad_ord = [t for t in ord_mis if not gap[t] < tol[t]]
    assert not bad_set, f"selected set differs on clear-margin tokens {bad_set[:10]}: margins {margin[bad_set[:10]]}"
    assert not bad_ord, f"selection order differs on tokens without a near tie {bad_ord[:10]}: gaps {gap[bad_ord[:10]]}"
    mism = np.where(~same_order)[0]
    return {"mismatch": mism, "set_mismatch": set_mis, "order_mismatch": ord_mis,
            "near_tie": np.where(margin < tol)[0], "below_1e-6": int((margin < 1e-6).sum()),
            "mismatch_margins": margin[set_mis]}


def check_permutation(cfg, gpu_idx: np.ndarray, offsets: np.ndarray, row_of: np.ndarray,
                      token_of: np.ndarray, n_grouped: int, n_ids: int, n_shared: int = 0,
                      T: int = 0) -> int:
    counts, off, row_o, tok_o, slot_o = oracle.group_tasks(gpu_idx, n_grouped, n_ids)
    R = int(off[-1])
    np.testing.assert_array_equal(offsets[:n_grouped + 1], off, err_msg="group offsets")
    np.testing.assert_array_equal(row_of, row_o, err_msg="row_of")
    np.testing.assert_array_equal(token_of[:R], tok_o, err_msg="token_of")
    for s in range(n_shared):   # shared groups: every token, in order
        assert offsets[n_grouped + 1 + s] == R + (s + 1) * T
        np.testing.assert_array_equal(token_of[R + s * T:R + (s + 1) * T], np.arange(T))
    return R


def assert_close(y_gpu: np.ndarray, y_ref: np.ndarray, dtype: str, what: str = "y") -> float:
    rms = math.sqrt(float((y_ref ** 2).mean()))
    err = float(np.abs(y_gpu - y_ref).max())
    assert err <= TOL[dtype] * rms, f"{what}: max|err| {err:.3e} > {TOL[dtype]} * rms {rms:.3e}"
    return err / rms


def check_swiglu_layer(cfg, inp: dict, tokens=None, check_sorted: bool = True, fused: bool = False,
                       gather: bool = False) -> dict:
    """Full check of a SwiGLU-kind layer; `tokens` limits the output comparison;
    `fused` runs the fused expert step (`gather`: with its own row gather, no
    x_sorted to check)."""
    dev = to_device(inp)
    r = run_gpu_fused(cfg, dev, gather=gather) if fused else run_gpu(cfg, dev)
    check_sorted = check_sorted and not (fused and gather)
    b = r["bufs"]
    T = cfg.T
    logits = b.logits.cpu().numpy().astype(np.float64)
    idx = b.idx.cpu().numpy()
    gate = b.gate.cpu().numpy().astype(np.float64)
    rep = check_swiglu_routing(cfg, inp, logits, idx, gate)
    n_ids = cfg.n_routed
    R = check_permutation(cfg, idx, b.offsets.cpu().numpy(), b.row_of.cpu().numpy(),
                          b.token_of.cpu().numpy(), cfg.n_ffn, n_ids, cfg.n_shared, T)
    total = R + cfg.n_shared * T
    fp8 = getattr(cfg, "expert_fp8", False)
    if check_sorted and total and fp8:
        # e4m3 codes and power-of-two scales of the permuted rows: bit-exact with
        # the oracle's quantization of the same rows (a power-of-two division is exact)
        cap = b.y_sorted.shape[0]
        off = (cap * cfg.d + 255) // 256 * 256
        codes = b.x_sorted[:total * cfg.d].view(total, cfg.d).cpu()
        scales = b.x_sorted[off:off + cap * 4].view(torch.float32)[:total].cpu().double().numpy()
        q_ref, s_ref = oracle.quantize_rows(inp["x"][b.token_of[:total].long().cpu()])
        np.testing.assert_array_equal(scales, s_ref, err_msg="x_sorted row scales")
        np.testing.assert_array_equal(codes.view(torch.float8_e4m3fn).double().numpy(), q_ref,
                                      err_msg="x_sorted e4m3 codes")
    elif check_sorted and total:
        tok = b.token_of[:total].long()
        assert torch.equal(b.x_sorted[:total], dev["x"][tok]), "x_sorted rows"
    if cfg.n_const:
        a_ref = oracle.const_mix(inp["x"], inp["w_const_mix"])
        assert np.abs(b.const_mix.cpu().numpy() - a_ref).max() <= 1e-5
    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, dtype=np.int32)
    y_gpu = b.y.float().cpu().numpy()[tokens].astype(np.float64)
    layer_ref = oracle.fp8_moe_tokens if fp8 else oracle.moe_tokens
    y_ref, _, _, _ = layer_ref(cfg, inp, tokens, idx_in=idx[tokens])
    rel = assert_close(y_gpu, y_ref, cfg.dtype)
    rep.update(rel_err=rel, R=R, n_tokens=len(tokens), rel_err_out=_out_err(r, tokens, y_ref))
    return rep


def _out_err(r, tokens, y_ref) -> float:
    """max |y_out - y_ref| / rms(y_ref) of the dtype output (reported)."""
    y = r.get("y16", r["bufs"].y)
    yo = y.float().cpu().numpy()[tokens].astype(np.float64)
    return float(np.abs(yo - y_ref).max() / np.sqrt((y_ref ** 2).mean()))


# ------------------------------------------------------------- atomic kind

def pk_error_bound(inp: dict, q: np.ndarray) -> np.ndarray:
    """Per-token bound of the fp32 error of the sub-key scores (each half)."""
    x = inp["x"].double().abs()
    wq = inp["w_query"].double().abs()
    d = x.shape[1]
    dq = wq.shape[0]
    dq_err = gamma(d) * (x @ wq.T).numpy() + 2.0 ** -23 * np.abs(q)   # q accumulation + split
    h = dq // 2
    kr = inp["subkeys_row"].double().abs().numpy()
    kc = inp["subkeys_col"].double().abs().numpy()
    er = gamma(h) * (np.abs(q[:, :h]) @ kr.T) + dq_err[:, :h] @ kr.T
    ec = gamma(h) * (np.abs(q[:, h:]) @ kc.T) + dq_err[:, h:] @ kc.T
    return np.stack([er.max(axis=1), ec.max(axis=1)], axis=1)


def check_atomic_layer(cfg, inp: dict, tokens=None) -> dict:
    dev = to_device(inp)
    r = run_gpu(cfg, dev)
    b = r["bufs"]
    T, K, rows = cfg.T, cfg.top_k, cfg.pk_rows
    sc_gpu = b.logits.cpu().numpy().astype(np.float64)
    sr_g, sc_g = sc_gpu[:, :rows], sc_gpu[:, rows:]
    idx = b.idx.cpu().numpy()
    gate = b.gate.cpu().numpy().astype(np.float64)
    # stage A
    idx_a, gate_a, _ = oracle.pk_select(sr_g, sc_g, cfg.pk_topk_half, K)
    np.testing.assert_array_equal(idx, idx_a, err_msg="stage A: product-key selection on GPU scores")
    assert np.abs(gate - gate_a).max() <= 2e-6
    # stage B
    sr, sc, q = oracle.pk_scores(inp["x"], inp["w_query"], inp["subkeys_row"], inp["subkeys_col"], want_q=True)
    eb = pk_error_bound(inp, q)
    assert (np.abs(sr_g - sr).max(axis=1) <= eb[:, 0]).all(), "row scores outside the error bound"
    assert (np.abs(sc_g - sc).max(axis=1) <= eb[:, 1]).all(), "column scores outside the error bound"
    idx_b, gate_b, mg = oracle.pk_select(sr, sc, cfg.pk_topk_half, K)
    e_r, e_c = np.abs(sr_g - sr).max(axis=1), np.abs(sc_g - sc).max(axis=1)
    cols = cfg.pk_cols
    tt = np.arange(T)[:, None]
    vals = sr[tt, idx_b // cols] + sc[tt, idx_b % cols]
    rep = _stage_b(idx, idx_b, mg.min(axis=1), vals, 2.0 * (e_r + e_c))
    # task order
    N = cfg.n_atomic
    counts, off, row_o, tok_o, slot_o = oracle.group_tasks(idx, N, N)
    np.testing.assert_array_equal(b.offsets.cpu().numpy(), off, err_msg="atomic offsets")
    flat_slot = tok_o.astype(np.int64) * K + slot_o
    np.testing.assert_array_equal(b.token_of.cpu().numpy()[:len(flat_slot)], flat_slot, err_msg="task order")
    np.testing.assert_array_equal(b.row_of.cpu().numpy(), row_o, err_msg="atomic row_of")
    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, dtype=np.int32)
    # outputs: oracle on the GPU's routing with gates from the fp64 scores of those experts
    g_ref = _pk_gates_for(sr, sc, idx[tokens], tokens, cfg.pk_cols)
    shared = {k_: inp[k_] for k_ in ("ws_gate", "ws_up", "ws_down")} if cfg.n_shared else None
    y_ref = oracle.atomic_tokens(inp["x"], inp["u"], inp["v"], tokens, idx[tokens], g_ref, shared=shared)
    y_gpu = b.y.float().cpu().numpy()[tokens].astype(np.float64)
    rel = assert_close(y_gpu, y_ref, "bf16")
    return rep | {"rel_err": rel, "rel_err_out": _out_err(r, tokens, y_ref)}


def _pk_gates_for(sr, sc, idx, tokens, cols):
    s = sr[tokens[:, None], idx // cols] + sc[tokens[:, None], idx % cols]
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)
