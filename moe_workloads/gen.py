"""Seeded synthetic inputs for the MoE layer workloads.

Recipe (the same for the CUDA path and the oracle):

* every tensor has its own CPU ``torch.Generator`` seeded with
  ``(seed << 32) | stream``; large tensors are drawn in row chunks, each chunk
  with its own stream, so a tensor never depends on the shape of another one
  (the weights of a workload are the same whatever its token count T);
* values are drawn as fp32 standard normals times the stated std, then cast
  round-to-nearest-even to bf16 for the bf16 workloads;
* weight std is 1/sqrt(fan_in): fan_in = d for the router, gate, up, constant
  mix and query matrices, H for the down matrices, 1024 for the atomic
  expert vectors u and v; sub-keys and the constant vectors v are N(0, 1);
  x is N(0, x_std^2); the previous layer's logits are N(0, 1) in fp32;
* the long-tail and MoE++ router biases are stored numbers (fp32), fitted by a
  script that uses only the oracle; they are loaded, not computed, here;
* FP8-expert workloads store each expert weight row (drawn as above, in bf16)
  as e4m3 codes of row / s with s = max|row| / 448 (fp32; torch's float8
  cast, nearest) and the row scale s: the stored weight is code * s.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
from pathlib import Path

import torch

from .configs import MoEConfig

GOLDEN_DIR = Path(__file__).resolve().parent.parent / "tests" / "golden"

# stream ids
_X, _WR, _WC, _CV, _ZP, _WQ, _KR, _KC = 1, 2, 3, 4, 5, 6, 7, 8
_U, _V = 1 << 20, 2 << 20
_EXPERT, _SHARED = 3 << 20, 4 << 20
_CHUNK_ROWS = 32768


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((int(seed) << 32) | int(stream))
    return g


def _normal(shape, std: float, seed: int, stream: int, dtype: torch.dtype, out=None) -> torch.Tensor:
    """fp32 N(0, std^2) draw in row chunks, cast to ``dtype`` (written into
    ``out`` when given)."""
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    inner = shape[1:]
    if out is None:
        out = torch.empty(shape, dtype=dtype)
    if rows == 0:
        return out
    buf = None
    for c, r0 in enumerate(range(0, rows, _CHUNK_ROWS)):
        r1 = min(rows, r0 + _CHUNK_ROWS)
        if buf is None or buf.shape[0] != r1 - r0:
            buf = torch.empty((r1 - r0,) + inner, dtype=torch.float32)
        buf.normal_(generator=_gen(seed, stream + c * 65536))
        if std != 1.0:
            buf.mul_(std)
        out[r0:r1].copy_(buf)
    return out


def _fill_parallel(jobs, seed: int, dt: torch.dtype) -> None:
    """Draw independent tensors on a thread pool (each has its own stream, so
    the values do not depend on the order or the number of threads)."""
    def one(job):
        dst, i, shape, std, stream = job
        _normal(shape, std, seed, stream, dt, out=dst[i])

    threads = max(1, min(len(jobs), os.cpu_count() or 1))
    prev = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, jobs))
    finally:
        torch.set_num_threads(prev)


def _to_e4m3_rows(w: torch.Tensor):
    """[..., K] weights -> (e4m3 codes as uint8, fp32 row scales [...])."""
    wf = w.to(torch.float32)
    s = wf.abs().amax(dim=-1) / 448.0
    s = torch.where(s > 0, s, torch.ones_like(s))
    codes = (wf / s.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), s.contiguous()


def _dt(cfg: MoEConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def expert_ids(cfg: MoEConfig) -> dict:
    """Router-row id ranges: FFN experts, then zero, copy, constant experts."""
    z0 = cfg.n_ffn
    c0 = z0 + cfg.n_zero
    k0 = c0 + cfg.n_copy
    return {"ffn": range(0, z0), "zero": range(z0, c0), "copy": range(c0, k0),
            "const": range(k0, k0 + cfg.n_const)}


def load_router_bias(cfg: MoEConfig) -> torch.Tensor | None:
    if cfg.router_bias is None:
        return None
    # an FP8-expert workload has the router (and so the bias) of its bf16 layer
    base = cfg.name[:-len("_fp8")] if cfg.expert_fp8 and cfg.name.endswith("_fp8") else cfg.name
    path = GOLDEN_DIR / f"{base}_router_bias.txt"
    vals = [float(l.split()[0]) for l in path.read_text().splitlines()
            if l.strip() and not l.lstrip().startswith("#")]
    if len(vals) != cfg.n_routed:
        raise ValueError(f"{path}: {len(vals)} values, expected {cfg.n_routed}")
    return torch.tensor(vals, dtype=torch.float32)


def make_router_weight(cfg: MoEConfig, seed: int = 0) -> torch.Tensor:
    """The router matrix W_r [n_routed, d] alone (same draw as in make_weights)."""
    return _normal((cfg.n_routed, cfg.d), cfg.d ** -0.5, seed, _WR, _dt(cfg))


def _shared_jobs(cfg: MoEConfig, w: dict, dt) -> list:
    """Allocate the always-on SwiGLU experts' weights in ``w``; their draws."""
    if not cfg.n_shared:
        return []
    d, S, Hs = cfg.d, cfg.n_shared, cfg.hidden_shared
    sg = torch.empty((S, Hs, d), dtype=dt)
    su = torch.empty((S, Hs, d), dtype=dt)
    sd = torch.empty((S, d, Hs), dtype=dt)
    jobs = []
    for s in range(S):
        base = _SHARED + s * 4 * 64
        jobs += [(sg, s, (Hs, d), d ** -0.5, base + 0), (su, s, (Hs, d), d ** -0.5, base + 64),
                 (sd, s, (d, Hs), Hs ** -0.5, base + 128)]
    w["ws_gate"], w["ws_up"], w["ws_down"] = sg, su, sd
    return jobs


def make_weights(cfg: MoEConfig, seed: int = 0) -> dict:
    dt = _dt(cfg)
    d = cfg.d
    w: dict = {}
    if cfg.kind == "atomic":
        dq = cfg.d_query
        w["w_query"] = _normal((dq, d), d ** -0.5, seed, _WQ, dt)
        w["subkeys_row"] = _normal((cfg.pk_rows, dq // 2), 1.0, seed, _KR, dt)
        w["subkeys_col"] = _normal((cfg.pk_cols, dq // 2), 1.0, seed, _KC, dt)
        w["u"] = torch.empty((cfg.n_atomic, d), dtype=dt)
        w["v"] = torch.empty((cfg.n_atomic, d), dtype=dt)
        # row chunks of u and v drawn in parallel (same streams as a serial draw)
        jobs = []
        for name, stream in (("u", _U), ("v", _V)):
            for c, r0 in enumerate(range(0, cfg.n_atomic, _CHUNK_ROWS)):
                r1 = min(cfg.n_atomic, r0 + _CHUNK_ROWS)
                jobs.append((w[name], slice(r0, r1), (r1 - r0, d), 1024 ** -0.5, stream + c * 65536))
        jobs += _shared_jobs(cfg, w, dt)
        _fill_parallel(jobs, seed, dt)
        return w
    H = cfg.hidden
    w["w_router"] = make_router_weight(cfg, seed)
    w["router_bias"] = load_router_bias(cfg)
    E = cfg.n_ffn
    wg = torch.empty((E, H, d), dtype=dt)
    wu = torch.empty((E, H, d), dtype=dt)
    wd = torch.empty((E, d, H), dtype=dt)
    jobs = []
    for e in range(E):
        base = _EXPERT + e * 4 * 64
        jobs += [(wg, e, (H, d), d ** -0.5, base + 0), (wu, e, (H, d), d ** -0.5, base + 64),
                 (wd, e, (d, H), H ** -0.5, base + 128)]
    jobs += _shared_jobs(cfg, w, dt)
    _fill_parallel(jobs, seed, dt)
    w["w_gate"], w["w_up"], w["w_down"] = wg, wu, wd
    if cfg.n_const:
        w["w_const_mix"] = _normal((cfg.n_const, 2, d), d ** -0.5, seed, _WC, dt)
        w["const_vec"] = _normal((cfg.n_const, d), 1.0, seed, _CV, dt)
    if cfg.expert_fp8:
        for name, sname in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down"),
                            ("ws_gate", "ss_gate"), ("ws_up", "ss_up"), ("ws_down", "ss_down")):
            if name in w:
                w[name], w[sname] = _to_e4m3_rows(w[name])
    return w


def make_activations(cfg: MoEConfig, seed: int = 0) -> dict:
    a = {"x": _normal((cfg.T, cfg.d), cfg.x_std, seed, _X, _dt(cfg))}
    if cfg.gating_residual:
        a["z_prev"] = _normal((cfg.T, cfg.n_routed), 1.0, seed, _ZP, torch.float32)
    return a


def make_inputs(cfg: MoEConfig, seed: int = 0) -> dict:
    out = make_weights(cfg, seed)
    out.update(make_activations(cfg, seed))
    return out


def flops_ffn(cfg: MoEConfig, rows: int) -> float:
    """Multiply-add FLOPs of the SwiGLU experts on ``rows`` expert rows."""
    return 6.0 * rows * cfg.d * cfg.hidden


def zipf_targets(cfg: MoEConfig) -> list:
    """Target tokens per expert for the long-tail workload: T*k*p_e with
    p_e proportional to (e+1)^-1.2, capped at T (one expert takes at most one
    slot per token) and the excess spread proportionally over the rest."""
    E, T, k = cfg.n_ffn, cfg.T, cfg.top_k
    p = [(e + 1) ** -1.2 for e in range(E)]
    total = T * k
    capped = [False] * E
    c = [0.0] * E
    while True:
        free = total - T * sum(capped)
        ps = sum(p[e] for e in range(E) if not capped[e])
        changed = False
        for e in range(E):
            c[e] = float(T) if capped[e] else free * p[e] / ps
            if not capped[e] and c[e] > T:
                capped[e] = True
                changed = True
        if not changed:
            return c

