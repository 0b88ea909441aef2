"""Writes the stored router biases of the long-tail and MoE++ workloads.

Uses only the fp64 oracle (router logits and top-k) on the seed-0 inputs.

* longtail_router_bias.txt -- per-expert bias b_e such that the number of
  tokens routed to expert e follows T*k*p_e, p_e proportional to
  (e+1)^-1.2 (Zipf, s = 1.2), capped at T tokens per expert with the excess
  spread over the rest.  The long-tail load itself is the FSE-DP page's
  Fig. 2 (tokens per expert, sorted, form a long tail).  Fit: 400 steps of
  b <- b + 0.3 (ln c_target - ln c_realised).
* moepp_router_bias.txt -- one scalar beta added to the logits of the four
  zero-computation experts (ids 16..19) so that 25% of the top-2 slots go to
  them (MoE++ page, "Approach": zero-computation experts take part in the
  routing; the share is a workload choice).  Bisection on beta.

Run:  python tests/golden/make_router_bias.py
"""

from __future__ import annotations

import sys
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
from moe_workloads import get_config  # noqa: E402
from moe_workloads.gen import make_activations, make_router_weight, zipf_targets  # noqa: E402

HERE = Path(__file__).resolve().parent


def _write(path: Path, header: str, vals) -> None:
    lines = ["# " + l for l in header.strip().splitlines()]
    lines += [repr(float(np.float32(v))) for v in vals]
    path.write_text("\n".join(lines) + "\n")


def fit_longtail():
    cfg = get_config("longtail")
    x = make_activations(cfg)["x"]
    z = oracle.router_logits(x, make_router_weight(cfg))
    target = np.array(zipf_targets(cfg))
    b = np.zeros(cfg.n_ffn)
    for _ in range(400):
        idx, _, _ = oracle.topk(z + b, cfg.top_k)
        c = np.bincount(idx.reshape(-1), minlength=cfg.n_ffn).astype(np.float64)
        b += 0.3 * (np.log(target) - np.log(np.maximum(c, 0.5)))
    b32 = b.astype(np.float32)
    idx, _, _ = oracle.topk(z + b32.astype(np.float64), cfg.top_k)
    c = np.bincount(idx.reshape(-1), minlength=cfg.n_ffn)
    hdr = (f"longtail router bias, {cfg.n_ffn} values (fp32), fitted on seed-0 fp64 logits.\n"
           f"target counts (rounded): {np.rint(target).astype(int).tolist()}\n"
           f"realised counts: {c.tolist()}\n"
           f"max |realised - target| = {np.abs(c - target).max():.1f}")
    _write(HERE / "longtail_router_bias.txt", hdr, b32)
    return c, target


def fit_moepp():
    cfg = get_config("moepp")
    a = make_activations(cfg)
    z = oracle.router_logits(a["x"], make_router_weight(cfg), z_prev=a["z_prev"])
    zc = np.zeros(cfg.n_routed)
    zc[cfg.n_ffn:] = 1.0

    def frac(beta):
        idx, _, _ = oracle.topk(z + beta * zc, cfg.top_k)
        return float((idx >= cfg.n_ffn).mean())

    lo, hi = -4.0, 4.0
    for _ in range(50):
        mid = 0.5 * (lo + hi)
        if frac(mid) < 0.25:
            lo = mid
        else:
            hi = mid
    beta = np.float32(0.5 * (lo + hi))
    f = frac(float(beta))
    hdr = (f"moepp router bias, {cfg.n_routed} values (fp32): 0 on the {cfg.n_ffn} FFN experts,\n"
           f"beta on the zero, copy and two constant experts.  beta = {float(beta)!r}\n"
           f"realised share of top-{cfg.top_k} slots on zero-computation experts: {f:.5f}\n"
           f"(share at beta = 0: {frac(0.0):.5f})")
    _write(HERE / "moepp_router_bias.txt", hdr, [0.0] * cfg.n_ffn + [beta] * 4)
    return f


if __name__ == "__main__":
    c, t = fit_longtail()
    print("longtail realised", c.tolist())
    print("moepp ZC share", fit_moepp())
