"""The five MoE layer workloads, named by what they are.

Every workload is one forward pass of one top-k routed MoE FFN layer.  The
shapes and distributions follow the workloads the pages study:

* ``tiny_f32``      : fp32 layer, T=64, d=128, 8 SwiGLU experts (H=256), top-2.
* ``mixtral``       : Mixtral-shaped bf16 layer, T=4096, d=4096, 8 experts
                      (H=14336), top-2, near-balanced load.
* ``longtail``      : fine-grained bf16 layer, T=2048, d=2048, 64 routed experts
                      (H=1408) at top-6 plus 2 always-on shared experts, with a
                      per-expert router bias giving a Zipf(1.2) long-tail load
                      (FSE-DP page, Fig. 2: long-tail tokens per expert).
* ``moepp``         : MoE++ heterogeneous bf16 layer, T=16384, d=2048, 16 FFN
                      experts (H=5632) + 1 zero, 1 copy, 2 constant experts,
                      top-2, gating residual from a previous layer's logits, a
                      bias giving ~25% of slots to zero-computation experts
                      (MoE++ page, "Approach").
* ``atomic``        : OmniMoE atomic experts, T=8192, d=1024, N=512x512 vector
                      experts, Cartesian-product router with top-32 per half and
                      top-64 overall (OmniMoE page, 2.1 and 2.2).
* ``omnimoe``       : the full OmniMoE layer: the ``atomic`` workload plus the
                      shared dense branch every token passes through (OmniMoE
                      page, 2.1 "Shared Dense MLP"), a SwiGLU FFN of hidden
                      width 2816 (8/3 d rounded up to a multiple of 128; the
                      page gives no size).
* ``mixtral_fp8``, ``longtail_fp8``, ``moepp_fp8``: the same layers with FP8
                      experts (PCoMoE page, "Improvements", 3: FP8 for the
                      expert computation, BF16 for the gating): each expert
                      weight row stored as e4m3 codes with an fp32 scale.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                     # tokens
    d: int                     # d_model
    top_k: int                 # k experts per token (atomic: K of the product router)
    dtype: str                 # "f32" or "bf16": x, weights and y
    kind: str = "swiglu"       # "swiglu" or "atomic"
    n_ffn: int = 0             # routed SwiGLU experts
    hidden: int = 0            # their hidden width H
    n_shared: int = 0          # always-on SwiGLU experts (weight 1)
    hidden_shared: int = 0
    n_zero: int = 0            # MoE++ zero-computation experts, ids follow the FFN ids
    n_copy: int = 0
    n_const: int = 0
    x_std: float = 1.0
    router_bias: str | None = None   # None, "zipf" (longtail) or "zc" (moepp)
    gating_residual: bool = False    # previous layer's logits added to this layer's
    # atomic experts with a Cartesian-product router
    pk_rows: int = 0
    pk_cols: int = 0
    pk_topk_half: int = 0
    d_query: int = 0
    expert_fp8: bool = False         # expert weights stored as e4m3 codes + fp32 row scales

    @property
    def n_routed(self) -> int:
        """Router rows: FFN experts then zero, copy and constant experts."""
        return self.n_ffn + self.n_zero + self.n_copy + self.n_const

    @property
    def n_atomic(self) -> int:
        return self.pk_rows * self.pk_cols

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


CONFIGS: dict[str, MoEConfig] = {
    "tiny_f32": MoEConfig(
        name="tiny_f32", T=64, d=128, top_k=2, dtype="f32",
        n_ffn=8, hidden=256, x_std=128 ** -0.5),
    "mixtral": MoEConfig(
        name="mixtral", T=4096, d=4096, top_k=2, dtype="bf16",
        n_ffn=8, hidden=14336),
    "longtail": MoEConfig(
        name="longtail", T=2048, d=2048, top_k=6, dtype="bf16",
        n_ffn=64, hidden=1408, n_shared=2, hidden_shared=1408,
        router_bias="zipf"),
    "moepp": MoEConfig(
        name="moepp", T=16384, d=2048, top_k=2, dtype="bf16",
        n_ffn=16, hidden=5632, n_zero=1, n_copy=1, n_const=2,
        router_bias="zc", gating_residual=True),
    "atomic": MoEConfig(
        name="atomic", T=8192, d=1024, top_k=64, dtype="bf16", kind="atomic",
        pk_rows=512, pk_cols=512, pk_topk_half=32, d_query=1024),
    "omnimoe": MoEConfig(
        name="omnimoe", T=8192, d=1024, top_k=64, dtype="bf16", kind="atomic",
        pk_rows=512, pk_cols=512, pk_topk_half=32, d_query=1024, n_shared=1, hidden_shared=2816),
}
for _base in ("mixtral", "longtail", "moepp"):
    CONFIGS[_base + "_fp8"] = dataclasses.replace(CONFIGS[_base], name=_base + "_fp8", expert_fp8=True)

ORDER = ["tiny_f32", "mixtral", "longtail", "moepp", "atomic", "omnimoe", "mixtral_fp8", "longtail_fp8",
         "moepp_fp8"]


def get_config(name: str) -> MoEConfig:
    return CONFIGS[name]


def scaled(cfg: MoEConfig, **changes) -> MoEConfig:
    """A copy of ``cfg`` with some fields changed (e.g. fewer tokens)."""
    return dataclasses.replace(cfg, **changes)
