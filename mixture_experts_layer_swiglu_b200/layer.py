"""Convenience wrappers over the C ABI: descriptors, buffer sets, a layer object.

Allocation of device buffers is done here with torch (the library itself
allocates nothing); every computation is a call into libmoe.so.
"""

from __future__ import annotations

import torch

from . import _abi as abi

_DT = {"f32": abi.MOE_F32, "bf16": abi.MOE_BF16, torch.float32: abi.MOE_F32, torch.bfloat16: abi.MOE_BF16}
_TORCH_DT = {abi.MOE_F32: torch.float32, abi.MOE_BF16: torch.bfloat16}


def make_desc(T: int, d_model: int, top_k: int, dtype="bf16", kind: str = "swiglu", n_ffn: int = 0,
              hidden: int = 0, n_shared: int = 0, hidden_shared: int = 0, n_zero: int = 0, n_copy: int = 0,
              n_const: int = 0, pk_rows: int = 0, pk_cols: int = 0, pk_topk_half: int = 0,
              d_query: int = 0, out_f32: bool = False, expert_fp8: bool = False) -> abi.MoELayerDesc:
    return abi.MoELayerDesc(
        T=T, d_model=d_model, top_k=top_k, dtype=_DT[dtype],
        kind=abi.MOE_EXPERT_SWIGLU if kind == "swiglu" else abi.MOE_EXPERT_ATOMIC_GELU,
        n_ffn=n_ffn, hidden=hidden, n_shared=n_shared, hidden_shared=hidden_shared, n_zero=n_zero,
        n_copy=n_copy, n_const=n_const, pk_rows=pk_rows, pk_cols=pk_cols, pk_topk_half=pk_topk_half,
        d_query=d_query, out_f32=int(bool(out_f32)), expert_fp8=int(bool(expert_fp8)))


def desc_from(cfg, T: int | None = None, out_f32: bool = False) -> abi.MoELayerDesc:
    """Descriptor from any object with the workload fields (T, d, top_k, ...)."""
    g = lambda n: getattr(cfg, n, 0) or 0  # noqa: E731
    return make_desc(T=cfg.T if T is None else T, d_model=cfg.d, top_k=cfg.top_k, dtype=cfg.dtype,
                     kind=cfg.kind, n_ffn=g("n_ffn"), hidden=g("hidden"), n_shared=g("n_shared"),
                     hidden_shared=g("hidden_shared"), n_zero=g("n_zero"), n_copy=g("n_copy"),
                     n_const=g("n_const"), pk_rows=g("pk_rows"), pk_cols=g("pk_cols"),
                     pk_topk_half=g("pk_topk_half"), d_query=g("d_query"), out_f32=out_f32,
                     expert_fp8=bool(g("expert_fp8")))


def torch_dtype(desc: abi.MoELayerDesc) -> torch.dtype:
    return _TORCH_DT[desc.dtype]


def out_dtype(desc: abi.MoELayerDesc) -> torch.dtype:
    return torch.float32 if desc.out_f32 else _TORCH_DT[desc.dtype]


def router_width(desc: abi.MoELayerDesc) -> int:
    if desc.kind == abi.MOE_EXPERT_SWIGLU:
        return desc.n_ffn + desc.n_zero + desc.n_copy + desc.n_const
    return desc.pk_rows + desc.pk_cols


class StageBuffers:
    """Device buffers for running the four stages one call at a time."""

    def __init__(self, desc: abi.MoELayerDesc, device="cuda"):
        T, k, d = desc.T, desc.top_k, desc.d_model
        cap = abi.moe_row_capacity(desc)
        groups = abi.moe_num_groups(desc)
        if cap < 0 or groups < 0:
            raise abi.MoEError("moe_row_capacity", abi.MOE_ERR_INVALID_ARG)
        i32, f32 = torch.int32, torch.float32
        dt = torch_dtype(desc)
        self.logits = torch.empty((T, router_width(desc)), dtype=f32, device=device)
        self.idx = torch.empty((T, k), dtype=i32, device=device)
        self.gate = torch.empty((T, k), dtype=f32, device=device)
        self.const_mix = torch.empty((T, max(desc.n_const, 0), 2), dtype=f32, device=device)
        self.offsets = torch.empty((groups + 1,), dtype=i32, device=device)
        self.row_of = torch.empty((T, k), dtype=i32, device=device)
        self.token_of = torch.empty((max(cap, 1),), dtype=i32, device=device)
        if desc.kind == abi.MOE_EXPERT_SWIGLU and desc.expert_fp8:
            # the rows' e4m3 codes, then (at a 256-byte boundary) their fp32 scales
            codes = (max(cap, 1) * d + 255) // 256 * 256
            self.x_sorted = torch.empty((codes + max(cap, 1) * 4,), dtype=torch.uint8, device=device)
            self.y_sorted = torch.empty((max(cap, 1), d), dtype=f32, device=device)
        elif desc.kind == abi.MOE_EXPERT_SWIGLU:
            self.x_sorted = torch.empty((max(cap, 1), d), dtype=dt, device=device)
            self.y_sorted = torch.empty((max(cap, 1), d), dtype=f32, device=device)
        else:
            self.x_sorted = None
            # c [T*k] fp32, then (full OmniMoE layer) the shared branch's [T, d] fp32 at a 256-byte boundary
            c_floats = (T * k * 4 + 255) // 256 * 64
            self.y_sorted = torch.empty((max(c_floats + desc.n_shared * T * d, 1),), dtype=f32, device=device)
        self.workspace = torch.empty((abi.moe_workspace_size(desc),), dtype=torch.uint8, device=device)
        fw = abi.moe_fused_workspace_size(desc)        # -1: the fused expert step does not apply
        self.fused_workspace = torch.empty((fw,), dtype=torch.uint8, device=device) if fw > 0 else None
        self.y = torch.empty((T, d), dtype=out_dtype(desc), device=device)


def run_stages(desc, weights, x, bufs: StageBuffers, prev_logits=None, stream=None, want_logits=True):
    """moe_route -> moe_permute -> moe_grouped_ffn -> moe_combine into bufs.y."""
    b = bufs
    ws = abi.weights_struct(weights)
    cm = b.const_mix if desc.n_const > 0 else None
    abi.moe_route(desc, ws, x, prev_logits, b.logits if want_logits else None, b.idx, b.gate, cm,
                  b.workspace, stream)
    abi.moe_permute(desc, b.idx, x, b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace, stream)
    abi.moe_grouped_ffn(desc, ws, b.x_sorted, b.offsets, b.token_of, x, b.gate, b.y_sorted, b.workspace,
                        stream)
    abi.moe_combine(desc, ws, b.y_sorted, b.offsets, b.row_of, b.idx, b.gate, cm, x, b.y, stream)
    return b.y


def _check_2d(name: str, t, rows: int, cols: int, dtype) -> None:
    if t is None:
        return
    if t.dim() != 2 or tuple(t.shape) != (rows, cols) or t.dtype != dtype:
        raise ValueError(f"{name}: expected a [{rows}, {cols}] {dtype} tensor, got {list(t.shape)} {t.dtype}")


class MoELayer:
    """One MoE FFN layer with device-resident weights; forward() = moe_layer_forward."""

    def __init__(self, desc: abi.MoELayerDesc, weights: dict):
        self.desc = desc
        self.weights = weights                       # keeps the tensors alive
        self._ws_struct = abi.weights_struct(weights)
        self._workspace = None

    def workspace(self, device) -> torch.Tensor:
        need = abi.moe_layer_workspace_size(self.desc)
        if need < 0:
            raise abi.MoEError("moe_layer_workspace_size", abi.MOE_ERR_INVALID_ARG)
        if self._workspace is None or self._workspace.numel() < need or self._workspace.device != device:
            self._workspace = torch.empty((need,), dtype=torch.uint8, device=device)
        return self._workspace

    def _check_io(self, x, prev_logits=None, logits_out=None, y=None) -> None:
        """The library reads and writes these through raw pointers sized by the
        descriptor, so their shapes and dtypes must be the descriptor's."""
        d = self.desc
        _check_2d("x", x, d.T, d.d_model, torch_dtype(d))
        _check_2d("y", y, d.T, d.d_model, out_dtype(d))
        if prev_logits is not None and d.kind != abi.MOE_EXPERT_SWIGLU:
            raise ValueError("prev_logits: the gating residual belongs to the SwiGLU kind")
        _check_2d("prev_logits", prev_logits, d.T, router_width(d), torch.float32)
        _check_2d("logits_out", logits_out, d.T, router_width(d), torch.float32)

    def forward(self, x: torch.Tensor, prev_logits=None, logits_out=None, y=None, stream=None):
        self._check_io(x, prev_logits, logits_out, y)
        if y is None:
            y = torch.empty(x.shape, dtype=out_dtype(self.desc), device=x.device)
        abi.moe_layer_forward(self.desc, self._ws_struct, x, prev_logits, y, logits_out,
                              self.workspace(x.device), stream)
        return y

    def forward_host(self, x_host: torch.Tensor, prev_logits=None, y_host=None, chunks: int = 0, stream=None,
                     device=None):
        """moe_layer_forward_host: x from host memory, y to host memory, the
        copies pipelined against the layer in token ranges.  Returns y_host
        (complete once `stream` reaches this point)."""
        self._check_io(x_host, prev_logits, None, y_host)
        device = torch.device(device or "cuda")
        if y_host is None:
            y_host = torch.empty(x_host.shape, dtype=out_dtype(self.desc), pin_memory=True)
        need = abi.moe_layer_host_workspace_size(self.desc, chunks)
        if need < 0:
            raise abi.MoEError("moe_layer_host_workspace_size", abi.MOE_ERR_INVALID_ARG)
        if getattr(self, "_host_ws", None) is None or self._host_ws.numel() < need or self._host_ws.device != device:
            self._host_ws = torch.empty((need,), dtype=torch.uint8, device=device)
        abi.moe_layer_forward_host(self.desc, self._ws_struct, x_host, prev_logits, y_host, chunks, self._host_ws,
                                   stream)
        return y_host

    __call__ = forward
