"""ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
CUDA tensors (or None for a NULL pointer).  Nothing here computes any part of
the layer; if the library cannot be loaded the import fails.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libmoe.so"

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_DEVICE_BOUNDS, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_F32, MOE_BF16 = 0, 1
MOE_EXPERT_SWIGLU, MOE_EXPERT_ATOMIC_GELU = 0, 1

EXPORTED = ("moe_num_groups", "moe_row_capacity", "moe_workspace_size", "moe_layer_workspace_size",
            "moe_route", "moe_permute", "moe_grouped_ffn", "moe_grouped_ffn_phase", "moe_combine",
            "moe_layer_forward", "moe_get_device_status", "moe_status_string",
            "moe_last_launch_count", "moe_permute_static", "moe_selftest_wait_timeout",
            "moe_layer_host_workspace_size", "moe_layer_forward_host", "moe_ep_expert_range", "moe_ep_owner",
            "moe_ep_plan", "moe_fused_workspace_size", "moe_fused_ffn_combine")


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class MoELayerDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "d_model", "top_k", "dtype", "kind", "n_ffn", "hidden", "n_shared", "hidden_shared",
        "n_zero", "n_copy", "n_const", "pk_rows", "pk_cols", "pk_topk_half", "d_query", "out_f32", "expert_fp8")]


class MoELayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_router", "router_bias", "w_const_mix", "const_vec", "w_gate", "w_up", "w_down",
        "ws_gate", "ws_up", "ws_down", "w_query", "subkeys_row", "subkeys_col", "u", "v",
        "s_gate", "s_up", "s_down", "ss_gate", "ss_up", "ss_down")]


_lib = None


def load(path: Path | str | None = None):
    """Load libmoe.so (building it in-tree with nvcc first if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    p = Path(path) if path else LIB_PATH
    if not p.exists():
        from . import build as _build
        _build.build()
    L = ctypes.CDLL(str(p))
    P, VP, I32, I64, SZ = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    D, W = P(MoELayerDesc), P(MoELayerWeights)
    for name in ("moe_num_groups", "moe_row_capacity", "moe_workspace_size", "moe_layer_workspace_size"):
        getattr(L, name).argtypes = [D]
        getattr(L, name).restype = I64
    L.moe_route.argtypes = [D, W, VP, VP, VP, VP, VP, VP, VP, SZ, VP]
    L.moe_permute.argtypes = [D, VP, VP, VP, VP, VP, VP, VP, SZ, VP]
    L.moe_permute_static.argtypes = [D, VP, VP, VP, VP, VP, VP, VP]
    L.moe_selftest_wait_timeout.argtypes = [ctypes.c_uint64, VP, VP]
    L.moe_grouped_ffn.argtypes = [D, W, VP, VP, VP, VP, VP, VP, VP, SZ, VP]
    L.moe_grouped_ffn_phase.argtypes = [D, W, ctypes.c_int, VP, VP, VP, VP, SZ, VP]
    L.moe_combine.argtypes = [D, W, VP, VP, VP, VP, VP, VP, VP, VP, VP]
    L.moe_layer_forward.argtypes = [D, W, VP, VP, VP, VP, VP, SZ, VP]
    L.moe_fused_workspace_size.argtypes = [D]
    L.moe_fused_workspace_size.restype = I64
    L.moe_fused_ffn_combine.argtypes = [D, W, ctypes.c_int, VP, VP, VP, VP, VP, VP, VP, VP, VP, VP, SZ, VP]
    L.moe_layer_host_workspace_size.argtypes = [D, ctypes.c_int]
    L.moe_layer_host_workspace_size.restype = I64
    L.moe_layer_forward_host.argtypes = [D, W, VP, VP, VP, ctypes.c_int, VP, SZ, VP]
    L.moe_get_device_status.argtypes = [P(ctypes.c_int), ctypes.c_int, VP]
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_last_launch_count.restype = I32
    L.moe_ep_expert_range.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P(I32), P(I32)]
    L.moe_ep_expert_range.restype = ctypes.c_int
    L.moe_ep_owner.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    L.moe_ep_owner.restype = I32
    L.moe_ep_plan.argtypes = [VP, ctypes.c_int, ctypes.c_int, ctypes.c_int, VP, VP, VP]
    L.moe_ep_plan.restype = I64
    for name in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_grouped_ffn_phase", "moe_combine",
                 "moe_layer_forward", "moe_get_device_status", "moe_permute_static", "moe_fused_ffn_combine",
                 "moe_selftest_wait_timeout", "moe_layer_forward_host"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def _p(t):
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libmoe takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return t.data_ptr()


def _hp(t):
    """Host pointer of a CPU tensor (None -> NULL); page-locked memory lets the copies overlap."""
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("moe_layer_forward_host takes host tensors")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return t.data_ptr()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoEError(fn, status)


def weights_struct(w: dict) -> MoELayerWeights:
    """MoELayerWeights from a dict of device tensors (missing keys -> NULL)."""
    s = MoELayerWeights()
    for name, _ in MoELayerWeights._fields_:
        setattr(s, name, _p(w.get(name)))
    return s


# ------------------------------------------------------------ entry points

def moe_num_groups(desc: MoELayerDesc) -> int:
    return int(load().moe_num_groups(ctypes.byref(desc)))


def moe_row_capacity(desc: MoELayerDesc) -> int:
    return int(load().moe_row_capacity(ctypes.byref(desc)))


def moe_workspace_size(desc: MoELayerDesc) -> int:
    return int(load().moe_workspace_size(ctypes.byref(desc)))


def moe_layer_workspace_size(desc: MoELayerDesc) -> int:
    return int(load().moe_layer_workspace_size(ctypes.byref(desc)))


def moe_route(desc, weights, x, prev_logits, logits_out, topk_idx, topk_gate, const_mix, workspace,
              stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_route", load().moe_route(ctypes.byref(desc), ctypes.byref(ws), _p(x), _p(prev_logits),
                                         _p(logits_out), _p(topk_idx), _p(topk_gate), _p(const_mix),
                                         _p(workspace), _nbytes(workspace), _stream(stream)))


def moe_permute(desc, topk_idx, x, expert_offsets, row_of, token_of, x_sorted, workspace,
                stream=None) -> None:
    _check("moe_permute", load().moe_permute(ctypes.byref(desc), _p(topk_idx), _p(x), _p(expert_offsets),
                                             _p(row_of), _p(token_of), _p(x_sorted), _p(workspace),
                                             _nbytes(workspace), _stream(stream)))


def moe_permute_static(desc, topk_idx, x, expert_offsets, row_of, token_of, x_sorted, stream=None) -> None:
    """moe_permute without a workspace (its scratch is a fixed array inside the library)."""
    _check("moe_permute_static", load().moe_permute_static(ctypes.byref(desc), _p(topk_idx), _p(x),
                                                           _p(expert_offsets), _p(row_of), _p(token_of),
                                                           _p(x_sorted), _stream(stream)))


def moe_grouped_ffn(desc, weights, x_sorted, expert_offsets, token_of, x, topk_gate, y_sorted, workspace,
                    stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_grouped_ffn", load().moe_grouped_ffn(ctypes.byref(desc), ctypes.byref(ws), _p(x_sorted),
                                                     _p(expert_offsets), _p(token_of), _p(x), _p(topk_gate),
                                                     _p(y_sorted), _p(workspace), _nbytes(workspace),
                                                     _stream(stream)))


def moe_grouped_ffn_phase(desc, weights, phase, x_sorted, expert_offsets, y_sorted, workspace,
                          stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_grouped_ffn_phase",
           load().moe_grouped_ffn_phase(ctypes.byref(desc), ctypes.byref(ws), int(phase), _p(x_sorted),
                                        _p(expert_offsets), _p(y_sorted), _p(workspace), _nbytes(workspace),
                                        _stream(stream)))


def moe_combine(desc, weights, y_sorted, expert_offsets, row_of, topk_idx, topk_gate, const_mix, x, y,
                stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_combine", load().moe_combine(ctypes.byref(desc), ctypes.byref(ws), _p(y_sorted),
                                             _p(expert_offsets), _p(row_of), _p(topk_idx), _p(topk_gate),
                                             _p(const_mix), _p(x), _p(y), _stream(stream)))


def moe_layer_forward(desc, weights, x, prev_logits, y, logits_out, workspace, stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_layer_forward", load().moe_layer_forward(ctypes.byref(desc), ctypes.byref(ws), _p(x),
                                                         _p(prev_logits), _p(y), _p(logits_out),
                                                         _p(workspace), _nbytes(workspace), _stream(stream)))


def moe_fused_workspace_size(desc: MoELayerDesc) -> int:
    """Workspace bytes of moe_fused_ffn_combine; -1 if the layer does not qualify."""
    return int(load().moe_fused_workspace_size(ctypes.byref(desc)))


def moe_fused_ffn_combine(desc, weights, phase, x, x_sorted, topk_idx, topk_gate, const_mix, expert_offsets,
                          row_of, token_of, y, workspace, stream=None) -> None:
    """x_sorted None: phase 1 gathers the token rows from x by its own loads."""
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_fused_ffn_combine",
           load().moe_fused_ffn_combine(ctypes.byref(desc), ctypes.byref(ws), int(phase), _p(x), _p(x_sorted),
                                        _p(topk_idx),
                                        _p(topk_gate), _p(const_mix), _p(expert_offsets), _p(row_of), _p(token_of),
                                        _p(y), _p(workspace), _nbytes(workspace), _stream(stream)))


def moe_layer_host_workspace_size(desc: MoELayerDesc, chunks: int = 0) -> int:
    return int(load().moe_layer_host_workspace_size(ctypes.byref(desc), int(chunks)))


def moe_layer_forward_host(desc, weights, x_host, prev_logits_host, y_host, chunks, workspace, stream=None) -> None:
    ws = weights if isinstance(weights, MoELayerWeights) else weights_struct(weights)
    _check("moe_layer_forward_host",
           load().moe_layer_forward_host(ctypes.byref(desc), ctypes.byref(ws), _hp(x_host), _hp(prev_logits_host),
                                         _hp(y_host), int(chunks), _p(workspace), _nbytes(workspace),
                                         _stream(stream)))


def moe_get_device_status(reset: bool = True, stream=None) -> int:
    out = ctypes.c_int(0)
    _check("moe_get_device_status", load().moe_get_device_status(ctypes.byref(out), int(bool(reset)),
                                                                 _stream(stream)))
    return int(out.value)


def moe_selftest_wait_timeout(limit_ns: int, waited_ok, stream=None) -> None:
    """Run the bounded-wait self-test kernel (see include/moe.h)."""
    _check("moe_selftest_wait_timeout", load().moe_selftest_wait_timeout(int(limit_ns), _p(waited_ok),
                                                                         _stream(stream)))


def moe_last_launch_count() -> int:
    return int(load().moe_last_launch_count())


# ------------------------------------------------------ expert parallelism (host)

def moe_ep_expert_range(G: int, E: int, rank: int) -> tuple[int, int]:
    lo, hi = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("moe_ep_expert_range", load().moe_ep_expert_range(int(G), int(E), int(rank), ctypes.byref(lo),
                                                              ctypes.byref(hi)))
    return int(lo.value), int(hi.value)


def moe_ep_owner(G: int, E: int, expert: int) -> int:
    r = int(load().moe_ep_owner(int(G), int(E), int(expert)))
    if r < 0:
        raise MoEError("moe_ep_owner", MOE_ERR_INVALID_ARG)
    return r


def moe_ep_plan(counts, rank: int):
    """counts: host int32 tensor [G, E].  Returns (recv_offsets [n_own, G],
    recv_counts [n_own, G], local_offsets [n_own + 1], rows received)."""
    if counts.is_cuda or counts.dtype != torch.int32 or counts.dim() != 2:
        raise ValueError("moe_ep_plan takes a host int32 [G, E] tensor")
    counts = counts.contiguous()
    G, E = counts.shape
    lo, hi = moe_ep_expert_range(G, E, rank)
    n_own = hi - lo
    ro = torch.zeros((max(n_own, 1), G), dtype=torch.int32)
    rc = torch.zeros((max(n_own, 1), G), dtype=torch.int32)
    lo_off = torch.zeros((n_own + 1,), dtype=torch.int32)
    total = int(load().moe_ep_plan(counts.data_ptr(), G, E, int(rank), ro.data_ptr(), rc.data_ptr(),
                                   lo_off.data_ptr()))
    if total < 0:
        raise MoEError("moe_ep_plan", MOE_ERR_INVALID_ARG)
    return ro[:n_own], rc[:n_own], lo_off, total
