"""fp64 CPU oracle of the top-k routed MoE FFN layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never calls it.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision, one token
at a time); this module only builds that file with gcc and marshals arrays.
Inputs are CPU torch tensors (fp32 or bf16, read exactly); outputs are numpy
float64 / int32 arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np
import torch

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "moe_oracle.c"
_LIB = _HERE / "liboracle.so"
_lib = None

_F64P = ctypes.POINTER(ctypes.c_double)
_I32P = ctypes.POINTER(ctypes.c_int32)
_VP = ctypes.c_void_p


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
                               "-shared", "-fPIC", "-std=c11", str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("T", "d", "top_k", "dt", "n_ffn", "hidden", "n_shared", "hidden_shared",
                 "n_zero", "n_copy", "n_const")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [ctypes.c_int]
        L.orc_router_logits.argtypes = [ctypes.c_int] * 4 + [_VP, _VP, _VP, _VP, _F64P]
        L.orc_topk.argtypes = [ctypes.c_int] * 3 + [_F64P, _I32P, _F64P, _F64P]
        L.orc_group_tasks.argtypes = [ctypes.c_int, ctypes.c_int, _I32P, ctypes.c_int,
                                      ctypes.c_int, _I32P, _I32P, _I32P, _I32P, _I32P]
        L.orc_group_tasks.restype = ctypes.c_long
        L.orc_moe_tokens.argtypes = [ctypes.POINTER(_Layer)] + [_VP] * 12 + [
            ctypes.c_int, _I32P, _I32P, _F64P, _I32P, _F64P, _F64P]
        L.orc_const_mix.argtypes = [ctypes.c_int] * 4 + [_VP, _VP, _F64P]
        L.orc_pk_scores.argtypes = [ctypes.c_int] * 6 + [_VP] * 4 + [_F64P] * 3
        L.orc_pk_select.argtypes = [ctypes.c_int] * 5 + [_F64P, _F64P, _I32P, _F64P, _F64P]
        L.orc_atomic_tokens.argtypes = [ctypes.c_int] * 3 + [_VP] * 3 + [
            ctypes.c_int, _I32P, _I32P, _F64P, _F64P]
        L.orc_omni_tokens.argtypes = [ctypes.c_int] * 3 + [_VP] * 3 + [ctypes.c_int] * 2 + [_VP] * 3 + [
            ctypes.c_int, _I32P, _I32P, _F64P, _F64P]
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_round.argtypes = [ctypes.c_double]
        L.orc_e4m3_round.restype = ctypes.c_double
        L.orc_pow2_scale.argtypes = [ctypes.c_double]
        L.orc_pow2_scale.restype = ctypes.c_double
        L.orc_quantize_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _VP, _F64P, _F64P]
        L.orc_fp8_moe_tokens.argtypes = [ctypes.POINTER(_Layer)] + [_VP] * 18 + [
            ctypes.c_int, _I32P, _I32P, _F64P, _I32P, _F64P, _F64P]
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().orc_num_threads())


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


# ----------------------------------------------------------------- helpers

def _dt(*ts) -> int:
    dts = {t.dtype for t in ts if t is not None}
    if dts == {torch.float32}:
        return 0
    if dts == {torch.bfloat16}:
        return 1
    raise TypeError(f"oracle inputs must all be fp32 or all bf16, got {dts}")


def _cpu(t):
    if t is None:
        return None
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    return t.contiguous()


def _vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _f64(a):
    return a.ctypes.data_as(_F64P)


def _i32(a):
    return None if a is None else a.ctypes.data_as(_I32P)


def _np_f64(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _np_i32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


# ------------------------------------------------------------------ router

def router_logits(x, w_router, bias=None, z_prev=None) -> np.ndarray:
    """fp64 logits z[t, e] = x_t . W_r[e] (+ bias[e]) (+ z_prev[t, e])."""
    x, w, bias, z_prev = _cpu(x), _cpu(w_router), _cpu(bias), _cpu(z_prev)
    T, d = x.shape
    E = w.shape[0]
    if bias is not None:
        bias = bias.to(torch.float32).contiguous()
    if z_prev is not None:
        z_prev = z_prev.to(torch.float32).contiguous()
    z = np.empty((T, E), np.float64)
    lib().orc_router_logits(T, d, E, _dt(x, w), _vp(x), _vp(w), _vp(bias), _vp(z_prev), _f64(z))
    return z


def topk(z, k: int):
    """Top-k of each row (ties to the lower index), softmax gates over the k,
    and the k-th minus (k+1)-th margin.  Returns (idx int32, gate f64, margin f64)."""
    z = _np_f64(z)
    T, E = z.shape
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float64)
    margin = np.empty((T,), np.float64)
    lib().orc_topk(T, E, k, _f64(z), _i32(idx), _f64(gate), _f64(margin))
    return idx, gate, margin


def group_tasks(idx, n_grouped: int, n_ids: int):
    """Expert-centric task order: (counts, offsets, row_of, token_of, slot_of)."""
    idx = _np_i32(idx)
    T, k = idx.shape
    counts = np.empty((n_grouped,), np.int32)
    offsets = np.empty((n_grouped + 1,), np.int32)
    row_of = np.empty((T, k), np.int32)
    token_of = np.empty((max(1, T * k),), np.int32)
    slot_of = np.empty((max(1, T * k),), np.int32)
    R = lib().orc_group_tasks(T, k, _i32(idx), n_grouped, n_ids, _i32(counts), _i32(offsets),
                              _i32(row_of), _i32(token_of), _i32(slot_of))
    if R < 0:
        raise ValueError("expert id out of range")
    return counts, offsets, row_of, token_of[:R].copy(), slot_of[:R].copy()


def const_mix(x, w_const_mix) -> np.ndarray:
    x, wc = _cpu(x), _cpu(w_const_mix)
    T, d = x.shape
    C = wc.shape[0]
    a = np.empty((T, C, 2), np.float64)
    lib().orc_const_mix(T, d, C, _dt(x, wc), _vp(x), _vp(wc), _f64(a))
    return a


def moe_tokens(cfg, inp: dict, tokens, idx_in=None):
    """Layer output y (fp64) for the listed tokens of a SwiGLU-kind workload.

    ``cfg`` carries the sizes (a MoEConfig); ``inp`` the tensors produced by
    the workload generator.  Returns (y [n, d], idx [n, k], gate [n, k],
    margin [n])."""
    tokens = _np_i32(tokens).reshape(-1)
    n = tokens.shape[0]
    x = _cpu(inp["x"])
    g = {k_: _cpu(inp.get(k_)) for k_ in ("w_router", "w_gate", "w_up", "w_down", "ws_gate",
                                          "ws_up", "ws_down", "w_const_mix", "const_vec")}
    bias = inp.get("router_bias")
    bias = None if bias is None else _cpu(bias).to(torch.float32).contiguous()
    zp = inp.get("z_prev")
    zp = None if zp is None else _cpu(zp).to(torch.float32).contiguous()
    dt = _dt(x, *[v for v in g.values() if v is not None])
    L = _Layer(T=x.shape[0], d=cfg.d, top_k=cfg.top_k, dt=dt, n_ffn=cfg.n_ffn,
               hidden=cfg.hidden, n_shared=cfg.n_shared, hidden_shared=cfg.hidden_shared,
               n_zero=cfg.n_zero, n_copy=cfg.n_copy, n_const=cfg.n_const)
    k = cfg.top_k
    y = np.empty((n, cfg.d), np.float64)
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k), np.float64)
    margin = np.empty((n,), np.float64)
    ii = None if idx_in is None else _np_i32(idx_in).reshape(n, k)
    lib().orc_moe_tokens(ctypes.byref(L), _vp(x), _vp(g["w_router"]), _vp(bias), _vp(zp),
                         _vp(g["w_gate"]), _vp(g["w_up"]), _vp(g["w_down"]),
                         _vp(g["ws_gate"]), _vp(g["ws_up"]), _vp(g["ws_down"]),
                         _vp(g["w_const_mix"]), _vp(g["const_vec"]),
                         n, _i32(tokens), _i32(ii), _f64(y), _i32(idx), _f64(gate), _f64(margin))
    return y, idx, gate, margin


# ------------------------------------------------- Cartesian-product router

def pk_scores(x, w_query, k_row, k_col, want_q: bool = False):
    """fp64 sub-key scores (s_row [T, rows], s_col [T, cols]) and optionally q."""
    x, wq, kr, kc = _cpu(x), _cpu(w_query), _cpu(k_row), _cpu(k_col)
    T, d = x.shape
    dq = wq.shape[0]
    rows, cols = kr.shape[0], kc.shape[0]
    sr = np.empty((T, rows), np.float64)
    sc = np.empty((T, cols), np.float64)
    q = np.empty((T, dq), np.float64)
    lib().orc_pk_scores(T, d, dq, rows, cols, _dt(x, wq, kr, kc), _vp(x), _vp(wq), _vp(kr),
                        _vp(kc), _f64(sr), _f64(sc), _f64(q))
    return (sr, sc, q) if want_q else (sr, sc)


def pk_select(s_row, s_col, kh: int, K: int):
    """Product-key top-K from sub-key scores: (idx int32 [T, K], gate f64 [T, K],
    margins f64 [T, 3] = row, column and candidate margins)."""
    sr, sc = _np_f64(s_row), _np_f64(s_col)
    T, rows = sr.shape
    cols = sc.shape[1]
    idx = np.empty((T, K), np.int32)
    gate = np.empty((T, K), np.float64)
    mg = np.empty((T, 3), np.float64)
    lib().orc_pk_select(T, rows, cols, kh, K, _f64(sr), _f64(sc), _i32(idx), _f64(gate), _f64(mg))
    return idx, gate, mg


def atomic_tokens(x, u, v, tokens, idx, gate, shared=None) -> np.ndarray:
    """y_t = sum_j g_j GELU(u_e . x_t) v_e for the listed tokens (fp64); with
    ``shared`` = dict(ws_gate, ws_up, ws_down) the shared dense SwiGLU
    branches are added (the full OmniMoE layer)."""
    x, u, v = _cpu(x), _cpu(u), _cpu(v)
    tokens = _np_i32(tokens).reshape(-1)
    n = tokens.shape[0]
    idx = _np_i32(idx).reshape(n, -1)
    K = idx.shape[1]
    gate = _np_f64(gate).reshape(n, K)
    d = x.shape[1]
    y = np.empty((n, d), np.float64)
    if shared is None:
        lib().orc_atomic_tokens(d, K, _dt(x, u, v), _vp(x), _vp(u), _vp(v), n, _i32(tokens),
                                _i32(idx), _f64(gate), _f64(y))
    else:
        sg, su, sd = (_cpu(shared[k_]) for k_ in ("ws_gate", "ws_up", "ws_down"))
        S, Hs = sg.shape[0], sg.shape[1]
        lib().orc_omni_tokens(d, K, _dt(x, u, v, sg, su, sd), _vp(x), _vp(u), _vp(v), S, Hs, _vp(sg), _vp(su),
                              _vp(sd), n, _i32(tokens), _i32(idx), _f64(gate), _f64(y))
    return y


# ------------------------------------------------------------- FP8 experts

def e4m3_decode(code: int) -> float:
    """Value of one e4m3 code (NaN for the NaN codes)."""
    return float(lib().orc_e4m3_decode(int(code) & 0xFF))


def e4m3_round(v: float) -> float:
    """Nearest e4m3 value (ties to even), saturated at +-448."""
    return float(lib().orc_e4m3_round(float(v)))


def pow2_scale(amax: float) -> float:
    """The smallest power of two s with 448 s >= amax (1 for amax == 0)."""
    return float(lib().orc_pow2_scale(float(amax)))


def quantize_rows(x):
    """Each row divided by its power-of-two scale and rounded to e4m3:
    (values [n, d] float64 on the e4m3 grid, scales [n])."""
    x = _cpu(x)
    n, d = x.shape
    q = np.empty((n, d), np.float64)
    sc = np.empty((n,), np.float64)
    lib().orc_quantize_rows(n, d, _dt(x), _vp(x), _f64(q), _f64(sc))
    return q, sc


def _u8(t):
    if t is None:
        return None
    t = _cpu(t)
    if t.dtype != torch.uint8:
        t = t.view(torch.uint8)
    return t


def fp8_moe_tokens(cfg, inp: dict, tokens, idx_in=None):
    """Layer output (fp64) for the listed tokens with FP8 experts: ``inp`` holds
    the e4m3 codes (w_gate8, w_up8, w_down8 and ws_*8 for shared experts, or
    under w_gate, ... themselves; uint8 or float8_e4m3fn tensors) and their
    fp32 row scales (s_gate, s_up, s_down, ss_*), plus x, the router and MoE++
    tensors as for moe_tokens.  Returns (y, idx, gate, margin)."""
    tokens = _np_i32(tokens).reshape(-1)
    n = tokens.shape[0]
    x = _cpu(inp["x"])
    g = {k_: _cpu(inp.get(k_)) for k_ in ("w_router", "w_const_mix", "const_vec")}
    def codes_of(name):   # the codes under name + "8", or under name itself when it holds codes
        c = inp.get(name + "8")
        if c is None and inp.get(name) is not None and inp[name].dtype in (torch.uint8, torch.float8_e4m3fn):
            c = inp[name]
        return _u8(c)
    codes = {k_ + "8": codes_of(k_) for k_ in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")}
    scales = {k_: (None if inp.get(k_) is None else _cpu(inp[k_]).to(torch.float32).contiguous())
              for k_ in ("s_gate", "s_up", "s_down", "ss_gate", "ss_up", "ss_down")}
    bias = inp.get("router_bias")
    bias = None if bias is None else _cpu(bias).to(torch.float32).contiguous()
    zp = inp.get("z_prev")
    zp = None if zp is None else _cpu(zp).to(torch.float32).contiguous()
    dt = _dt(x, *[v for v in g.values() if v is not None])
    L = _Layer(T=x.shape[0], d=cfg.d, top_k=cfg.top_k, dt=dt, n_ffn=cfg.n_ffn,
               hidden=cfg.hidden, n_shared=cfg.n_shared, hidden_shared=cfg.hidden_shared,
               n_zero=cfg.n_zero, n_copy=cfg.n_copy, n_const=cfg.n_const)
    k = cfg.top_k
    y = np.empty((n, cfg.d), np.float64)
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k), np.float64)
    margin = np.empty((n,), np.float64)
    ii = None if idx_in is None else _np_i32(idx_in).reshape(n, k)
    lib().orc_fp8_moe_tokens(ctypes.byref(L), _vp(x), _vp(g["w_router"]), _vp(bias), _vp(zp),
                             _vp(codes["w_gate8"]), _vp(scales["s_gate"]), _vp(codes["w_up8"]), _vp(scales["s_up"]),
                             _vp(codes["w_down8"]), _vp(scales["s_down"]),
                             _vp(codes["ws_gate8"]), _vp(scales["ss_gate"]), _vp(codes["ws_up8"]),
                             _vp(scales["ss_up"]), _vp(codes["ws_down8"]), _vp(scales["ss_down"]),
                             _vp(g["w_const_mix"]), _vp(g["const_vec"]),
                             n, _i32(tokens), _i32(ii), _f64(y), _i32(idx), _f64(gate), _f64(margin))
    return y, idx, gate, margin
