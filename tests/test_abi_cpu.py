"""The C-ABI library on a machine without a GPU: it loads, exports every
entry point include/moe.h declares, and its host-side logic (descriptor
checks, sizes, argument errors) answers without touching a device."""

from __future__ import annotations

import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


def _declared():
    text = (ROOT / "include" / "moe.h").read_text()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def abi():
    from mixture_experts_layer_swiglu_b200 import _abi
    return _abi


def test_library_exports_every_declared_symbol(abi):
    lib = abi.load()
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(abi.EXPORTED)


def _desc(abi, **kw):
    from mixture_experts_layer_swiglu_b200.layer import make_desc
    return make_desc(**kw)


def test_sizes_and_groups(abi):
    d = _desc(abi, T=4096, d_model=4096, top_k=2, n_ffn=8, hidden=14336)
    assert abi.moe_num_groups(d) == 8
    assert abi.moe_row_capacity(d) == 8192
    ws = abi.moe_workspace_size(d)
    assert ws >= 8192 * 14336 * 2          # the hidden activation
    # the layer's two-pass step holds x_sorted (bf16) and y_sorted (fp32) beside the scratch
    assert abi.moe_layer_workspace_size(d) > ws + 8192 * 4096 * (2 + 4)
    # the fused step: h and the [T, d] fp32 accumulator
    assert abi.moe_fused_workspace_size(d) >= 8192 * 14336 * 2 + 4096 * 4096 * 4
    s = _desc(abi, T=2048, d_model=2048, top_k=6, n_ffn=64, hidden=1408, n_shared=2, hidden_shared=1408)
    assert abi.moe_num_groups(s) == 66 and abi.moe_row_capacity(s) == 2048 * 6 + 2 * 2048
    assert abi.moe_fused_workspace_size(s) == -1        # shared experts, k = 6: the two-pass combine
    assert abi.moe_layer_workspace_size(s) > 2 * (2048 * 6 + 2 * 2048) * 2048 * 2
    a = _desc(abi, T=8192, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=512,
              pk_topk_half=32, d_query=1024)
    assert abi.moe_num_groups(a) == 512 * 512 and abi.moe_row_capacity(a) == 8192 * 64
    o = _desc(abi, T=8192, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=512,
              pk_topk_half=32, d_query=1024, n_shared=1, hidden_shared=2816)
    # the full layer: the shared branch's fp32 output after the task coefficients
    assert abi.moe_num_groups(o) == 512 * 512
    assert abi.moe_layer_workspace_size(o) >= abi.moe_layer_workspace_size(a) + 8192 * 1024 * 4


@pytest.mark.parametrize("bad", [
    dict(T=-1, d_model=256, top_k=2, n_ffn=4, hidden=256),
    dict(T=8, d_model=256, top_k=5, n_ffn=4, hidden=256),                  # k > experts
    dict(T=8, d_model=200, top_k=2, n_ffn=4, hidden=256),                  # d not a multiple of 64 (bf16)
    dict(T=8, d_model=256, top_k=2, n_ffn=4, hidden=200),                  # H not a multiple of 128
    dict(T=8, d_model=256, top_k=2, n_ffn=4, hidden=256, n_shared=1, hidden_shared=128),
    dict(T=8, d_model=256, top_k=33, n_ffn=64, hidden=256),                # k > 32
    dict(T=8, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=256, pk_topk_half=32,
         d_query=1024),                                                   # rows != cols
    dict(T=8, d_model=1024, top_k=2000, kind="atomic", pk_rows=512, pk_cols=512, pk_topk_half=32,
         d_query=1024),                                                   # K > kh^2
    dict(T=8, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=512, pk_topk_half=32,
         d_query=1024, n_shared=2, hidden_shared=1024),                   # one shared branch at most
    dict(T=8, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=512, pk_topk_half=32,
         d_query=1024, n_shared=1, hidden_shared=1000),                   # shared width not a multiple of 128
    dict(T=8, d_model=1024, top_k=64, kind="atomic", pk_rows=512, pk_cols=512, pk_topk_half=32,
         d_query=1024, n_shared=0, hidden_shared=1024),                   # width without a branch
])
def test_rejected_descriptors(abi, bad):
    d = _desc(abi, **bad)
    assert abi.moe_workspace_size(d) == -1
    assert abi.moe_layer_workspace_size(d) == -1
    assert abi.moe_layer_host_workspace_size(d, 0) == -1


def test_host_call_workspace_follows_the_token_ranges(abi):
    d = _desc(abi, T=4096, d_model=4096, top_k=2, n_ffn=8, hidden=14336)
    one = _desc(abi, T=2048, d_model=4096, top_k=2, n_ffn=8, hidden=14336)
    two = abi.moe_layer_host_workspace_size(d, 0)           # automatic: 2 ranges of 2048 tokens
    assert two == abi.moe_layer_host_workspace_size(d, 2)
    # one range's layer workspace plus double-buffered x, y and router-logit staging
    staging = 2 * (2048 * 4096 * 2 * 2 + 2048 * 8 * 4)
    assert two >= abi.moe_layer_workspace_size(one) + staging
    assert abi.moe_layer_host_workspace_size(d, 1) > two     # one range holds the whole batch
    assert abi.moe_layer_host_workspace_size(d, 100) == abi.moe_layer_host_workspace_size(d, 8)


def test_argument_errors_without_a_device(abi):
    lib = abi.load()
    d = _desc(abi, T=8, d_model=256, top_k=2, n_ffn=4, hidden=256)
    w = abi.MoELayerWeights()
    # null descriptor / null pointers are rejected on the host, nothing launched
    assert lib.moe_route(None, ctypes.byref(w), None, None, None, None, None, None, None, 0, None) == 1
    assert lib.moe_route(ctypes.byref(d), ctypes.byref(w), None, None, None, None, None, None, None, 0,
                         None) == 1
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), 16, None, 16, None, None, 0, None) == 3
    assert lib.moe_grouped_ffn_phase(ctypes.byref(d), ctypes.byref(w), 3, 16, 16, 16, 16, 1 << 20, None) == 1
    assert lib.moe_layer_forward_host(ctypes.byref(d), ctypes.byref(w), None, None, None, 0, None, 0, None) == 1
    assert lib.moe_layer_forward_host(ctypes.byref(d), ctypes.byref(w), 16, None, 16, 0, 16, 0, None) == 3
    a = _desc(abi, T=8, d_model=256, top_k=4, kind="atomic", pk_rows=32, pk_cols=32, pk_topk_half=4, d_query=64)
    assert lib.moe_layer_forward_host(ctypes.byref(a), ctypes.byref(w), 16, 16, 16, 0, 16, 1 << 30, None) == 1
    assert lib.moe_last_launch_count() == 0
    assert abi.status_string(3) == "workspace too small"


def test_layer_object_rejects_buffers_that_disagree_with_the_descriptor():
    """MoELayer hands raw pointers to the library, sized by the descriptor: a
    tensor of another shape or dtype is refused before any device work."""
    import torch

    from mixture_experts_layer_swiglu_b200 import layer as L

    desc = L.make_desc(T=8, d_model=256, top_k=2, dtype="bf16", n_ffn=4, hidden=256, n_zero=1)
    lay = L.MoELayer(desc, {})
    bf, f32 = torch.bfloat16, torch.float32
    bad_calls = [
        lambda: lay.forward(torch.zeros(9, 256, dtype=bf)),                           # rows
        lambda: lay.forward(torch.zeros(8, 128, dtype=bf)),                           # width
        lambda: lay.forward(torch.zeros(8, 256, dtype=f32)),                          # dtype
        lambda: lay.forward(torch.zeros(8 * 256, dtype=bf)),                          # rank
        lambda: lay.forward(torch.zeros(8, 256, dtype=bf), y=torch.zeros(8, 256, dtype=f32)),
        lambda: lay.forward(torch.zeros(8, 256, dtype=bf), prev_logits=torch.zeros(8, 4, dtype=f32)),
        lambda: lay.forward(torch.zeros(8, 256, dtype=bf), logits_out=torch.zeros(8, 5, dtype=bf)),
        lambda: lay.forward_host(torch.zeros(8, 256, dtype=bf), y_host=torch.zeros(7, 256, dtype=bf)),
    ]
    for call in bad_calls:
        with pytest.raises(ValueError, match="expected a"):
            call()
    # the right shapes pass the check and reach the device-pointer step (host tensors here)
    with pytest.raises(ValueError, match="CUDA tensors"):
        lay.forward(torch.zeros(8, 256, dtype=bf), prev_logits=torch.zeros(8, 5, dtype=f32))
    atomic = L.make_desc(T=8, d_model=256, top_k=4, dtype="bf16", kind="atomic", pk_rows=32, pk_cols=32,
                         pk_topk_half=4, d_query=64)
    with pytest.raises(ValueError, match="gating residual"):
        L.MoELayer(atomic, {}).forward(torch.zeros(8, 256, dtype=bf), prev_logits=torch.zeros(8, 64, dtype=f32))
