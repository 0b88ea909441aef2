"""moe_permute_static: the permutation for callers that cannot allocate device
memory (a plugin whose host framework owns all device memory, a service whose
memory budget is fixed at start-up).  It must give exactly what moe_permute
gives with a caller-allocated workspace, call after call, although its
scratch array keeps whatever the previous call left in it.

This file is collected last on purpose: a run that stops at the first
failure has then already run every other test.
"""

from __future__ import annotations

import pytest
import torch

from moe_workloads import get_config, make_inputs, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_swiglu_b200 as moe
    from parity import to_device


def _routed(cfg):
    """Device inputs, descriptor, and the router's indices for a workload."""
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    b = moe.StageBuffers(desc)
    cm = b.const_mix if desc.n_const > 0 else None
    moe.moe_route(desc, inp, inp["x"], inp.get("z_prev"), None, b.idx, b.gate, cm, b.workspace)
    return inp, desc, b


def _with_workspace(inp, desc, b):
    moe.moe_permute(desc, b.idx, inp["x"], b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace)
    torch.cuda.synchronize()
    return b.offsets.clone(), b.row_of.clone(), b.token_of.clone(), b.x_sorted.clone()


def _static(inp, desc, b):
    off = torch.full_like(b.offsets, -7)          # poison: every entry must be written
    row = torch.full_like(b.row_of, -7)
    tok = torch.full_like(b.token_of, -7)
    xs = torch.zeros_like(b.x_sorted)
    moe.moe_permute_static(desc, b.idx, inp["x"], off, row, tok, xs)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    return off, row, tok, xs


def _assert_same(ref, got):
    off_r, row_r, tok_r, xs_r = ref
    off_g, row_g, tok_g, xs_g = got
    assert torch.equal(off_g, off_r)
    assert torch.equal(row_g, row_r)
    n = int(off_r[-1].item())                     # rows written (routed + shared)
    assert torch.equal(tok_g[:n], tok_r[:n])
    assert torch.equal(xs_g[:n], xs_r[:n])


def test_static_scratch_permute_matches_workspace_permute_twice():
    a = _routed(scaled(get_config("longtail"), T=300))                 # 64 experts + 2 shared
    bcase = _routed(scaled(get_config("moepp"), T=700, hidden=640))    # zero-computation slots
    ref_a = _with_workspace(*a)
    ref_b = _with_workspace(*bcase)
    # two calls in a row on different routings, then the first again: what
    # one call leaves in the shared array must not leak into the next
    _assert_same(ref_a, _static(*a))
    _assert_same(ref_b, _static(*bcase))
    _assert_same(ref_a, _static(*a))


def test_static_scratch_permute_rejects_sizes_beyond_its_array():
    dev = torch.device("cuda")
    too_big = moe.make_desc(T=257 * 256, d_model=256, top_k=2, n_ffn=256, hidden=256)  # 257*256 > 65536
    assert moe.moe_row_capacity(too_big) > 0                                            # a valid layer
    idx = torch.zeros((1, 2), dtype=torch.int32, device=dev)
    buf = torch.zeros((1024, 256), dtype=torch.bfloat16, device=dev)
    i32 = torch.zeros((4096,), dtype=torch.int32, device=dev)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_permute_static(too_big, idx, buf, i32, i32, i32, buf)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED
    fits = moe.make_desc(T=256 * 256, d_model=256, top_k=2, n_ffn=256, hidden=256)     # exactly 65536
    assert moe.moe_row_capacity(fits) > 0
    atomic = moe.make_desc(T=8, d_model=256, top_k=4, kind="atomic", pk_rows=32, pk_cols=32,
                           pk_topk_half=4, d_query=64)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_permute_static(atomic, idx, buf, i32, i32, i32, None)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def test_static_scratch_permute_at_its_size_limit():
    # ceil(T / 256) * n_ffn = 65536 exactly: every entry of the array is used
    # once, so an off-by-one in the size check or the kernels' indexing shows
    dev = torch.device("cuda")
    T, k, E, d = 256 * 256, 2, 256, 256
    desc = moe.make_desc(T=T, d_model=d, top_k=k, n_ffn=E, hidden=256)
    g = torch.Generator(device=dev).manual_seed(5)
    first = torch.randint(0, E, (T,), device=dev, generator=g, dtype=torch.int32)
    second = (first + torch.randint(1, E, (T,), device=dev, generator=g, dtype=torch.int32)) % E
    x = torch.randn((T, d), device=dev, generator=g).to(torch.bfloat16)
    b = moe.StageBuffers(desc, device=dev)
    b.idx.copy_(torch.stack([first, second], dim=1))        # two distinct experts per token
    ref = _with_workspace({"x": x}, desc, b)
    got = _static({"x": x}, desc, b)
    _assert_same(ref, got)
    assert int(ref[0][-1].item()) == T * k
