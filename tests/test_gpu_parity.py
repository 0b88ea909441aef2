"""CUDA path (through the C ABI) vs the fp64 oracle, element by element.

Small cases compare every output; the full-size workloads compare routing and
the permutation for every token and the outputs of sampled tokens.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from moe_workloads import get_config, make_inputs, scaled

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_swiglu_b200 as moe  # noqa: E402
    from parity import check_atomic_layer, check_swiglu_layer, run_gpu, to_device  # noqa: E402


@pytest.fixture(autouse=True)
def _clean_status():
    if torch.cuda.is_available():
        moe.moe_get_device_status(reset=True)
    yield


def _report(name: str, rep: dict) -> None:
    print(f"\n{name}: margin<1e-6 {rep['below_1e-6']}, boundary within error {len(rep['near_tie'])}, "
          f"set mismatches {len(rep['set_mismatch'])} (margins {np.round(rep['mismatch_margins'][:6], 9)}), "
          f"order-only mismatches {len(rep['order_mismatch'])}, "
          f"fp32 result err/rms {rep['rel_err']:.3e}, dtype output err/rms {rep['rel_err_out']:.3e}"
          + (f", routed rows {rep['R']}" if "R" in rep else ""))


def _sample(T: int, n: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, size=min(n, T), replace=False).tolist()) | {0, T - 1}
    return np.array(sorted(s), dtype=np.int32)


# ------------------------------------------------------------ small, every output

def test_tiny_f32_full_layer():
    cfg = get_config("tiny_f32")
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["rel_err"] <= 1e-4


def test_f32_layer_long_k_ragged():
    """fp32 layer whose K exceeds one 256-element staging step of the FMA
    GEMMs, with ragged tails everywhere: d = 264 (gate/up K in steps of 256
    and 8; down N = 4 x 64 + 8), H = 300 (down K 256 + 44; gate/up N =
    4 x 64 + 44), 300 rows over 8 experts (row tiles of 32 with short ends)."""
    cfg = scaled(get_config("tiny_f32"), T=150, d=264, hidden=300)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["rel_err"] <= 1e-4


def test_mixtral_shaped_small_ragged():
    cfg = scaled(get_config("mixtral"), T=333, d=512, hidden=1024)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["R"] == 333 * 2


def test_longtail_shared_experts():
    cfg = scaled(get_config("longtail"), T=200)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["R"] == 200 * 6


def test_moepp_zero_copy_const_residual():
    cfg = scaled(get_config("moepp"), T=300, hidden=640)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["R"] < 300 * 2          # some slots went to zero-computation experts


def test_atomic_small_grid():
    cfg = scaled(get_config("atomic"), T=100, d=256, pk_rows=64, pk_cols=64, pk_topk_half=16,
                 top_k=32, d_query=128)
    check_atomic_layer(cfg, make_inputs(cfg))


@pytest.mark.parametrize("T", [100, 700])      # single-CTA and CTA-pair shared GEMMs
def test_full_omnimoe_layer_small(T):
    """Atomic experts plus the shared dense SwiGLU branch."""
    cfg = scaled(get_config("omnimoe"), T=T, d=256, pk_rows=64, pk_cols=64, pk_topk_half=16,
                 top_k=32, d_query=128, hidden_shared=384)
    check_atomic_layer(cfg, make_inputs(cfg))


@pytest.mark.parametrize("E,T,d", [(2, 600, 512), (4, 1100, 2048), (2, 513, 512)])
def test_cta_pair_gemm_ragged_groups(E, T, d):
    """>= 512 rows per expert on average: the grouped GEMMs run on CTA pairs;
    group sizes are not multiples of 256.  d = 2048 takes the token-column
    form for the SwiGLU GEMM too (d = 512: row tiles for it)."""
    cfg = scaled(get_config("mixtral"), T=T, d=d, hidden=1024, n_ffn=E)
    check_swiglu_layer(cfg, make_inputs(cfg))


def test_cta_pair_gemm_nearly_empty_group():
    """CTA-pair GEMMs with one group of ~1090 rows and one of a few rows:
    the small group's token tile is narrower than 32 rows (MMA N = 16)."""
    cfg = scaled(get_config("mixtral"), T=1100, d=2048, hidden=1024, n_ffn=2, top_k=1)
    inp = make_inputs(cfg)
    inp["router_bias"] = torch.tensor([3.5, 0.0])
    rep = check_swiglu_layer(cfg, inp)
    assert rep["R"] == 1100


def test_atomic_cta_pair_router():
    cfg = scaled(get_config("atomic"), T=600, d=256, pk_rows=64, pk_cols=64, pk_topk_half=16,
                 top_k=32, d_query=128)
    check_atomic_layer(cfg, make_inputs(cfg))


def test_more_groups_than_the_token_column_table():
    """255 routed experts and 2 shared ones, 257 groups (the token-column tile
    table holds 256): the grouped GEMMs take the row-tiled forms; the router
    has more than 64 rows."""
    cfg = scaled(get_config("mixtral"), T=700, d=2048, hidden=256, n_ffn=255, n_shared=2, hidden_shared=256, top_k=4)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["R"] == 700 * 4


def test_more_destination_rows_than_the_one_launch_permutation_holds():
    """top-7 plus 2 shared experts: 9 destination rows per token, more than the
    one-launch permutation keeps per token, so the four-kernel form runs."""
    cfg = scaled(get_config("longtail"), T=300, top_k=7)
    rep = check_swiglu_layer(cfg, make_inputs(cfg))
    assert rep["R"] == 300 * 7


@pytest.mark.parametrize("T", [1, 2, 127, 129])
def test_bf16_token_counts_across_tile_edges(T):
    cfg = scaled(get_config("mixtral"), T=T, d=256, hidden=384, n_ffn=4)
    check_swiglu_layer(cfg, make_inputs(cfg))


def test_all_tokens_one_expert_and_empty_experts():
    cfg = scaled(get_config("mixtral"), T=300, d=256, hidden=256, n_ffn=6, top_k=1)
    inp = make_inputs(cfg)
    inp["router_bias"] = torch.tensor([0, 0, 0, 50.0, 0, 0])     # every token picks expert 3
    rep = check_swiglu_layer(cfg, inp)
    assert rep["R"] == 300


def test_empty_batch_is_a_no_op():
    cfg = scaled(get_config("mixtral"), T=0, d=256, hidden=256, n_ffn=4)
    inp = to_device(make_inputs(scaled(cfg, T=1)))
    desc = moe.desc_from(cfg)
    x = inp["x"][:0]
    y = torch.empty_like(x)
    layer = moe.MoELayer(desc, inp)
    layer.forward(x, y=y)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == moe.MOE_OK


def test_layer_forward_equals_stages():
    cfg = scaled(get_config("longtail"), T=150)
    inp = to_device(make_inputs(cfg))
    r = run_gpu(cfg, inp)
    layer = moe.MoELayer(r["desc"], inp)
    y = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(y, r["bufs"].y)


@pytest.mark.parametrize("name,T,changes", [("moepp", 700, {"hidden": 640}), ("atomic", 300, {})])
def test_cuda_graph_replay_matches_eager(name, T, changes):
    """The layer's launches captured once in a CUDA graph and replayed give
    the eager result bit for bit, also after the input changes in place."""
    cfg = scaled(get_config(name), T=T, **changes)
    inp = to_device(make_inputs(cfg))
    layer = moe.MoELayer(moe.desc_from(cfg), inp)
    x, zp = inp["x"], inp.get("z_prev")
    y = layer.forward(x, prev_logits=zp)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward(x, prev_logits=zp, y=y)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, prev_logits=zp, y=y)
    for trial in range(2):
        if trial:
            x.copy_(torch.roll(x, shifts=1, dims=0))
        ref = layer.forward(x, prev_logits=zp).clone()
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, ref)
    del g
    assert moe.moe_get_device_status() == moe.MOE_OK


@pytest.mark.parametrize("name,T,changes,chunks", [
    ("moepp", 700, {"hidden": 640}, 3),        # gating residual from host memory, ragged last range
    ("atomic", 1000, {}, 4),
    ("mixtral", 600, {"d": 512, "hidden": 512}, 0),
    ("tiny_f32", 64, {}, 2),
    ("longtail", 300, {}, 3),                    # shared experts: their groups hold every token of a range
    ("mixtral_fp8", 600, {"d": 512, "hidden": 512}, 2),   # e4m3 experts
])
def test_host_call_equals_device_call(name, T, changes, chunks):
    """moe_layer_forward_host (host buffers, copies pipelined over token
    ranges) gives moe_layer_forward's output bit for bit."""
    cfg = scaled(get_config(name), T=T, **changes)
    inp = make_inputs(cfg)
    dev = to_device(inp)
    layer = moe.MoELayer(moe.desc_from(cfg), dev)
    ref = layer.forward(dev["x"], prev_logits=dev.get("z_prev"))
    x_host = inp["x"].contiguous().pin_memory()
    zp_host = inp["z_prev"].contiguous().pin_memory() if "z_prev" in inp else None
    y_host = layer.forward_host(x_host, prev_logits=zp_host, chunks=chunks)
    torch.cuda.synchronize()
    assert torch.equal(y_host, ref.cpu())
    assert moe.moe_get_device_status() == moe.MOE_OK


def test_invalid_expert_id_sets_bounds_status():
    cfg = scaled(get_config("mixtral"), T=64, d=256, hidden=256, n_ffn=4)
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    b = moe.StageBuffers(desc)
    idx = torch.zeros((64, 2), dtype=torch.int32, device="cuda")
    idx[:, 1] = 1
    idx[5, 1] = 7            # out of range: 4 experts
    moe.moe_permute(desc, idx, inp["x"], b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace)
    assert moe.moe_get_device_status(reset=True) == moe.MOE_ERR_DEVICE_BOUNDS
    idx[5, 1] = 0            # same expert twice in one token
    moe.moe_permute(desc, idx, inp["x"], b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace)
    assert moe.moe_get_device_status(reset=True) == moe.MOE_ERR_DEVICE_BOUNDS
    idx[5, 1] = 1
    moe.moe_permute(desc, idx, inp["x"], b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace)
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK


def test_bounded_wait_times_out_and_context_survives():
    """A wait on a barrier nothing arrives on gives up after its limit: the
    kernel returns, the status reads MOE_ERR_TIMEOUT, and the next layer call
    on the same context runs and is correct."""
    import time
    ok = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.moe_selftest_wait_timeout(50_000_000, ok)          # 50 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.5
    assert int(ok.item()) == 0
    assert moe.moe_get_device_status(reset=True) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    cfg = scaled(get_config("mixtral"), T=40, d=256, hidden=256, n_ffn=4)
    check_swiglu_layer(cfg, make_inputs(cfg))


def test_argument_errors_return_before_launch():
    cfg = scaled(get_config("mixtral"), T=8, d=256, hidden=256, n_ffn=4)
    inp = to_device(make_inputs(cfg))
    desc = moe.desc_from(cfg)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.moe_layer_forward(desc, inp, inp["x"], None, torch.empty_like(inp["x"]), None, small)
    assert e.value.status == moe.MOE_ERR_WORKSPACE
    bad = moe.desc_from(scaled(cfg, hidden=200))       # hidden not a multiple of 128 on bf16
    assert moe.moe_layer_workspace_size(bad) == -1


# ------------------------------------------------------------ full-size workloads

def test_mixtral_full_size_sampled():
    cfg = get_config("mixtral")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 12), check_sorted=True)
    _report("mixtral", rep)


def test_longtail_full_size_sampled():
    cfg = get_config("longtail")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 24))
    _report("longtail", rep)


def test_moepp_full_size_sampled():
    cfg = get_config("moepp")
    rep = check_swiglu_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 24))
    _report("moepp", rep)


def test_atomic_full_size_sampled():
    cfg = get_config("atomic")
    rep = check_atomic_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 48))
    _report("atomic", rep)


def test_omnimoe_full_size_sampled():
    cfg = get_config("omnimoe")
    rep = check_atomic_layer(cfg, make_inputs(cfg), tokens=_sample(cfg.T, 48))
    _report("omnimoe", rep)
