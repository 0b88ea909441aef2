"""Benchmark of the MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one rank per GPU)

A step is one pass of the whole hot path -- router + top-k, histogram / scan
/ permutation, grouped gate/up GEMM with SwiGLU, grouped down GEMM, combine --
over one batch of the Mixtral-shaped workload (T=4096 tokens, d=4096, 8 SwiGLU
experts of hidden 14336, top-2, bf16, seeded synthetic inputs).  Ranks run
independent token batches on replicated weights (no collective on the data
path; weak scaling); `value` is the tokens of all ranks per second, time
being the max over ranks of the summed per-step device times.

Prints one JSON line (rank 0).  Extra keys: per-kernel times, the roofline of
the dominant kernel, the fp64 oracle timed on the host cores (cpu_baseline),
the end-to-end figure through moe_layer_forward with host buffers (e2e), the
SM clocks seen during the timed region, and the number of our kernels
launched in it.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

from moe_workloads import get_config, make_activations, make_weights  # noqa: E402

METRIC = "MoE-layer tokens/sec on 1 B200; % of bf16 tensor / HBM roofline"
WORKLOAD = "mixtral"
L2_FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--oracle-tokens", type=int, default=0,
                   help="tokens in the CPU oracle sample (0: sized to ~15 s)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--tokens", type=int, default=0, help="override T (profiling a smaller case)")
    p.add_argument("--experts", type=int, default=0, help="override the expert count (profiling)")
    p.add_argument("--workload", default=WORKLOAD,
                   help="tiny_f32 | mixtral | longtail | moepp | atomic | omnimoe (default: the Mixtral-shaped layer)")
    p.add_argument("--no-library-ref", action="store_true", help="skip the cuBLAS same-shape reference")
    p.add_argument("--no-workloads", action="store_true",
                   help="time only --workload (skip the per-workload lines of the other layers)")
    return p.parse_args()


def bench_config(args):
    from moe_workloads import scaled
    cfg = get_config(args.workload)
    ch = {}
    if args.tokens:
        ch["T"] = args.tokens
    if args.experts:
        ch["n_ffn"] = args.experts
    return scaled(cfg, **ch) if ch else cfg


def workload_config(cfg) -> dict:
    if cfg.kind == "atomic":
        name = f"{cfg.name}_T{cfg.T}_d{cfg.d}_N{cfg.pk_rows}x{cfg.pk_cols}_K{cfg.top_k}_half{cfg.pk_topk_half}"
        shape = {"experts": cfg.n_atomic, "d_query": cfg.d_query, "router": "Cartesian product, top-K of top-half^2"}
        if cfg.n_shared:
            name += f"_shared{cfg.hidden_shared}"
            shape["shared_dense_hidden"] = cfg.hidden_shared
    else:
        name = f"{cfg.name}_T{cfg.T}_d{cfg.d}_E{cfg.n_ffn}_H{cfg.hidden}_k{cfg.top_k}"
        if cfg.n_shared:
            name += f"_S{cfg.n_shared}"
        if cfg.n_zero + cfg.n_copy + cfg.n_const:
            name += f"_zc{cfg.n_zero + cfg.n_copy + cfg.n_const}"
        shape = {"experts": cfg.n_ffn, "hidden": cfg.hidden, "shared": cfg.n_shared,
                 "zero_copy_const": [cfg.n_zero, cfg.n_copy, cfg.n_const], "router": "softmax over top-k"}
    return {"workload": name, "T_per_gpu": cfg.T, "d_model": cfg.d, "top_k": cfg.top_k, **shape,
            "parallelism": "token-sharded replicas",
            "l2": "flushed between steps (256 MiB write outside the step events)",
            "timing": "CUDA events around each step; the step is fully queued before its first event"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and throttle reasons of one GPU, sampled every 20 ms via NVML
    (read-only queries)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:   # match the CUDA device to the NVML device by PCI address
                p = torch.cuda.get_device_properties(index)
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:   # noqa: BLE001
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:   # noqa: BLE001
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._reasons_fn(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:   # noqa: BLE001
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self) -> dict:
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, inp, toks) -> None:
    """The whole layer for the listed tokens with the fp64 oracle."""
    import oracle
    if cfg.kind == "atomic":
        xs = inp["x"][torch.from_numpy(toks).long()]
        sr, sc = oracle.pk_scores(xs, inp["w_query"], inp["subkeys_row"], inp["subkeys_col"])
        idx, gate, _ = oracle.pk_select(sr, sc, cfg.pk_topk_half, cfg.top_k)
        shared = {k_: inp[k_] for k_ in ("ws_gate", "ws_up", "ws_down")} if cfg.n_shared else None
        oracle.atomic_tokens(inp["x"], inp["u"], inp["v"], toks, idx, gate, shared=shared)
    else:
        oracle.moe_tokens(cfg, inp, toks)


def cpu_oracle_leg(cfg, inp, n_tokens: int, seconds: float = 15.0, single_seconds: float = 5.0) -> dict:
    """The fp64 oracle as it stands on a bounded sample of the workload's
    tokens (routing + experts of each token): on all host cores (OpenMP over
    tokens), then on one thread."""
    import numpy as np

    import oracle
    threads = oracle.num_threads()

    def timed(n: int, nthreads: int, budget: float):
        """tokens/s of the oracle on n evenly spaced tokens (n <= 0: sized to
        about `budget` seconds from a small probe)."""
        oracle.set_num_threads(nthreads)
        try:
            if n <= 0:
                t0 = time.perf_counter()
                oracle_sample(cfg, inp, np.arange(nthreads, dtype=np.int32))
                per_tok = (time.perf_counter() - t0) / nthreads
                n = int(max(nthreads, min(cfg.T, budget / max(per_tok, 1e-6))))
            toks = np.linspace(0, cfg.T - 1, n).astype(np.int32)
            t0 = time.perf_counter()
            oracle_sample(cfg, inp, toks)
            return n, time.perf_counter() - t0
        finally:
            oracle.set_num_threads(threads)

    n_all, el_all = timed(n_tokens, threads, seconds)
    n_one, el_one = timed(0, 1, single_seconds)
    return {"value": n_all / el_all, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_all} of the {cfg.T} tokens (evenly spaced), full routing + experts per token, "
                      f"{el_all:.1f} s on {threads} threads (OpenMP over tokens)",
            "single_thread": {"value": n_one / el_one, "unit": "tokens/s", "cores": 1,
                              "sample": f"{n_one} of the {cfg.T} tokens (evenly spaced), {el_one:.1f} s"}}


# ------------------------------------------------------------------- ranks

def reduce_max_over_ranks(dist, values, device) -> list:
    """Time-like values of this rank -> their maximum over all ranks (every
    rank takes part; a single process returns its own values)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput: the tokens of all ranks per second of the
    slowest rank's step time (weak scaling: every rank has its own batch)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------- ours

def stage_names(cfg) -> list:
    if cfg.kind == "atomic":
        shared = ["shared_gate_up_gemm", "shared_down_gemm"] if cfg.n_shared else []
        return ["router", "permute", "expert_dot"] + shared + ["expert_combine"]
    return ["router", "permute", "gate_up_gemm", "down_gemm", "combine"]


def work_model(cfg, R_total: int, R_ffn: int, touched: int, fused: bool = False) -> dict:
    """Algorithmic work of each stage: ("tensor", FLOPs) or ("hbm", bytes).
    Fused expert step: the combine stage reads the [T, d] fp32 accumulator
    the down GEMM formed (no y_sorted)."""
    d, T, k, e = cfg.d, cfg.T, cfg.top_k, cfg.elt_bytes
    if cfg.kind == "atomic":
        dq, N = cfg.d_query, cfg.n_atomic
        return {
            # q = W_q x, then each half of q (dq / 2 wide) against its sub-keys: the
            # method's own work (the kernels' three-part bf16 split of q, which
            # triples the score GEMM's K, is reported as router_split_flops)
            "router": ("tensor", 2.0 * T * d * dq + 2.0 * T * (dq // 2) * (cfg.pk_rows + cfg.pk_cols)),
            "permute": ("hbm", T * k * 4 * 6 + N * 4 * 5),
            # each touched expert's u (phase A) and v (phase B) row once, x read
            # once, y written once (the token-centric phase B moves more: it
            # gathers a v row per slot, with L2 hits for rows shared in time)
            "expert_dot": ("hbm", touched * d * e + T * d * e + T * k * 12),
            "expert_combine": ("hbm", touched * d * e + T * d * e + T * k * 8 + cfg.n_shared * T * d * 4),
            "shared_gate_up_gemm": ("tensor", 4.0 * T * d * cfg.hidden_shared),
            "shared_down_gemm": ("tensor", 2.0 * T * d * cfg.hidden_shared),
        }
    H = cfg.hidden
    E_r = cfg.n_routed
    router = T * d * e + (E_r + 2 * cfg.n_const) * d * e + T * k * 8 + T * cfg.n_const * 8
    if cfg.gating_residual:
        router += T * E_r * 4
    zc_x = T * d * e if (cfg.n_copy + cfg.n_const) else 0
    if fused:
        return {
            "router": ("hbm", router),
            "permute": ("hbm", T * d * e + R_total * d * e + T * k * 12),
            "gate_up_gemm": ("tensor", 4.0 * R_total * d * H),
            "down_gemm": ("tensor", 2.0 * R_total * d * H),
            "combine": ("hbm", T * d * 4 + T * d * e + zc_x + T * k * 12),
        }
    return {
        "router": ("hbm", router),
        "permute": ("hbm", T * d * e + R_total * d * (1 if cfg.expert_fp8 else e) + T * k * 12),
        "gate_up_gemm": ("tensor", 4.0 * R_total * d * H),
        "down_gemm": ("tensor", 2.0 * R_total * d * H),
        "combine": ("hbm", R_total * d * 4 + T * d * e + zc_x + T * k * 12),
    }


class Peaks:
    """Roofline denominators: MEASURED_PEAKS.json when present, else the fallback."""

    def __init__(self):
        peaks = {}
        pk = ROOT / "MEASURED_PEAKS.json"
        if pk.exists():
            peaks = json.loads(pk.read_text())
        self.tf = peaks.get("bf16_tflops")
        self.tf_sus = peaks.get("bf16_tflops_sustained")
        self.tf_src = "of measured (MEASURED_PEAKS.json, burst)" if self.tf else "of fallback"
        self.tf = self.tf or 1590.0
        self.hbm = peaks.get("hbm_gbs")
        self.hbm_src = "of measured (MEASURED_PEAKS.json)" if self.hbm else "of fallback"
        self.hbm = self.hbm or 6650.0


class Workload:
    """One layer's weights, inputs and stage buffers on the device, and its
    hot path as a list of C-ABI calls (route, permute, expert GEMMs, combine)."""

    def __init__(self, cfg, dev, rank: int):
        import mixture_experts_layer_swiglu_b200 as moe
        self.moe, self.cfg, self.dev = moe, cfg, dev
        self.w_cpu = make_weights(cfg, seed=0)
        self.a_cpu = make_activations(cfg, seed=rank)          # each rank its own tokens
        self.w = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.w_cpu.items()}
        self.x = self.a_cpu["x"].to(dev)
        self.zp = self.a_cpu["z_prev"].to(dev) if "z_prev" in self.a_cpu else None
        self.desc = moe.desc_from(cfg)
        self.desc_atomic = moe.desc_from(cfg)      # the same layer without its shared branch
        self.desc_atomic.n_shared, self.desc_atomic.hidden_shared = 0, 0
        self.ws = moe.weights_struct(self.w)
        self.b = moe.StageBuffers(self.desc, device=dev)
        self.atomic = cfg.kind == "atomic"
        # moe_layer_forward's path is the two-pass expert step; the fused one is
        # timed beside it where it applies
        self.fused = False
        self.fused_ok = self.b.fused_workspace is not None

    def calls(self, st, fused=None):
        moe, cfg, b, x, ws, desc = self.moe, self.cfg, self.b, self.x, self.ws, self.desc
        fused = self.fused if fused is None else fused
        cm = b.const_mix if cfg.n_const else None
        c = [lambda: moe.moe_route(desc, ws, x, self.zp, None, b.idx, b.gate, cm, b.workspace, st),
             lambda: moe.moe_permute(desc, b.idx, x, b.offsets, b.row_of, b.token_of, b.x_sorted, b.workspace,
                                     st)]
        if fused:   # the combine in the down GEMM's epilogue, then the finish
            for ph in (1, 2, 3):
                c.append(lambda ph=ph: moe.moe_fused_ffn_combine(desc, ws, ph, x, b.x_sorted, b.idx, b.gate, cm,
                                                                 b.offsets, b.row_of, b.token_of, b.y,
                                                                 b.fused_workspace, st))
            return c
        if self.atomic:   # the atomic step alone, then the shared dense branch's two GEMMs (if any)
            c.append(lambda: moe.moe_grouped_ffn(self.desc_atomic, ws, None, b.offsets, b.token_of, x, b.gate,
                                                 b.y_sorted, b.workspace, st))
            if cfg.n_shared:
                c.append(lambda: moe.moe_grouped_ffn_phase(desc, ws, 1, x, b.offsets, b.y_sorted, b.workspace, st))
                c.append(lambda: moe.moe_grouped_ffn_phase(desc, ws, 2, x, b.offsets, b.y_sorted, b.workspace, st))
        else:
            c.append(lambda: moe.moe_grouped_ffn_phase(desc, ws, 1, b.x_sorted, b.offsets, b.y_sorted,
                                                       b.workspace, st))
            c.append(lambda: moe.moe_grouped_ffn_phase(desc, ws, 2, b.x_sorted, b.offsets, b.y_sorted,
                                                       b.workspace, st))
        c.append(lambda: moe.moe_combine(desc, ws, b.y_sorted, b.offsets, b.row_of, b.idx, b.gate, cm, x, b.y, st))
        return c


def time_workload(wl: Workload, K: int, warmup: int, dist, flush, want_graph: bool, fused=None) -> dict:
    """Warm-up, then K timed steps (L2 flushed and a GPU sleep before each,
    outside the events; CUDA events between the stages on the launching
    stream; SM clocks sampled meanwhile); times reduced to their maximum over
    ranks.  Every rank takes the same collective steps."""
    moe, dev = wl.moe, wl.dev
    stream = torch.cuda.current_stream(dev)
    fused = wl.fused if fused is None else fused
    stage_calls = wl.calls(stream, fused)
    names = stage_names(wl.cfg)
    nst = len(stage_calls)

    def step(ev=None):
        """One pass of the hot path; events between the stages if given."""
        launches = 0
        for j, f in enumerate(stage_calls):
            if ev:
                ev[j].record(stream)
            f()
            launches += moe.moe_last_launch_count()
        if ev:
            ev[nst].record(stream)
        return launches

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(K)]
    # ~0.5 ms of GPU sleep after each flush, outside the events: the host has
    # queued the whole step before the device reaches the first event, so the
    # events time the device, not the Python launch path.
    sleep_cycles = int(0.5e-3 * torch.cuda.get_device_properties(dev).clock_rate * 1e3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    launches = 0
    with ClockSampler(dev.index) as clk:
        for i in range(K):
            flush.zero_()
            torch.cuda._sleep(sleep_cycles)
            launches += step(evs[i])
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    status = moe.moe_get_device_status(reset=True)
    assert status == moe.MOE_OK, moe.status_string(status)
    per = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)] for j, n in enumerate(names)}
    total_ms = sum(evs[i][0].elapsed_time(evs[i][nst]) for i in range(K))
    off = wl.b.offsets.cpu()
    R_total = int(off[-1].item())
    R_ffn = int(off[wl.cfg.n_ffn].item()) if not wl.atomic else R_total
    touched = int((off[1:] > off[:-1]).sum().item()) if wl.atomic else 0
    graph_ms = graph_step_ms(lambda st: wl.calls(st, fused), stream, flush, sleep_cycles, K) if want_graph else 0.0
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    mean = {n: sum(v) / K for n, v in per.items()}
    red = reduce_max_over_ranks(dist, [total_ms, graph_ms] + [mean[n] for n in names], dev)
    return {"names": names, "ms_step": red[0] / K, "graph_ms": red[1],
            "mean": {n: red[2 + j] for j, n in enumerate(names)}, "launches": launches,
            "clocks": clk.summary(), "R_total": R_total, "R_ffn": R_ffn, "touched": touched, "fused": fused}


FP8_OVER_BF16 = 2.0     # dense e4m3 / bf16 tensor throughput (nominal 4.5 / 2.25 PFLOP/s)


def kernel_table(cfg, t: dict, peaks: Peaks) -> dict:
    """Per-stage time, share of the step and fraction of its roofline (the
    expert GEMMs of an FP8-expert layer against the e4m3 peak: the measured
    bf16 peak times the nominal ratio)."""
    work = work_model(cfg, t["R_total"], t["R_ffn"], t["touched"], t["fused"])
    fp8 = getattr(cfg, "expert_fp8", False)
    kern = {}
    for n in t["names"]:
        ms = t["mean"][n]
        unit, amount = work[n]
        kern[n] = {"ms": round(ms, 4), "share": round(ms / t["ms_step"], 4)}
        if unit == "tensor":
            peak = peaks.tf * (FP8_OVER_BF16 if fp8 and n in ("gate_up_gemm", "down_gemm") else 1.0)
            kern[n]["tflops"] = round(amount / (ms / 1e3) / 1e12, 1)
            kern[n]["tensor_frac"] = round(kern[n]["tflops"] / peak, 4)
            if peak != peaks.tf:
                kern[n]["peak"] = f"e4m3: {FP8_OVER_BF16:g} x the bf16 peak"
        else:
            kern[n]["gbs"] = round(amount / (ms / 1e3) / 1e9, 1)
            kern[n]["hbm_frac"] = round(kern[n]["gbs"] / peaks.hbm, 4)
    if cfg.kind == "atomic":   # what the three-part split of q costs on top of the method's work
        kern["router"]["router_split_flops"] = 2.0 * cfg.T * cfg.d * cfg.d_query + \
            2.0 * cfg.T * (3 * cfg.d_query // 2) * (cfg.pk_rows + cfg.pk_cols)
    return kern


def workload_line(cfg, t: dict, world: int, peaks: Peaks) -> dict:
    """The compact per-workload entry of the JSON line's `workloads` map."""
    return {"config": workload_config(cfg)["workload"], "dtype": cfg.dtype, "ms_per_step": round(t["ms_step"], 4),
            "value": round(job_value(world, cfg.T, t["ms_step"]), 1), "unit": "tokens/s",
            "graph": {"ms_per_step": round(t["graph_ms"], 4),
                      "value": round(job_value(world, cfg.T, t["graph_ms"]), 1)},
            "expert_step": "fused" if t["fused"] else "two-pass",
            "kernels": kernel_table(cfg, t, peaks), "gpu_launches": t["launches"], "clocks": t["clocks"],
            "rows": {"grouped": t["R_total"], "ffn": t["R_ffn"], "touched_experts": t["touched"]}}


def run_ours(args, rank: int, world: int, dist) -> dict | None:
    import mixture_experts_layer_swiglu_b200 as moe

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    cfg = bench_config(args)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    peaks = Peaks()
    K = args.steps

    wl = Workload(cfg, dev, rank)
    t = time_workload(wl, K, args.warmup, dist, flush, want_graph=True)
    sleep_cycles = int(0.5e-3 * torch.cuda.get_device_properties(dev).clock_rate * 1e3)

    # end to end through the public call with host buffers: moe_layer_forward_host
    # copies x (and the previous layer's router logits) in and y out inside the
    # timed region, pipelined against the layer over token ranges
    x_host = wl.a_cpu["x"].pin_memory()
    zp_host = wl.a_cpu["z_prev"].contiguous().pin_memory() if "z_prev" in wl.a_cpu else None
    y_host = torch.empty(x_host.shape, dtype=moe.out_dtype(wl.desc)).pin_memory()
    layer = moe.MoELayer(wl.desc, wl.w)
    for _ in range(2):
        layer.forward_host(x_host, prev_logits=zp_host, y_host=y_host, stream=stream, device=dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    KE = max(3, K // 4)
    e2e_ms = 0.0
    for _ in range(KE):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        e0.record(stream)
        layer.forward_host(x_host, prev_logits=zp_host, y_host=y_host, stream=stream, device=dev)
        e1.record(stream)
        e1.synchronize()
        e2e_ms += e0.elapsed_time(e1)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(reset=True) == moe.MOE_OK
    e2e_ms = reduce_max_over_ranks(dist, [e2e_ms / KE], dev)[0]
    del layer

    # the fused expert step (combine in the down GEMM's epilogue) on the same
    # workload, for comparison with the two-pass one the layer takes
    fused_alt = None
    if wl.fused_ok:
        fused_alt = time_workload(wl, K, args.warmup, dist, flush, want_graph=False, fused=True)

    cublas = None
    if wl.atomic is False and cfg.dtype == "bf16" and rank == 0 and not args.no_library_ref:
        cublas = library_reference(cfg, t["R_total"], dev)

    # every other workload, timed the same way (each rank runs them all, so the
    # collective steps stay in step)
    others = {}
    if not args.no_workloads and not args.tokens and not args.experts:
        from moe_workloads.configs import ORDER
        for name in ORDER:
            if name == cfg.name:
                continue
            c2 = get_config(name)
            w2 = Workload(c2, dev, rank)
            t2 = time_workload(w2, K, args.warmup, dist, flush, want_graph=True)
            others[name] = workload_line(c2, t2, world, peaks)
            del w2
            torch.cuda.empty_cache()
    if rank != 0:
        return None

    kern = kernel_table(cfg, t, peaks)
    work = work_model(cfg, t["R_total"], t["R_ffn"], t["touched"], t["fused"])
    ms_step = t["ms_step"]
    value = job_value(world, cfg.T, ms_step)
    names = t["names"]
    dom = max(names, key=lambda n: t["mean"][n])
    unit, amount = work[dom]
    dom_s = t["mean"][dom] / 1e3
    if unit == "tensor":
        roof = {"bound": "tensor", "kernel": dom, "achieved": round(amount / dom_s / 1e12, 1), "peak": peaks.tf,
                "unit": "TFLOP/s", "peak_source": peaks.tf_src, "flops_per_launch": amount}
        if peaks.tf_sus:
            roof["frac_of_sustained"] = round(roof["achieved"] / peaks.tf_sus, 4)
    else:
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(amount / dom_s / 1e9, 1), "peak": peaks.hbm,
                "unit": "GB/s", "peak_source": peaks.hbm_src, "bytes_per_launch": amount}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    roof["traffic"] = _ncu_traffic(dom, cfg.name)
    h2d = x_host.numel() * x_host.element_size() + (zp_host.numel() * 4 if zp_host is not None else 0)
    d2h = y_host.numel() * y_host.element_size()
    flops = sum(a for u, a in work.values() if u == "tensor")
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) x, N(0,1/fan_in) weights)",
        "config": workload_config(cfg),
        "roofline": roof,
        "kernels": kern,
        "step_tflops": round(flops / (ms_step / 1e3) / 1e12, 1),
        "rows": {"grouped": t["R_total"], "ffn": t["R_ffn"], "touched_experts": t["touched"]},
        "e2e": {"value": round(job_value(world, cfg.T, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "moe_layer_forward_host: x (and previous router logits) from pinned host, y to pinned "
                        "host, copies pipelined against the layer over token ranges"},
        "graph": {"ms_per_step": round(t["graph_ms"], 4),
                  "value": round(job_value(world, cfg.T, t["graph_ms"]), 1), "unit": "tokens/s",
                  "how": "the same step captured once in a CUDA graph and replayed; L2 flushed before each replay"},
        "gpu_launches": t["launches"],
        "clocks": t["clocks"],
    }
    out["config"]["expert_step"] = "fused (combine in the down GEMM's epilogue)" if t["fused"] \
        else "two-pass (permuted copy, expert GEMMs, combine kernel)"
    if fused_alt:
        out["fused_step"] = {"ms_per_step": round(fused_alt["ms_step"], 4),
                             "value": round(job_value(world, cfg.T, fused_alt["ms_step"]), 1),
                             "kernels": kernel_table(cfg, fused_alt, peaks),
                             "note": "moe_fused_ffn_combine: accumulator zeroed in the gate/up epilogue, gated "
                                     "atomic adds in the down GEMM's epilogue, finish kernel; not the layer's path"}
    if cublas:
        out["library_reference"] = cublas
    if others:
        out["workloads"] = others
    if world == 1 and not args.no_cpu_baseline:
        w_cpu = dict(wl.w_cpu)
        w_cpu.update(wl.a_cpu)
        out["cpu_baseline"] = cpu_oracle_leg(cfg, w_cpu, args.oracle_tokens)
    return out


def graph_step_ms(calls, stream, flush, sleep_cycles: int, K: int) -> float:
    """Mean device time of one step replayed from a CUDA graph (the step's
    launches captured once), timed like the eager steps: L2 flush and a GPU
    sleep before each replay, CUDA events around it."""
    side = torch.cuda.Stream(device=stream.device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for f in calls(side):      # warm the capture stream's path once
            f()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for f in calls(side):
            f()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        evs[i][0].record(stream)
        g.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / K
    del g
    return ms


def library_reference(cfg, R_total: int, dev) -> dict:
    """cuBLAS (torch.bmm) on the same GEMM shapes with the rows split evenly
    over the experts: context for the grouped tcgen05 GEMMs, not part of the
    timed step."""
    E = cfg.n_ffn + cfg.n_shared
    m = max(1, R_total // max(E, 1))
    d, H = cfg.d, cfg.hidden
    g = torch.Generator(device=dev).manual_seed(1)
    A = torch.randn((E, m, d), device=dev, generator=g).to(torch.bfloat16)
    B = torch.randn((E, d, 2 * H), device=dev, generator=g).to(torch.bfloat16)
    Hh = torch.randn((E, m, H), device=dev, generator=g).to(torch.bfloat16)
    D = torch.randn((E, H, d), device=dev, generator=g).to(torch.bfloat16)
    out = {}
    for name, a, bm, fl in (("gate_up_bmm", A, B, 2.0 * E * m * d * 2 * H), ("down_bmm", Hh, D, 2.0 * E * m * H * d)):
        for _ in range(3):
            torch.bmm(a, bm)
        ts = []
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.bmm(a, bm)
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        out[name] = {"ms": round(ms, 4), "tflops": round(fl / (ms / 1e3) / 1e12, 1),
                     "shape": f"{E} x [{m}, {a.shape[2]}] @ [{bm.shape[1]}, {bm.shape[2]}]"}
    del A, B, Hh, D
    torch.cuda.empty_cache()
    return out


def _ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, when
    the summary was taken from the current source of the file that holds the
    kernel (its `source:` line names the file and its sha256); else null: a
    changed kernel has no counters yet."""
    import hashlib
    f = ROOT / "profiles" / f"{kernel}_{workload}.md"
    if not f.exists():
        return None
    traffic, src_ok = None, False
    for line in f.read_text().splitlines():
        if line.startswith("dram_bytes_per_launch:"):
            try:
                traffic = float(line.split(":", 1)[1].split()[0])
            except ValueError:
                return None
        elif line.startswith("source:"):
            parts = line.split()
            if len(parts) == 3 and parts[2].startswith("sha256:"):
                src = ROOT / "mixture_experts_layer_swiglu_b200" / parts[1]
                src_ok = src.exists() and hashlib.sha256(src.read_bytes()).hexdigest() == parts[2][7:]
    return traffic if src_ok else None


# -------------------------------------------------------------- reference

def run_reference(args, rank: int, world: int) -> dict | None:
    """The reference arm: the fp64 CPU oracle on the host cores, each step a
    bounded sample of the same workload."""
    if rank != 0:
        return None
    import numpy as np

    import oracle
    cfg = bench_config(args)
    inp = make_weights(cfg, seed=0)
    inp.update(make_activations(cfg, seed=0))
    n = args.oracle_tokens or max(8, oracle.num_threads())
    rng = np.random.default_rng(0)
    for _ in range(min(args.warmup, 1)):
        oracle_sample(cfg, inp, rng.choice(cfg.T, n, replace=False).astype(np.int32))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(cfg, inp, rng.choice(cfg.T, n, replace=False).astype(np.int32))
    el = time.perf_counter() - t0
    value = n * args.steps / el
    base = {"value": round(value, 3), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} random tokens of the {cfg.T} per step (routing + experts per token)"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(cfg),
            "cpu_baseline": base,
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        out = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime

            import torch.distributed as dist
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        out = run_ours(args, rank, world, dist)
        if dist:
            dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
