#!/usr/bin/env python
"""Benchmark of the top-k MoE FFN layer forward on B200.

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]
                    [--preset v3 --tokens 9440] [--no-sweep] [--no-cpu] [--no-parity]

One step = one whole layer forward (RMSNorm, router, top-k, permutation,
grouped gate/up and down GEMMs, combine) over one batch of T synthetic tokens,
through the C ABI (moe_layer_forward).  Default workload: the largest
single-GPU configuration, the DeepSeek-V3-shaped layer (d 7168, 256 routed
experts with a Zipf(1.1)-skewed select-mode bias, top-8, expert hidden 2048, one
shared expert, bf16) at T = 9440 tokens, the batch where this layer crosses from
memory- to compute-bound.  With N > 1 (torchrun) every rank runs its own batch
on its own GPU with replicated weights -- token data parallelism, no collective
on the data path (weak scaling); the step time is the max over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle (the
only reference this layer has) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_synth  # noqa: E402
from moe_layer_fp32_b200 import roofline as R  # noqa: E402

METRIC = "MoE-layer tokens/s (decode & prefill); % of HBM / tensor-core roofline"
KERNEL_NAMES_TC = ["rmsnorm", "router", "route_topk", "permute", "gather", "gateup_gemm",
                   "down_gemm", "combine"]
KERNEL_NAMES_SIMT = ["rmsnorm", "router", "route_topk", "permute", "gateup_simt", "down_simt",
                     "combine"]


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--preset", default="v3")
    p.add_argument("--tokens", type=int, default=9440)
    p.add_argument("--no-sweep", action="store_true",
                   help="skip the other configurations (decode and prefill batches)")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-parity", action="store_true")
    p.add_argument("--prefill-tiles", choices=["auto", "single", "pair"], default="auto",
                   help="bf16 prefill tiles: chosen by rows per expert (auto), 128-token tiles "
                        "on single CTAs, or 256-token tiles on CTA pairs")
    return p.parse_args()


def workload_name(sh, T):
    names = {"olmoe": "OLMoE-1B-7B-shaped", "v2lite": "DeepSeek-V2-Lite-shaped",
             "qwen3_int4": "Qwen3-30B-A3B-shaped (int4 experts)",
             "qwen3_int8": "Qwen3-30B-A3B-shaped (int8 experts)",
             "qwen3_fp8": "Qwen3-30B-A3B-shaped (fp8 experts)", "v3": "DeepSeek-V3-shaped",
             "v3_e32": "DeepSeek-V3-shaped (32 experts)", "tiny": "Tiny"}
    kind = "decode" if T <= 64 else "prefill"
    return f"{names.get(sh.name, sh.name)} MoE layer forward, {kind} T={T}"


def config_dict(sh, T, world):
    return {"workload": workload_name(sh, T), "T_per_gpu": T, "global_batch": T * world,
            "d": sh.d, "E": sh.E, "k": sh.k, "f": sh.f, "n_shared": sh.n_shared,
            "expert_dtype": sh.expert, "router_dtype": sh.router, "bias_mode": sh.bias_mode,
            "capacity_factor": sh.capacity_factor, "renormalize": sh.renormalize,
            "parallelism": f"replicas x{world} (token data parallel, no collective)",
            "l2": "not flushed; inputs larger than L2 (126 MB): the routed experts' weights "
                  "total %.0f MB and every step streams the touched ones from HBM" % (
                      R.expert_bytes(sh.expert, sh.d, sh.f, sh.group_size) * sh.E / 1e6)}


# --------------------------------------------------------------------- clocks
class Clocks:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# --------------------------------------------------------------------- helpers
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, ms_local: float, world: int):
    """Whole-job throughput: the units all ranks processed over the slowest rank's
    time (ms).  Returns (units/s, slowest ms)."""
    ms_max = max_over_ranks(ms_local, world)
    return units_per_rank * world / (ms_max / 1e3), ms_max


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


def time_oracle(li, x, n_tokens, reps=1):
    """Oracle on the first n_tokens rows of the batch (routing over that
    sub-batch); returns seconds per call."""
    from oracle import moe_oracle as O
    xs = x[:n_tokens]
    t0 = time.perf_counter()
    for _ in range(reps):
        O.layer_from_inputs(li, xs)
    return (time.perf_counter() - t0) / reps


def routing_stats(sh, T, counts):
    """(kept rows, touched experts) of one batch from its per-expert counts."""
    cnt = counts.cpu().numpy()
    cap = None
    if sh.capacity_factor > 0:
        import math
        cap = math.ceil(float(np.float32(sh.capacity_factor)) * T * sh.k / sh.E)
    kept = int(np.minimum(cnt, cap).sum()) if cap else int(cnt.sum())
    return kept, int((cnt > 0).sum())


# --------------------------------------------------------------------- our arm
def run_ours(args):
    import moe_layer_fp32_b200 as M
    world, rank, local = dist_setup(args)
    sh = moe_synth.PRESETS[args.preset]
    T, K, W = args.tokens, args.steps, max(args.warmup, 3)
    dev = torch.device("cuda", local)
    li_host = moe_synth.make_layer(sh)
    li = li_host.to(dev)
    x_host = moe_synth.make_x(sh, T, stream=T + 7919 * rank)
    x = x_host.to(dev)
    layer = M.MoELayer(li, T)            # output in the activation dtype (bf16)
    layer.cfg.prefill_tiles = {"auto": 0, "single": 1, "pair": 2}[args.prefill_tiles]
    cfg = layer.cfg
    L = M.moe_layer_launch_count(cfg)
    n_steps = M.moe_layer_step_count(cfg)
    names = KERNEL_NAMES_TC if sh.expert != "f32" else KERNEL_NAMES_SIMT
    assert len(names) == n_steps

    # routing statistics of this batch (touched experts, kept rows) for the roofline
    counts = torch.empty(sh.E, dtype=torch.int32, device=dev)
    out = layer.forward(x, counts=counts)
    torch.cuda.synchronize()
    kept, touched = routing_stats(sh, T, counts)

    for _ in range(W):
        layer.forward(x, out)
    barrier(world)

    # profiled steps: per-kernel events on up to 256 evenly spread steps
    n_prof = min(K, 256)
    prof_steps = set(np.linspace(0, K - 1, n_prof).round().astype(int).tolist())
    evs = {s: [torch.cuda.Event(enable_timing=True) for _ in range(n_steps + 1)]
           for s in prof_steps}
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    start.record()
    for s in range(K):
        if s in prof_steps:
            M.moe_layer_forward_profiled(cfg, layer.w, x, out, layer.ws, evs[s])
        else:
            layer.forward(x, out)
    end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    assert M.moe_get_device_status(layer.ws) == 0, "device error word set"
    value, ms_max = aggregate_throughput(T * K, ms, world)
    per_kernel = {n: float(np.mean([evs[s][i].elapsed_time(evs[s][i + 1]) for s in prof_steps]))
                  for i, n in enumerate(names)}

    # the peak that applies to a kernel timed inside this loop (burst or sustained)
    peaks = R.measured_peaks()
    tc_peak, peak_label = R.tensor_peak(peaks, ms_max / 1e3, clk.get("sm_mhz"))
    dom = max(per_kernel, key=per_kernel.get)
    dom_ms = per_kernel[dom]
    if dom in ("gateup_gemm", "down_gemm", "router"):
        if dom == "gateup_gemm":
            fl = R.gateup_flops(sh, T, kept)
        elif dom == "down_gemm":
            fl = 2.0 * sh.d * sh.f * (kept + sh.n_shared * T)
        else:
            fl = 2.0 * T * sh.d * sh.E
        ach = fl / (dom_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": round(ach, 2),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(ach / tc_peak, 4),
                "peak_source": peak_label,
                "algorithmic_per_launch": fl, "avg_launch_us": round(dom_ms * 1e3, 2),
                "traffic": read_traffic(dom, sh, T)}
    else:
        nb = R.layer_bytes(sh, T, touched)
        ach = nb / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                "peak_source": f"{peaks['source']} hbm_gbs (copy kernel)",
                "avg_launch_us": round(dom_ms * 1e3, 2), "traffic": None}
    # whole-layer roofline (slower of flops at the tensor peak and bytes over HBM)
    fl_layer = R.layer_flops(sh, T, kept)
    by_layer = R.layer_bytes(sh, T, touched)
    t_roof = R.roofline_time(fl_layer, by_layer, tc_peak * 1e12, peaks["hbm_gbs"] * 1e9)
    layer_roof = {"t_roof_us": round(t_roof * 1e6, 2), "t_step_us": round(ms_max / K * 1e3, 2),
                  "frac": round(t_roof / (ms_max / K / 1e3), 4),
                  "bound": "tensor" if fl_layer / (tc_peak * 1e12)
                  > by_layer / (peaks["hbm_gbs"] * 1e9) else "hbm",
                  "peak_tflops": tc_peak, "peak_gbs": peaks["hbm_gbs"],
                  "flops": fl_layer, "bytes": by_layer, "touched_experts": touched,
                  "kept_rows": kept}

    # end to end through the C ABI with host buffers
    e2e = run_e2e(M, layer, x_host, sh, T, min(K, 100), world)

    res = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
           "steps": K, "warmup": W, "ms_per_step": round(ms_max / K, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,1) tokens, fan-in-scaled random expert weights)",
           "config": dict(config_dict(sh, T, world), prefill_tiles=args.prefill_tiles),
           "roofline": roof, "layer_roofline": layer_roof,
           "e2e": e2e, "gpu_launches": L * K, "launches_per_step": L, "clocks": clk,
           "kernels_avg_us": {k: round(v * 1e3, 2) for k, v in per_kernel.items()}}
    if rank == 0 and world == 1 and not args.no_parity:
        res["parity"] = parity_sample(M, layer, li_host, x_host, x, sh, T)
    if rank == 0 and world == 1 and not args.no_sweep:
        res["sweep"] = run_sweep(M, dev, sh, T, li)
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(li_host, x_host, sh, T)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def run_e2e(M, layer, x_host, sh, T, K, world):
    """The same layer through the C ABI from host memory: every step copies its
    batch from pinned host memory to the device, runs the layer, and copies the
    result back to pinned host memory, all inside the timed region.  Copies run on
    a second stream with two device buffers each way, so that the transfers of
    steps i-1 and i+1 overlap the layer of step i (each step's own copies still
    precede and follow its layer)."""
    xp = x_host.pin_memory()
    outp = [torch.empty(x_host.shape, dtype=layer.out_dtype).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(xp, device="cuda") for _ in range(2)]
    od = [torch.empty(x_host.shape, dtype=layer.out_dtype, device="cuda") for _ in range(2)]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        with torch.cuda.stream(copy):
            xd[0].copy_(xp, non_blocking=True)
            in_ready[0].record(copy)
        for i in range(n):
            b = i & 1
            if i + 1 < n:                       # next step's input, on the copy stream
                nb = (i + 1) & 1
                with torch.cuda.stream(copy):
                    if i >= 1:
                        copy.wait_event(in_free[nb])
                    xd[nb].copy_(xp, non_blocking=True)
                    in_ready[nb].record(copy)
            comp.wait_event(in_ready[b])
            if i >= 2:
                comp.wait_event(out_free[b])
            layer.forward(xd[b], od[b], stream=comp)
            in_free[b].record(comp)
            out_ready[b].record(comp)
            with torch.cuda.stream(copy):       # this step's result back to the host
                copy.wait_event(out_ready[b])
                outp[b].copy_(od[b], non_blocking=True)
                out_free[b].record(copy)
        comp.wait_stream(copy)

    run(3)
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    copy.wait_event(s)                          # no copy starts before the timed region
    run(K)
    e.record(comp)
    torch.cuda.synchronize()
    value, _ = aggregate_throughput(T * K, s.elapsed_time(e), world)
    return {"value": round(value, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(xp.numel() * xp.element_size()),
            "d2h_bytes_per_step": int(outp[0].numel() * outp[0].element_size()), "steps": K,
            "copies": "pinned host buffers; copy-in of step i+1 and copy-out of step i-1 "
                      "overlap the layer of step i on a second stream"}


def parity_sample(M, layer, li_host, x_host, x, sh, T, n_rows=8):
    """This batch's output (FP32, the layer the bench times) against the oracle on
    sampled rows: the oracle routes the whole batch itself (route mismatches and
    drift) and is then re-run with the GPU's routes on the sampled rows (output
    error over RMS(out) and over RMS(out - x))."""
    from moe_layer_fp32_b200.drift import route_drift
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    l32 = M.MoELayer(layer.inputs, T, out_dtype="f32")
    idx = torch.empty(T, sh.k, dtype=torch.int32, device=x.device)
    out = l32.forward(x, topk_idx=idx).float().cpu().numpy()
    gi = idx.cpu().numpy()
    del l32
    r = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, T - 1], r.choice(T, min(T, n_rows) - 2 if T > 2 else 0,
                                                           replace=False)]))
    own = O.layer_from_inputs(li_host, x_host, tokens=[0])
    rep = O.layer_from_inputs(li_host, x_host, forced_idx=gi, tokens=rows)
    diff = (np.sort(gi, 1) != np.sort(own["idx"], 1)).any(1)
    x64 = x_host.float().numpy().astype(np.float64)[rows]
    err = float(np.max(np.abs(out[rows] - rep["out"])))
    return {"rows": int(rows.size), "route_mismatches": int(diff.sum()),
            "max_margin_of_mismatch": float(own["margin"][diff].max()) if diff.any() else 0.0,
            "drift": route_drift(gi, own["idx"]),
            "err_over_rms_out": err / float(np.sqrt(np.mean(rep["out"] ** 2))),
            "err_over_rms_delta": err / float(np.sqrt(np.mean((rep["out"] - x64) ** 2))),
            "oracle_s": round(time.perf_counter() - t0, 1)}


def time_layer(M, layer, x, n):
    """(stream-launched us, CUDA-graph-replayed us) per layer call."""
    o = layer.forward(x)
    for _ in range(10):
        layer.forward(x, o)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(n):
        layer.forward(x, o)
    e.record()
    torch.cuda.synchronize()
    us_stream = s.elapsed_time(e) / n * 1e3
    us_graph = None
    try:
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream()
        with torch.cuda.stream(st):
            layer.forward(x, o, stream=st)
            st.synchronize()
            with torch.cuda.graph(g, stream=st):
                layer.forward(x, o, stream=st)
        for _ in range(10):
            g.replay()
        torch.cuda.synchronize()
        s.record()
        for _ in range(n):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        us_graph = s.elapsed_time(e) / n * 1e3
        del g
    except Exception as ex:  # capture problems are reported, not hidden
        us_graph = f"capture failed: {ex}"
    return us_stream, us_graph


SWEEP = [("olmoe", 1), ("olmoe", 16), ("olmoe", 64), ("olmoe", 4096), ("v2lite", 32),
         ("v2lite", 8192), ("qwen3_int4", 1), ("qwen3_int4", 64), ("qwen3_int4", 16384),
         ("qwen3_int8", 1), ("qwen3_int8", 64), ("qwen3_int8", 16384), ("qwen3_fp8", 1),
         ("qwen3_fp8", 64), ("qwen3_fp8", 16384), ("v3", 32), ("v3", 256),
         ("v3", 9440), ("tiny", 64)]


def run_sweep(M, dev, head_sh, head_T, head_li):
    """Every other configuration: whole-layer time, stream-launched and replayed
    from a CUDA graph, and the fraction of the layer roofline (the slower of the
    flops at the bf16 peak that applies to the loop and the touched-weight bytes
    at the measured HBM bandwidth)."""
    peaks = R.measured_peaks()
    bw = peaks["hbm_gbs"] * 1e9
    rows = []
    cache = {head_sh.name: head_li}
    for name in dict.fromkeys(n for n, _ in SWEEP):
        sh = moe_synth.PRESETS[name]
        li = cache.get(name)
        if li is None:
            li = moe_synth.make_layer(sh).to(dev)
        for pname, T in SWEEP:
            if pname != name or (name == head_sh.name and T == head_T):
                continue
            x = moe_synth.make_x(sh, T).to(dev)
            layer = M.MoELayer(li, T)
            counts = torch.empty(sh.E, dtype=torch.int32, device=dev)
            layer.forward(x, counts=counts)
            torch.cuda.synchronize()
            kept, touched = routing_stats(sh, T, counts)
            n = 40 if T >= 4096 else 400
            us_s, us_g = time_layer(M, layer, x, n)
            best = min(us_s, us_g) if isinstance(us_g, float) else us_s
            pf, _ = R.tensor_peak(peaks, best * n / 1e6)
            fl, nb = R.layer_flops(sh, T, kept), R.layer_bytes(sh, T, touched)
            t_roof = R.roofline_time(fl, nb, pf * 1e12, bw)
            rows.append({"workload": workload_name(sh, T), "T": T, "touched": touched,
                         "kept": kept, "launches": M.moe_layer_launch_count(layer.cfg),
                         "us_stream": round(us_s, 1),
                         "us_graph": round(us_g, 1) if isinstance(us_g, float) else us_g,
                         "tokens_per_s": round(T / (best / 1e6), 1),
                         "roofline_us": round(t_roof * 1e6, 1),
                         "bound": "tensor" if fl / (pf * 1e12) > nb / bw else "hbm",
                         "frac": round(t_roof * 1e6 / best, 4)})
            del layer
        if name != head_sh.name:
            del li
        torch.cuda.empty_cache()
    return rows


def cpu_baseline(li_host, x_host, sh, T):
    """The oracle, as it stands, on the host cores: the first tokens of the same
    batch (routing over that sub-batch, every expert they touch), once on all
    the threads numpy's BLAS uses and once on a single thread."""
    n = min(T, 32 if sh.d >= 4096 else 512)
    sec = time_oracle(li_host, x_host, n)
    res = {"value": round(n / sec, 2), "unit": "tokens/s", "cores": cpu_threads(),
           "kind": "oracle", "sample": f"first {n} of the {T} tokens of the timed batch, one "
                                       f"call ({sec:.1f} s), numpy float64"}
    try:
        import threadpoolctl
        n1 = max(1, n // 4)
        with threadpoolctl.threadpool_limits(limits=1):
            sec1 = time_oracle(li_host, x_host, n1)
        res["single_thread"] = {"value": round(n1 / sec1, 2), "unit": "tokens/s", "cores": 1,
                                "sample": f"first {n1} tokens, one call ({sec1:.1f} s)"}
    except Exception as ex:  # reported, not hidden
        res["single_thread"] = f"unavailable: {ex}"
    return res


# --------------------------------------------------------------------- traffic
def code_of(text):
    """CUDA source without its // comments, trailing blanks and empty lines: what
    the compiler sees (the kernel sources hold no // inside string literals)."""
    lines = []
    for line in text.splitlines():
        i = line.find("//")
        if i >= 0:
            line = line[:i]
        line = line.rstrip()
        if line:
            lines.append(line)
    return "\n".join(lines) + "\n"


def kernel_source_digest():
    """First 16 hex digits of the SHA-256 of the GEMM kernel sources' code
    (common.cuh, then gemm_tc.cuh), comments excluded."""
    import hashlib
    src = os.path.join(ROOT, "moe_layer_fp32_b200", "csrc")
    h = hashlib.sha256()
    for f in ("common.cuh", "gemm_tc.cuh"):
        with open(os.path.join(src, f)) as fh:
            h.update(code_of(fh.read()).encode())
    return h.hexdigest()[:16]


def read_traffic(kernel, sh, T):
    """DRAM bytes per launch of this kernel from the committed ncu summary, if
    that summary was taken on the current kernel code."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{sh.name}_T{T}.md")
    if not os.path.exists(path):
        return None
    digest = kernel_source_digest()
    vals = {}
    with open(path) as fh:
        for line in fh:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != digest:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------- reference arm
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sh = moe_synth.PRESETS[args.preset]
    T, K, W = args.tokens, args.steps, max(args.warmup, 3)
    li = moe_synth.make_layer(sh)
    x = moe_synth.make_x(sh, T)
    # size each step's sample so the whole run takes a few minutes
    probe = time_oracle(li, x, 1)
    target_s = 150.0   # seconds for the whole reference run
    per_step = target_s / (K + W)
    n_tok = 1
    if per_step > 2 * probe:
        n_tok = int(min(T, max(1, (per_step / probe))))
    for _ in range(W):
        time_oracle(li, x, n_tok)
    t0 = time.perf_counter()
    for _ in range(K):
        time_oracle(li, x, n_tok)
    sec = time.perf_counter() - t0
    value = n_tok * K / sec
    cores = cpu_threads()
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
           "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(sec / K * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded N(0,1) tokens, fan-in-scaled random expert weights)",
           "config": config_dict(sh, T, 1),
           "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                            "kind": "oracle",
                            "sample": f"each step: the oracle on the first {n_tok} token(s) of "
                                      f"the T={T} batch (routing over that sub-batch)"},
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
