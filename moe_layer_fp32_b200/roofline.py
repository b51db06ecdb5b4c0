"""Roofline arithmetic for the MoE layer (host logic, no device code).

* Algorithmic bytes of one layer forward: the expert weights of every expert
  that received at least one kept token, the shared experts, the router, and
  x in / out out.  Intermediates (gathered rows, h, per-assignment outputs) are
  implementation cost and are not counted.  ("MoE at the inference level ...",
  Arithmetic intensity: the weight stream sets the bytes; "MoE Research",
  section 7 A: experts touched at batch B is E (1 - (1 - k/E)^B).)
* Algorithmic flops: 6 d f per kept (token, expert) pair and per shared-expert
  token (three GEMMs of 2 d f), plus 2 T d E for the router.
* Roofline time: max(flops / tensor peak, bytes / HBM bandwidth).

Also the pages' own arithmetic (Amdahl ceiling, all-to-all bytes, ridge batch),
used to pin these helpers against the numbers the pages print.
"""
from __future__ import annotations

import json
import os
from typing import Optional, Sequence

BYTES_PER_WEIGHT = {"f32": 4.0, "bf16": 2.0, "int8": 1.0, "fp8": 1.0, "int4": 0.5}


def scale_bytes_per_expert(expert: str, d: int, f: int, group: int = 128) -> float:
    """bf16 scale bytes of one expert's three matrices."""
    if expert in ("int8", "fp8"):
        return 2.0 * (f + f + d)                      # per output column
    if expert == "int4":
        return 2.0 * (2 * (d // group) * f + (f // group) * d)
    return 0.0


def expert_bytes(expert: str, d: int, f: int, group: int = 128) -> float:
    return 3.0 * d * f * BYTES_PER_WEIGHT[expert] + scale_bytes_per_expert(expert, d, f, group)


def layer_bytes(shape, T: int, touched: int, out_bytes: Optional[float] = None) -> float:
    act = 2.0 if shape.act == "bf16" else 4.0
    ob = act if out_bytes is None else out_bytes
    eb = expert_bytes(shape.expert, shape.d, shape.f, shape.group_size)
    router = shape.d * shape.E * (2.0 if shape.router == "bf16" else 4.0)
    return touched * eb + shape.n_shared * eb + router + T * shape.d * (act + ob)


def layer_flops(shape, T: int, kept: int) -> float:
    return 6.0 * shape.d * shape.f * (kept + shape.n_shared * T) + 2.0 * T * shape.d * shape.E


def gateup_flops(shape, T: int, kept: int) -> float:
    """flops of the gate/up grouped GEMM: two GEMMs of 2 d f per row."""
    return 4.0 * shape.d * shape.f * (kept + shape.n_shared * T)


def gateup_bytes(shape, T: int, kept: int, touched: int) -> float:
    """Algorithmic bytes of the gate/up GEMM: gate+up weights of the touched
    (and shared) experts, the gathered activation rows in, the bf16 h rows out."""
    w = 2.0 * shape.d * shape.f * BYTES_PER_WEIGHT[shape.expert]
    rows = kept + shape.n_shared * T
    return (touched + shape.n_shared) * w + rows * shape.d * 2.0 + rows * shape.f * 2.0


def roofline_time(flops: float, nbytes: float, peak_flops: float, peak_bw: float) -> float:
    return max(flops / peak_flops, nbytes / peak_bw)


def experts_touched_expected(E: int, k: int, B: int) -> float:
    return E * (1.0 - (1.0 - k / E) ** B)


# --------------------------------------------------------------- page arithmetic
def amdahl(f: float, s: float) -> float:
    """Overall speedup when a fraction f of the time runs s times faster."""
    return 1.0 / ((1.0 - f) + f / s)


def all_to_all_bytes(B: int, k: int, d: int, bytes_per_elem: int = 2) -> int:
    return B * k * d * bytes_per_elem


def ridge_batch(ridge_flop_per_byte: float, E: int, k: int) -> float:
    """Batch at which k/E-sparse MoE decode reaches the ridge (AI = B k / E)."""
    return ridge_flop_per_byte * E / k


# --------------------------------------------------------------- peaks
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# a timed loop at least this long runs into the power cap: the sustained peak
# applies; a shorter one is a burst
SUSTAINED_AFTER_S = 2.0


def tensor_peak(peaks: dict, timed_loop_s: float, sm_mhz=None) -> tuple:
    """(bf16 TFLOP/s, label) that applies to a kernel timed inside a loop of
    ``timed_loop_s`` seconds: the burst figure (a cuBLAS GEMM timed alone) for a
    short loop, the sustained one (the same GEMM back to back for seconds, under
    the power cap) for a loop of SUSTAINED_AFTER_S or more."""
    src = peaks.get("source", "measured")
    clk = f", median SM clock {sm_mhz:.0f} MHz" if sm_mhz else ""
    if timed_loop_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks:
        return (float(peaks["bf16_tflops_sustained"]),
                f"{src} bf16_tflops_sustained: the timed loop ran {timed_loop_s * 1e3:.0f} ms "
                f"(>= {SUSTAINED_AFTER_S:.0f} s, power-capped regime{clk})")
    return (float(peaks["bf16_tflops"]),
            f"{src} bf16_tflops (burst): the timed loop ran {timed_loop_s * 1e3:.0f} ms "
            f"(< {SUSTAINED_AFTER_S:.0f} s{clk})")


def measured_peaks(path: Optional[str] = None) -> dict:
    """Peaks measured on this kind of GPU (MEASURED_PEAKS.json at the repository
    root: a copy-kernel HBM bandwidth and cuBLAS bf16 throughput), else the
    fallback figures above."""
    path = path or os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                                "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return dict(d, source="measured")
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")
