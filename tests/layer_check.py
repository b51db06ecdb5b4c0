"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and the
CPU oracle on the same seeded inputs, and compare them.

Tolerances (each derived from the arithmetic of the path):
* routing indices, counts, offsets, permutation: bit-exact given the same FP32
  logits; end to end, a token may differ from the oracle's selection only where
  the oracle's k-th/(k+1)-th key margin is below 1e-4;
* bf16 experts: max|out - out_oracle| / RMS(out_oracle) <= 1e-2 on the FP32
  layer output, against the oracle re-run with the GPU's routes; int8 / int4
  / fp8 experts: <= 3e-2 (the same oracle, same dequantised weights); fp32 experts:
  <= 1e-5.  The ratio against RMS(out_oracle - x) (the MoE delta alone) is
  reported beside it and held under DELTA_GUARD.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

import moe_layer_fp32_b200 as M
import moe_synth
from moe_layer_fp32_b200.drift import route_drift
from oracle import moe_oracle as O

ROUTE_MARGIN = 1e-4
TOL = {"f32": 1e-5, "bf16": 1e-2, "int8": 3e-2, "int4": 3e-2, "fp8": 3e-2}
DELTA_GUARD = {"f32": 1e-4, "bf16": 3e-2, "int8": 6e-2, "int4": 6e-2, "fp8": 6e-2}


def inputs_on_device(shape, T, x_stream=None):
    li = moe_synth.make_layer(shape)
    x = moe_synth.make_x(shape, T, x_stream)
    return li, x, li.to("cuda"), x.cuda()


@dataclass
class LayerResult:
    out: np.ndarray            # [T, d] fp32 (GPU)
    logits: np.ndarray
    idx: np.ndarray
    counts: np.ndarray
    mismatched: int            # tokens whose selection differs from the oracle's
    max_margin_mismatch: float
    err_ratio: float           # max|out - ref| / RMS(ref) on the compared rows
    err_ratio_delta: float     # max|out - ref| / RMS(ref - x)
    rows: np.ndarray
    drift: dict                # swaps per token and Jaccard against the oracle's routes


def route_mismatches(gpu_idx, oracle_idx):
    a = np.sort(gpu_idx, axis=1)
    b = np.sort(oracle_idx, axis=1)
    return np.nonzero((a != b).any(axis=1))[0]


def run_layer(shape, T, tokens: Optional[Sequence[int]] = None, x_stream=None,
              out_dtype="f32", data=None) -> LayerResult:
    li, x, dli, dx = data if data is not None else inputs_on_device(shape, T, x_stream)
    layer = M.MoELayer(dli, T, out_dtype=out_dtype)
    logits = torch.empty(T, shape.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, shape.k, dtype=torch.int32, device="cuda")
    counts = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    out = layer.forward(dx, logits=logits, topk_idx=idx, counts=counts)
    assert M.moe_get_device_status(layer.ws) == 0
    out = out.float().cpu().numpy()
    gi = idx.cpu().numpy()
    gl = logits.cpu().numpy()
    gc = counts.cpu().numpy()
    # oracle with its own routing (full batch; experts on the sampled rows only)
    own = O.layer_from_inputs(li, x, tokens=[0])
    mism = route_mismatches(gi, own["idx"])
    mmax = float(own["margin"][mism].max()) if mism.size else 0.0
    # replay the GPU's routes through the oracle for the output comparison
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    rep = O.layer_from_inputs(li, x, forced_idx=gi, tokens=rows)
    np.testing.assert_array_equal(gc, rep["counts"])
    x64 = x.float().numpy().astype(np.float64)[rows]
    delta = rep["out"] - x64
    rms_d = float(np.sqrt(np.mean(delta ** 2)))
    rms_o = float(np.sqrt(np.mean(rep["out"] ** 2)))
    err = float(np.max(np.abs(out[rows] - rep["out"])))
    return LayerResult(out, gl, gi, gc, int(mism.size), mmax, err / rms_o, err / rms_d, rows,
                       route_drift(gi, own["idx"]))


def sample_rows(T, n=48, seed=0):
    if T <= n:
        return np.arange(T)
    r = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, T - 1], r.choice(T, n - 2, replace=False)]))
