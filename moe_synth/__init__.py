"""Seeded synthetic inputs for the top-k Mixture-of-Experts FFN layer forward.

This module draws the inputs that both the CUDA path and the CPU oracle consume.
It holds none of the layer's own arithmetic: it draws random tensors, encodes
expert weights into the int8 / int4 storage formats, and builds the per-expert
router bias that skews expert popularity.

Recipe (every tensor draws from its own PCG64 stream,
``SeedSequence([seed, tensor_id, chunk])``):

* ``x ~ N(0, 1)`` per element, rounded to bf16 (round-to-nearest-even) or kept
  fp32; each token count T draws from its own stream (chunk = T).
* RMSNorm gain ``gamma = 1`` (fp32).
* Router ``W_r ~ N(0, 1/d)``, experts ``W_gate, W_up ~ N(0, 1/d)`` and
  ``W_down ~ N(0, 1/f)`` (fan-in scaling), one stream per expert.
* Router bias:
  - ``logit`` mode (OLMoE-shaped): ``bias_e = beta * z_e``, ``z ~ N(0,1)``; beta is
    the constant ``OLMOE_BIAS_BETA`` found by ``oracle/calibrate_bias.py`` so that
    the busiest expert carries about 1.5x the mean load at T = 4096.
  - ``select`` mode (DeepSeek-V3-shaped): Zipf(1.1) popularity
    ``p_r ~ r^-1.1`` over a seeded permutation of the experts,
    ``bias_e = ln p_e - mean(ln p)``.
* int8 weights: symmetric, one bf16 scale per output column,
  ``s = bf16(max|w| / 127)``, ``q = clamp(rint(w / s), -127, 127)``.
* Quantised codes (int8, int4, fp8) are stored with the reduction dim K
  contiguous, i.e. as the transpose of the [K, N] weight: ``[E, N, K]`` (int4:
  ``[E, N, K/2]``), so that one output feature's codes of a K block are adjacent.
* fp8 weights: FP8 E4M3 codes, one bf16 scale per output column,
  ``s = bf16(max|w| / 448)``, ``q = e4m3(w / s)`` (round to nearest even).
* int4 weights: symmetric, groups of ``group_size`` along the reduction (K) dim,
  ``s = bf16(max|w| / 7)``, ``q = clamp(rint(w / s), -8, 7)``; two values per byte
  along the contiguous (K) dim, eight per 4-byte word: nibble j of the
  little-endian word holds code 8w + (0, 2, 4, 6, 1, 3, 5, 7)[j].

Weight layouts follow the layer's statement of the problem: ``W_r[d, E]``,
``W_gate/W_up[E, d, f]``, ``W_down[E, f, d]``; shared experts ``[S, d, f]`` and
``[S, f, d]``; quantised codes transposed (``[E, f, d]`` and ``[E, d, f]``, int4
with the last dim halved).  int8 / fp8 scales are ``[E, f]`` (gate/up) and
``[E, d]`` (down); int4 scales are ``[E, d/G, f]`` (gate/up) and ``[E, f/G, d]``
(down).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np
import torch

# beta for the OLMoE-shaped logit-mode bias; written by oracle/calibrate_bias.py
OLMOE_BIAS_BETA = 0.1044921875

# stream ids, one per tensor
_TID = dict(x=1, w_router=3, bias_z=4, w_gate=5, w_up=6, w_down=7,
            sh_gate=8, sh_up=9, sh_down=10, zipf_perm=11)


@dataclass(frozen=True)
class LayerShape:
    """One MoE layer configuration (sizes, dtypes and routing options)."""
    name: str
    d: int                      # model dim
    E: int                      # routed experts
    k: int                      # experts per token
    f: int                      # expert hidden dim
    n_shared: int = 0           # always-on shared experts (hidden f each)
    act: str = "bf16"           # x / out dtype: "bf16" | "f32"
    router: str = "bf16"        # router weight dtype: "bf16" | "f32"
    expert: str = "bf16"        # "f32" | "bf16" | "int8" | "int4" | "fp8"
    renormalize: bool = True    # gates renormalised over the selected k
    bias_mode: str = "none"     # "none" | "logit" | "select"
    capacity_factor: float = 0.0  # <= 0: uncapped
    rms_eps: float = 1e-6
    group_size: int = 128       # int4 group along K
    seed: int = 0
    tokens: Tuple[int, ...] = (64,)
    routing: str = "topk"       # "topk" | "expert_choice"

    def with_(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)


PRESETS: Dict[str, LayerShape] = {
    # Tiny layer: fp32 weights, renormalised gates, uncapped, seed 0
    "tiny": LayerShape("tiny", d=256, E=8, k=2, f=512, act="f32", router="f32",
                       expert="f32", renormalize=True, seed=0, tokens=(64,)),
    # OLMoE-1B-7B-shaped layer with a logit-mode bias (busiest expert ~1.5x mean)
    "olmoe": LayerShape("olmoe", d=2048, E=64, k=8, f=1024, bias_mode="logit",
                        seed=1, tokens=(1, 16, 64, 4096)),
    # DeepSeek-V2-Lite-shaped layer: 2 shared experts, capacity-factor mode
    "v2lite": LayerShape("v2lite", d=2048, E=64, k=6, f=1408, n_shared=2,
                         capacity_factor=1.25, seed=2, tokens=(32, 8192)),
    # Qwen3-30B-A3B-shaped layer, int4 g128 experts, bf16 router
    "qwen3_int4": LayerShape("qwen3_int4", d=2048, E=128, k=8, f=768, expert="int4",
                             seed=3, tokens=(1, 64, 16384)),
    # the same layer with int8 per-channel experts
    "qwen3_int8": LayerShape("qwen3_int8", d=2048, E=128, k=8, f=768, expert="int8",
                             seed=3, tokens=(1, 64, 16384)),
    # the same layer with FP8 (E4M3) per-channel experts
    "qwen3_fp8": LayerShape("qwen3_fp8", d=2048, E=128, k=8, f=768, expert="fp8",
                            seed=3, tokens=(1, 64, 16384)),
    # DeepSeek-V3-shaped layer: 1 shared expert, Zipf(1.1) select-mode bias
    "v3": LayerShape("v3", d=7168, E=256, k=8, f=2048, n_shared=1, bias_mode="select",
                     seed=4, tokens=(32, 256, 9440)),
    # profiling case of the V3-shaped expert GEMMs: the same d, f, k, shared expert and
    # select-mode bias over 32 experts (2.9 GB of weights), T = 1184 giving the same
    # 296 rows per expert on average as the V3-shaped T = 9440 batch
    "v3_e32": LayerShape("v3_e32", d=7168, E=32, k=8, f=2048, n_shared=1,
                         bias_mode="select", seed=4, tokens=(1184,)),
}


def _rng(seed: int, tid: int, chunk: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, tid, chunk]))


def _normal(seed: int, tid: int, chunk: int, shape, std: float) -> np.ndarray:
    a = _rng(seed, tid, chunk).standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(std)
    return a


def _to_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(a)
    if dtype == "bf16":
        return t.to(torch.bfloat16)       # round-to-nearest-even
    if dtype == "f32":
        return t.to(torch.float32)
    raise ValueError(dtype)


def make_x(shape: LayerShape, T: int, stream: Optional[int] = None) -> torch.Tensor:
    """x[T, d] ~ N(0,1) in the activation dtype (host tensor)."""
    chunk = T if stream is None else stream
    return _to_dtype(_normal(shape.seed, _TID["x"], chunk, (T, shape.d), 1.0), shape.act)


def make_gamma(shape: LayerShape) -> torch.Tensor:
    return torch.ones(shape.d, dtype=torch.float32)


def make_router(shape: LayerShape) -> torch.Tensor:
    w = _normal(shape.seed, _TID["w_router"], 0, (shape.d, shape.E), shape.d ** -0.5)
    return _to_dtype(w, shape.router)


def make_router_bias(shape: LayerShape) -> Optional[torch.Tensor]:
    if shape.bias_mode == "none":
        return None
    if shape.bias_mode == "logit":
        z = _rng(101, _TID["bias_z"]).standard_normal(shape.E)
        return torch.tensor(OLMOE_BIAS_BETA * z, dtype=torch.float32)
    if shape.bias_mode == "select":
        perm = _rng(shape.seed, _TID["zipf_perm"]).permutation(shape.E)
        ranks = np.empty(shape.E, dtype=np.float64)
        ranks[perm] = np.arange(1, shape.E + 1, dtype=np.float64)
        logp = -1.1 * np.log(ranks)
        logp -= np.log(np.exp(logp).sum())
        return torch.tensor(logp - logp.mean(), dtype=torch.float32)
    raise ValueError(shape.bias_mode)


def master_expert(shape: LayerShape, which: str, e: int, shared: bool = False) -> np.ndarray:
    """fp32 master weights of one expert matrix before rounding / quantisation.

    ``which`` is "gate", "up" or "down"; gate/up are [d, f], down is [f, d].
    """
    tid = _TID[("sh_" if shared else "w_") + which]
    if which in ("gate", "up"):
        return _normal(shape.seed, tid, e, (shape.d, shape.f), shape.d ** -0.5)
    return _normal(shape.seed, tid, e, (shape.f, shape.d), shape.f ** -0.5)


def quantize_int8(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """w[K, N] fp32 -> (q int8 stored [N, K], s bf16 [N]); one scale per output
    column.  The codes are stored with K contiguous (the transpose of w)."""
    amax = w.abs().amax(dim=0)
    s = (amax / 127.0).to(torch.bfloat16)
    s = torch.where(s.float() > 0, s, torch.ones_like(s))
    q = torch.round(w / s.float()).clamp_(-127, 127).to(torch.int8)
    return q.t().contiguous(), s


def quantize_fp8(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """w[K, N] fp32 -> (q uint8 FP8 E4M3 codes stored [N, K], s bf16 [N]); one scale
    per output column, ``s = bf16(max|w| / 448)``, ``q = e4m3(w / s)`` rounded to
    nearest even and clamped to the largest finite code (448); K contiguous."""
    amax = w.abs().amax(dim=0)
    s = (amax / 448.0).to(torch.bfloat16)
    s = torch.where(s.float() > 0, s, torch.ones_like(s))
    q = (w / s.float()).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).t().contiguous(), s


def quantize_int4(w: torch.Tensor, group: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """w[K, N] fp32 -> (packed uint8 [N, K/2], s bf16 [K/group, N]).

    Groups of ``group`` rows along K share a scale per column.  The codes are
    stored with K contiguous (the transpose of w), eight codes per 4-byte word:
    nibble j of the little-endian word holds code 8w + (0, 2, 4, 6, 1, 3, 5, 7)[j]
    (the even codes in the low nibbles of its bytes, the odd ones in the high).
    """
    K, N = w.shape
    wg = w.view(K // group, group, N)
    amax = wg.abs().amax(dim=1)
    s = (amax / 7.0).to(torch.bfloat16)
    s = torch.where(s.float() > 0, s, torch.ones_like(s))
    q = torch.round(wg / s.float().unsqueeze(1)).clamp_(-8, 7).to(torch.int16).view(K, N)
    qt = q.t().contiguous().view(N, K // 8, 8)
    nib = qt[:, :, [0, 2, 4, 6, 1, 3, 5, 7]].reshape(N, K) & 0xF   # nibble j of each word
    lo = nib[:, 0::2]
    hi = nib[:, 1::2] << 4
    return (lo | hi).to(torch.uint8).contiguous(), s


def _encode(shape: LayerShape, w: np.ndarray):
    """Round or quantise one [K, N] matrix to the expert storage dtype."""
    if shape.expert in ("bf16", "f32"):
        return (_to_dtype(w, shape.expert), None)
    t = torch.from_numpy(w)
    if shape.expert == "int8":
        return quantize_int8(t)
    if shape.expert == "fp8":
        return quantize_fp8(t)
    if shape.expert == "int4":
        return quantize_int4(t, shape.group_size)
    raise ValueError(shape.expert)


def make_expert_stack(shape: LayerShape, which: str, shared: bool = False,
                      experts: Optional[range] = None, device="cpu"):
    """Stacked weights (and scales, None for f32/bf16) for one matrix kind."""
    n = shape.n_shared if shared else shape.E
    ids = list(range(n) if experts is None else experts)
    ws, ss = [], []

    def one(e):
        return _encode(shape, master_expert(shape, which, e, shared))

    # experts draw from independent streams: generate them on a few host threads
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for q, s in ex.map(one, ids):
            ws.append(q.to(device))
            if s is not None:
                ss.append(s.to(device))
    W = torch.stack(ws) if ws else None
    S = torch.stack(ss) if ss else None
    return W, S


@dataclass
class LayerInputs:
    shape: LayerShape
    gamma: torch.Tensor
    w_router: torch.Tensor
    router_bias: Optional[torch.Tensor]
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    s_gate: Optional[torch.Tensor] = None
    s_up: Optional[torch.Tensor] = None
    s_down: Optional[torch.Tensor] = None
    sh_gate: Optional[torch.Tensor] = None
    sh_up: Optional[torch.Tensor] = None
    sh_down: Optional[torch.Tensor] = None
    sh_s_gate: Optional[torch.Tensor] = None
    sh_s_up: Optional[torch.Tensor] = None
    sh_s_down: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "LayerInputs":
        kw = {}
        for fld in dataclasses.fields(self):
            v = getattr(self, fld.name)
            kw[fld.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return LayerInputs(**kw)


def make_layer(shape: LayerShape, device="cpu") -> LayerInputs:
    """All weights of one layer (host tensors unless ``device`` says otherwise)."""
    g, sg = make_expert_stack(shape, "gate", device=device)
    u, su = make_expert_stack(shape, "up", device=device)
    dn, sd = make_expert_stack(shape, "down", device=device)
    li = LayerInputs(shape, make_gamma(shape).to(device), make_router(shape).to(device),
                     None, g, u, dn, sg, su, sd)
    b = make_router_bias(shape)
    li.router_bias = None if b is None else b.to(device)
    if shape.n_shared:
        li.sh_gate, li.sh_s_gate = make_expert_stack(shape, "gate", True, device=device)
        li.sh_up, li.sh_s_up = make_expert_stack(shape, "up", True, device=device)
        li.sh_down, li.sh_s_down = make_expert_stack(shape, "down", True, device=device)
    return li
