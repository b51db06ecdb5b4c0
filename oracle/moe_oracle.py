"""CPU oracle for the top-k Mixture-of-Experts FFN layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm call it.  It shares no code with the CUDA library.

Plain numpy in float64.  Where the layer fixes a narrower type (the bf16
activations the expert GEMMs consume, the FP32 router logits on which the
top-k decision is taken) the oracle rounds to that type explicitly, once, with
round-to-nearest-even.

Sources (page title, then section):

* "MoE: dynamism the compiler cannot remove", natural implementation: the
  router's logits give each token its top-k experts and weights, each selected
  expert's output for the token is weighted by its gate and added to the
  token's output row.  ``moe_layer`` evaluates exactly that definition: every
  kept assignment (t, j) contributes ``g[t, j] * FFN_{idx[t, j]}(xn[t])`` to row
  t, summed in j order after the residual and the shared experts.
* same page, capacity section: each expert holds at most ``C * T*k/E`` tokens;
  overflow tokens skip the FFN and pass through on the residual.
* picx.dev summary of the moe-ceilings study, Sub-study 1 (FusedSoftmax):
  gate probabilities are accumulated in FP32 before the top-k.
* same summary, Theoretical Foundation: the top-k selection is discrete; a
  perturbation smaller than the smallest logit margin changes nothing.
* "MoE Research", section 2: shared (always-on) experts; per-expert bias terms
  (auxiliary-loss-free balancing).
* "MoE at the inference level ...", Workarounds: gather -> grouped GEMM ->
  scatter; int4 expert weights.

Readings where the pages are silent:

* RMSNorm: ``xn = x * (mean(x^2) + eps)^-1/2 * gamma``, computed in float64 and
  rounded once to the activation dtype (bf16 or fp32) -- the experts and the
  router consume that tensor.
* Selection key: FP32 ``logit (+ bias)``; descending, ties to the lower expert
  index; ``idx[t, :]`` is emitted in that order.
* Gates: softmax over all E of the FP32 logits (bias included only in "logit"
  mode), evaluated in float64; optionally renormalised over the selected k.
* Capacity: ``cap = ceil(C*T*k/E)`` in double; slots are ranked in flat order
  ``a = t*k + j`` and slot ``a`` is kept iff its rank within its expert is
  ``< cap``.  Kept slots keep their gate (no re-renormalisation).
* Expert: SwiGLU, ``y = (silu(xn Wg) * (xn Wu)) Wd``.
* Combine: ``out = x + sum_s shared_s(xn) + sum_{kept j} g_j * y_j``.
* fp8 weights (E4M3 codes with one bf16 scale per output column, "MoE at the
  inference level", Workarounds: int4/fp8 expert weights) dequantise the same
  way, ``bf16(e4m3(q) * s)``.
* int8 and int4 weights dequantise to ``bf16(q * s)`` (the exact product rounded
  once to bf16): the layer's tensor-core GEMMs consume bf16 weights.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

BIAS_NONE, BIAS_LOGIT, BIAS_SELECT = "none", "logit", "select"


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------
def round_to_format(a, mant_bits: int, min_exp: int = -126) -> np.ndarray:
    """Round float64 values to a binary format with ``mant_bits`` stored mantissa
    bits and minimum normal exponent ``min_exp`` (round-to-nearest-even).

    bf16: mant_bits=7; fp32: mant_bits=23; both have min_exp=-126.  The grid
    spacing at |a| in [2^e, 2^(e+1)) is 2^(max(e, min_exp) - mant_bits); scaling
    by a power of two is exact, and ``np.round`` rounds half to even.
    """
    a = np.asarray(a, dtype=np.float64)
    _, ex = np.frexp(a)                      # a = m * 2^ex, 0.5 <= |m| < 1
    e = np.maximum(ex.astype(np.int64) - 1, min_exp)
    spacing = np.ldexp(1.0, e - mant_bits)
    out = np.round(a / spacing) * spacing
    return np.where(a == 0, a, out)


def round_bf16(a) -> np.ndarray:
    return round_to_format(a, 7)


def round_f32(a) -> np.ndarray:
    return round_to_format(a, 23)


def round_act(a, act: str) -> np.ndarray:
    return round_bf16(a) if act == "bf16" else round_f32(a)


# ---------------------------------------------------------------------------
# a1: RMSNorm
# ---------------------------------------------------------------------------
def rmsnorm(x, gamma, eps: float, act: str) -> np.ndarray:
    """Pre-norm RMSNorm of each token row, rounded once to the activation dtype.

    ``eps`` is taken as the fp32 value the layer's configuration carries.
    """
    x = np.asarray(x, dtype=np.float64)
    eps = float(np.float32(eps))
    ms = np.sum(x * x, axis=1) / x.shape[1]
    r = 1.0 / np.sqrt(ms + eps)
    xn = (x * r[:, None]) * np.asarray(gamma, dtype=np.float64)[None, :]
    return round_act(xn, act)


# ---------------------------------------------------------------------------
# a2: router GEMM
# ---------------------------------------------------------------------------
def router_logits(xn, w_router) -> np.ndarray:
    """logits[T, E] = xn[T, d] . W_r[d, E] in float64."""
    return np.asarray(xn, np.float64) @ np.asarray(w_router, np.float64)


# ---------------------------------------------------------------------------
# a3: selection key, top-k, softmax gates
# ---------------------------------------------------------------------------
def selection_keys(logits32, bias, bias_mode: str):
    """(keys, softmax inputs), both FP32.  NaN keys order below every number."""
    l = np.asarray(logits32, dtype=np.float32)
    if bias_mode == BIAS_NONE or bias is None:
        s, p_in = l, l
    else:
        b = np.asarray(bias, dtype=np.float32)[None, :]
        s = (l + b).astype(np.float32)
        p_in = s if bias_mode == BIAS_LOGIT else l
    s = np.where(np.isnan(s), np.float32(-np.inf), s)
    return s, p_in


def topk_sorted(keys, k: int):
    """Full sort of every row by (key descending, expert ascending); first k.

    Returns (idx[T, k] int32, margin[T] float64) where margin is the gap between
    the k-th and (k+1)-th keys (inf when k == E).
    """
    keys = np.asarray(keys, dtype=np.float32)
    T, E = keys.shape
    experts = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((experts, -keys.astype(np.float64)), axis=1)
    idx = order[:, :k].astype(np.int32)
    ks = np.take_along_axis(keys, order, axis=1).astype(np.float64)
    if k < E:
        margin = ks[:, k - 1] - ks[:, k]
    else:
        margin = np.full(T, np.inf)
    return idx, margin


def softmax64(p_in) -> np.ndarray:
    p = np.asarray(p_in, dtype=np.float64)
    m = np.max(p, axis=1, keepdims=True)
    e = np.exp(p - m)
    return e / np.sum(e, axis=1, keepdims=True)


def route(logits32, bias, k: int, bias_mode: str, renormalize: bool,
          forced_idx=None):
    """Top-k routing of FP32 logits.

    Returns dict(idx, gates, margin, probs).  With ``forced_idx`` the selection
    is replaced by the given indices (route replay) and only the gates are
    computed.
    """
    keys, p_in = selection_keys(logits32, bias, bias_mode)
    idx, margin = topk_sorted(keys, k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, dtype=np.int32)
    probs = softmax64(p_in)
    gates = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    if renormalize:
        gates = gates / np.sum(gates, axis=1, keepdims=True)
    return dict(idx=idx, gates=gates, margin=margin, probs=probs, keys=keys)


# ---------------------------------------------------------------------------
# expert-choice routing (the inverted assignment)
# ---------------------------------------------------------------------------
def expert_choice_capacity(capacity_factor: float, T: int, k: int, E: int) -> int:
    """Tokens each expert picks: ceil(C * T*k/E) with C = 1 when the factor is <= 0
    (the balanced case, C = 1.0 exact), at most T."""
    c = float(np.float32(capacity_factor))
    if c <= 0:
        c = 1.0
    return int(min(T, math.ceil(c * T * k / E)))


def expert_choice_scores(logits32, bias, bias_mode: str) -> np.ndarray:
    """Affinity of every (token, expert): the softmax over the experts of the FP32
    logits (plus the bias in "logit" mode), in float64, as FP32 values."""
    if bias_mode == BIAS_SELECT:
        raise ValueError("expert-choice routing takes no selection-only bias")
    _, p_in = selection_keys(logits32, bias, bias_mode)
    return round_f32(softmax64(p_in))


def expert_choice_select(scores32, C: int) -> Dict[str, np.ndarray]:
    """Each expert e picks the C tokens with the largest score[t, e] (ties to the
    lower token; NaN scores below every number).

    tok[e, c]    the c-th picked token of expert e, in ascending token order
    gate[e, c]   its score (the gate of that assignment)
    slot[t, e]   e*C + c if token t was picked by e, else -1
    margin[e]    gap between the C-th and (C+1)-th largest scores of e (inf if C == T)
    """
    s = np.asarray(scores32, dtype=np.float32)
    T, E = s.shape
    key = np.where(np.isnan(s), -np.inf, s).astype(np.float64)
    tok = np.empty((E, C), dtype=np.int64)
    gate = np.empty((E, C), dtype=np.float64)
    slot = np.full((T, E), -1, dtype=np.int64)
    margin = np.full(E, np.inf)
    tokens = np.arange(T)
    for e in range(E):
        order = np.lexsort((tokens, -key[:, e]))          # score descending, token ascending
        picked = np.sort(order[:C])
        tok[e] = picked
        gate[e] = s[picked, e]
        slot[picked, e] = e * C + np.arange(C)
        if C < T:
            margin[e] = key[order[C - 1], e] - key[order[C], e]
    return dict(tok=tok.astype(np.int32), gate=gate, slot=slot.astype(np.int32), margin=margin)


def moe_layer_expert_choice(x, gamma, w_router, router_bias, experts: "Weights", *, k: int,
                            act: str = "bf16", rms_eps: float = 1e-6,
                            bias_mode: str = BIAS_NONE, capacity_factor: float = 0.0,
                            shared: Optional["Weights"] = None, n_shared: int = 0,
                            forced_scores=None, tokens: Optional[Sequence[int]] = None,
                            residual: bool = True) -> Dict[str, np.ndarray]:
    """Forward of one MoE layer under expert-choice routing ("MoE: dynamism the
    compiler cannot remove", capacity section: instead of each token picking k
    experts, each expert picks its top T*k/E tokens, so every expert holds exactly
    C = T*k/E rows; a token may get several experts or none):

        out[t] = x[t] + sum_s FFN_s(xn_t) + sum_{e : t picked by e} score[t, e] FFN_e(xn_t)

    with the routed terms added in ascending e.  ``forced_scores`` replaces the
    oracle's FP32 scores by given ones (selection replay)."""
    x64 = np.asarray(x, np.float64)
    T, d = x64.shape
    E = np.asarray(w_router).shape[1]
    xn = rmsnorm(x64, gamma, rms_eps, act)
    logits = router_logits(xn, w_router)
    logits32 = logits.astype(np.float32)
    scores = expert_choice_scores(logits32, router_bias, bias_mode)
    if forced_scores is not None:
        scores = np.asarray(forced_scores, dtype=np.float32)
    C = expert_choice_capacity(capacity_factor, T, k, E)
    sel = expert_choice_select(scores, C)
    rows = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    where = np.full(T, -1, dtype=np.int64)
    where[rows] = np.arange(rows.size)
    out = x64[rows].copy() if residual else np.zeros((rows.size, d))
    for s_ in range(n_shared):
        out += shared.ffn(s_, xn[rows])
    for e in range(E):                                   # routed terms in ascending e
        t_sel = sel["tok"][e][where[sel["tok"][e]] >= 0]
        if t_sel.size == 0:
            continue
        g = sel["gate"][e][where[sel["tok"][e]] >= 0]
        out[where[t_sel]] += g[:, None] * experts.ffn(e, xn[t_sel])
    return dict(out=out, xn=xn, logits=logits, logits32=logits32, scores=scores, C=C, **sel)


# ---------------------------------------------------------------------------
# a4 / a5: histogram, scan, capacity and the stable permutation
# ---------------------------------------------------------------------------
def capacity(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """Per-expert capacity ceil(C*T*k/E) (None when uncapped, C <= 0)."""
    c = float(np.float32(capacity_factor))
    if c <= 0:
        return None
    return int(math.ceil(c * T * k / E))


def permute(idx, E: int, capacity_factor: float = 0.0) -> Dict[str, np.ndarray]:
    """Counting sort of the flat assignments ``a = t*k + j`` by expert.

    counts[e]      assignments routed to e (before capacity)
    offsets[E+1]   exclusive scan of kept[e] = min(counts[e], cap)
    slot_of[a]     offsets[e] + rank(a) if kept, else -1
    perm_assign[s] the assignment stored in slot s (token = a // k)
    dropped        sum_e max(0, counts[e] - cap)
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    order = np.argsort(flat, kind="stable")           # by expert, then by a
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.empty_like(flat)
    rank[order] = np.arange(flat.size) - first[flat[order]]
    cap = capacity(capacity_factor, T, k, E)
    kept = counts if cap is None else np.minimum(counts, cap)
    offsets = np.concatenate([[0], np.cumsum(kept)]).astype(np.int64)
    keep = np.ones(flat.size, bool) if cap is None else rank < cap
    slot_of = np.where(keep, offsets[flat] + rank, -1)
    perm_assign = np.empty(int(offsets[-1]), dtype=np.int64)
    perm_assign[slot_of[keep]] = np.nonzero(keep)[0]
    dropped = int(np.sum(counts - kept))
    return dict(counts=counts.astype(np.int32), offsets=offsets.astype(np.int32),
                slot_of=slot_of.astype(np.int32), perm_assign=perm_assign.astype(np.int32),
                dropped=dropped, cap=cap, rank=rank.astype(np.int32))


# ---------------------------------------------------------------------------
# expert weights as the layer sees them
# ---------------------------------------------------------------------------
# Nibble j of each little-endian 4-byte word of int4 codes holds code 8w + INT4_ORDER[j]
# of that word's eight: the even codes in the low nibbles of the four bytes, the odd
# ones in the high nibbles (byte 0: codes 0 and 2, byte 1: 4 and 6, byte 2: 1 and 3,
# byte 3: 5 and 7).
INT4_ORDER = (0, 2, 4, 6, 1, 3, 5, 7)


def unpack_int4(packed) -> np.ndarray:
    """uint8 [R, C/2] -> int [R, C] (C a multiple of 8), two's complement nibbles
    in the word order INT4_ORDER."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    R, nb = p.shape
    nib = np.empty((R, nb * 2), dtype=np.int64)
    nib[:, 0::2] = p & 0xF            # nibble 2b of the stream: low half of byte b
    nib[:, 1::2] = (p >> 4) & 0xF
    nib = nib.reshape(R, nb // 4, 8)
    q = np.empty_like(nib)
    q[:, :, list(INT4_ORDER)] = nib   # nibble j -> code INT4_ORDER[j]
    q = q.reshape(R, nb * 2)
    return np.where(q >= 8, q - 16, q)


def dequant_int8(q, s) -> np.ndarray:
    """w[K, N] = bf16(q[n, k] * s[n]) from codes stored K-contiguous, q[N, K]."""
    return round_bf16(np.asarray(q, np.float64).T * np.asarray(s, np.float64)[None, :])


def dequant_int4(packed, s, group: int) -> np.ndarray:
    """w[K, N] = bf16(q[n, k] * s[k // group, n]) from packed codes stored
    K-contiguous, packed[N, K/2]."""
    q = unpack_int4(packed).astype(np.float64).T
    sk = np.repeat(np.asarray(s, np.float64), group, axis=0)
    return round_bf16(q * sk)


def decode_e4m3(codes) -> np.ndarray:
    """FP8 E4M3 codes (uint8) -> float64, from the format's definition: bit 7 sign,
    bits 6..3 biased exponent (bias 7), bits 2..0 mantissa; exponent 0 encodes the
    subnormals m/8 * 2^-6; this variant has no infinities and exponent 15 with
    mantissa 7 encodes NaN (largest finite value 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


def dequant_fp8(q, s) -> np.ndarray:
    """w[K, N] = bf16(e4m3(q[n, k]) * s[n]) from codes stored K-contiguous, q[N, K]."""
    return round_bf16(decode_e4m3(q).T * np.asarray(s, np.float64)[None, :])


def expert_matrix(w, s, expert_dtype: str, group: int = 128) -> np.ndarray:
    """One expert's [K, N] weight matrix in float64."""
    if expert_dtype in ("bf16", "f32"):
        return np.asarray(w, np.float64)
    if expert_dtype == "int8":
        return dequant_int8(w, s)
    if expert_dtype == "fp8":
        return dequant_fp8(w, s)
    if expert_dtype == "int4":
        return dequant_int4(w, s, group)
    raise ValueError(expert_dtype)


# ---------------------------------------------------------------------------
# a6 / a7: the SwiGLU expert
# ---------------------------------------------------------------------------
def silu(u) -> np.ndarray:
    with np.errstate(over="ignore"):
        return u / (1.0 + np.exp(-u))


def expert_ffn(X, wg, wu, wd) -> np.ndarray:
    """y = (silu(X Wg) * (X Wu)) Wd for X[M, d], Wg/Wu[d, f], Wd[f, d]."""
    X = np.asarray(X, np.float64)
    h = silu(X @ wg) * (X @ wu)
    return h @ wd


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------
class Weights:
    """Expert weights (stacked per expert, numpy arrays or host torch tensors);
    each matrix is converted to float64 (dequantised for int8 / int4) when it is
    used, one expert at a time."""

    def __init__(self, expert_dtype: str, group: int, gate, up, down,
                 s_gate=None, s_up=None, s_down=None):
        self.dt, self.group = expert_dtype, group
        self.src = dict(gate=(gate, s_gate), up=(up, s_up), down=(down, s_down))

    def get(self, which: str, e: int) -> np.ndarray:
        w, s = self.src[which]
        return expert_matrix(_npy(w[e]), None if s is None else _npy(s[e]), self.dt, self.group)

    def ffn(self, e: int, X) -> np.ndarray:
        return expert_ffn(X, self.get("gate", e), self.get("up", e), self.get("down", e))


def moe_layer(x, gamma, w_router, router_bias, experts: Weights, *, k: int,
              act: str = "bf16", rms_eps: float = 1e-6, bias_mode: str = BIAS_NONE,
              renormalize: bool = True, capacity_factor: float = 0.0,
              shared: Optional[Weights] = None, n_shared: int = 0,
              forced_idx=None, tokens: Optional[Sequence[int]] = None,
              residual: bool = True) -> Dict[str, np.ndarray]:
    """Forward of one MoE layer.

    Routing, histogram and permutation always run over all T tokens (capacity
    couples the tokens); with ``tokens`` given, expert outputs and ``out`` are
    evaluated for those token rows only (``out`` is then ``[len(tokens), d]``).
    """
    x64 = np.asarray(x, np.float64)
    T, d = x64.shape
    E = np.asarray(w_router).shape[1]
    xn = rmsnorm(x64, gamma, rms_eps, act)
    logits = router_logits(xn, w_router)
    logits32 = logits.astype(np.float32)
    r = route(logits32, router_bias, k, bias_mode, renormalize, forced_idx)
    p = permute(r["idx"], E, capacity_factor)

    rows = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    where = np.full(T, -1, dtype=np.int64)
    where[rows] = np.arange(rows.size)
    out = x64[rows].copy() if residual else np.zeros((rows.size, d))

    # y[t, j] = FFN_{idx[t, j]}(xn[t]) for every kept assignment of the evaluated
    # rows; each row's FFN is independent of the others, so the rows that share an
    # expert are evaluated together (one matmul per weight matrix)
    kept = (p["slot_of"].reshape(T, k) >= 0) & (where[:, None] >= 0)
    y = np.zeros((rows.size, k, d))
    for e in np.unique(r["idx"][kept]):
        t_sel, j_sel = np.nonzero(kept & (r["idx"] == e))
        y[where[t_sel], j_sel] = experts.ffn(int(e), xn[t_sel])
    for s in range(n_shared):                            # always-on experts, gate 1
        out += shared.ffn(s, xn[rows])
    g = np.where(kept[rows], r["gates"][rows], 0.0)
    for j in range(k):                                   # routed outputs in j order
        out += g[:, j, None] * y[:, j]
    return dict(out=out, xn=xn, logits=logits, logits32=logits32, **r, **p)


def moe_layer_dense(x, gamma, w_router, router_bias, experts: Weights, *, k: int,
                    act: str = "bf16", rms_eps: float = 1e-6, bias_mode: str = BIAS_NONE,
                    renormalize: bool = True, capacity_factor: float = 0.0,
                    shared: Optional[Weights] = None, n_shared: int = 0) -> np.ndarray:
    """Brute force: every expert on every token, masked by the kept top-k set.

    Used to pin ``moe_layer`` on tiny inputs; token by token, no permutation.
    """
    x64 = np.asarray(x, np.float64)
    T, d = x64.shape
    E = np.asarray(w_router).shape[1]
    xn = rmsnorm(x64, gamma, rms_eps, act)
    logits32 = router_logits(xn, w_router).astype(np.float32)
    r = route(logits32, router_bias, k, bias_mode, renormalize)
    slot_of = permute(r["idx"], E, capacity_factor)["slot_of"].reshape(T, k)
    out = x64.copy()
    for t in range(T):
        for e in range(E):
            y = experts.ffn(e, xn[t:t + 1])[0]
            w = 0.0
            for j in range(k):
                if r["idx"][t, j] == e and slot_of[t, j] >= 0:
                    w += r["gates"][t, j]
            out[t] += w * y
        for s in range(n_shared):
            out[t] += shared.ffn(s, xn[t:t + 1])[0]
    return out


def _npy(t):
    """numpy view of a host tensor (floating types widened to float32, which is
    exact for bf16); numpy arrays pass through."""
    if t is None or isinstance(t, np.ndarray):
        return t
    return t.float().numpy() if t.is_floating_point() else t.numpy()


def weights_from_inputs(li, shared: bool = False) -> Optional[Weights]:
    """Expert weights of a ``moe_synth.LayerInputs`` (host tensors); integer
    storage stays integer."""
    sh = li.shape
    if shared and not sh.n_shared:
        return None
    pre = "sh_" if shared else ""
    get = lambda n: getattr(li, pre + n)   # noqa: E731  (converted per expert when used)
    return Weights(sh.expert, sh.group_size, get("w_gate" if not shared else "gate"),
                   get("w_up" if not shared else "up"), get("w_down" if not shared else "down"),
                   get("s_gate"), get("s_up"), get("s_down"))


def layer_expert_choice_from_inputs(li, x, **kw) -> Dict[str, np.ndarray]:
    """Run ``moe_layer_expert_choice`` on a ``moe_synth.LayerInputs``."""
    sh = li.shape
    args = dict(k=sh.k, act=sh.act, rms_eps=sh.rms_eps, bias_mode=sh.bias_mode,
                capacity_factor=sh.capacity_factor, shared=weights_from_inputs(li, shared=True),
                n_shared=sh.n_shared)
    args.update(kw)
    return moe_layer_expert_choice(_npy(x), _npy(li.gamma), _npy(li.w_router),
                                   _npy(li.router_bias), weights_from_inputs(li), **args)


def layer_from_inputs(li, x, **kw) -> Dict[str, np.ndarray]:
    """Run ``moe_layer`` on a ``moe_synth.LayerInputs`` (host tensors)."""
    sh = li.shape
    npy = _npy
    experts = weights_from_inputs(li)
    shared = weights_from_inputs(li, shared=True)
    args = dict(k=sh.k, act=sh.act, rms_eps=sh.rms_eps, bias_mode=sh.bias_mode,
                renormalize=sh.renormalize, capacity_factor=sh.capacity_factor,
                shared=shared, n_shared=sh.n_shared)
    args.update(kw)
    return moe_layer(npy(x), npy(li.gamma), npy(li.w_router), npy(li.router_bias),
                     experts, **args)
