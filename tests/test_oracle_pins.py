"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- a library routine, a closed form, brute force on tiny inputs, an
invariant the pages state, or a statistic with a known expectation.

CPU only; sized to run in seconds.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_synth
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------
def test_round_bf16_matches_torch_on_f32_inputs():
    r = rng(0)
    a = np.concatenate([r.standard_normal(20000) * 10.0 ** r.integers(-40, 38, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 1e-39, -3e-42]])
    a32 = a.astype(np.float32)
    ref = torch.from_numpy(a32).to(torch.bfloat16).double().numpy()
    got = O.round_bf16(a32.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_round_f32_matches_numpy_cast():
    r = rng(1)
    a = r.standard_normal(20000) * 10.0 ** r.integers(-44, 38, 20000)
    np.testing.assert_array_equal(O.round_f32(a), a.astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# a1 RMSNorm, a2 router
# ---------------------------------------------------------------------------
def test_rmsnorm_matches_torch_rms_norm():
    r = rng(2)
    x = r.standard_normal((37, 96))
    g = r.uniform(0.5, 1.5, 96)
    eps = 1e-6
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(g),
                                       eps=float(np.float32(eps))).numpy()
    got = O.rmsnorm(x, g, eps, "f32")
    np.testing.assert_allclose(got, ref, rtol=2 ** -23, atol=0)
    # bf16 output is the bf16 rounding of the same values
    np.testing.assert_allclose(O.rmsnorm(x, g, eps, "bf16"), ref, rtol=2 ** -8, atol=0)


def test_rmsnorm_eps_matters_for_tiny_rows():
    x = np.full((1, 4), 1e-4)
    xn = O.rmsnorm(x, np.ones(4), 1e-6, "f32")
    # closed form: 1e-4 / sqrt(1e-8 + eps32)
    eps = float(np.float32(1e-6))
    assert xn[0, 0] == pytest.approx(1e-4 / math.sqrt(1e-8 + eps), rel=1e-7)


def test_router_picks_row_of_basis_token():
    """x = a * e_i normalises to sqrt(d) * e_i, so logits = xn_i * W_r[i, :]."""
    d, E = 24, 7
    r = rng(3)
    w = r.standard_normal((d, E))
    rows = [0, 5, 23]
    x = np.zeros((3, d))
    for t, i in enumerate(rows):
        x[t, i] = 3.0 + t
    xn = O.rmsnorm(x, np.ones(d), 1e-6, "f32")
    l = O.router_logits(xn, w)
    for t, i in enumerate(rows):
        a = 3.0 + t
        eps = float(np.float32(1e-6))
        assert xn[t, i] == pytest.approx(a / math.sqrt(a * a / d + eps), rel=1e-7)
        np.testing.assert_array_equal(l[t], xn[t, i] * w[i])


# ---------------------------------------------------------------------------
# a3 softmax / top-k / bias / renormalisation
# ---------------------------------------------------------------------------
def test_softmax_matches_torch():
    r = rng(4)
    p = r.standard_normal((50, 64)) * 4
    np.testing.assert_allclose(O.softmax64(p), torch.softmax(torch.from_numpy(p), -1).numpy(),
                               rtol=1e-14, atol=1e-300)


def brute_topk(keys, k):
    """Rank by counting: expert e has rank = #experts that beat it."""
    T, E = keys.shape
    idx = np.zeros((T, k), np.int32)
    for t in range(T):
        for e in range(E):
            better = sum(1 for o in range(E)
                         if keys[t, o] > keys[t, e] or (keys[t, o] == keys[t, e] and o < e))
            if better < k:
                idx[t, better] = e
    return idx


@pytest.mark.parametrize("E,k", [(8, 2), (9, 9), (16, 5), (12, 1)])
def test_topk_matches_rank_by_counting_with_ties(E, k):
    r = rng(5 + E + k)
    keys = r.integers(-3, 4, size=(40, E)).astype(np.float32)   # many ties
    idx, margin = O.topk_sorted(keys, k)
    np.testing.assert_array_equal(idx, brute_topk(keys, k))
    if k < E:
        srt = -np.sort(-keys.astype(np.float64), axis=1)
        np.testing.assert_array_equal(margin, srt[:, k - 1] - srt[:, k])


def test_topk_set_is_best_subset_by_enumeration():
    r = rng(6)
    keys = r.standard_normal((25, 7)).astype(np.float32)
    idx, _ = O.topk_sorted(keys, 3)
    for t in range(25):
        best = max(itertools.combinations(range(7), 3),
                   key=lambda s: sum(float(keys[t, e]) for e in s))
        assert set(idx[t]) == set(best)


def test_topk_matches_torch_topk_values():
    r = rng(7)
    keys = r.standard_normal((100, 64)).astype(np.float32)
    idx, _ = O.topk_sorted(keys, 8)
    tv, ti = torch.topk(torch.from_numpy(keys), 8, dim=1)
    np.testing.assert_array_equal(idx, ti.numpy())


def test_nan_keys_are_never_preferred():
    keys = np.array([[np.nan, 0.5, -1.0, np.nan, 2.0]], np.float32)
    s, _ = O.selection_keys(keys, None, O.BIAS_NONE)
    idx, _ = O.topk_sorted(s, 3)
    assert list(idx[0]) == [4, 1, 2]


def test_gates_renormalised_and_bias_modes():
    r = rng(8)
    l = r.standard_normal((30, 16)).astype(np.float32)
    b = (r.standard_normal(16) * 2).astype(np.float32)
    sel = O.route(l, b, 4, O.BIAS_SELECT, True)
    np.testing.assert_allclose(sel["gates"].sum(1), 1.0, rtol=1e-14)
    # select mode: chosen by l + b, weighted by softmax(l)
    p = torch.softmax(torch.from_numpy(l.astype(np.float64)), -1).numpy()
    ref = np.take_along_axis(p, sel["idx"].astype(np.int64), 1)
    np.testing.assert_allclose(sel["gates"], ref / ref.sum(1, keepdims=True), rtol=1e-13)
    np.testing.assert_array_equal(sel["idx"], brute_topk((l + b[None]).astype(np.float32), 4))
    # logit mode: bias is part of the logits for both selection and gates
    lg = O.route(l, b, 4, O.BIAS_LOGIT, False)
    pb = torch.softmax(torch.from_numpy((l + b[None]).astype(np.float32).astype(np.float64)), -1)
    np.testing.assert_allclose(lg["gates"], np.take_along_axis(pb.numpy(), lg["idx"].astype(np.int64), 1),
                               rtol=1e-13)
    # without renormalisation the gates are the plain probabilities (sum < 1)
    assert np.all(lg["gates"].sum(1) < 1.0)


# ---------------------------------------------------------------------------
# a4 / a5 histogram, scan, capacity, permutation
# ---------------------------------------------------------------------------
def brute_permute(idx, E, cap):
    T, k = idx.shape
    flat = [int(v) for v in idx.reshape(-1)]
    counts = [flat.count(e) for e in range(E)]
    kept = [c if cap is None else min(c, cap) for c in counts]
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + kept[e])
    slot_of, perm = [], [None] * offsets[-1]
    for a, e in enumerate(flat):
        rank = sum(1 for b in range(a) if flat[b] == e)
        if cap is None or rank < cap:
            slot_of.append(offsets[e] + rank)
            perm[offsets[e] + rank] = a
        else:
            slot_of.append(-1)
    return counts, offsets, slot_of, perm


@pytest.mark.parametrize("C", [0.0, 0.5, 1.0, 1.25])
def test_permute_matches_brute_force(C):
    r = rng(9)
    T, k, E = 23, 3, 6
    idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)])
    got = O.permute(idx, E, C)
    cap = O.capacity(C, T, k, E)
    counts, offsets, slot_of, perm = brute_permute(idx, E, cap)
    assert list(got["counts"]) == counts
    assert list(got["offsets"]) == offsets
    assert list(got["slot_of"]) == slot_of
    assert list(got["perm_assign"]) == perm


def test_permute_invariants_and_drop_count():
    r = rng(10)
    T, k, E = 500, 6, 64
    # skewed routing so that capacity binds
    pop = np.arange(1, E + 1) ** -1.1
    idx = np.stack([r.choice(E, k, replace=False, p=pop / pop.sum()) for _ in range(T)])
    for C in (0.0, 1.0, 1.25, 1.5, 100.0):
        p = O.permute(idx, E, C)
        assert p["counts"].sum() == T * k
        cap = O.capacity(C, T, k, E)
        kept = p["counts"] if cap is None else np.minimum(p["counts"], cap)
        assert p["offsets"][-1] == kept.sum()
        assert p["dropped"] == int(np.sum(np.maximum(0, p["counts"] - (cap or 10 ** 9))))
        # bijection between kept assignments and slots
        kept_a = np.nonzero(p["slot_of"] >= 0)[0]
        assert sorted(p["slot_of"][kept_a]) == list(range(p["offsets"][-1]))
        np.testing.assert_array_equal(p["perm_assign"][p["slot_of"][kept_a]], kept_a)
        # each slot lies in its expert's segment
        e_of = idx.reshape(-1)[p["perm_assign"]]
        seg = np.searchsorted(p["offsets"], np.arange(p["offsets"][-1]), side="right") - 1
        np.testing.assert_array_equal(e_of, seg)
        if C == 100.0:
            assert p["dropped"] == 0


def test_capacity_values_for_the_v2lite_shape():
    # C * T*k / E rows per expert, rounded up: T=32, k=6, E=64 and T=8192
    assert [O.capacity(c, 32, 6, 64) for c in (1.0, 1.25, 1.5)] == [3, 4, 5]
    assert [O.capacity(c, 8192, 6, 64) for c in (1.0, 1.25, 1.5)] == [768, 960, 1152]
    assert O.capacity(0.0, 32, 6, 64) is None


def test_padding_fraction_at_capacity_one_and_a_half():
    g = json.load(open(os.path.join(GOLDEN, "page_arithmetic.json")))["capacity"]
    # with perfectly balanced routing every expert fills T*k/E of its C*T*k/E rows
    C = g["C_padding"]
    T, k, E = 4096, 8, 64
    cap = O.capacity(C, T, k, E)
    assert (cap - T * k / E) / cap == pytest.approx(g["printed_padding_fraction"], abs=1e-3)


# ---------------------------------------------------------------------------
# weight formats
# ---------------------------------------------------------------------------
def test_int4_unpack_fixture():
    g = json.load(open(os.path.join(GOLDEN, "int4_packing.json")))
    np.testing.assert_array_equal(O.unpack_int4(np.array(g["packed"], np.uint8)),
                                  np.array(g["values"]))


def test_quantised_weights_within_quantisation_bound():
    w = torch.from_numpy(rng(11).standard_normal((256, 64)).astype(np.float32)) * 0.05
    q8, s8 = moe_synth.quantize_int8(w)
    dq8 = O.dequant_int8(q8.numpy(), s8.float().numpy())
    bound8 = 0.5 * s8.float().numpy()[None, :] + np.abs(dq8) * 2.0 ** -8
    assert np.all(np.abs(dq8 - w.numpy()) <= bound8 * (1 + 1e-6))
    np.testing.assert_array_equal(dq8, O.round_bf16(dq8))
    p4, s4 = moe_synth.quantize_int4(w, 128)
    dq4 = O.dequant_int4(p4.numpy(), s4.float().numpy(), 128)
    s_full = np.repeat(s4.float().numpy(), 128, axis=0)
    bound = 0.5 * s_full + np.abs(dq4) * 2.0 ** -8
    assert np.all(np.abs(dq4 - w.numpy()) <= bound * (1 + 1e-6))
    # the dequantised int4 weight is a bf16 value
    np.testing.assert_array_equal(dq4, O.round_bf16(dq4))


def test_e4m3_decode_matches_torch_float8_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.decode_e4m3(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # closed forms: 1.0, the largest finite value, the smallest subnormal, a sign
    assert O.decode_e4m3([0x38])[0] == 1.0 and O.decode_e4m3([0x7E])[0] == 448.0
    assert O.decode_e4m3([0x01])[0] == 2.0 ** -9 and O.decode_e4m3([0xB8])[0] == -1.0
    assert np.isnan(O.decode_e4m3([0x7F, 0xFF])).all()


def test_fp8_weights_within_quantisation_bound():
    w = torch.from_numpy(rng(13).standard_normal((256, 64)).astype(np.float32)) * 0.05
    q, s = moe_synth.quantize_fp8(w)
    dq = O.dequant_fp8(q.numpy(), s.float().numpy())
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normals, absolute
    # <= 2^-10 s below the normal range; then one bf16 rounding of q*s
    sf = s.float().numpy()[None, :]
    bound = np.abs(w.numpy()) * 2.0 ** -4 + sf * 2.0 ** -10 + np.abs(dq) * 2.0 ** -8
    assert np.all(np.abs(dq - w.numpy()) <= bound * (1 + 1e-6))
    np.testing.assert_array_equal(dq, O.round_bf16(dq))
    # each output column's maximum maps to (nearly) the largest code; the codes are
    # stored K-contiguous, one row per output column
    assert np.all(np.abs(O.decode_e4m3(q.numpy())).max(axis=1) >= 416)


# ---------------------------------------------------------------------------
# a6 / a7 expert FFN, a8 combine, the whole layer
# ---------------------------------------------------------------------------
def tiny_layer(seed=12, d=32, E=6, f=48, S=0, dtype="f32"):
    r = rng(seed)
    wg = r.standard_normal((E, d, f)) / math.sqrt(d)
    wu = r.standard_normal((E, d, f)) / math.sqrt(d)
    wd = r.standard_normal((E, f, d)) / math.sqrt(f)
    wr = r.standard_normal((d, E)) / math.sqrt(d)
    sh = None
    if S:
        sh = O.Weights(dtype, 128, r.standard_normal((S, d, f)) / math.sqrt(d),
                       r.standard_normal((S, d, f)) / math.sqrt(d),
                       r.standard_normal((S, f, d)) / math.sqrt(f))
    return O.Weights(dtype, 128, wg, wu, wd), wr, sh


def test_expert_ffn_matches_torch_swiglu():
    r = rng(13)
    X = r.standard_normal((9, 32))
    wg, wu, wd = r.standard_normal((32, 40)), r.standard_normal((32, 40)), r.standard_normal((40, 32))
    Xt = torch.from_numpy(X)
    ref = (torch.nn.functional.silu(Xt @ torch.from_numpy(wg)) * (Xt @ torch.from_numpy(wu))) \
        @ torch.from_numpy(wd)
    np.testing.assert_allclose(O.expert_ffn(X, wg, wu, wd), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_single_expert_layer_is_a_dense_ffn():
    """E = 1, k = 1, renormalised: out = x + SwiGLU(RMSNorm(x))."""
    ex, wr, _ = tiny_layer(E=1)
    x = rng(14).standard_normal((10, 32))
    res = O.moe_layer(x, np.ones(32), wr, None, ex, k=1, act="f32", renormalize=True)
    xt = torch.from_numpy(x)
    xn = torch.nn.functional.rms_norm(xt, (32,), eps=float(np.float32(1e-6)))
    g, u, dn = (torch.from_numpy(ex.get(w, 0)) for w in ("gate", "up", "down"))
    ref = xt + (torch.nn.functional.silu(xn @ g) * (xn @ u)) @ dn
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-6, atol=1e-6)


def test_all_experts_selected_is_softmax_weighted_mixture():
    """k = E with renormalisation: out = x + sum_e softmax(l)_e FFN_e(xn)."""
    ex, wr, _ = tiny_layer(E=5)
    x = rng(15).standard_normal((8, 32))
    res = O.moe_layer(x, np.ones(32), wr, None, ex, k=5, act="f32")
    xn = res["xn"]
    p = torch.softmax(torch.from_numpy(res["logits32"].astype(np.float64)), -1)
    ys = torch.stack([torch.from_numpy(ex.ffn(e, xn)) for e in range(5)])   # [E, T, d]
    ref = torch.from_numpy(x) + torch.einsum("te,etd->td", p, ys)
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("C,S,mode", [(0.0, 0, "none"), (0.0, 2, "logit"),
                                      (0.75, 1, "select"), (1.0, 0, "none")])
def test_sparse_layer_equals_dense_brute_force(C, S, mode):
    ex, wr, sh = tiny_layer(S=S)
    r = rng(16)
    x = r.standard_normal((14, 32))
    b = r.standard_normal(6).astype(np.float32) if mode != "none" else None
    kw = dict(k=2, act="bf16", bias_mode=mode, renormalize=(mode != "logit"),
              capacity_factor=C, shared=sh, n_shared=S)
    sparse = O.moe_layer(x, np.ones(32), wr, b, ex, **kw)["out"]
    dense = O.moe_layer_dense(x, np.ones(32), wr, b, ex, **kw)
    np.testing.assert_allclose(sparse, dense, rtol=1e-12, atol=1e-12)


def test_fully_dropped_token_passes_through_on_residual():
    ex, wr, sh = tiny_layer(S=1)
    x = rng(17).standard_normal((40, 32))
    res = O.moe_layer(x, np.ones(32), wr, None, ex, k=2, act="f32", capacity_factor=0.05,
                      shared=sh, n_shared=1)
    dropped = np.nonzero((res["slot_of"].reshape(40, 2) < 0).all(1))[0]
    assert dropped.size > 0
    ref = x[dropped] + sh.ffn(0, res["xn"][dropped])
    np.testing.assert_array_equal(res["out"][dropped], ref)


def test_replaying_own_routes_is_bitwise_identical():
    """Causal route replay control: replaying the run's own routes returns the
    baseline exactly (picx.dev summary, Sub-study 2)."""
    ex, wr, sh = tiny_layer(S=1)
    x = rng(18).standard_normal((20, 32))
    a = O.moe_layer(x, np.ones(32), wr, None, ex, k=3, act="bf16", shared=sh, n_shared=1)
    b = O.moe_layer(x, np.ones(32), wr, None, ex, k=3, act="bf16", shared=sh, n_shared=1,
                    forced_idx=a["idx"])
    np.testing.assert_array_equal(a["out"], b["out"])


def test_token_subset_matches_full_rows():
    ex, wr, sh = tiny_layer(S=1)
    x = rng(19).standard_normal((30, 32))
    kw = dict(k=2, act="bf16", capacity_factor=1.0, shared=sh, n_shared=1)
    full = O.moe_layer(x, np.ones(32), wr, None, ex, **kw)["out"]
    rows = [29, 3, 17]
    sub = O.moe_layer(x, np.ones(32), wr, None, ex, tokens=rows, **kw)["out"]
    # BLAS may block a different row count differently: agree to rounding
    np.testing.assert_allclose(sub, full[rows], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------------------
# statistics the pages fix
# ---------------------------------------------------------------------------
def test_experts_touched_matches_formula():
    """With i.i.d. logits every token picks a uniform k-subset, so the expected
    number of distinct experts touched at batch B is E (1 - (1 - k/E)^B)
    ("MoE Research", section 7 exercise A)."""
    E, k, trials = 64, 8, 300
    r = rng(20)
    for B in json.load(open(os.path.join(GOLDEN, "page_arithmetic.json")))["experts_touched"]["batches"]:
        touched = []
        for _ in range(trials):
            l = r.standard_normal((B, E)).astype(np.float32)
            idx = O.route(l, None, k, O.BIAS_NONE, True)["idx"]
            touched.append(np.unique(idx).size)
        touched = np.array(touched, float)
        expect = E * (1 - (1 - k / E) ** B)
        se = max(touched.std(ddof=1), 0.5) / math.sqrt(trials)
        assert abs(touched.mean() - expect) < 5 * se, (B, touched.mean(), expect)


def test_olmoe_bias_gives_one_and_a_half_times_mean_load():
    sh = moe_synth.PRESETS["olmoe"]
    x = moe_synth.make_x(sh, 4096).float().numpy()
    xn = O.rmsnorm(x, np.ones(sh.d), sh.rms_eps, sh.act)
    l32 = O.router_logits(xn, moe_synth.make_router(sh).float().numpy()).astype(np.float32)
    r = O.route(l32, moe_synth.make_router_bias(sh).numpy(), sh.k, O.BIAS_LOGIT, True)
    c = O.permute(r["idx"], sh.E)["counts"]
    assert c.max() / c.mean() == pytest.approx(1.5, abs=0.05)
