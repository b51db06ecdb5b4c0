"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Every test here needs a B200."""
import dataclasses

import numpy as np
import pytest
import torch

import moe_layer_fp32_b200 as M
import moe_synth
from moe_synth import LayerShape
from oracle import moe_oracle as O
from tests.layer_check import (DELTA_GUARD, ROUTE_MARGIN, TOL, inputs_on_device, run_layer,
                               sample_rows)

pytestmark = pytest.mark.gpu

# small shapes: several tiles, ragged tails, every routing option
SMALL = {
    "bf16_plain": LayerShape("bf16_plain", d=256, E=16, k=4, f=256, seed=11),
    "bf16_shared_cap": LayerShape("bf16_shared_cap", d=384, E=32, k=6, f=384, n_shared=2,
                                  capacity_factor=1.25, bias_mode="logit", seed=12),
    "bf16_select_tc_router": LayerShape("bf16_select", d=256, E=64, k=8, f=128, n_shared=1,
                                        bias_mode="select", renormalize=False, seed=13),
    "bf16_prefill_tiles": LayerShape("bf16_prefill", d=512, E=8, k=2, f=640, seed=14),
    "f32_tiny": moe_synth.PRESETS["tiny"],
    "int4_decode": LayerShape("int4_decode", d=256, E=16, k=4, f=384, n_shared=1,
                              expert="int4", seed=15),
    "int8_decode": LayerShape("int8_decode", d=384, E=32, k=6, f=256, expert="int8",
                              bias_mode="logit", seed=16),
    "int4_prefill": LayerShape("int4_prefill", d=512, E=8, k=2, f=384, expert="int4",
                               capacity_factor=1.25, seed=17),
    "int8_prefill": LayerShape("int8_prefill", d=384, E=8, k=2, f=512, n_shared=1,
                               expert="int8", seed=18),
    # tensor-core router with K split into 4 parts (partial logits added by the route)
    "bf16_tc_router_split": LayerShape("bf16_router_split", d=1024, E=64, k=4, f=256, seed=20),
    # prefill tiles under Zipf-skewed routing and a shared expert: 256-token pair
    # tiles whose odd CTA holds no rows, tiles with a few rows, experts with none
    "bf16_prefill_skew": LayerShape("bf16_prefill_skew", d=256, E=16, k=4, f=384, n_shared=1,
                                    bias_mode="select", seed=21),
    # FP8 (E4M3) experts: decode tiles (in-loop dequantisation, split K) and
    # prefill tiles (dequantised once), with a shared expert and capacity
    "fp8_decode": LayerShape("fp8_decode", d=384, E=32, k=6, f=256, n_shared=1, expert="fp8",
                             bias_mode="logit", seed=22),
    "fp8_prefill": LayerShape("fp8_prefill", d=512, E=8, k=2, f=384, expert="fp8",
                              capacity_factor=1.25, seed=23),
    # quantised decode tiles that fill the SMs (64 experts x 3 feature tiles): the
    # direct orientation with 128-token tiles, expanded weights in shared memory
    "int4_decode_direct": LayerShape("int4_decode_direct", d=256, E=64, k=8, f=384, n_shared=1,
                                     expert="int4", seed=26),
    "int8_decode_direct": LayerShape("int8_decode_direct", d=256, E=64, k=6, f=384,
                                     expert="int8", bias_mode="logit", seed=27),
    # FP32 experts with f not a multiple of 4 (scalar weight columns in gate/up)
    "f32_odd_f": LayerShape("f32_odd_f", d=136, E=6, k=2, f=130, n_shared=1, act="f32",
                            router="f32", expert="f32", capacity_factor=1.5,
                            bias_mode="logit", seed=19),
}
SMALL_T = {"bf16_plain": 100, "bf16_shared_cap": 77, "bf16_select_tc_router": 200,
           "bf16_prefill_tiles": 1000, "f32_tiny": 64, "int4_decode": 20, "int8_decode": 50,
           "int4_prefill": 900, "int8_prefill": 700, "f32_odd_f": 37,
           "bf16_tc_router_split": 300, "bf16_prefill_skew": 700, "fp8_decode": 40,
           "fp8_prefill": 800, "int4_decode_direct": 40, "int8_decode_direct": 61}


@pytest.fixture(autouse=True)
def _dev(cuda_device):
    yield


def tdev(a, dtype):
    return torch.as_tensor(a, dtype=dtype).cuda()


# --------------------------------------------------------------------- a1 + a2
@pytest.mark.parametrize("name", ["bf16_plain", "bf16_select_tc_router", "bf16_tc_router_split",
                                  "f32_tiny", "f32_odd_f"])
def test_rmsnorm_bitexact_and_router(name):
    sh, T = SMALL[name], SMALL_T[name]
    li, x, dli, dx = inputs_on_device(sh, T)
    cfg = M.make_config(sh, T)
    ws = M.alloc_workspace(cfg)
    act = torch.bfloat16 if sh.act == "bf16" else torch.float32
    xn = torch.empty(T, sh.d, dtype=act, device="cuda")
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    M.moe_rmsnorm_router(cfg, M.make_weights(dli), dx, xn, logits, ws)
    ref_xn = O.rmsnorm(x.float().numpy(), li.gamma.numpy(), sh.rms_eps, sh.act)
    np.testing.assert_array_equal(xn.float().cpu().numpy().astype(np.float64), ref_xn)
    wr = li.w_router.float().numpy().astype(np.float64)
    ref_l = O.router_logits(ref_xn, wr)
    # FP32 accumulation of d exact products: |err| <= d 2^-24 sum|xn_i w_ie|
    bound = sh.d * 2.0 ** -24 * (np.abs(ref_xn) @ np.abs(wr)) + 1e-30
    assert np.all(np.abs(logits.cpu().numpy() - ref_l) <= bound)


# --------------------------------------------------------------------- a3
@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (64, 6), (128, 8), (256, 8), (512, 32), (33, 1)])
@pytest.mark.parametrize("mode", ["none", "logit", "select"])
@pytest.mark.parametrize("renorm", [True, False])
def test_route_bitexact_given_logits(E, k, mode, renorm):
    r = np.random.default_rng(E * 100 + k)
    T = 300
    logits = r.standard_normal((T, E)).astype(np.float32)
    logits[: T // 3] = np.round(logits[: T // 3] * 2)          # many exact ties
    logits[5, : E // 2] = np.nan                                # NaN keys
    bias = (r.standard_normal(E) * 0.5).astype(np.float32) if mode != "none" else None
    sh = LayerShape("r", d=256, E=E, k=k, f=256, bias_mode=mode, renormalize=renorm,
                    act="f32", router="f32", expert="f32")
    cfg = M.make_config(sh, T)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    M.moe_route(cfg, tdev(logits, torch.float32), None if bias is None else tdev(bias, torch.float32),
                idx, gate)
    ref = O.route(logits, bias, k, mode, renorm)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    ok = np.isfinite(ref["gates"]).all(1)
    ok[5] = False
    # softmax over E in FP32 (expf within 2 ulp, a sum of E terms): rtol (E + k + 8) 2^-24
    np.testing.assert_allclose(gate.cpu().numpy()[ok], ref["gates"][ok],
                               rtol=(E + k + 8) * 2.0 ** -24, atol=1e-30)


# --------------------------------------------------------------------- a4 + a5
@pytest.mark.parametrize("full_ws", [False, True])
@pytest.mark.parametrize("T,k,E,C", [(1, 1, 8, 0.0), (1, 8, 64, 0.0), (37, 6, 64, 1.0),
                                     (32, 6, 64, 1.25), (500, 8, 64, 1.5), (4096, 8, 64, 0.0),
                                     (16384, 8, 128, 0.0), (9440, 8, 256, 1.0), (1000, 3, 512, 0.5),
                                     (6000, 6, 512, 1.25), (513, 8, 64, 0.0)])
def test_permute_bitexact(T, k, E, C, full_ws):
    """full_ws: with a whole workspace, batches above 4096 assignments take the
    three-kernel multi-CTA path; with only the error word, the one-CTA kernel."""
    r = np.random.default_rng(T + E)
    pop = np.arange(1, E + 1, dtype=np.float64) ** -1.1
    pop /= pop.sum()
    idx = np.stack([r.choice(E, k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)
    sh = LayerShape("p", d=256, E=E, k=k, f=256, capacity_factor=C)
    cfg = M.make_config(sh, T)
    n = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    slot = torch.empty(n, dtype=torch.int32, device="cuda")
    dropped = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg) if full_ws else torch.zeros(256, dtype=torch.uint8, device="cuda")
    M.moe_permute(cfg, tdev(idx, torch.int32), counts, offsets, perm, slot, dropped, ws)
    ref = O.permute(idx, E, C)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(slot.cpu().numpy(), ref["slot_of"])
    kept = int(ref["offsets"][-1])
    np.testing.assert_array_equal(perm.cpu().numpy()[:kept], ref["perm_assign"])
    assert int(dropped.item()) == ref["dropped"]
    assert M.moe_get_device_status(ws) == 0


def test_permute_flags_out_of_range_expert():
    T, k, E = 10, 2, 8
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[3, 1] = 8
    idx[7, 0] = -1
    cfg = M.make_config(LayerShape("p", d=256, E=E, k=k, f=256), T)
    outs = [torch.empty(E, dtype=torch.int32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda")] + \
           [torch.empty(T * k, dtype=torch.int32, device="cuda") for _ in range(2)] + \
           [torch.empty(1, dtype=torch.int32, device="cuda")]
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    M.moe_permute(cfg, tdev(idx, torch.int32), *outs, ws)
    assert M.moe_get_device_status(ws) == 1
    slot = outs[3].cpu().numpy()
    assert slot[3 * k + 1] == -1 and slot[7 * k + 0] == -1
    assert outs[0].cpu().numpy().sum() == T * k - 2


# --------------------------------------------------------------------- a6 + a7
@pytest.mark.parametrize("name", ["bf16_plain", "bf16_shared_cap", "bf16_prefill_tiles", "f32_tiny",
                                  "int4_decode", "int8_decode", "int4_prefill", "int8_prefill",
                                  "bf16_prefill_skew", "fp8_decode", "fp8_prefill",
                                  "int4_decode_direct", "int8_decode_direct"])
def test_grouped_ffn_matches_oracle_per_assignment(name):
    sh, T = SMALL[name], SMALL_T[name]
    li, x, dli, dx = inputs_on_device(sh, T)
    own = O.layer_from_inputs(li, x, tokens=[0])
    cfg = M.make_config(sh, T)
    ws = M.alloc_workspace(cfg)
    act = torch.bfloat16 if sh.act == "bf16" else torch.float32
    xn = tdev(own["xn"], act)
    y = torch.zeros(T * sh.k, sh.d, dtype=torch.float32, device="cuda")
    ys = torch.zeros(max(sh.n_shared, 1), T, sh.d, dtype=torch.float32, device="cuda")
    M.moe_grouped_ffn(cfg, M.make_weights(dli), xn, tdev(own["offsets"], torch.int32),
                      tdev(own["perm_assign"], torch.int32),
                      tdev(own["gates"].reshape(-1), torch.float32), y,
                      ys if sh.n_shared else None, ws)
    assert M.moe_get_device_status(ws) == 0
    y = y.cpu().numpy()
    ex = O.weights_from_inputs(li)
    kept = np.nonzero(own["slot_of"] >= 0)[0]
    ref = np.zeros((T * sh.k, sh.d))
    bound = np.zeros((T * sh.k, sh.d))
    flat_idx = own["idx"].reshape(-1)
    gates = own["gates"].reshape(-1)
    # The tensor-core path rounds h = silu(u) v to bf16 before the down GEMM
    # (relative error <= 2^-9 per element); with FP32 accumulation elsewhere the
    # error of y_n is bounded by 2^-8 g sum_i |h_i Wd[i, n]| (2^-9 doubled for the
    # FP32 sums).  The fp32 path keeps h in FP32: bound 2^-16 g sum_i |h_i Wd[i, n]|.
    rel = 2.0 ** -8 if sh.expert != "f32" else 2.0 ** -16

    def ffn_and_bound(W, e, X):
        u, v = X @ W.get("gate", e), X @ W.get("up", e)
        h = O.silu(u) * v
        return h @ W.get("down", e), np.abs(h) @ np.abs(W.get("down", e))

    for e in range(sh.E):
        a = kept[flat_idx[kept] == e]
        if a.size:
            yv, bv = ffn_and_bound(ex, e, own["xn"][a // sh.k])
            ref[a] = gates[a, None] * yv
            bound[a] = rel * gates[a, None] * bv
    assert np.all(np.abs(y[kept] - ref[kept]) <= bound[kept] + 1e-30)
    rms = np.sqrt(np.mean(ref[kept] ** 2))
    print(f"{name}: max|dy|/rms(y) = {np.max(np.abs(y[kept] - ref[kept])) / rms:.3e}")
    if sh.n_shared:
        shw = O.weights_from_inputs(li, shared=True)
        ysn = ys.cpu().numpy()
        for s in range(sh.n_shared):
            rs, bs = ffn_and_bound(shw, s, own["xn"])
            assert np.all(np.abs(ysn[s] - rs) <= rel * bs + 1e-30)


def test_direct_tile_row_boundaries():
    """128-token tiles around the 64-row and 128-row boundaries: experts receiving
    exactly 1, 63, 64, 65, 127, 128, 129 and 0 rows (k = 1, every token routed by
    hand), so that tiles of at most 64 rows (M = 64 MMAs over a 64-row copy), full
    and ragged 128-row tiles and a one-row tail all occur in both GEMMs; every row
    within the bound of the per-assignment test."""
    counts = [1, 63, 64, 65, 127, 128, 129, 0]
    T = sum(counts)
    sh = LayerShape("rows", d=256, E=len(counts), k=1, f=512, seed=7, tokens=(T,))
    li, x, dli, dx = inputs_on_device(sh, T)
    cfg = M.make_config(sh, T)
    ws = M.alloc_workspace(cfg)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.arange(T, dtype=np.int32)            # slot s holds token s (k = 1)
    gates = np.random.default_rng(11).uniform(0.1, 1.0, T).astype(np.float32)
    y = torch.zeros(T, sh.d, dtype=torch.float32, device="cuda")
    M.moe_grouped_ffn(cfg, M.make_weights(dli), dx, tdev(offsets, torch.int32),
                      tdev(perm, torch.int32), tdev(gates, torch.float32), y, None, ws)
    assert M.moe_get_device_status(ws) == 0
    y = y.cpu().numpy()
    ex = O.weights_from_inputs(li)
    xf = x.float().numpy().astype(np.float64)
    rel = 2.0 ** -8   # bf16 h, FP32 sums (the per-assignment test's bound)
    for e, (a0, a1) in enumerate(zip(offsets[:-1], offsets[1:])):
        if a1 == a0:
            continue
        X = xf[a0:a1]
        h = O.silu(X @ ex.get("gate", e)) * (X @ ex.get("up", e))
        ref = gates[a0:a1, None] * (h @ ex.get("down", e))
        bound = rel * gates[a0:a1, None] * (np.abs(h) @ np.abs(ex.get("down", e)))
        assert np.all(np.abs(y[a0:a1] - ref) <= bound + 1e-30), (e, counts[e])


# --------------------------------------------------------------------- a8
def test_combine_sums_in_fixed_order():
    T, d, k, S = 33, 256, 3, 2
    r = np.random.default_rng(5)
    y = r.standard_normal((T * k, d)).astype(np.float32)
    ys = r.standard_normal((S, T, d)).astype(np.float32)
    slot = np.where(r.random(T * k) < 0.3, -1, np.arange(T * k)).astype(np.int32)
    x = r.standard_normal((T, d)).astype(np.float32)
    sh = LayerShape("c", d=d, E=8, k=k, f=256, n_shared=S)
    cfg = M.make_config(sh, T, out_dtype="f32")
    out = torch.empty(T, d, dtype=torch.float32, device="cuda")
    M.moe_combine(cfg, tdev(y, torch.float32), tdev(slot, torch.int32), tdev(ys, torch.float32),
                  tdev(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), torch.bfloat16), out)
    xb = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    ref = xb + ys.astype(np.float64).sum(0) + \
        np.where((slot >= 0)[:, None], y, 0).reshape(T, k, d).astype(np.float64).sum(1)
    terms = np.abs(xb) + np.abs(ys).sum(0) + np.abs(y).reshape(T, k, d).sum(1)
    assert np.all(np.abs(out.cpu().numpy() - ref) <= (k + S + 1) * 2.0 ** -24 * terms + 1e-30)


# --------------------------------------------------------------------- whole layer
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_matches_oracle(name):
    sh, T = SMALL[name], SMALL_T[name]
    res = run_layer(sh, T)
    assert res.max_margin_mismatch < ROUTE_MARGIN, (res.mismatched, res.max_margin_mismatch)
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    assert res.err_ratio_delta <= DELTA_GUARD[sh.expert], res.err_ratio_delta
    print(f"{name}: err/rms(out) {res.err_ratio:.3e}  err/rms(delta) {res.err_ratio_delta:.3e}")


def test_layer_routing_bitexact_given_gpu_logits():
    sh, T = SMALL["bf16_shared_cap"], SMALL_T["bf16_shared_cap"]
    res = run_layer(sh, T)
    bias = moe_synth.make_router_bias(sh)
    ref = O.route(res.logits, None if bias is None else bias.numpy(), sh.k, sh.bias_mode,
                  sh.renormalize)
    np.testing.assert_array_equal(res.idx, ref["idx"])


def test_layer_is_deterministic_and_replayable():
    """Two runs are bitwise identical, and the five-call chain fed the layer's own
    routes (its routed rows rounded to bf16 as the fused call stores them)
    reproduces the fused call bitwise (route replay control, picx.dev
    summary Sub-study 2)."""
    sh, T = SMALL["bf16_shared_cap"], SMALL_T["bf16_shared_cap"]
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    o1 = layer.forward(dx).clone()
    o2 = layer.forward(dx).clone()
    assert torch.equal(o1, o2)
    cfg, w = layer.cfg, layer.w
    ws = M.alloc_workspace(cfg)
    xn = torch.empty(T, sh.d, dtype=torch.bfloat16, device="cuda")
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    M.moe_rmsnorm_router(cfg, w, dx, xn, logits, ws)
    idx = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T * sh.k, dtype=torch.float32, device="cuda")
    M.moe_route(cfg, logits, dli.router_bias, idx, gate)
    counts = torch.empty(sh.E, dtype=torch.int32, device="cuda")
    offs = torch.empty(sh.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    slot = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    drop = torch.empty(1, dtype=torch.int32, device="cuda")
    M.moe_permute(cfg, idx, counts, offs, perm, slot, drop, ws)
    y = torch.empty(T * sh.k, sh.d, dtype=torch.float32, device="cuda")
    ys = torch.empty(sh.n_shared, T, sh.d, dtype=torch.float32, device="cuda")
    M.moe_grouped_ffn(cfg, w, xn, offs, perm, gate, y, ys, ws)
    o3 = torch.empty(T, sh.d, dtype=torch.float32, device="cuda")
    # inside the layer the gated routed rows of tensor-core experts are stored in
    # bf16: the round-to-nearest-even of the same FP32 rows this entry point returns
    y_layer = y.to(torch.bfloat16).to(torch.float32) if sh.expert != "f32" else y
    M.moe_combine(cfg, y_layer, slot, ys, dx, o3)
    assert M.moe_get_device_status(ws) == 0
    assert torch.equal(o1, o3)


@pytest.mark.parametrize("T", [16, 100, 700])
def test_dropped_tokens_and_combine(T):
    """With no shared expert, k = 2 and a capacity of half the mean load, half the
    assignments are dropped and many tokens keep no row at all; their output must
    be the residual exactly, and every token the oracle's value.  T = 16 is the
    single-launch layer (decode tiles), 100 the kernel chain with decode tiles,
    700 the chain with prefill tiles.  The combine entry point fed the layer's
    routed rows (rounded to bf16 as the layer keeps them) gives the same bits."""
    sh = LayerShape("drop_no_shared", d=256, E=8, k=2, f=256, capacity_factor=0.5, seed=25)
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    # one launch; or RMSNorm, router, route, permutation, [row gather], gate/up, down,
    # combine
    assert M.moe_layer_launch_count(layer.cfg) == {16: 1, 100: 7, 700: 8}[T]
    out = layer.forward(dx).clone()
    assert M.moe_get_device_status(layer.ws) == 0
    res = run_layer(sh, T, data=(li, x, dli, dx))
    assert res.max_margin_mismatch < ROUTE_MARGIN
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    # tokens without a kept row: out == residual, bit for bit
    cap = int(np.ceil(0.5 * T * sh.k / sh.E))
    flat = res.idx.reshape(-1)                       # assignment a = t*k + j
    rank = np.zeros(flat.size, dtype=np.int64)
    seen = np.zeros(sh.E, dtype=np.int64)
    for a, e in enumerate(flat):
        rank[a] = seen[e]
        seen[e] += 1
    kept = (rank < cap).reshape(T, sh.k)
    empty = ~kept.any(axis=1)
    assert empty.any(), "the capacity must leave some tokens without a row"
    xf = dx.float().cpu().numpy()
    np.testing.assert_array_equal(out.cpu().numpy()[empty], xf[empty])
    # the separate combine over the layer's own routed rows gives the same bits
    cfg, w = layer.cfg, layer.w
    ws = M.alloc_workspace(cfg)
    xn = torch.empty(T, sh.d, dtype=torch.bfloat16, device="cuda")
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    M.moe_rmsnorm_router(cfg, w, dx, xn, logits, ws)
    idx_d = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T * sh.k, dtype=torch.float32, device="cuda")
    M.moe_route(cfg, logits, dli.router_bias, idx_d, gate)
    counts_d = torch.empty(sh.E, dtype=torch.int32, device="cuda")
    offs = torch.empty(sh.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    slot = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    drop = torch.empty(1, dtype=torch.int32, device="cuda")
    M.moe_permute(cfg, idx_d, counts_d, offs, perm, slot, drop, ws)
    y = torch.empty(T * sh.k, sh.d, dtype=torch.float32, device="cuda")
    M.moe_grouped_ffn(cfg, w, xn, offs, perm, gate, y, None, ws)
    o2 = torch.empty(T, sh.d, dtype=torch.float32, device="cuda")
    M.moe_combine(cfg, y.to(torch.bfloat16).to(torch.float32), slot, None, dx, o2)
    assert M.moe_get_device_status(ws) == 0
    assert torch.equal(out, o2)


def test_bf16_output_is_rounding_of_fp32_output():
    sh, T = SMALL["bf16_plain"], SMALL_T["bf16_plain"]
    li, x, dli, dx = inputs_on_device(sh, T)
    o32 = M.MoELayer(dli, T, out_dtype="f32").forward(dx)
    o16 = M.MoELayer(dli, T, out_dtype="bf16").forward(dx)
    assert torch.equal(o16, o32.to(torch.bfloat16))


# --------------------------------------------------------------------- full sizes
FULL = [("olmoe", 1), ("olmoe", 16), ("olmoe", 64), ("olmoe", 4096),
        ("v2lite", 32), ("v2lite", 8192), ("qwen3_int4", 1), ("qwen3_int4", 64),
        ("qwen3_int4", 16384), ("qwen3_int8", 1), ("qwen3_int8", 64), ("qwen3_int8", 16384),
        ("qwen3_fp8", 1), ("qwen3_fp8", 64), ("qwen3_fp8", 16384)]


@pytest.mark.parametrize("preset,T", FULL)
def test_full_size_layer_sampled(preset, T):
    sh = moe_synth.PRESETS[preset]
    res = run_layer(sh, T, tokens=sample_rows(T))
    assert res.max_margin_mismatch < ROUTE_MARGIN, (res.mismatched, res.max_margin_mismatch)
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    assert res.err_ratio_delta <= DELTA_GUARD[sh.expert], res.err_ratio_delta
    print(f"{preset} T={T}: mismatched routes {res.mismatched} (max margin "
          f"{res.max_margin_mismatch:.2e}), swaps/token {res.drift['swaps_per_token']:.4f}, "
          f"err/rms(out) {res.err_ratio:.3e}, "
          f"err/rms(delta) {res.err_ratio_delta:.3e}")


@pytest.fixture(scope="module")
def v2lite_weights():
    li = moe_synth.make_layer(moe_synth.PRESETS["v2lite"])
    yield li, li.to("cuda")


@pytest.mark.parametrize("T", [32, 8192])
@pytest.mark.parametrize("C", [1.0, 1.5])
def test_v2lite_capacity_factors(C, T, v2lite_weights):
    """Capacity C in {1.0, 1.5} (the preset's 1.25 is in the full-size list) at the
    decode and the prefill batch: at T = 8192 the caps of 768 / 1152 rows drop
    slots of many experts across the multi-CTA permutation."""
    sh = moe_synth.PRESETS["v2lite"].with_(capacity_factor=C)
    li, dli = v2lite_weights
    li, dli = dataclasses.replace(li, shape=sh), dataclasses.replace(dli, shape=sh)
    x = moe_synth.make_x(sh, T)
    res = run_layer(sh, T, tokens=sample_rows(T), data=(li, x, dli, x.cuda()))
    assert res.max_margin_mismatch < ROUTE_MARGIN, (res.mismatched, res.max_margin_mismatch)
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    assert res.err_ratio_delta <= DELTA_GUARD[sh.expert], res.err_ratio_delta
    print(f"v2lite C={C} T={T}: mismatched routes {res.mismatched}, swaps/token "
          f"{res.drift['swaps_per_token']:.4f}, err/rms(out) {res.err_ratio:.3e}, "
          f"err/rms(delta) {res.err_ratio_delta:.3e}")


@pytest.fixture(scope="module")
def v3_weights():
    li = moe_synth.make_layer(moe_synth.PRESETS["v3"])
    yield li, li.to("cuda")


@pytest.mark.parametrize("T", [32, 256, 9440])
def test_v3_full_size_sampled(T, v3_weights):
    """The DeepSeek-V3-shaped layer (d 7168, 256 experts with Zipf(1.1)-skewed
    select-mode bias, 1 shared expert; 22.5 GB of bf16 weights, generated once
    for the module) at the decode, crossover and compute-bound batches."""
    sh = moe_synth.PRESETS["v3"]
    li, dli = v3_weights
    x = moe_synth.make_x(sh, T)
    res = run_layer(sh, T, tokens=sample_rows(T, 16), data=(li, x, dli, x.cuda()))
    assert res.max_margin_mismatch < ROUTE_MARGIN, (res.mismatched, res.max_margin_mismatch)
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    assert res.err_ratio_delta <= DELTA_GUARD[sh.expert], res.err_ratio_delta
    print(f"v3 T={T}: mismatched routes {res.mismatched} (max margin "
          f"{res.max_margin_mismatch:.2e}), swaps/token {res.drift['swaps_per_token']:.4f}, "
          f"Jaccard {res.drift['jaccard']:.6f}, err/rms(out) {res.err_ratio:.3e}, "
          f"err/rms(delta) {res.err_ratio_delta:.3e}")


# --------------------------------------------------------------------- alignment
def _offset_copy(t):
    """A copy of ``t`` whose data starts one element past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = buf[1:].view(t.shape)
    v.copy_(t)
    return v


def test_misaligned_tensors():
    """Tensors aligned only to their element type take the scalar kernels and give
    the same results; tensor-core operands must be 16-byte aligned."""
    sh, T = SMALL["bf16_shared_cap"], SMALL_T["bf16_shared_cap"]
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    lg = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    ref = layer.forward(dx, logits=lg).clone()
    # input and output off a 16-byte boundary: scalar RMSNorm and combine, same bits
    xm = _offset_copy(dx)
    om = _offset_copy(torch.empty_like(ref))
    layer.forward(xm, om)
    assert torch.equal(om, ref)
    assert M.moe_get_device_status(layer.ws) == 0
    # router weights off a boundary: the CUDA-core split router, same logits up to
    # the order of the FP32 additions
    dli2 = dataclasses.replace(dli, w_router=_offset_copy(dli.w_router))
    layer2 = M.MoELayer(dli2, T, out_dtype="f32")
    lg2 = torch.empty_like(lg)
    layer2.forward(dx, logits=lg2)
    assert M.moe_get_device_status(layer2.ws) == 0
    torch.testing.assert_close(lg2, lg, rtol=1e-5, atol=1e-5)
    # a misaligned TMA operand is an argument error, found before any launch
    cfg, w = layer.cfg, layer.w
    ws = M.alloc_workspace(cfg)
    xn = _offset_copy(torch.zeros(T, sh.d, dtype=torch.bfloat16, device="cuda"))
    offs = torch.zeros(sh.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.zeros(T * sh.k, dtype=torch.int32, device="cuda")
    gate = torch.zeros(T * sh.k, dtype=torch.float32, device="cuda")
    y = torch.empty(T * sh.k, sh.d, dtype=torch.float32, device="cuda")
    ys = torch.empty(sh.n_shared, T, sh.d, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as e:
        M.moe_grouped_ffn(cfg, w, xn, offs, perm, gate, y, ys, ws)
    assert e.value.status == M.MOE_ERR_INVALID


# --------------------------------------------------------------------- single launch
DECODE_ONE_LAUNCH = {
    "olmoe_like": (LayerShape("d1", d=2048, E=64, k=8, f=1024, bias_mode="logit", seed=51), 1),
    "shared_cap": (LayerShape("d2", d=1024, E=32, k=6, f=512, n_shared=2, capacity_factor=1.0,
                              seed=52), 32),
    "select_256": (LayerShape("d3", d=768, E=256, k=8, f=256, n_shared=1, bias_mode="select",
                              seed=53), 17),
    "wide_tiles": (LayerShape("d4", d=512, E=8, k=8, f=384, seed=54), 32),
}


@pytest.mark.parametrize("name", list(DECODE_ONE_LAUNCH))
def test_single_launch_decode_layer_equals_the_kernel_chain(name):
    """Decode batches of bf16 experts run as one cooperative launch; the profiled
    entry point runs the same layer as a chain of kernels.  The two give the same
    bits (the RMSNorm sum of squares of bf16 inputs is exact in double, and the
    GEMM tiles are the same), the same routes, and the oracle's result."""
    sh, T = DECODE_ONE_LAUNCH[name]
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    assert M.moe_layer_launch_count(layer.cfg) == 1
    idx = torch.empty(T, sh.k, dtype=torch.int32, device="cuda")
    one = layer.forward(dx, topk_idx=idx).clone()
    assert M.moe_get_device_status(layer.ws) == 0
    evs = [torch.cuda.Event(enable_timing=True)
           for _ in range(M.moe_layer_step_count(layer.cfg) + 1)]
    chain = torch.empty_like(one)
    M.moe_layer_forward_profiled(layer.cfg, layer.w, dx, chain, layer.ws, evs)
    assert M.moe_get_device_status(layer.ws) == 0
    assert torch.equal(one, chain)
    # and twice in a row (the grid-barrier words are left ready for the next call)
    again = layer.forward(dx)
    assert torch.equal(again, one)
    res = run_layer(sh, T)
    assert res.max_margin_mismatch < ROUTE_MARGIN
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio
    print(f"{name}: err/rms(out) {res.err_ratio:.3e}, err/rms(delta) {res.err_ratio_delta:.3e}")


PREFILL_TILES = {
    "bf16_prefill_tiles": (SMALL["bf16_prefill_tiles"], 1000),
    "bf16_prefill_skew": (SMALL["bf16_prefill_skew"], 700),
    # several full tiles per expert and a ragged last one on each (1500 x 4 / 8 =
    # 750 mean rows: 2 pair tiles + 238, 5 single tiles + 110), capacity-cut
    "bf16_many_tiles": (LayerShape("bf16_many_tiles", d=256, E=8, k=4, f=256, n_shared=1,
                                   capacity_factor=1.1, seed=24), 1500),
    # quantised weights expanded into shared memory, on CTA pairs or single CTAs
    # (550 / 600 / 560 rows per expert; quantised experts take single CTAs by default)
    "int4_pairs": (LayerShape("int4_pairs", d=256, E=8, k=4, f=384, n_shared=1, expert="int4",
                              seed=28), 1100),
    "int8_pairs": (LayerShape("int8_pairs", d=384, E=8, k=4, f=256, expert="int8",
                              capacity_factor=1.1, seed=29), 1200),
    "fp8_pairs": (LayerShape("fp8_pairs", d=256, E=8, k=4, f=256, n_shared=1, expert="fp8",
                             seed=30), 1120),
}


@pytest.mark.parametrize("name", list(PREFILL_TILES))
def test_prefill_pair_and_single_tiles_give_the_same_bits(name):
    """moe_config.prefill_tiles picks 256-token tiles on CTA pairs (2) or 128-token
    tiles on single CTAs (1) for prefill batches (0: chosen by the rows per
    expert), bf16 or quantised.  Each output element is one FP32 dot product accumulated in the same
    k order either way, so the layer outputs agree bit for bit; the result is
    checked against the oracle."""
    sh, T = PREFILL_TILES[name]
    data = inputs_on_device(sh, T)
    li, x, dli, dx = data
    layer = M.MoELayer(dli, T, out_dtype="f32")
    assert layer.cfg.prefill_tiles == 0
    auto = layer.forward(dx).clone()
    assert M.moe_get_device_status(layer.ws) == 0
    layer.cfg.prefill_tiles = 2
    pair = layer.forward(dx).clone()
    assert M.moe_get_device_status(layer.ws) == 0
    layer.cfg.prefill_tiles = 1
    single = layer.forward(dx).clone()
    assert M.moe_get_device_status(layer.ws) == 0
    assert torch.equal(pair, single)
    assert torch.equal(auto, single)
    assert M.moe_layer_launch_count(layer.cfg) >= 8
    res = run_layer(sh, T, tokens=sample_rows(T), data=data)
    assert res.max_margin_mismatch < ROUTE_MARGIN
    assert res.err_ratio <= TOL[sh.expert], res.err_ratio


def test_precision_of_bf16_rows_against_fp32_rows():
    """The layer forward keeps the gated routed rows in bf16 between the down GEMM
    and the combine; the grouped-FFN + combine entry points keep them in FP32.
    Both are measured against the oracle on the MoE delta (out - x), the stricter
    denominator: the bf16 rows may add at most their own rounding (relative 2^-9
    per row, summed over k rows) to the error the FP32 rows have, which comes from
    h rounded to bf16 before the down GEMM."""
    sh, T = LayerShape("prec", d=1024, E=32, k=8, f=512, seed=61), 512
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    idx = torch.empty(T, sh.k, dtype=torch.int32, device="cuda")
    fused = layer.forward(dx, topk_idx=idx).cpu().numpy()
    cfg, w = layer.cfg, layer.w
    ws = M.alloc_workspace(cfg)
    xn = torch.empty(T, sh.d, dtype=torch.bfloat16, device="cuda")
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    M.moe_rmsnorm_router(cfg, w, dx, xn, logits, ws)
    tidx = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T * sh.k, dtype=torch.float32, device="cuda")
    M.moe_route(cfg, logits, dli.router_bias, tidx, gate)
    counts = torch.empty(sh.E, dtype=torch.int32, device="cuda")
    offs = torch.empty(sh.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    slot = torch.empty(T * sh.k, dtype=torch.int32, device="cuda")
    drop = torch.empty(1, dtype=torch.int32, device="cuda")
    M.moe_permute(cfg, tidx, counts, offs, perm, slot, drop, ws)
    y = torch.empty(T * sh.k, sh.d, dtype=torch.float32, device="cuda")
    M.moe_grouped_ffn(cfg, w, xn, offs, perm, gate, y, None, ws)
    chain = torch.empty(T, sh.d, dtype=torch.float32, device="cuda")
    M.moe_combine(cfg, y, slot, None, dx, chain)
    chain = chain.cpu().numpy()
    rep = O.layer_from_inputs(li, x, forced_idx=idx.cpu().numpy())
    delta = rep["out"] - x.float().numpy().astype(np.float64)
    rd = float(np.sqrt(np.mean(delta ** 2)))
    e_fused = float(np.max(np.abs(fused - rep["out"]))) / rd
    e_chain = float(np.max(np.abs(chain - rep["out"]))) / rd
    print(f"err/rms(delta): bf16 rows {e_fused:.3e}, FP32 rows {e_chain:.3e}")
    assert e_chain <= DELTA_GUARD["bf16"] and e_fused <= DELTA_GUARD["bf16"]
    # the bf16 rows' own rounding: |y_a| 2^-9 summed over the k rows of a token
    bound = sh.k * 2.0 ** -9 * float(np.max(np.abs(y.cpu().numpy()))) / rd
    assert e_fused <= e_chain + bound
