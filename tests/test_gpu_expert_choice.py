"""Expert-choice routing on the GPU ("MoE: dynamism the compiler cannot remove",
capacity section: each expert picks its top T*k/E tokens) against the oracle.

* scores: the FP32 softmax over the experts, within (E + 8) 2^-24 relative of the
  oracle's float64 softmax;
* picks: given the GPU's own FP32 scores, bit-exact to the oracle's selection
  (tokens, slots, gates), ties included;
* whole layer: the oracle re-run with the GPU's scores (selection replay), within
  the tolerances of the top-k layer; picks that differ from the oracle's own
  scores are counted and allowed only at near-ties."""
import numpy as np
import pytest
import torch

import moe_layer_fp32_b200 as M
import moe_synth
from moe_synth import LayerShape
from oracle import moe_oracle as O
from tests.layer_check import DELTA_GUARD, TOL, inputs_on_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _dev(cuda_device):
    yield


def ec_shape(name, **kw):
    return LayerShape(name, routing="expert_choice", **kw)


def route_ec(cfg, logits, bias, ws):
    T, E = logits.shape
    C = M.moe_expert_choice_capacity(cfg)
    scores = torch.empty(T, E, dtype=torch.float32, device="cuda")
    tok = torch.full((E * C,), -7, dtype=torch.int32, device="cuda")
    gate = torch.empty(E * C, dtype=torch.float32, device="cuda")
    slot = torch.empty(T, E, dtype=torch.int32, device="cuda")
    M.moe_route_expert_choice(cfg, logits, bias, scores, tok, gate, slot, ws)
    return C, scores.cpu().numpy(), tok.cpu().numpy(), gate.cpu().numpy(), slot.cpu().numpy()


@pytest.mark.parametrize("T,E,k,cf", [(1, 8, 2, 0.0), (37, 8, 2, 0.0), (300, 64, 8, 0.0),
                                      (1000, 64, 6, 1.25), (5000, 256, 8, 0.0),
                                      (2048, 128, 1, 2.0), (20, 16, 8, 4.0)])
@pytest.mark.parametrize("mode", ["none", "logit"])
def test_expert_choice_picks_bitexact_given_scores(T, E, k, cf, mode):
    r = np.random.default_rng(T * 7 + E)
    logits = r.standard_normal((T, E)).astype(np.float32)
    dup = r.choice(T, T // 4, replace=True)
    logits[dup] = logits[r.choice(T, dup.size, replace=True)]   # repeated rows: tied scores
    bias = (r.standard_normal(E) * 0.5).astype(np.float32) if mode == "logit" else None
    sh = ec_shape("ec", d=256, E=E, k=k, f=256, bias_mode=mode, capacity_factor=cf)
    cfg = M.make_config(sh, T)
    ws = M.alloc_workspace(cfg)
    dl = torch.as_tensor(logits).cuda()
    db = None if bias is None else torch.as_tensor(bias).cuda()
    C, sc, tok, gate, slot = route_ec(cfg, dl, db, ws)
    assert C == O.expert_choice_capacity(cf, T, k, E)
    ref_sc = O.expert_choice_scores(logits, bias, mode)
    np.testing.assert_allclose(sc, ref_sc, rtol=(E + 8) * 2.0 ** -24, atol=1e-38)
    ref = O.expert_choice_select(sc, C)                  # the oracle's rule on the GPU's scores
    np.testing.assert_array_equal(tok.reshape(E, C), ref["tok"])
    np.testing.assert_array_equal(slot, ref["slot"])
    np.testing.assert_array_equal(gate.reshape(E, C).astype(np.float64), ref["gate"])
    assert M.moe_get_device_status(ws) == 0


EC_LAYERS = {
    # decode tiles (in-GEMM gather), 1 shared expert, logit bias
    "ec_decode": (ec_shape("ec_decode", d=256, E=16, k=2, f=256, n_shared=1, bias_mode="logit",
                           seed=41), 64),
    # prefill tiles (gathered rows, CTA-pair GEMM), capacity factor 1.25
    "ec_prefill": (ec_shape("ec_prefill", d=512, E=8, k=2, f=384, capacity_factor=1.25,
                            seed=42), 1100),
    # int4 and fp8 experts
    "ec_int4": (ec_shape("ec_int4", d=256, E=16, k=4, f=384, expert="int4", seed=43), 48),
    "ec_fp8": (ec_shape("ec_fp8", d=384, E=8, k=2, f=256, n_shared=1, expert="fp8", seed=44), 700),
}


@pytest.mark.parametrize("name", list(EC_LAYERS))
def test_expert_choice_layer_matches_oracle(name):
    sh, T = EC_LAYERS[name]
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    counts = torch.empty(sh.E, dtype=torch.int32, device="cuda")
    out = layer.forward(dx, counts=counts).cpu().numpy()
    assert M.moe_get_device_status(layer.ws) == 0
    C = M.moe_expert_choice_capacity(layer.cfg)
    assert (counts.cpu().numpy() == C).all()
    # the layer's own scores: the same RMSNorm and router, then the routing step
    ws = M.alloc_workspace(layer.cfg)
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    M.moe_rmsnorm_router(layer.cfg, layer.w, dx, None, logits, ws)
    _, sc, tok, gate, slot = route_ec(layer.cfg, logits, dli.router_bias, ws)
    own = O.layer_expert_choice_from_inputs(li, x, tokens=[0])
    rep = O.layer_expert_choice_from_inputs(li, x, forced_scores=sc)
    np.testing.assert_array_equal(slot, rep["slot"])
    # picks against the oracle's own scores: differences only at near-ties
    moved = np.nonzero((own["slot"] >= 0) != (slot >= 0))
    if moved[0].size:
        assert own["margin"][np.unique(moved[1])].max() < 1e-6
    delta = rep["out"] - x.float().numpy().astype(np.float64)
    err = np.max(np.abs(out - rep["out"]))
    ratio = err / np.sqrt(np.mean(rep["out"] ** 2))
    ratio_d = err / np.sqrt(np.mean(delta ** 2))
    print(f"{name}: C {C}, picks moved {moved[0].size}, err/rms(out) {ratio:.3e}, "
          f"err/rms(delta) {ratio_d:.3e}")
    assert ratio <= TOL[sh.expert], ratio
    assert ratio_d <= DELTA_GUARD[sh.expert], ratio_d


def test_expert_choice_rejects_what_it_does_not_take():
    sh = ec_shape("ec_bad", d=256, E=16, k=2, f=256, bias_mode="select")
    assert M.moe_workspace_size(M.make_config(sh, 8)) == 0
    sh2 = ec_shape("ec_f32", d=256, E=16, k=2, f=256, act="f32", router="f32", expert="f32")
    assert M.moe_workspace_size(M.make_config(sh2, 8)) == 0
