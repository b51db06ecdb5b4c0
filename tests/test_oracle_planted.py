"""Plant plausible mistakes in the oracle (CPU only) and check that a pin in
test_oracle_pins.py catches each one: a dropped term, a wrong index or tie
rule, a transposed or mis-scaled operand."""
import numpy as np
import pytest

from oracle import moe_oracle as O
from tests import test_oracle_expert_choice as EC
from tests import test_oracle_pins as P


def _rms_sum_not_mean(x, gamma, eps, act):
    x = np.asarray(x, np.float64)
    r = 1.0 / np.sqrt(np.sum(x * x, axis=1) + float(np.float32(eps)))
    return O.round_act(x * r[:, None] * gamma, act)


def _rms_no_eps(x, gamma, eps, act):
    x = np.asarray(x, np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=1))
    return O.round_act(x * r[:, None] * gamma, act)


def _ffn_no_up(X, wg, wu, wd):
    return O.silu(np.asarray(X) @ wg) @ wd


def _ffn_sigmoid_gate(X, wg, wu, wd):
    u = np.asarray(X) @ wg
    return (1.0 / (1.0 + np.exp(-u)) * (np.asarray(X) @ wu)) @ wd


def _ffn_swapped_gate_up(X, wg, wu, wd):
    return O.silu(np.asarray(X) @ wu) * (np.asarray(X) @ wg) @ wd


def _topk_ties_high(keys, k):
    keys = np.asarray(keys, np.float32)
    T, E = keys.shape
    experts = np.broadcast_to(-np.arange(E), (T, E))
    order = np.lexsort((experts, -keys.astype(np.float64)), axis=1)
    ks = np.take_along_axis(keys, order, axis=1).astype(np.float64)
    margin = ks[:, k - 1] - ks[:, k] if k < E else np.full(T, np.inf)
    return order[:, :k].astype(np.int32), margin


_real_softmax = O.softmax64


def _softmax_no_shift_wrong_axis(p):
    p = np.asarray(p, np.float64)
    e = np.exp(p)
    return e / np.sum(e, axis=0, keepdims=True)


_real_permute = O.permute


def _permute_keeps_one_extra(idx, E, capacity_factor=0.0):
    c = O.capacity(capacity_factor, *np.asarray(idx).shape, E)
    if c is None:
        return _real_permute(idx, E, capacity_factor)
    # off by one: rank <= cap kept, i.e. the capacity of c + 1 rows
    T, k = np.asarray(idx).shape
    return _real_permute(idx, E, (c + 0.5) * E / (T * k))


def _route_gates_unrenormalised(logits32, bias, k, bias_mode, renormalize, forced_idx=None):
    return _real_route(logits32, bias, k, bias_mode, False, forced_idx)


_real_route = O.route


_real_ec_select = O.expert_choice_select


def _ec_ties_to_higher_token(scores32, C):
    s = np.asarray(scores32, np.float32)
    r = _real_ec_select(s[::-1], C)             # reversed token order: ties go high
    T = s.shape[0]
    tok = np.sort(T - 1 - r["tok"], axis=1).astype(np.int32)
    return dict(r, tok=tok, gate=np.take_along_axis(s.T, tok, axis=1).astype(np.float64))


def _ec_decode_e4m3_bias_8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return np.where(c & 0x80, -1.0, 1.0) * mag


MUTANTS = [
    ("rmsnorm", _rms_sum_not_mean, P.test_rmsnorm_matches_torch_rms_norm),
    ("rmsnorm", _rms_no_eps, P.test_rmsnorm_eps_matters_for_tiny_rows),
    ("expert_ffn", _ffn_no_up, P.test_expert_ffn_matches_torch_swiglu),
    ("expert_ffn", _ffn_sigmoid_gate, P.test_single_expert_layer_is_a_dense_ffn),
    ("expert_ffn", _ffn_swapped_gate_up, P.test_expert_ffn_matches_torch_swiglu),
    ("topk_sorted", _topk_ties_high,
     lambda: P.test_topk_matches_rank_by_counting_with_ties(8, 2)),
    ("softmax64", _softmax_no_shift_wrong_axis, P.test_softmax_matches_torch),
    ("permute", _permute_keeps_one_extra, lambda: P.test_permute_matches_brute_force(1.0)),
    ("route", _route_gates_unrenormalised, P.test_gates_renormalised_and_bias_modes),
    ("expert_choice_select", _ec_ties_to_higher_token,
     EC.test_selection_matches_a_library_sort_with_ties),
    ("decode_e4m3", _ec_decode_e4m3_bias_8, P.test_e4m3_decode_matches_torch_float8_on_every_code),
]


@pytest.mark.parametrize("name,mutant,pin", MUTANTS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pin):
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()
