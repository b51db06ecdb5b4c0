"""Pins for the oracle's expert-choice routing ("MoE: dynamism the compiler
cannot remove", capacity section: each expert picks its top T*k/E tokens; load is
balanced by construction, a token may get several experts or none).  CPU only."""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O


def rng(seed):
    return np.random.default_rng(seed)


def test_capacity_is_tk_over_e():
    assert O.expert_choice_capacity(0.0, 4096, 8, 64) == 512          # C = 1.0 exact
    assert O.expert_choice_capacity(0.0, 10, 3, 4) == math.ceil(7.5)
    assert O.expert_choice_capacity(1.25, 64, 2, 8) == 20
    assert O.expert_choice_capacity(4.0, 10, 8, 4) == 10              # at most T


def test_selection_matches_a_library_sort_with_ties():
    r = rng(1)
    T, E, C = 37, 6, 9
    s = r.random((T, E)).astype(np.float32)
    s[:12] = np.round(s[:12] * 4) / 4                                  # many exact ties
    s[3, 2] = np.nan
    sel = O.expert_choice_select(s, C)
    for e in range(E):
        keyed = [(-(-np.inf if np.isnan(s[t, e]) else float(s[t, e])), t) for t in range(T)]
        best = sorted(t for _, t in sorted(keyed)[:C])
        assert list(sel["tok"][e]) == best
        np.testing.assert_array_equal(sel["gate"][e], s[best, e].astype(np.float64))


def test_selection_by_brute_force_on_tiny_inputs():
    """The picked set is the only C-subset whose every member beats every
    non-member under (score descending, token ascending)."""
    r = rng(2)
    T, E, C = 7, 3, 3
    s = (r.integers(0, 4, (T, E)) / 4).astype(np.float32)
    sel = O.expert_choice_select(s, C)
    import itertools
    for e in range(E):
        ok = [c for c in itertools.combinations(range(T), C)
              if all((s[a, e], -a) > (s[b, e], -b) for a in c for b in range(T) if b not in c)]
        assert len(ok) == 1 and tuple(sel["tok"][e]) == ok[0]


def test_load_is_balanced_and_the_slot_map_is_consistent():
    r = rng(3)
    T, E, k = 200, 16, 4
    s = O.expert_choice_scores(r.standard_normal((T, E)).astype(np.float32), None, "none")
    C = O.expert_choice_capacity(0.0, T, k, E)
    sel = O.expert_choice_select(s, C)
    slot = sel["slot"]
    assert ((slot >= 0).sum(axis=0) == C).all()                        # every expert: C rows
    assert (slot >= 0).sum() == E * C == T * k
    flat = slot[slot >= 0]
    assert np.array_equal(np.sort(flat), np.arange(E * C))            # a bijection on slots
    for e in range(E):
        assert (slot[sel["tok"][e], e] == e * C + np.arange(C)).all()
    # some tokens get more than k experts and some none (nothing forces k per token)
    per_token = (slot >= 0).sum(axis=1)
    assert per_token.sum() == T * k


def test_scores_are_fp32_softmax_rows():
    r = rng(4)
    l = r.standard_normal((30, 12)).astype(np.float32)
    sc = O.expert_choice_scores(l, None, "none")
    np.testing.assert_allclose(sc.sum(axis=1), 1.0, rtol=12 * 2.0 ** -24)
    np.testing.assert_array_equal(sc, sc.astype(np.float32).astype(np.float64))
    with pytest.raises(ValueError):
        O.expert_choice_scores(l, np.zeros(12, np.float32), "select")


def _tiny_layer(seed=5, d=16, E=5, f=24, S=1):
    r = rng(seed)
    ws = [r.standard_normal((E, d, f)) / math.sqrt(d), r.standard_normal((E, d, f)) / math.sqrt(d),
          r.standard_normal((E, f, d)) / math.sqrt(f)]
    sh = [r.standard_normal((S, d, f)) / math.sqrt(d), r.standard_normal((S, d, f)) / math.sqrt(d),
          r.standard_normal((S, f, d)) / math.sqrt(f)]
    wr = r.standard_normal((d, E)) / math.sqrt(d)
    return O.Weights("f32", 128, *ws), O.Weights("f32", 128, *sh), wr


def test_layer_equals_dense_brute_force():
    experts, shared, wr = _tiny_layer()
    T, d, E, k = 11, 16, 5, 2
    x = rng(6).standard_normal((T, d))
    g = np.ones(d)
    res = O.moe_layer_expert_choice(x, g, wr, None, experts, k=k, act="f32", shared=shared,
                                    n_shared=1)
    xn = O.rmsnorm(x, g, 1e-6, "f32")
    sc = O.expert_choice_scores(O.router_logits(xn, wr).astype(np.float32), None, "none")
    sel = O.expert_choice_select(sc, O.expert_choice_capacity(0.0, T, k, E))
    dense = x.copy()
    for t in range(T):
        dense[t] += shared.ffn(0, xn[t:t + 1])[0]
        for e in range(E):
            if sel["slot"][t, e] >= 0:
                dense[t] += sc[t, e] * experts.ffn(e, xn[t:t + 1])[0]
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-12)


def test_every_expert_taking_every_token_is_the_dense_softmax_mixture():
    """k = E gives C = T: every expert picks every token, which is the top-k layer
    with k = E and unrenormalised gates (all experts, softmax weights)."""
    experts, _, wr = _tiny_layer(S=1)
    T, d, E = 9, 16, 5
    x = rng(7).standard_normal((T, d))
    g = np.ones(d)
    ec = O.moe_layer_expert_choice(x, g, wr, None, experts, k=E, act="f32")
    tk = O.moe_layer(x, g, wr, None, experts, k=E, act="f32", renormalize=False)
    assert ec["C"] == T
    # the expert-choice gates are the FP32 scores (relative rounding <= 2^-24), the
    # top-k gates the float64 softmax
    xn = O.rmsnorm(x, g, 1e-6, "f32")
    mag = sum(tk["probs"][:, e:e + 1] * np.abs(experts.ffn(e, xn)) for e in range(E))
    assert np.all(np.abs(ec["out"] - tk["out"]) <= 2.0 ** -24 * mag + 1e-14)
