"""Route-drift metrics (swaps per token, Jaccard) on hand-worked cases."""
import numpy as np
import pytest

from moe_layer_fp32_b200.drift import route_drift


def test_identical_routes_have_no_drift():
    a = np.array([[3, 1, 7], [0, 2, 5]])
    r = route_drift(a, a[:, ::-1])            # order within a row does not matter
    assert r["swaps_per_token"] == 0 and r["jaccard"] == 1 and r["tokens_changed"] == 0


def test_hand_worked_swaps_and_jaccard():
    a = np.array([[0, 1, 2, 3], [4, 5, 6, 7], [0, 1, 2, 3]])
    b = np.array([[0, 1, 2, 9], [4, 5, 10, 11], [12, 13, 14, 15]])
    r = route_drift(a, b)
    # swaps 1, 2, 4 -> mean 7/3; Jaccard 3/5, 2/6, 0/8 -> mean (0.6 + 1/3 + 0) / 3
    assert r["swaps_per_token"] == pytest.approx(7 / 3)
    assert r["selection_shift"] == pytest.approx(7 / 12)
    assert r["jaccard"] == pytest.approx((0.6 + 1 / 3) / 3)
    assert r["tokens_changed"] == 3 and r["max_swaps"] == 4


def test_swaps_equal_k_times_shift_on_random_routes():
    rng = np.random.default_rng(0)
    E, k, T = 64, 8, 500
    a = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    b = a.copy()
    # move exactly m experts of each row to ids outside the row
    m = rng.integers(0, k + 1, T)
    for t in range(T):
        free = np.setdiff1d(np.arange(E), a[t])
        b[t, :m[t]] = rng.choice(free, m[t], replace=False)
    r = route_drift(a, b)
    assert r["swaps_per_token"] == pytest.approx(m.mean())
    assert r["swaps_per_token"] == pytest.approx(k * r["selection_shift"])
    assert r["jaccard"] == pytest.approx(np.mean((k - m) / (k + m)))


def test_shape_mismatch_is_an_error():
    with pytest.raises(ValueError):
        route_drift(np.zeros((2, 3)), np.zeros((2, 4)))
