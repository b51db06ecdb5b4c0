"""Route drift between two top-k selections of the same tokens (host logic).

picx.dev summary of the moe-ceilings study, Sub-study 2 (causal route replay)
and Results: a change to the router's arithmetic is judged by how many of a
token's k selected experts it swaps, "swaps per token = k x selection shift".
For selections A_t and B_t of token t (sets of k expert ids):

* swaps_t   = k - |A_t intersect B_t|  (experts of A_t that B_t replaced);
* jaccard_t = |A_t intersect B_t| / |A_t union B_t|;
* shift_t   = swaps_t / k              (the fraction of the selection that moved).

The report averages them over tokens and counts the tokens with any swap.
"""
from __future__ import annotations

import numpy as np


def route_drift(idx_a, idx_b) -> dict:
    """Drift between two routings ``idx[T, k]`` (order within a row ignored)."""
    a = np.asarray(idx_a, dtype=np.int64)
    b = np.asarray(idx_b, dtype=np.int64)
    if a.shape != b.shape or a.ndim != 2:
        raise ValueError("both routings must be [T, k] of the same shape")
    T, k = a.shape
    if T == 0:
        return dict(tokens=0, k=k, swaps_per_token=0.0, selection_shift=0.0, jaccard=1.0,
                    tokens_changed=0, max_swaps=0)
    # |A intersect B| per row: each id of A found in B (ids within a row are distinct)
    inter = (a[:, :, None] == b[:, None, :]).any(axis=2).sum(axis=1)
    swaps = k - inter
    jac = inter / (2 * k - inter)
    return dict(tokens=int(T), k=int(k), swaps_per_token=float(swaps.mean()),
                selection_shift=float(swaps.mean() / k), jaccard=float(jac.mean()),
                tokens_changed=int((swaps > 0).sum()), max_swaps=int(swaps.max()))
