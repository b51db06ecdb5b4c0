"""moe_permute_static, the permutation for callers that cannot allocate device
memory (an engine plugin that is handed only its input and output tensors, or a
server whose device memory is all reserved when it starts).  Its scratch is an
array built into the library, so it takes no workspace.

Checked through the C ABI against moe_permute with a full workspace, on two
calls in a row (the built-in array keeps the previous call's contents, which
must not leak into the next result).  Outputs are integers: bit-exact, the
tolerance every permutation test here uses.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import moe_layer_fp32_b200 as M
from moe_synth import LayerShape

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _dev(cuda_device):
    yield


def skewed_routes(T, k, E, seed):
    r = np.random.default_rng(seed)
    pop = np.arange(1, E + 1, dtype=np.float64) ** -1.1
    pop /= pop.sum()
    return np.stack([r.choice(E, k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)


def outputs(T, k, E, fill):
    n = T * k
    return [torch.full((E,), fill, dtype=torch.int32, device="cuda"),
            torch.full((E + 1,), fill, dtype=torch.int32, device="cuda"),
            torch.full((n,), fill, dtype=torch.int32, device="cuda"),
            torch.full((n,), fill, dtype=torch.int32, device="cuda"),
            torch.full((1,), fill, dtype=torch.int32, device="cuda")]


@pytest.mark.parametrize("T,k,E,C", [(16384, 8, 128, 0.0), (9440, 8, 256, 1.0),
                                     (6000, 6, 512, 1.25), (37, 6, 64, 1.25)])
def test_static_permute_matches_workspace_permute_twice(T, k, E, C):
    cfg = M.make_config(LayerShape("p", d=256, E=E, k=k, f=256, capacity_factor=C), T)
    ref = outputs(T, k, E, -5)
    ws = M.alloc_workspace(cfg)
    # two routings, so the second static call starts from the first one's leftovers
    for call, seed in enumerate((T + E, T + E + 1)):
        idx = torch.as_tensor(skewed_routes(T, k, E, seed)).cuda()
        M.moe_permute(cfg, idx, *ref[:4], ref[4], ws)
        got = outputs(T, k, E, 7 + call)
        M.moe_permute_static(cfg, idx, *got)
        torch.cuda.synchronize()
        kept = int(ref[1][E].item())
        for name, a, b in zip(("counts", "offsets", "perm_assign", "slot_of", "n_dropped"),
                              ref, got):
            if name == "perm_assign":
                a, b = a[:kept], b[:kept]
            assert torch.equal(a, b), (call, name)
    assert M.moe_get_device_status(ws) == 0


def test_static_permute_rejects_batches_beyond_its_scratch():
    # E * ceil(T*k / 2048) = 512 * 513 > 262144 int32 counters: refused, nothing launched
    T, k, E = 131329, 8, 512
    cfg = M.make_config(LayerShape("p", d=256, E=E, k=k, f=256), T)
    dummy = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_permute_static(cfg, dummy, dummy, dummy, dummy, dummy, dummy)
    assert ei.value.status == M.MOE_ERR_WORKSPACE


@pytest.mark.parametrize("T,k,E", [(40, 6, 64), (9440, 8, 256)])
def test_static_permute_drops_out_of_range_ids_like_moe_permute(T, k, E):
    """Expert ids outside [0, E) are dropped (slot -1) by both entry points; the
    static one has no workspace for the error word, so it reports nothing and
    returns MOE_OK.  T*k = 240 takes the one-CTA kernel, 75520 the three-kernel
    path."""
    cfg = M.make_config(LayerShape("p", d=256, E=E, k=k, f=256, capacity_factor=1.25), T)
    idx_h = skewed_routes(T, k, E, 99)
    bad = np.zeros(T * k, bool)
    flat = idx_h.reshape(-1)
    r = np.random.default_rng(3)
    for a in r.choice(T * k, 12, replace=False):
        flat[a] = -1 if a % 2 else E
        bad[a] = True
    idx = torch.as_tensor(idx_h).cuda()
    ref = outputs(T, k, E, -5)
    ws = M.alloc_workspace(cfg)
    M.moe_permute(cfg, idx, *ref[:4], ref[4], ws)
    assert M.moe_get_device_status(ws) == 1          # the workspace entry point reports
    got = outputs(T, k, E, 7)
    M.moe_permute_static(cfg, idx, *got)             # raises unless MOE_OK
    torch.cuda.synchronize()
    slot = got[3].cpu().numpy()
    assert np.all(slot[bad] == -1)
    assert int(got[0].sum().item()) == T * k - int(bad.sum())
    kept = int(ref[1][E].item())
    for name, a, b in zip(("counts", "offsets", "perm_assign", "slot_of", "n_dropped"), ref, got):
        if name == "perm_assign":
            a, b = a[:kept], b[:kept]
        assert torch.equal(a, b), name
