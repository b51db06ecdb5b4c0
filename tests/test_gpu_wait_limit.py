"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

Every wait of the tensor-core kernels' pipelines is bounded by
moe_config.wait_kcycles.  With a limit of 1024 clock cycles (about half a
microsecond) the first accumulator wait of the epilogue cannot be met -- a tile's
main loop alone takes far longer -- so the kernel must give up: record device
error 2, drain its own copies and MMAs, free its TMEM and return.  The test then
checks that the context is still usable: the status is read on the host, and the
next call with the default limit gives bit for bit the result of a call made
before the time-out."""
import ctypes

import pytest
import torch

import moe_layer_fp32_b200 as M
from moe_synth import LayerShape
from tests.layer_check import inputs_on_device

pytestmark = pytest.mark.gpu

CASES = {
    # 128-token (prefill) tiles, bf16 experts, 2 shared experts
    "bf16_prefill": (LayerShape("wl_prefill", d=1024, E=8, k=2, f=512, n_shared=2, seed=31), 600),
    # 16-token tiles with the in-GEMM row gather
    "bf16_decode": (LayerShape("wl_decode", d=1024, E=32, k=4, f=512, seed=32), 24),
    # int4 decode tiles: dequantisation warps and split K
    "int4_decode": (LayerShape("wl_int4", d=1024, E=16, k=4, f=512, expert="int4", seed=33), 8),
}


@pytest.fixture(autouse=True)
def _dev(cuda_device):
    yield


@pytest.mark.parametrize("name", list(CASES))
def test_wait_limit_runs_out_and_the_next_call_is_exact(name):
    sh, T = CASES[name]
    li, x, dli, dx = inputs_on_device(sh, T)
    layer = M.MoELayer(dli, T, out_dtype="f32")
    ref = layer.forward(dx).clone()
    assert M.moe_get_device_status(layer.ws) == 0

    short = M.make_config(sh, T, out_dtype="f32")
    short.wait_kcycles = 1
    out = torch.empty_like(ref)
    M.moe_layer_forward(short, layer.w, dx, out, layer.ws)
    assert M.moe_get_device_status(layer.ws) == 2          # a wait ran out

    M.moe_clear_device_status(layer.ws)
    again = layer.forward(dx)
    assert M.moe_get_device_status(layer.ws) == 0
    assert torch.equal(again, ref)


def test_negative_wait_limit_is_an_argument_error():
    sh, T = CASES["bf16_decode"]
    cfg = M.make_config(sh, T)
    cfg.wait_kcycles = -1
    assert M.moe_workspace_size(cfg) == 0
