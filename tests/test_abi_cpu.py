"""The C-ABI library on a host without a GPU: it builds for sm_100a, loads,
exports every function include/moe.h declares, agrees with the binding's
struct layouts, and validates arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import moe_layer_fp32_b200 as M
import moe_synth
from moe_layer_fp32_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(moe_\w+)\s*\(", text, re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_layer_forward",
              "moe_workspace_size", "moe_get_device_status", "moe_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    fields_c = [f for f, _ in M.MoeConfig._fields_]
    fields_w = [f for f, _ in M.MoeWeights._fields_]
    body = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', 'int main(void){',
            'printf("%zu %zu\\n", sizeof(moe_config), sizeof(moe_weights));']
    body += [f'printf("%zu\\n", offsetof(moe_config, {f}));' for f in fields_c]
    body += [f'printf("%zu\\n", offsetof(moe_weights, {f}));' for f in fields_w]
    body += ["return 0;}"]
    src.write_text("\n".join(body))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", str(src), "-o", str(exe)], check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                           check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(M.MoeConfig) and vals[1] == ctypes.sizeof(M.MoeWeights)
    offs = [getattr(M.MoeConfig, f).offset for f in fields_c] + \
           [getattr(M.MoeWeights, f).offset for f in fields_w]
    assert vals[2:] == offs


@pytest.mark.parametrize("preset", ["tiny", "olmoe", "v2lite", "v3"])
def test_workspace_size_for_presets(lib, preset):
    sh = moe_synth.PRESETS[preset]
    for T in sh.tokens:
        n = M.moe_workspace_size(M.make_config(sh, T))
        assert n > 0 and n % 256 == 0
        # the routed output rows and hidden rows are both in there (bf16 for
        # tensor-core experts, FP32 for FP32 experts)
        eb = 4 if sh.expert == "f32" else 2
        assert n >= T * sh.k * (sh.d + sh.f) * eb


def test_invalid_configs_are_rejected_on_the_host(lib):
    sh = moe_synth.PRESETS["olmoe"]
    bad = [dict(k=65), dict(k=0), dict(T=0), dict(E=0), dict(d=100), dict(n_shared=9),
           dict(prefill_tiles=3), dict(prefill_tiles=-1), dict(wait_kcycles=-1)]
    for b in bad:
        cfg = M.make_config(sh, 16)
        for kk, v in b.items():
            setattr(cfg, kk, v)
        assert M.moe_workspace_size(cfg) == 0
        s = lib.moe_route(ctypes.byref(cfg), None, None, None, None, None)
        assert s == M.MOE_ERR_INVALID
    cfg = M.make_config(sh, 16)
    cfg.f = 1000                          # not a multiple of 128 for bf16 experts
    assert lib.moe_layer_forward(ctypes.byref(cfg), None, None, None, None, 0, None, None, None,
                                 None) == M.MOE_ERR_UNSUPPORTED
    cfg = M.make_config(sh, 16)
    w = M.MoeWeights()
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), None, None, None, 0, None,
                                 None, None, None) == M.MOE_ERR_INVALID


def test_workspace_checks(lib):
    sh = moe_synth.PRESETS["olmoe"]
    cfg = M.make_config(sh, 16)
    w = M.MoeWeights(rms_gamma=256, w_router=256, router_bias=256)
    p = ctypes.c_void_p(1 << 20)
    n = M.moe_workspace_size(cfg)
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), p, p, None, n, None, None,
                                 None, None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), p, p, p, n - 256, None,
                                 None, None, None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), p,
                                 p, ctypes.c_void_p((1 << 20) + 8), n, None, None, None,
                                 None) == M.MOE_ERR_WORKSPACE


def test_status_strings(lib):
    assert M.status_string(0) == "MOE_OK"
    assert M.status_string(3) == "MOE_ERR_WORKSPACE"
    assert M.status_string(99) == "MOE_ERR_UNKNOWN"


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(M, "_lib", None)
    monkeypatch.setattr(M, "LIB_PATH", "/nonexistent/libmoe_b200.so")
    with pytest.raises(ImportError):
        M.lib()


def test_make_weights_maps_every_layer_tensor():
    import types
    sh = moe_synth.PRESETS["v2lite"]
    names = ["gamma", "w_router", "router_bias", "w_gate", "w_up", "w_down", "sh_gate", "sh_up",
             "sh_down"]
    li = types.SimpleNamespace(**{n: types.SimpleNamespace(data_ptr=lambda i=i: 4096 * (i + 1))
                                  for i, n in enumerate(names)})
    w = M.make_weights(li)
    assert w.rms_gamma == 4096 and w.w_router == 8192 and w.sh_down == 4096 * 9
    assert w.s_gate is None and w.sh_s_gate is None


# (preset, T) -> kernel launches per layer call.  Decode batches (T <= 32) of bf16
# experts run as one cooperative launch.  Otherwise six always run (RMSNorm,
# router, route, gate/up, down, combine); the permutation adds 0 (it shares the
# routing launch up to 32 tokens), 1 (one CTA, T*k <= 4096) or 3 (count / scan /
# rank); tensor-core experts add the row gather unless bf16 decode tiles (<= 32
# rows per expert on average) gather inside the GEMM (quantised weights are
# expanded inside the GEMM at every batch).
LAUNCHES = [("tiny", 64, 7), ("olmoe", 1, 1), ("olmoe", 16, 1), ("olmoe", 64, 7),
            ("olmoe", 4096, 10), ("v2lite", 32, 1), ("v2lite", 8192, 10),
            ("qwen3_int4", 1, 7), ("qwen3_int4", 64, 8), ("qwen3_int4", 16384, 10),
            ("qwen3_int8", 16384, 10), ("qwen3_fp8", 64, 8), ("qwen3_fp8", 16384, 10),
            ("v3", 32, 1), ("v3", 256, 7), ("v3", 9440, 10)]


@pytest.mark.parametrize("preset,T,n", LAUNCHES)
def test_launch_and_step_counts(lib, preset, T, n):
    sh = moe_synth.PRESETS[preset]
    cfg = M.make_config(sh, T)
    assert M.moe_layer_launch_count(cfg) == n
    # profiled steps: 7 for FP32 experts, 8 with the [dequantise + gather] step
    assert M.moe_layer_step_count(cfg) == (7 if sh.expert == "f32" else 8)


def test_expert_choice_configuration_on_the_host(lib):
    sh = moe_synth.PRESETS["olmoe"].with_(routing="expert_choice", bias_mode="logit")
    cfg = M.make_config(sh, 4096)
    assert M.moe_expert_choice_capacity(cfg) == 4096 * 8 // 64
    assert M.moe_workspace_size(cfg) > 0
    # rmsnorm, router, scores, picks, gather, gate/up, down, combine
    assert M.moe_layer_launch_count(cfg) == 8
    cfg.capacity_factor = 1.5
    assert M.moe_expert_choice_capacity(cfg) == 768
    # a selection-only bias and FP32 experts are refused; top-k configs have no C
    assert M.moe_workspace_size(M.make_config(sh.with_(bias_mode="select"), 16)) == 0
    assert M.moe_expert_choice_capacity(M.make_config(moe_synth.PRESETS["olmoe"], 16)) == 0
    bad = M.make_config(sh, 16)
    bad.routing = 2
    assert M.moe_workspace_size(bad) == 0
