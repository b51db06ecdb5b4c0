"""The harness's roofline helpers against the arithmetic the pages print."""
import json
import os

import pytest

import moe_synth
from moe_layer_fp32_b200 import roofline as R

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_arithmetic.json")))


def test_amdahl_brackets_the_printed_ceiling():
    g = G["amdahl"]
    lo, hi = (R.amdahl(g["f"], s) for s in g["isolated_speedups"])
    assert lo == pytest.approx(1.069, abs=5e-4) and hi == pytest.approx(1.075, abs=5e-4)
    assert lo <= g["printed_ceiling"] <= hi
    assert R.amdahl(g["f"], 1e12) == pytest.approx(1 / (1 - g["f"]), rel=1e-9)


def test_all_to_all_bytes():
    g = G["all_to_all"]
    b = R.all_to_all_bytes(g["B"], g["k"], g["d"], g["bytes_per_elem"])
    assert b == 3670016
    assert b / 1e6 == pytest.approx(g["printed_MB"], abs=0.005)


def test_ridge_batch():
    g = G["ridge"]
    assert R.ridge_batch(g["h100_ridge_flop_per_byte"], g["E"], g["k"]) == g["printed_batch"]


def test_experts_touched_limits():
    assert R.experts_touched_expected(64, 8, 1) == pytest.approx(8)
    assert R.experts_touched_expected(64, 8, 10 ** 6) == pytest.approx(64)


def test_layer_bytes_and_flops_for_the_olmoe_shape():
    sh = moe_synth.PRESETS["olmoe"]
    # T = 1: 8 experts of 3 * 2048 * 1024 bf16 weights (+ router, x, out) ~ 101 MB
    b = R.layer_bytes(sh, 1, touched=8)
    assert b == pytest.approx(8 * 3 * 2048 * 1024 * 2 + 2048 * 64 * 2 + 2048 * 4)
    assert 100e6 < b < 102e6
    f = R.layer_flops(sh, 4096, kept=4096 * 8)
    assert f == pytest.approx(6 * 2048 * 1024 * 4096 * 8 + 2 * 4096 * 2048 * 64)
    assert 410e9 < f < 416e9


def test_int4_bytes_include_scales():
    sh = moe_synth.PRESETS["qwen3_int4"]
    eb = R.expert_bytes("int4", sh.d, sh.f, 128)
    assert eb == 3 * 2048 * 768 * 0.5 + 2 * (2 * 16 * 768 + 6 * 2048)


def test_peaks_fallback(tmp_path):
    p = R.measured_peaks(str(tmp_path / "missing.json"))
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0


def test_tensor_peak_follows_the_timed_loop_length():
    peaks = {"bf16_tflops": 1610.9, "bf16_tflops_sustained": 1393.5, "source": "measured"}
    v, label = R.tensor_peak(peaks, 0.2, 1965.0)
    assert v == 1610.9 and "burst" in label and "200 ms" in label
    v, label = R.tensor_peak(peaks, 5.0)
    assert v == 1393.5 and "sustained" in label


def test_kernel_digest_ignores_comments_only():
    """The traffic figures stay tied to the kernel code: a comment edit keeps the
    digest, a code edit changes it."""
    import bench
    code = "int a = 1;  // one\n// a note\n\nint b = 2;\n"
    assert bench.code_of(code) == bench.code_of("int a = 1;\nint b = 2;   // two\n")
    assert bench.code_of(code) != bench.code_of("int a = 1;\nint b = 3;\n")
