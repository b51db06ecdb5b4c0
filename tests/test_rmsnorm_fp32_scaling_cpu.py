"""The RMSNorm kernels scale x r gamma in FP32 where that provably gives the bf16
of the double product, and in double elsewhere.  The claim they rest on: with x a
bf16 value, r32 = fl32(r) and two FP32 products, y32 lies within 3 units in the
last place of the exact product, so y32 and the double product round to the same
bf16 whenever the 16 low bits of y32 are more than 8 units from the rounding
midpoint 0x8000 (exponent field 2..252).  Checked here over every finite bf16 x
and scales across twelve decades, on the CPU (the GPU bit-exact RMSNorm tests check
the kernels themselves)."""
import numpy as np
import torch


def _bf16_bits_rne_from_f64(v):
    """bf16 bits of float64 values, one round-to-nearest-even on the double bits."""
    b = v.view(np.uint64).copy()
    b = b + np.uint64(0xFFFFFFFFFFF) + ((b >> np.uint64(45)) & np.uint64(1))
    b &= ~np.uint64(0x1FFFFFFFFFFF)
    # 8 significant bits now: exact in FP32 (beyond its range only where the caller
    # does not look), whose top half is the bf16
    with np.errstate(over="ignore"):
        f32 = b.view(np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def test_fp32_scaling_is_certified_where_claimed():
    rng = np.random.default_rng(5)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.int16)
    x = torch.from_numpy(bits).view(torch.bfloat16).float().numpy()
    x = x[np.isfinite(x)]
    certified = 0
    for it in range(40):
        r = float(1.0 / np.sqrt(10.0 ** rng.uniform(-6, 6)))
        g = np.float32(rng.uniform(-3, 3) if it % 2 else 10.0 ** rng.uniform(-3, 3))
        with np.errstate(over="ignore"):
            y = (x * np.float32(r)).astype(np.float32) * g
        u = y.astype(np.float32).view(np.uint32)
        low, ex = u & 0xFFFF, (u >> 23) & 0xFF
        ok = (ex > 1) & (ex < 253) & ((low < 0x8000 - 8) | (low > 0x8000 + 8))
        fast = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
        yd = (x.astype(np.float64) * r) * np.float64(g)
        normal = (np.abs(yd) >= 2.0 ** -126) & (np.abs(yd) < 2.0 ** 127)
        exact = _bf16_bits_rne_from_f64(yd).view(np.int16)
        m = ok & normal
        assert np.array_equal(fast.numpy()[m], exact[m])
        certified += int(m.sum())
    assert certified > 2_000_000
