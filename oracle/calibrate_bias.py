"""Find the OLMoE-shaped logit-mode bias scale beta (test infrastructure).

The OLMoE-shaped workload skews expert popularity with ``bias_e = beta * z_e``
so that the busiest expert carries about 1.5x the mean load ("MoE: dynamism the
compiler cannot remove", capacity section: a busiest expert at 1.3-1.8x the
mean is common).  This script bisects beta on the T = 4096 batch using only the
oracle's routing and prints it; ``moe_synth.OLMOE_BIAS_BETA`` holds the result,
rounded to a multiple of 2^-10, and ``tests/test_oracle_pins.py`` re-checks it.

    python -m oracle.calibrate_bias
"""
import numpy as np

import moe_synth
from oracle import moe_oracle as O


def load_ratio(beta: float, T: int = 4096) -> float:
    sh = moe_synth.PRESETS["olmoe"]
    x = moe_synth.make_x(sh, T).float().numpy()
    wr = moe_synth.make_router(sh).float().numpy()
    z = np.random.default_rng(np.random.SeedSequence([101, 4, 0])).standard_normal(sh.E)
    bias = (beta * z).astype(np.float32)
    xn = O.rmsnorm(x, np.ones(sh.d), sh.rms_eps, sh.act)
    l32 = O.router_logits(xn, wr).astype(np.float32)
    r = O.route(l32, bias, sh.k, O.BIAS_LOGIT, sh.renormalize)
    counts = O.permute(r["idx"], sh.E)["counts"]
    return float(counts.max() / counts.mean())


def main():
    lo, hi = 0.0, 2.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if load_ratio(mid) < 1.5:
            lo = mid
        else:
            hi = mid
    beta = round(0.5 * (lo + hi) * 1024) / 1024
    print(f"beta = {beta!r}  ratio = {load_ratio(beta):.4f}")


if __name__ == "__main__":
    main()
