"""Sweep the per-bpw target RMS of the scaled, transformed weights.

Prints, for each bits-per-weight setting, the relative reconstruction MSE of the
oracle's encode -> decode on Gaussian rows as a function of sigma_t, where the
global scale is s = rms(W) / sigma_t.  The minimisers, rounded to 0.05, are the
SIGMA_T constants of decode_gemm_e8_b200/synth.py.  Test infrastructure: calls
only the oracle.

    python -m oracle.sigma_sweep
"""
from __future__ import annotations

import numpy as np

from oracle import oracle as orc


def sweep(N: int = 64, K: int = 1024, seed: int = 12345):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    rms = float(np.sqrt(np.mean(W.astype(np.float64) ** 2)))
    res = {}
    for bpw in (2, 3, 4):
        rows = []
        for sig in (0.70, 0.75, 0.80, 0.85, 0.90, 0.95, 1.00, 1.05, 1.10):
            s = float(np.float32(rms / sig))
            i1, i2 = orc.encode(W, bpw, 7, s)
            wd = orc.bf16_bits_to_f32(orc.decode(i1, i2, N, K, bpw, 7, s)).astype(np.float64)
            mse = float(np.mean((wd - W) ** 2) / rms ** 2)
            rows.append((sig, mse))
            print("bpw %d sigma_t %.2f  rel-mse %.5f" % (bpw, sig, mse), flush=True)
        res[bpw] = min(rows, key=lambda r: r[1])[0]
    print("argmin:", res)
    return res


if __name__ == "__main__":
    sweep()
