"""Coefficients of the FMA-pipe exponential in exp2_poly.cuh.

A degree-4 polynomial p(f) ~ 2^f on [-1/2, 1/2], fitted by the Remez
exchange algorithm on the relative error (p(f) - 2^f) / 2^f, then rounded to
FP32; the script reports the maximum relative error of the FP32 coefficients
evaluated in FP32 Horner form with fused multiply-adds.

    python quantized_attention_quant_b200/csrc/fit_exp2_poly.py
"""

import numpy as np


def remez_exp2(deg, iters=30, lo=-0.5, hi=0.5):
    n = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the n reference points
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            a[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        c = np.linalg.solve(a, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # the new reference: the extremum of each sign-alternating run
        sign = np.sign(err)
        edges = np.nonzero(sign[1:] != sign[:-1])[0] + 1
        runs = np.split(np.arange(len(grid)), edges)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) == n:
            x = grid[ext]
    return c


def fp32_horner_error(c32, lo=-0.5, hi=0.5):
    f = np.linspace(lo, hi, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        # a fused multiply-add: the product is exact in FP64, one rounding to FP32
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
    t = np.exp2(f.astype(np.float64))
    return float(np.abs((p.astype(np.float64) - t) / t).max())


if __name__ == "__main__":
    c32 = remez_exp2(4).astype(np.float32)
    for k, (v, b) in enumerate(zip(c32, c32.view(np.uint32))):
        print(f"constexpr unsigned kExp2C{k} = 0x{int(b):08x}u;  // {float(v):.9g}")
    e = fp32_horner_error(c32)
    print(f"max relative error {e:.3e} (2^{np.log2(e):.2f})")
