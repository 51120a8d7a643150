"""Fit Swish-like starting coefficients for the KAT-S-shaped workload.

The FlashKAT notes (section "Loss / training strategy") say the second GR-KAN
layer of each block starts as Swish, but print no coefficients. This script
fits them: degree-5 numerator a_0..a_5 and degree-4 denominator b_1..b_4 so that
P(x)/(1+|Q(x)|) approximates swish(x) = x / (1 + exp(-x)) on [-4, 4].

Method: linearised least squares in float64. With s = swish(x) and assuming
1 + Q(x) > 0 on the grid, P(x) - s(x)(1 + Q(x)) = 0 is linear in (a, b), so
minimise sum_k (P(x_k) - s(x_k) Q(x_k) - s(x_k))^2 over 1001 uniform points.
The fit is then checked with the absolute value in place.

Run:  python synth/fit_swish.py      (writes synth/swish_fit.json)
"""
import json
import os

import numpy as np


def fit(npts=1001, lo=-4.0, hi=4.0, m=5, n=4):
    x = np.linspace(lo, hi, npts, dtype=np.float64)
    s = x / (1.0 + np.exp(-x))
    cols = [x**i for i in range(m + 1)] + [-s * x**j for j in range(1, n + 1)]
    A = np.stack(cols, axis=1)
    theta, *_ = np.linalg.lstsq(A, s, rcond=None)
    a = theta[: m + 1]
    b = theta[m + 1:]
    P = sum(a[i] * x**i for i in range(m + 1))
    Q = sum(b[j - 1] * x**j for j in range(1, n + 1))
    approx = P / (1.0 + np.abs(Q))
    return a, b, float(np.max(np.abs(approx - s))), float(np.min(1.0 + Q))


def main():
    a, b, err, min_den = fit()
    out = {
        "target": "swish(x) = x / (1 + exp(-x)) on [-4, 4], 1001 uniform points",
        "method": "float64 linearised least squares, see fit_swish.py",
        "a": [float(v) for v in a],
        "b": [float(v) for v in b],
        "max_abs_err_on_grid": err,
        "min_1_plus_Q_on_grid": min_den,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "swish_fit.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
