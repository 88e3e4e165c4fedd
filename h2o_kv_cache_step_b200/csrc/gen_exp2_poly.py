"""Coefficients of the polynomial 2^f, f in [-1/2, 1/2], used by the
FMA-pipe exp2 in tc_ptx.cuh (exp2_poly3 / exp2_poly4).

Method: least-squares fit of the RELATIVE error at 4096 Chebyshev nodes of
[-1/2, 1/2] (a near-minimax fit), coefficients rounded to float32, then the
float32 Horner evaluation is checked against numpy's exp2 in float64.
Run: python h2o_kv_cache_step_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def fit(deg, n=4096):
    k = np.arange(n)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * n))     # Chebyshev nodes in [-1/2, 1/2]
    y = np.exp2(f)
    A = np.stack([f ** j for j in range(deg + 1)], axis=1) / y[:, None]   # relative weighting
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return c.astype(np.float32)


def horner32(c, f):
    f = f.astype(np.float32)
    r = np.full_like(f, c[-1])
    for a in c[-2::-1]:
        r = (r * f + a).astype(np.float32)
    return r


if __name__ == "__main__":
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    for deg in (3, 4):
        c = fit(deg)
        err = np.abs(horner32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max()
        print(f"degree {deg}: max rel err {err:.3e}")
        print("  " + ", ".join(f"{float(a):.9e}f" for a in c))
