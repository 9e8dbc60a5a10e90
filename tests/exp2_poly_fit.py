"""Derivation of the polynomial the prefill kernel uses to compute part of its exponentials on the
FMA pipe instead of the MUFU unit.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-0.5, 0.5]; 2^f is approximated by the degree-3
polynomial that minimises the maximum relative error on [-0.5, 0.5], found with the Remez exchange
algorithm (E. Remez, 1934). Running this file prints the coefficients rounded to fp32 and the error
of the fp32 Horner evaluation; exact_attention_139_b200/csrc/sm100.cuh holds the same four numbers (a CPU test checks that
they match this fit and the bound).
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
INTERVAL = (-0.5, 0.5)


def remez(deg: int = DEGREE, a: float = INTERVAL[0], b: float = INTERVAL[1], iters: int = 30):
    n = deg + 2
    x = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (b - a) / 2 + (a + b) / 2
    t = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[: deg + 1]
        err = (np.polyval(c[::-1], t) - np.exp2(t)) / np.exp2(t)
        idx = [0] + [i for i in range(1, len(t) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(t) - 1]
        sel = []
        for xi, vi in zip(t[idx], err[idx]):
            if sel and np.sign(vi) == np.sign(sel[-1][1]):
                if abs(vi) > abs(sel[-1][1]):
                    sel[-1] = (xi, vi)
            else:
                sel.append((xi, vi))
        while len(sel) > n:
            sel.pop(0 if abs(sel[0][1]) < abs(sel[-1][1]) else -1)
        if len(sel) < n:
            break
        x = np.array([s[0] for s in sel])
    return c


def fp32_coefficients():
    return [float(np.float32(v)) for v in remez()]


def horner_fp32(coeffs, f):
    f = np.asarray(f, dtype=np.float32)
    r = np.float32(coeffs[-1])
    for ck in coeffs[-2::-1]:
        r = (r * f + np.float32(ck)).astype(np.float32)
    return r


def max_rel_error(coeffs):
    f = np.linspace(INTERVAL[0], INTERVAL[1], 1000001)
    return float(np.max(np.abs(horner_fp32(coeffs, f).astype(np.float64) / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fp32_coefficients()
    print("coefficients (c0..c3):", c)
    print("max relative error of the fp32 Horner evaluation:", max_rel_error(c))
