"""Derives the coefficients of the software 2^x used by the attention kernel.

Minimax (Remez exchange) fit of 2^f on [-1/2, 1/2] for *relative* error with a
polynomial of degree 3, then the fp32-rounded coefficients are re-evaluated with fp32
Horner steps to report the error actually obtained.  The range [-1/2, 1/2] is what
remains after the exact reduction x = rint(x) + f.

    python exact_attention_146_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def remez_exp2(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 40):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        fx = 2.0 ** x
        A = np.zeros((n, n))
        for i in range(deg + 1):
            A[:, i] = x ** i
        A[:, deg + 1] = (-1.0) ** k * fx
        c = np.linalg.solve(A, fx)[: deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        turn = np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1
        cand = np.concatenate([[0], turn, [len(grid) - 1]])
        if len(cand) != n:
            cand = np.sort(cand[np.argsort(-np.abs(err[cand]))[:n]])
        x = grid[cand]
    return c


def fp32_horner_rel_error(c32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ci in c32[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    exact = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs(p.astype(np.float64) - exact) / exact))


if __name__ == "__main__":
    c32 = remez_exp2(3).astype(np.float32)
    print("coefficients c0..c3:", [repr(float(v)) for v in c32])
    print("max relative error (fp32 Horner):", fp32_horner_rel_error(c32))
