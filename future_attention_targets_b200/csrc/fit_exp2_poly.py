"""Fits the polynomial of the software exp2 used on the FMA pipe.

The kernels evaluate 2^y for part of their exponentials without the
multi-function unit: Cody-Waite range reduction y = n + f with n = floor(y)
and f in [0, 1), then 2^f ~ p(f), then 2^n * p(f) by adding n to the
exponent field.  p(f) = 1 + f (c1 + f (c2 + ...)): the constant term is
pinned to exactly 1 so that p(0) = 1 and the result for the clamped lower
end is exact.  The free coefficients minimise the maximum relative error
|p(f) / 2^f - 1| on [0, 1] (Remez exchange on a dense grid).  Two degrees:
4 (3.0e-6; kP1..kP4) for the row logsumexp, whose lse is an output, and 3
(8.6e-5; kT1..kT3) for the transposed pass, whose error only reaches the
targets (held to 2e-3) and whose cheaper evaluation lets more pairs leave
the MUFU.

Run:  python fit_exp2_poly.py      prints both coefficient sets (as C hex
floats) and the error of their float32 Horner evaluation.
"""
from __future__ import annotations

import numpy as np

DEGREES = (4, 3)


def _basis(f, degree):
    # error(f) = (1 + sum_k c_k f^k) / 2^f - 1 = sum_k c_k f^k 2^-f - (1 - 2^-f)
    return np.stack([f ** k * 2.0 ** -f for k in range(1, degree + 1)], axis=1), 1.0 - 2.0 ** -f


def remez(degree: int, iters: int = 30, grid: int = 200001):
    x = np.linspace(0.0, 1.0, grid)[1:]
    n_ref = degree + 1
    ref = 0.5 - 0.5 * np.cos(np.pi * (np.arange(n_ref) + 1) / n_ref)   # in (0, 1]
    c = None
    for _ in range(iters):
        A, g = _basis(ref, degree)
        M = np.hstack([A, ((-1.0) ** np.arange(n_ref))[:, None]])
        sol = np.linalg.solve(M, g)
        c, E = sol[:degree], sol[degree]
        B, gx = _basis(x, degree)
        err = B @ c - gx
        # local extrema of err, keep an alternating set of n_ref with the largest |err|
        idx = [0] + [i for i in range(1, len(x) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(x) - 1]
        idx = np.array(sorted(set(idx)))
        # merge runs of the same sign, keeping the largest of each run
        picked = []
        for i in idx:
            if picked and np.sign(err[i]) == np.sign(err[picked[-1]]):
                if abs(err[i]) > abs(err[picked[-1]]):
                    picked[-1] = i
            else:
                picked.append(i)
        while len(picked) > n_ref:
            # drop the smaller end
            if abs(err[picked[0]]) < abs(err[picked[-1]]):
                picked.pop(0)
            else:
                picked.pop()
        if len(picked) < n_ref:
            break
        ref = x[np.array(picked)]
    B, gx = _basis(x, degree)
    return c, float(np.max(np.abs(B @ c - gx)))


def fp32_horner_error(c32: np.ndarray, samples: int = 2_000_001) -> float:
    f = np.linspace(0.0, 1.0, samples, dtype=np.float32)[:-1].astype(np.float64)
    p = np.full_like(f, c32[-1], dtype=np.float64)
    for ck in c32[-2::-1]:
        p = np.float32(p * f + ck).astype(np.float64)           # fma rounded once to fp32
    p = np.float32(p * f + 1.0).astype(np.float64)
    return float(np.max(np.abs(p / 2.0 ** f - 1.0)))


def main():
    for degree in DEGREES:
        c, e = remez(degree)
        c32 = c.astype(np.float32)
        print(f"degree {degree}")
        print(f"  minimax relative error (exact arithmetic): {e:.3e}")
        print(f"  float32 Horner relative error:             {fp32_horner_error(c32):.3e}")
        for k, v in enumerate(c32, start=1):
            print(f"  c{k} = {float(v).hex()}f  // {float(v):.9g}")


if __name__ == "__main__":
    main()
