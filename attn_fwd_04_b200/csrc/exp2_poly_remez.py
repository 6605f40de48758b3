"""Fit the polynomial the forward kernel uses to evaluate part of its
exponentials on the FMA pipe instead of the special-function unit.

    python -m attn_fwd_04_b200.csrc.exp2_poly_remez [degree]

Method (Cody and Waite style range reduction, then a minimax polynomial):
    2^x = 2^j * 2^f,  j = round(x),  f = x - j in [-1/2, 1/2]
and 2^f is replaced by the degree-n polynomial p that minimises the maximum
*relative* error max |p(f) / 2^f - 1| over [-1/2, 1/2].  The polynomial is
found with the Remez exchange algorithm (E. Remez, 1934), written out below:
solve the linear system p(x_i) - 2^x_i = (-1)^i E 2^x_i on n+2 reference
points, move the references to the extrema of the new error curve, repeat
until the equioscillation levels agree.

The kernel's constants (kExp2P0 .. kExp2P3 in fwd_sm100.cu) are this script's
output rounded to fp32; tests/test_exp2_poly.py checks that they match and
that the fp32 evaluation, with the kernel's range reduction, stays within the
error bound printed here.
"""
import sys

import mpmath
import numpy as np

mpmath.mp.dps = 40


def _target(x):
    return mpmath.power(2, x)


def _solve(refs, n):
    """Coefficients c_0..c_n and level E with (p(x_i) - g(x_i)) / g(x_i) = (-1)^i E."""
    m = n + 2
    A = mpmath.matrix(m, m)
    b = mpmath.matrix(m, 1)
    for i, x in enumerate(refs):
        g = _target(x)
        for k in range(n + 1):
            A[i, k] = mpmath.power(x, k)
        A[i, n + 1] = -((-1) ** i) * g
        b[i] = g
    sol = mpmath.lu_solve(A, b)
    return [sol[k] for k in range(n + 1)], sol[n + 1]


def _rel_err(c, x):
    p = mpmath.mpf(0)
    for k in reversed(range(len(c))):
        p = p * x + c[k]
    return p / _target(x) - 1


def remez(n: int, lo=-0.5, hi=0.5, iters=30, grid=4000):
    lo, hi = mpmath.mpf(lo), mpmath.mpf(hi)
    m = n + 2
    # Chebyshev extrema as the first references
    refs = [(lo + hi) / 2 - (hi - lo) / 2 * mpmath.cos(mpmath.pi * i / (m - 1)) for i in range(m)]
    xs = [lo + (hi - lo) * i / grid for i in range(grid + 1)]
    for _ in range(iters):
        c, E = _solve(refs, n)
        errs = [_rel_err(c, x) for x in xs]
        # one extremum per sign run of the error curve
        new = []
        run_start = 0
        for i in range(1, len(xs) + 1):
            if i == len(xs) or mpmath.sign(errs[i]) != mpmath.sign(errs[run_start]):
                seg = range(run_start, i)
                best = max(seg, key=lambda k: abs(errs[k]))
                new.append(xs[best])
                run_start = i
        if len(new) > m:  # keep the m largest, alternating
            while len(new) > m:
                ends = [abs(_rel_err(c, new[0])), abs(_rel_err(c, new[-1]))]
                new = new[1:] if ends[0] < ends[1] else new[:-1]
        if len(new) == m:
            refs = new
        emax = max(abs(e) for e in errs)
        if emax - abs(E) < mpmath.mpf("1e-12") * emax:
            break
    return [float(x) for x in c], float(emax)


def fp32_eval_error(c32, samples=200001):
    """Max relative error of the fp32 Horner evaluation against exact 2^f."""
    f = np.linspace(-0.5, 0.5, samples, dtype=np.float32)
    p = np.full_like(f, c32[-1])
    for k in reversed(range(len(c32) - 1)):
        p = (p * f + np.float32(c32[k])).astype(np.float32)
    exact = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) / exact - 1)))


if __name__ == "__main__":
    n = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez(n)
    c32 = [float(np.float32(x)) for x in c]
    print(f"degree {n}: minimax relative error {e:.3e}; fp32 evaluation {fp32_eval_error(c32):.3e}")
    print("coefficients c0..cn (fp32):")
    for k, x in enumerate(c32):
        print(f"  c{k} = {x!r}f")
