"""Fits the polynomial the kernel uses to compute 2^x on the FMA pipe.

Method: Cody-Waite style range reduction x = n + f with n = round(x) and
f in [-1/2, 1/2], so 2^x = 2^n * 2^f; 2^n goes into the exponent field and
2^f is a degree-3 polynomial. Its coefficients minimise the maximum
*relative* error on [-1/2, 1/2] and come from the Remez exchange algorithm
(E. Ya. Remez, 1934) run here in float64: solve for the polynomial that
equioscillates on a reference set, move the reference to the extrema of the
new error curve, repeat until the levelled error settles. The coefficients
are then rounded to float32 and the error is measured again with float32
Horner arithmetic, as the kernel evaluates it.

Usage: python fit_exp2_poly.py   (prints the coefficients and error bounds)
"""

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree=DEGREE, iters=30):
    n = degree + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i, unknowns c_0..c_d and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        b = 2.0 ** ref
        sol = np.linalg.solve(A, b)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum of |err| in each sign-alternating run
        sign = np.sign(err)
        runs = np.split(np.arange(grid.size), np.nonzero(np.diff(sign))[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest errors
        while len(ext) > n:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        ref = grid[ext]
    return coef


def horner_f32(coef32, f):
    p = np.float32(coef32[-1])
    for c in coef32[-2::-1]:
        p = np.float32(np.float32(p * f) + np.float32(c))  # one rounding per FMA is finer
    return p


def exp2_emulated_f32(x, coef32):
    """Float32 model of the kernel's emulated 2^x for x in [-126, 16]."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, np.float32(coef32[-1]))
    for c in coef32[-2::-1]:
        p = (p * f + np.float32(c)).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + \
        ((t.view(np.uint32).astype(np.uint64) << np.uint64(23)) & np.uint64(0xFFFFFFFF))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def main():
    coef = remez_relative()
    coef32 = coef.astype(np.float32)
    grid = np.linspace(LO, HI, 400001)
    e64 = np.max(np.abs(np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0))
    x = np.linspace(-125.0, 9.0, 2000001).astype(np.float32)
    y = exp2_emulated_f32(x, coef32).astype(np.float64)
    e32 = np.max(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0))
    print("degree", DEGREE)
    for i, c in enumerate(coef32):
        print(f"c{i} = {float(c):.9e}f  (0x{c.view(np.uint32):08x})")
    print(f"max relative error: float64 poly {e64:.3e}; float32 kernel model on [-125, 9] {e32:.3e}")
    print(f"largest relative rounding of P: bf16 {2.0 ** -8:.3e}, fp16 {2.0 ** -11:.3e}")


if __name__ == "__main__":
    main()
