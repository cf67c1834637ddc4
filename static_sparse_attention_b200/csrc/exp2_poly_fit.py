"""Derive the polynomial the forward kernel uses for part of its exp2 work.

Method (our own derivation, standard numerics): range reduction in the style of
Cody and Waite -- x = j + f with j = round(x) an integer and f in [-1/2, 1/2],
2^x = 2^j * 2^f, the 2^j factor applied by adding j to the float's exponent
field -- and a degree-3 polynomial for 2^f fitted by the Remez exchange
algorithm to minimise the maximum RELATIVE error on [-1/2, 1/2].

The kernel rounds the result to bf16 (8 significant bits, relative spacing
2^-7), so a relative error around 1e-4 is far below what the rounding adds.

    python static_sparse_attention_b200/csrc/exp2_poly_fit.py
prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the error bound.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    target = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (deg + 1))
    dense = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - t(x_i) = (-1)^i E t(x_i) for the relative error
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * target(xi)
        sol = np.linalg.solve(A, target(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], dense) - target(dense)) / target(dense)
        # new reference: the extrema of the error, one per sign run
        sign_change = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = np.concatenate([[0], sign_change + 1, [len(dense)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) != deg + 2:
            break
        x = dense[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    f32 = np.float32(c)
    dense = np.linspace(LO, HI, 200001).astype(np.float32)
    # evaluate in fp32 Horner form, as the kernel does
    p = ((f32[3] * dense + f32[2]) * dense + f32[1]) * dense + f32[0]
    e32 = float(np.max(np.abs(p.astype(np.float64) / np.exp2(dense.astype(np.float64)) - 1)))
    for i, ci in enumerate(f32):
        print(f"c{i} = {ci!r}  ({float(ci).hex()})")
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 Horner)")
