"""Fits the cubic that the attention kernel uses for 2^x on the FMA pipe.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a cubic c0 + c1 f + c2 f^2 + c3 f^3 whose maximum relative
error over [-1/2, 1/2] is minimised with Lawson's iteratively reweighted
least-squares algorithm (C. L. Lawson, "Contributions to the theory of
linear least maximum approximation", 1961) on a dense Chebyshev grid.  2^n is
applied by adding n to the float's exponent field.

The softmax probabilities that use it are rounded to bfloat16 (relative step
2^-8), so a relative error near 1e-4 is far below the output tolerance.

    python block_sparse_attention_coarse_b200/csrc/fit_exp2_poly.py
prints the coefficients (as float32 hex literals) that isa_common.cuh holds.
"""
import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, iters: int = 200):
    n = 4001
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)       # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w) / y                                      # relative error weights
        c, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    return c, float(np.max(np.abs(V @ c - y) / y))


def eval_f32(c, x):
    """The kernel's float32 evaluation, for checking the error bound."""
    c = np.asarray(c, np.float32)
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)                               # 1.5 * 2^23
    t = x + magic
    n = t - magic                                                # round to nearest integer
    fr = x - n
    p = ((c[3] * fr + c[2]) * fr + c[1]) * fr + c[0]
    bits = p.view(np.uint32).astype(np.int64) + (n.astype(np.int64) << 23)
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, e = fit()
    c32 = np.asarray(c, np.float32)
    print("max relative error (float64 coefficients):", e)
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v)!r:>24}  0x{int(np.float32(v).view(np.uint32)):08X}")
    xs = np.linspace(-125, 0, 2_000_001, dtype=np.float32)
    rel = np.abs(eval_f32(c32, xs).astype(np.float64) - np.exp2(xs.astype(np.float64))) / np.exp2(xs.astype(np.float64))
    print("max relative error, float32 evaluation on [-125, 0]:", rel.max())
