"""Derives the coefficients of the polynomial exp2 used by the attention
kernel's softmax (`exp2_poly` in sm100.cuh), and its error bound.

Method (Cody-Waite style range reduction with a minimax polynomial): write
x = n + f with n = round(x) and f in [-1/2, 1/2], so 2^x = 2^n * 2^f. The
factor 2^n is applied by adding n to the float's exponent field; 2^f is a
degree-3 polynomial whose coefficients minimise the maximum relative error
on [-1/2, 1/2], found here by the Remez exchange algorithm.

    python -m paged_kv_cache_frame_b200.csrc.exp2_poly
"""
import numpy as np


def remez_rel(deg=3, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.concatenate(([0], np.where(np.diff(s) != 0)[0] + 1, [len(grid)]))
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in
               (np.arange(idx[i], idx[i + 1]) for i in range(len(idx) - 1))]
        if len(ext) != deg + 2:
            break
        x = grid[np.array(ext)]
    return c, float(np.max(np.abs(err)))


COEFFS = (9.999280572e-01, 6.932609677e-01, 2.426111251e-01, 5.517166853e-02)


def emulate(x):
    """Bit-exact float32 replay of the device sequence in `exp2_poly2`: clamp,
    round with the 1.5 * 2^23 shifter, Horner in float32 with fused
    multiply-adds (replayed in float64, then rounded once, which is exact for
    one FMA), exponent-field add."""
    f32 = np.float32
    x = np.maximum(np.asarray(x, dtype=f32), f32(-126.0))
    kr = f32(12582912.0)
    j = (x + kr).astype(f32)
    n = (j - kr).astype(f32)
    f = (n.astype(np.float64) * -1.0 + x.astype(np.float64)).astype(f32)
    c0, c1, c2, c3 = (f32(c) for c in COEFFS)
    fma = lambda a, b, c: (a.astype(np.float64) * np.float64(b) + np.float64(c)).astype(f32) \
        if np.ndim(b) == 0 else (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(f32)
    p = fma(f, c3, c2)
    p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c1)).astype(f32)
    p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c0)).astype(f32)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.astype(np.int32).view(f32)


def verify(lo=-200.0, hi=9.0, n=2000001):
    """Max relative error of the emulated device exp2 against exp2 in float64
    over [-125, hi], and the finiteness/positivity of every result in [lo, hi]."""
    x = np.linspace(lo, hi, n, dtype=np.float32)
    y = emulate(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0), "non-finite or negative result"
    m = x >= -125.0
    rel = np.abs(y[m].astype(np.float64) / np.exp2(x[m].astype(np.float64)) - 1.0)
    return float(rel.max())


if __name__ == "__main__":
    c, e = remez_rel()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 1000001)
    p = ((c32[3] * g.astype(np.float32) + c32[2]) * g.astype(np.float32) + c32[1]) * g.astype(np.float32) + c32[0]
    e32 = float(np.max(np.abs(p.astype(np.float64) / np.exp2(g) - 1)))
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v):.9e}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 Horner)")
    print(f"device sequence (emulated) over [-125, 9]: {verify():.3e}")
