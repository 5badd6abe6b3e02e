"""Fit the polynomial used by the attention kernel's FMA-pipe exp2.

exp2(x) = 2^n * 2^f with n = rint(x), f = x - n in [-1/2, 1/2]; 2^f is
approximated by a degree-3 polynomial minimising the maximum RELATIVE error on
[-1/2, 1/2] (Remez exchange, written here from the textbook algorithm: solve for
the polynomial that equi-oscillates on the current reference points, move the
reference to the extrema of the new error, repeat). The coefficients printed are
the ones in attn.cu (kExp2C0..kExp2C3); P is rounded to bf16 (relative step
2^-8) right after, so a relative error near 1e-4 is far below what is kept.

    python fit_exp2_poly.py
"""
import numpy as np


def remez_rel(deg=3, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    ref = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # sum_k c_k x^k - f(x) = (-1)^i E f(x)   (relative error E)
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:deg + 1]
        xs = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], xs) - f(xs)) / f(xs)
        # new reference: the extremum of each sign run of the error
        sign = np.sign(err)
        cuts = np.where(np.diff(sign) != 0)[0]
        bounds = np.r_[0, cuts + 1, len(xs)]
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest errors
        ext = np.array(ext)
        best = max(range(len(ext) - n + 1), key=lambda s: np.abs(err[ext[s:s + n]]).min())
        ref = xs[ext[best:best + n]]
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_rel()
    c32 = c.astype(np.float32)
    xs = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c32[3] * xs + c32[2]) * xs + c32[1]) * xs + c32[0]
    rel = np.abs(p.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1).max()
    for i, v in enumerate(c32):
        print(f"kExp2C{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error: fit {e:.3e}, fp32 Horner {rel:.3e}")
