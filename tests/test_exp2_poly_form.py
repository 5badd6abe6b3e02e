"""The attention kernel computes one exponential in four on the FMA pipe: for
x = n + f with n = rint(x) and f in [-1/2, 1/2], 2^x = 2^n * p(f), with p a cubic
fitted to 2^f by minimax in relative error (Remez exchange). The kernel states a
relative error of 7.5e-5 for p on [-1/2, 1/2]. This reads the compiled constants
from the source and checks that bound against numpy's exp2 on a dense grid, both
for the polynomial in fp64 and for the kernel's whole fp32 sequence (the shift
that rounds to n, Horner in fp32, the exponent added to the bits), so a mistyped
coefficient or a wrong step fails here on the CPU."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs():
    src = open(os.path.join(ROOT, "learned_token_pruning_gemm_b200", "csrc", "attn.cu")).read()
    c = dict(re.findall(r"constexpr float kExp2C(\d) = (-?[0-9.]+)f;", src))
    assert sorted(c) == ["0", "1", "2", "3"]
    return [np.float32(float(c[str(i)])) for i in range(4)]


def test_polynomial_relative_error_bound():
    c = [float(v) for v in _coeffs()]
    f = np.linspace(-0.5, 0.5, 400001)
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()
    # minimax: the error equi-oscillates, so both ends and the interior reach near the bound
    assert rel[0] > 5e-5 and rel[-1] > 5e-5


def _exp2_fma_fp32(x):
    """The kernel's sequence, step by step in fp32 (numpy float32 rounds every op)."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)            # 1.5 * 2^23: adding it rounds to an integer
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    fr = (x - n).astype(np.float32)
    p = (c3 * fr + c2).astype(np.float32)     # fmaf rounds once; two roundings here are
    p = (p * fr + c1).astype(np.float32)      # within 2^-23 relative of it
    p = (p * fr + c0).astype(np.float32)
    # n sits in t's low mantissa bits; shifting t's bits by 23 puts it in the
    # exponent field (the shift constant's bits vanish modulo 2^32)
    tb = t.view(np.uint32)
    ni = tb.astype(np.int64) - 0x4B400000
    assert np.array_equal((ni << 23) & 0xFFFFFFFF, (tb.astype(np.int64) << 23) & 0xFFFFFFFF)
    return (p.view(np.uint32) + (tb << np.uint32(23))).view(np.float32)


def test_fp32_sequence_matches_exp2():
    x = np.concatenate([np.linspace(-120.0, 8.0, 500001), np.array([-0.5, 0.5, 0.0, 8.0])])
    got = _exp2_fma_fp32(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float32).astype(np.float64)) - 1.0)
    assert rel.max() <= 8e-5, rel.max()
    # below -125 the input is clamped: a tiny positive weight, never inf or NaN
    low = _exp2_fma_fp32(np.array([-200.0, -1e30], np.float32))
    assert np.all(np.isfinite(low)) and np.all(low >= 0) and np.all(low < 1e-37)
