"""The bf16 gate epilogue evaluates erf with Abramowitz & Stegun, Handbook of
Mathematical Functions, eq. 7.1.26 (|error| <= 1.5e-7). This checks the constants
compiled into the kernel against that published bound (fp64 evaluation of the
same form, compared with math.erf on a dense grid), so a mistyped coefficient
fails here on the CPU. The kernel's end result is checked against the oracle by
the GPU gate tests."""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _constants():
    src = open(os.path.join(ROOT, "learned_token_pruning_gemm_b200", "csrc", "gate.cu")).read()
    c = dict(re.findall(r"constexpr float kAs(P|A\d) = (-?[0-9.]+)f;", src))
    return {k: float(v) for k, v in c.items()}


def test_as_7_1_26_error_bound():
    c = _constants()
    assert set(c) == {"P", "A1", "A2", "A3", "A4", "A5"}
    x = np.linspace(-6.0, 6.0, 240001)
    ax = np.abs(x)
    t = 1.0 / (1.0 + c["P"] * ax)
    poly = t * (c["A1"] + t * (c["A2"] + t * (c["A3"] + t * (c["A4"] + t * c["A5"]))))
    approx = np.sign(x) * (1.0 - poly * np.exp(-ax * ax))
    exact = np.array([math.erf(v) for v in x])
    err = np.abs(approx - exact).max()
    # the published bound, with room for the constants' fp32 rounding
    assert err <= 1.6e-7, err
    # the resulting GELU error stays far below the gate's 1e-4 score tolerance
    u = x * math.sqrt(2.0)
    assert np.abs(0.5 * u * (approx - exact)).max() < 1e-6
