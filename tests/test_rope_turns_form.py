"""The projection kernel forms each rotary angle pos * theta_i in turns: F_i =
theta_i / (2 pi) rounded to a 64-bit fixed-point fraction, the integer product
pos * F_i taken modulo 2^64 (so modulo one turn), its top 32 bits rounded to 23 as
a float in [1, 2], and x = 2 pi (turns - 1/2) in fp32, whose sine and cosine are
the negated sine and cosine of the angle. This repeats that sequence on the CPU
(Python integers for the fixed point, numpy float32 for every fp32 step) and
checks x against the angle computed in 60-digit decimal arithmetic, for positions
up to 2^31 - 1, so a wrong shift, a dropped rounding bit or a wrong constant
fails here rather than only through the GPU parity tests. The kernel's own lines
(taken from qkv.cu as it stands and compiled for the host) must match the mirror
bit for bit, so the checks hold for the code that runs."""
import decimal
import math
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

D = decimal.Decimal
decimal.getcontext().prec = 60


def _pi():
    # Machin: pi = 16 atan(1/5) - 4 atan(1/239), each by its Taylor series
    def atan_inv(n):
        x, n2, k, s, term = D(1) / n, D(n) * n, 1, D(0), D(1) / n
        while term != 0:
            s += term / k if (k // 2) % 2 == 0 else -term / k
            term /= n2
            k += 2
        return s
    return 16 * atan_inv(5) - 4 * atan_inv(239)


PI = _pi()


def _theta(i, base, dh=128):
    return (D(-2 * i) / dh * D(base).ln()).exp()


def _kernel_x(p, i, base, dh=128):
    # F_i from the fp64 frequency, as the kernel's prologue does
    t = math.exp(-2.0 * i / dh * math.log(base)) * 0.15915494309189535
    F = int(round(math.ldexp(t, 64)))
    assert 0 < F < 2 ** 64
    fx = (p * F) % 2 ** 64                      # two's complement product, low 64 bits
    fr = fx >> 32
    m = ((fr + 256) % 2 ** 32) >> 9              # 23 bits, rounded; a carry wraps to 0
    f1 = np.uint32(0x3F800000 + m).view(np.float32)
    return np.float32(np.float32(f1 - np.float32(1.5)) * np.float32(6.28318530717958648))


def _true_x(p, i, base):
    # the angle less pi, reduced to [-pi, pi)
    a = (D(p) * _theta(i, base)) % (2 * PI)
    x = a - PI
    return x


def test_turns_match_the_exact_angle():
    rng = np.random.default_rng(5)
    pos = [0, 1, 2, 3, 127, 128, 16383, 65536, 131071, 10 ** 6, 2 ** 24 - 1, 2 ** 31 - 1]
    pos += [int(v) for v in rng.integers(0, 2 ** 31 - 1, 40)]
    worst = 0.0
    for base in (1e4, 1e6):
        for i in (0, 1, 2, 17, 31, 32, 50, 63):
            for p in pos:
                got = D(float(_kernel_x(p, i, base)))
                d = abs(got - _true_x(p, i, base))
                d = min(d, 2 * PI - d)              # angles equal modulo 2 pi
                # 2^-24 turn from the 23-bit rounding, two fp32 roundings of |x| <= pi,
                # and the fp64 frequency's own error times the position
                bound = 2 * math.pi * 2.0 ** -24 + 2 * math.pi * 2.0 ** -24 + p * 1.6e-17 * 2 * math.pi
                assert float(d) <= bound, (p, i, base, float(d), bound)
                worst = max(worst, float(d))
    assert worst > 1e-8   # the check is not vacuous


def test_sine_and_cosine_of_the_turn_form():
    # sin/cos of x = angle - pi are the negated sine and cosine of the angle
    for p, i in [(5, 0), (1000, 3), (123457, 10), (2 ** 31 - 1, 63)]:
        x = float(_kernel_x(p, i, 1e6))
        a = float(_true_x(p, i, 1e6) + PI)
        assert abs(-math.cos(x) - math.cos(a)) < 1e-6
        assert abs(-math.sin(x) - math.sin(a)) < 1e-6


def test_negative_positions_wrap_like_the_kernel():
    # the product is taken on the sign-extended position, so -p is the mirror angle
    for p, i in [(1, 0), (77, 5), (10 ** 6, 40)]:
        x1 = float(_kernel_x(p, i, 1e6))
        x2 = float(_kernel_x((-p) % 2 ** 64, i, 1e6))
        # angle(-p) = -angle(p): x2 + pi = -(x1 + pi) mod 2 pi
        d = (x2 + math.pi + x1 + math.pi) % (2 * math.pi)
        assert min(d, 2 * math.pi - d) < 2e-6


def test_kernel_source_matches_the_mirror(tmp_path):
    # the projection kernel's own lines (the frequency's fixed point in the prologue,
    # then the turn, its rounding and the angle), compiled for the host, must give
    # the mirror's x bit for bit: the accuracy checks above then hold for the kernel
    import re
    import shutil
    import subprocess
    import ctypes
    if shutil.which("g++") is None:
        import pytest
        pytest.skip("g++ not available")
    src = open(os.path.join(ROOT, "learned_token_pruning_gemm_b200", "csrc", "qkv.cu")).read()
    inv = re.search(r"constexpr double kInvTwoPi = ([0-9.e+-]+);", src).group(1)
    turn = re.search(r"S\.turn\[i\] = (__double2ull_rn\(.*?\));", src).group(1)
    lines = re.search(r"(const uint64_t fx = .*?const float x = [^;]*;)", src, re.S).group(1)
    lines = re.sub(r"S\.turn\[[^\]]*\]", "F", lines)
    code = f"""
#include <cmath>
#include <cstdint>
#include <cstring>
static inline float __uint_as_float(uint32_t u) {{ float f; std::memcpy(&f, &u, 4); return f; }}
static inline unsigned long long __double2ull_rn(double d) {{ return (unsigned long long)std::nearbyint(d); }}
constexpr int kDh = 128;
extern "C" float kernel_x(int p, int i, double log_base) {{
  constexpr double kInvTwoPi = {inv};
  const uint64_t F = {turn};
  {lines}
  return x;
}}
"""
    (tmp_path / "angle.cpp").write_text(code)
    lib = str(tmp_path / "libangle.so")
    subprocess.check_call(["g++", "-O2", "-ffp-contract=off", "-shared", "-fPIC", "-o", lib,
                           str(tmp_path / "angle.cpp")])
    f = ctypes.CDLL(lib).kernel_x
    f.restype, f.argtypes = ctypes.c_float, [ctypes.c_int, ctypes.c_int, ctypes.c_double]
    rng = np.random.default_rng(9)
    pos = [0, 1, 127, 16383, 10 ** 6, 2 ** 31 - 1] + [int(v) for v in rng.integers(0, 2 ** 31 - 1, 30)]
    for base in (1e4, 1e6):
        for i in (0, 1, 17, 33, 63):
            for p in pos:
                assert np.float32(f(p, i, math.log(base))) == _kernel_x(p, i, base), (p, i, base)
