"""The selection kernel ranks scores by a 32-bit key (its radix passes run on the
key's bytes): NaN ranks lowest, -0 equals +0, and every other float keeps its
order. This compiles the kernel's own key function, taken from the source as it
stands, for the host (gcc) and checks it against that order on every class of
float32 value (zeros, denormals, normals, infinities, NaNs with any payload and
sign) and on random values, pairwise: key order must equal score order exactly,
and +inf must stay below the kernel's "above every key" sentinel 0xFFFFFFFF."""
import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def score_key(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(os.path.join(ROOT, "learned_token_pruning_gemm_b200", "csrc", "select.cu")).read()
    m = re.search(r"__device__ __forceinline__ uint32_t score_key\(float f\) \{(.*?)\n\}", src, re.S)
    assert m, "score_key not found in select.cu"
    c = ("#include <stdint.h>\n#include <string.h>\n"
         "static inline uint32_t __float_as_uint(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }\n"
         "uint32_t score_key(float f) {" + m.group(1) + "\n}\n")
    d = tmp_path_factory.mktemp("key")
    (d / "key.c").write_text(c)
    lib = str(d / "libkey.so")
    subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", "-o", lib, str(d / "key.c")])
    f = ctypes.CDLL(lib).score_key
    f.restype, f.argtypes = ctypes.c_uint32, [ctypes.c_float]
    return f


def _values():
    bits = [0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x007FFFFF, 0x807FFFFF,
            0x00800000, 0x80800000, 0x3F800000, 0xBF800000, 0x7F7FFFFF, 0xFF7FFFFF,
            0x7F800000, 0xFF800000,                                  # +-inf
            0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF800001, 0x7FFFFFFF, 0xFFFFFFFF]  # NaNs
    rng = np.random.default_rng(3)
    rand = np.concatenate([rng.standard_normal(600), rng.uniform(-1e-30, 1e-30, 200),
                           rng.uniform(-3e38, 3e38, 200), np.round(rng.standard_normal(200), 1)])
    vals = np.concatenate([np.array(bits, dtype=np.uint32).view(np.float32),
                           rand.astype(np.float32),
                           rng.integers(0, 2 ** 32, 800, dtype=np.uint64).astype(np.uint32).view(np.float32)])
    return vals


def test_key_order_is_score_order(score_key):
    v = _values()
    keys = np.array([score_key(float(x)) for x in v], dtype=np.uint64)
    nan = np.isnan(v)
    # the order the selection defines: NaN below everything, -0 == +0, else the value
    with np.errstate(invalid="ignore"):   # signalling NaN payloads widen with a warning
        rank = np.where(nan, -np.inf, v.astype(np.float64))
    lo = np.where(nan, 0, 1)               # NaN strictly below -inf
    a_lt = (lo[:, None] < lo[None, :]) | ((lo[:, None] == lo[None, :]) & (rank[:, None] < rank[None, :]))
    a_eq = (lo[:, None] == lo[None, :]) & ((rank[:, None] == rank[None, :]) | (nan[:, None] & nan[None, :]))
    assert np.array_equal(keys[:, None] < keys[None, :], a_lt)
    assert np.array_equal(keys[:, None] == keys[None, :], a_eq)


def test_special_keys(score_key):
    f32 = lambda b: float(np.array([b], dtype=np.uint32).view(np.float32)[0])
    assert score_key(0.0) == score_key(-0.0)
    for nan_bits in (0x7FC00000, 0xFFC00000, 0x7F800001, 0xFFFFFFFF):
        assert score_key(f32(nan_bits)) == 0                 # the lowest key
    assert score_key(f32(0xFF800000)) > 0                     # -inf above every NaN
    assert score_key(f32(0x7F800000)) == 0xFF800000            # +inf, the largest key
    assert score_key(f32(0x7F800000)) < 0xFFFFFFFF             # below the sentinel
