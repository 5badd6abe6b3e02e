"""ctypes loader for libtokengate.so (the C ABI declared in include/tg.h).

There is no fallback: if the shared library is missing or fails to load, every
call raises. Build it with `python -m learned_token_pruning_gemm_b200.build`.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# TG_DEBUG=1 in the environment selects the debug library (index checks on every
# data-dependent global access, TG_ERR_DEBUG_BOUNDS instead of a fault)
LIB_PATH = os.path.join(_HERE, "libtokengate_debug.so" if os.environ.get("TG_DEBUG") == "1"
                        else "libtokengate.so")

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F32 = ctypes.c_float
INT = ctypes.c_int

# (name, restype, argtypes) for every symbol the header declares
SIGNATURES = {
    "tg_abi_version": (INT, []),
    "tg_debug_build": (INT, []),
    "tg_status_string": (ctypes.c_char_p, [INT]),
    "tg_gate_score": (INT, [P, INT, I64, INT, P, P, P, F32, INT, P, P]),
    "tg_select_topk": (INT, [P, P, P, P, P, INT, I64, I64, INT, P, P, P, P, P]),
    "tg_compact_kv": (INT, [P, P, P, INT, P, I64, I64, P]),
    "tg_gated_attention": (INT, [P, P, P, INT, P, P, P, P, INT, I64, INT, INT, INT, INT, P, P, P]),
    "tg_gated_attention_bwd_workspace_size": (ctypes.c_size_t, [INT, INT, I64, INT, INT, INT, INT]),
    "tg_gated_attention_bwd": (INT, [P, P, P, P, P, INT, P, P, P, P, P, INT, I64, INT, INT, INT,
                                     INT, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
    "tg_qkv_rope": (INT, [P, I64, INT, P, INT, INT, INT, F32, P, P, P, P, P]),
    "tg_compact_qkv_rope": (INT, [P, I64, INT, P, I64, P, P, INT, INT, INT, F32, P, P, P, P, P]),
    "tg_cache_append": (INT, [P, P, P, INT, INT, INT, INT, P, P, P, P, P]),
    "tg_gated_decode_workspace_size": (ctypes.c_size_t, [INT, INT, INT, INT]),
    "tg_gated_decode": (INT, [P, P, P, P, P, INT, INT, INT, INT, INT, INT, P, P, P, P,
                              ctypes.c_size_t, P]),
    "tg_gated_decode_noalloc": (INT, [P, P, P, P, P, INT, INT, INT, INT, INT, INT, P, P, P, P]),
    "tg_gated_delta_rule_workspace_size": (ctypes.c_size_t, [INT, I64, INT, INT]),
    "tg_gated_delta_rule": (INT, [P, P, P, INT, P, P, P, INT, I64, INT, INT, INT, INT, P, P,
                                  ctypes.c_size_t, P]),
    "tg_device_status": (INT, [P, INT]),
    "tg_selftest_bounded_wait": (INT, [I64, P]),
}

_lib = None


class TokenGateError(RuntimeError):
    pass


def load(path: str = LIB_PATH):
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise TokenGateError(
                f"{path} not found: build the CUDA library first "
                "(python -m learned_token_pruning_gemm_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(status: int, what: str) -> None:
    if status != 0:
        name = load().tg_status_string(status).decode()
        raise TokenGateError(f"{what} failed: {name} ({status})")
