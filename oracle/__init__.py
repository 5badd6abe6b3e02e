"""ctypes wrapper of the fp64 CPU oracle (oracle.cpp).

TEST INFRASTRUCTURE: only tests/, the smoke check and bench.py's CPU-baseline and
reference legs use it. The CUDA path never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle_tg.so")
_lib = None

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F32 = ctypes.c_float


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_gate_score.argtypes = [P, ctypes.c_int, I64, ctypes.c_int, P, P, P, F32,
                                        ctypes.c_int, P, P]
        L.oracle_gate_score.restype = None
        L.oracle_select_topk.argtypes = [P, P, P, P, P, ctypes.c_int, P, P]
        L.oracle_select_topk.restype = I64
        L.oracle_gather_rows.argtypes = [P, I64, P, I64, P]
        L.oracle_gather_rows.restype = None
        L.oracle_gated_attention.argtypes = [P, P, P, ctypes.c_int, P, P, P, P, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, P, I64, P]
        L.oracle_gated_attention.restype = None
        L.oracle_qkv_rope.argtypes = [P, ctypes.c_int, I64, ctypes.c_int, P, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P, I64, P,
                                      P, P]
        L.oracle_qkv_rope.restype = None
        L.oracle_gated_decode.argtypes = [P, P, P, ctypes.c_int, P, P, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          P, P, P]
        L.oracle_gated_decode.restype = None
        L.oracle_gated_attention_bwd.argtypes = [P, P, P, P, ctypes.c_int, P, P, P, P,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, P, P, P, P, P, P]
        L.oracle_gated_attention_bwd.restype = None
        L.oracle_gated_delta_rule.argtypes = [P, P, P, ctypes.c_int, P, P, P, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        L.oracle_gated_delta_rule.restype = None
        _lib = L
    return _lib


def _ptr(a) -> int:
    return a.ctypes.data if isinstance(a, np.ndarray) else a.data_ptr()


def _raw(t: torch.Tensor):
    """(contiguous CPU tensor, dtype code): f32 -> 0, bf16 -> 1 (bits read as-is)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t, 0
    if t.dtype == torch.bfloat16:
        return t, 1
    raise TypeError(f"oracle: unsupported dtype {t.dtype}")


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _f32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def gate_score(x: torch.Tensor, w1: torch.Tensor, b1, w2, b2: float):
    """s_i = b2 + w2 . GELU(W1 x_i + b1); returns (fp64 scores, fp32 rounding)."""
    xr, dt = _raw(x)
    w1r, dt2 = _raw(w1)
    assert dt == dt2
    n, d = xr.shape
    h = w1r.shape[0]
    assert w1r.shape[1] == d
    b1a, w2a = _f32(b1), _f32(w2)
    s64 = np.empty(n, np.float64)
    s32 = np.empty(n, np.float32)
    lib().oracle_gate_score(_ptr(xr), dt, n, d, _ptr(w1r), _ptr(b1a), _ptr(w2a), float(b2), h,
                            _ptr(s64), _ptr(s32))
    return s64, s32


def select_topk(scores, cu_seqlens, doc_begin, doc_end, k_doc):
    """Returns (kept global row ids, ascending; cu_kept[B+1])."""
    s = _f32(scores)
    cu = _i32(cu_seqlens)
    db, de, kd = _i32(doc_begin), _i32(doc_end), _i32(k_doc)
    B = len(db)
    out = np.empty(int(cu[-1]), np.int32)
    cuk = np.empty(B + 1, np.int32)
    n = lib().oracle_select_topk(_ptr(s), _ptr(cu), _ptr(db), _ptr(de), _ptr(kd), B, _ptr(out),
                                 _ptr(cuk))
    if n < 0:
        raise ValueError("oracle_select_topk: bad span")
    return out[:n].copy(), cuk


def gather_rows(src: np.ndarray, kept_idx) -> np.ndarray:
    src = np.ascontiguousarray(src)
    idx = _i32(kept_idx)
    row_bytes = src.strides[0]
    dst = np.empty((len(idx),) + src.shape[1:], src.dtype)
    lib().oracle_gather_rows(_ptr(src), row_bytes, _ptr(idx), len(idx), _ptr(dst))
    return dst


def gated_attention(q, k, v, s_kept, gain, tau, cu_kept, rows=None) -> np.ndarray:
    """O [K, hq, dh] fp64 (rows not in `rows` are left as NaN)."""
    qr, dt = _raw(q)
    kr, _ = _raw(k)
    vr, _ = _raw(v)
    K, hq, dh = qr.shape
    hkv = kr.shape[1]
    s, g, t = _f32(s_kept), _f32(gain), _f32(tau)
    cu = _i32(cu_kept)
    out = np.full((K, hq, dh), np.nan, np.float64)
    if rows is None:
        rp, nr = None, 0
    else:
        ra = _i32(rows)
        rp, nr = _ptr(ra), len(ra)
    lib().oracle_gated_attention(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(s), _ptr(g), _ptr(t),
                                 _ptr(cu), len(cu) - 1, hq, hkv, dh, rp, nr, _ptr(out))
    return out


def qkv_rope(xc: torch.Tensor, w: torch.Tensor, hq: int, hkv: int, dh: int, base: float, pos,
             rows=None):
    """(q [n,hq,dh], k [n,hkv,dh], v [n,hkv,dh]) fp64: y = W xc split per head, q and k
    rotated at pos (rotate-half RoPE). Rows not in `rows` are left as NaN."""
    xr, dt = _raw(xc)
    wr, dt2 = _raw(w)
    assert dt == dt2
    n, d = xr.shape
    assert wr.shape == ((hq + 2 * hkv) * dh, d)
    pa = _i32(pos)
    assert len(pa) == n
    q = np.full((n, hq, dh), np.nan)
    k = np.full((n, hkv, dh), np.nan)
    v = np.full((n, hkv, dh), np.nan)
    if rows is None:
        rp, nr = None, 0
    else:
        ra = _i32(rows)
        rp, nr = _ptr(ra), len(ra)
    lib().oracle_qkv_rope(_ptr(xr), dt, n, d, _ptr(wr), hq, hkv, dh, float(base), _ptr(pa), rp,
                          nr, _ptr(q), _ptr(k), _ptr(v))
    return q, k, v


def gated_decode(q, k_cache, v_cache, s_cache, cache_len, gain, tau) -> np.ndarray:
    """One query row per sequence over its cache rows j < cache_len[b]:
    q [B, hq, dh], k/v cache [B, cap, hkv, dh], s cache [B, cap] -> O [B, hq, dh] fp64."""
    qr, dt = _raw(q)
    kr, dt2 = _raw(k_cache)
    vr, dt3 = _raw(v_cache)
    assert dt == dt2 == dt3
    B, hq, dh = qr.shape
    Bk, cap, hkv, dh2 = kr.shape
    assert Bk == B and dh2 == dh and tuple(vr.shape) == tuple(kr.shape)
    s = _f32(s_cache).reshape(B, cap)
    ln = _i32(cache_len)
    assert len(ln) == B and (ln <= cap).all()
    g, t = _f32(gain), _f32(tau)
    out = np.empty((B, hq, dh), np.float64)
    lib().oracle_gated_decode(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(s), _ptr(ln), B, cap, hq,
                              hkv, dh, _ptr(g), _ptr(t), _ptr(out))
    return out


def gated_attention_bwd(q, k, v, dout, s_kept, gain, tau, cu_kept):
    """Gradients of the gated attention for upstream dout: returns fp64
    (dq [K,hq,dh], dk [K,hkv,dh], dv [K,hkv,dh], ds [K], dgain [hq], dtau [hq])."""
    qr, dt = _raw(q)
    kr, dt2 = _raw(k)
    vr, dt3 = _raw(v)
    dr, dt4 = _raw(dout)
    assert dt == dt2 == dt3 == dt4
    K, hq, dh = qr.shape
    hkv = kr.shape[1]
    s, g, t = _f32(s_kept), _f32(gain), _f32(tau)
    cu = _i32(cu_kept)
    dq = np.empty((K, hq, dh))
    dk = np.empty((K, hkv, dh))
    dv = np.empty((K, hkv, dh))
    ds = np.empty(K)
    dg = np.empty(hq)
    dtau = np.empty(hq)
    lib().oracle_gated_attention_bwd(_ptr(qr), _ptr(kr), _ptr(vr), _ptr(dr), dt, _ptr(s), _ptr(g),
                                     _ptr(t), _ptr(cu), len(cu) - 1, hq, hkv, dh, _ptr(dq),
                                     _ptr(dk), _ptr(dv), _ptr(ds), _ptr(dg), _ptr(dtau))
    return dq, dk, dv, ds, dg, dtau


def gated_delta_rule(q, k, v, alpha, beta, cu_seqlens) -> np.ndarray:
    """Gated delta rule per sequence and head (state reset at each sequence):
    q, k [T, H, dk], v [T, H, dv], alpha/beta [T, H] -> o [T, H, dv] fp64."""
    qr, dt = _raw(q)
    kr, dt2 = _raw(k)
    vr, dt3 = _raw(v)
    assert dt == dt2 == dt3
    T, H, dk = qr.shape
    dv = vr.shape[2]
    a = _f32(alpha).reshape(T, H)
    b = _f32(beta).reshape(T, H)
    cu = _i32(cu_seqlens)
    out = np.zeros((T, H, dv), np.float64)
    lib().oracle_gated_delta_rule(_ptr(qr), _ptr(kr), _ptr(vr), dt, _ptr(a), _ptr(b), _ptr(cu),
                                  len(cu) - 1, H, dk, dv, _ptr(out))
    return out
