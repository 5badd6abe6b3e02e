"""Python binding of the C ABI: argument marshalling over torch CUDA tensors.

Every function here checks shapes/dtypes, passes raw device pointers and the
current torch stream to libtokengate.so, and raises TokenGateError on a non-OK
status. All arithmetic happens in the CUDA kernels.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import TokenGateError, check

TG_F32, TG_BF16 = 0, 1
_DT = {torch.float32: TG_F32, torch.bfloat16: TG_BF16}


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TokenGateError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise TokenGateError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TokenGateError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _numel(t: torch.Tensor, n: int, name: str) -> None:
    if t.numel() != n:
        raise TokenGateError(f"{name} must have {n} elements, got {t.numel()}")


def _shape(t: torch.Tensor, shape, name: str, dtype=None) -> None:
    if tuple(t.shape) != tuple(shape):
        raise TokenGateError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TokenGateError(f"{name} must be {dtype}, got {t.dtype}")


def abi_version() -> int:
    return _lib.load().tg_abi_version()


def gate_score(x: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: float,
               out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """s = b2 + w2 . GELU(W1 x + b1) per token. x [N, d], w1 [h, d] (same dtype)."""
    n, d = x.shape
    h = w1.shape[0]
    if w1.shape != (h, d) or w1.dtype != x.dtype or x.dtype not in _DT:
        raise TokenGateError("gate_score: x [N,d] and w1 [h,d] must share a dtype (f32/bf16)")
    _numel(b1, h, "b1")
    _numel(w2, h, "w2")
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=x.device)
    _numel(out, n, "scores")
    st = _lib.load().tg_gate_score(_cuda(x, "x"), _DT[x.dtype], n, d, _cuda(w1, "w1"),
                                   _cuda(b1, "b1", torch.float32), _cuda(w2, "w2", torch.float32),
                                   float(b2), h, _cuda(out, "scores", torch.float32), _stream(stream))
    check(st, "tg_gate_score")
    return out


def select_topk(scores: torch.Tensor, cu_seqlens: torch.Tensor, doc_begin: torch.Tensor,
                doc_end: torch.Tensor, k_doc: torch.Tensor, total_kept: int, max_seqlen: int,
                kept_idx: Optional[torch.Tensor] = None, kept_scores: Optional[torch.Tensor] = None,
                cu_kept: Optional[torch.Tensor] = None, want_scores: bool = True,
                kept_pos: Optional[torch.Tensor] = None, want_pos: bool = False, stream=None):
    """Returns (kept_idx int32 [total_kept], kept_scores f32 [total_kept] or None,
    cu_kept int32 [B+1]); with want_pos (or kept_pos given) also kept_pos int32
    [total_kept], the kept rows' positions within their sequences, as a 4th item."""
    B = doc_begin.numel()
    dev = scores.device
    total_kept = int(total_kept)
    _numel(cu_seqlens, B + 1, "cu_seqlens")
    _numel(doc_end, B, "doc_end")
    _numel(k_doc, B, "k_doc")
    if kept_idx is None:
        kept_idx = torch.empty(total_kept, dtype=torch.int32, device=dev)
    if kept_scores is None and want_scores:
        kept_scores = torch.empty(total_kept, dtype=torch.float32, device=dev)
    if kept_pos is None and want_pos:
        kept_pos = torch.empty(total_kept, dtype=torch.int32, device=dev)
    if cu_kept is None:
        cu_kept = torch.empty(B + 1, dtype=torch.int32, device=dev)
    _numel(kept_idx, total_kept, "kept_idx")
    if kept_scores is not None:
        _numel(kept_scores, total_kept, "kept_scores")
    if kept_pos is not None:
        _numel(kept_pos, total_kept, "kept_pos")
    _numel(cu_kept, B + 1, "cu_kept")
    st = _lib.load().tg_select_topk(
        _cuda(scores, "scores", torch.float32), _cuda(cu_seqlens, "cu_seqlens", torch.int32),
        _cuda(doc_begin, "doc_begin", torch.int32), _cuda(doc_end, "doc_end", torch.int32),
        _cuda(k_doc, "k_doc", torch.int32), B, scores.numel(), total_kept, int(max_seqlen),
        _cuda(kept_idx, "kept_idx", torch.int32),
        _cuda(kept_scores, "kept_scores", torch.float32) if kept_scores is not None else None,
        _cuda(kept_pos, "kept_pos", torch.int32) if kept_pos is not None else None,
        _cuda(cu_kept, "cu_kept", torch.int32), _stream(stream))
    check(st, "tg_select_topk")
    if kept_pos is not None:
        return kept_idx, kept_scores, cu_kept, kept_pos
    return kept_idx, kept_scores, cu_kept


def compact_rows(srcs: Sequence[torch.Tensor], kept_idx: torch.Tensor,
                 outs: Optional[Sequence[torch.Tensor]] = None, stream=None):
    """dst[t][r] = src[t][kept_idx[r]] for every tensor (rows = first dim)."""
    n = kept_idx.numel()
    if not srcs:
        raise TokenGateError("compact_rows: at least one source tensor")
    if outs is None:
        outs = [torch.empty((n,) + tuple(s.shape[1:]), dtype=s.dtype, device=s.device) for s in srcs]
    k = len(srcs)
    if len(outs) != k:
        raise TokenGateError("compact_rows: one output per source")
    for s, o in zip(srcs, outs):
        if o.shape[1:] != s.shape[1:] or o.dtype != s.dtype or o.shape[0] != n:
            raise TokenGateError("compact_rows: output shape/dtype mismatch")
    src_arr = (ctypes.c_void_p * k)(*[_cuda(s, "src") for s in srcs])
    dst_arr = (ctypes.c_void_p * k)(*[_cuda(o, "dst") for o in outs])
    rb = (ctypes.c_int64 * k)(*[math.prod(s.shape[1:]) * s.element_size() for s in srcs])
    n_src = min(s.shape[0] for s in srcs)
    st = _lib.load().tg_compact_kv(src_arr, dst_arr, rb, k, _cuda(kept_idx, "kept_idx", torch.int32),
                                   n, n_src, _stream(stream))
    check(st, "tg_compact_kv")
    return list(outs)


def gated_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s_kept: torch.Tensor,
                    gain: torch.Tensor, tau: torch.Tensor, cu_kept: torch.Tensor, max_kept: int,
                    out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Token-gated causal GQA attention. q [K,Hq,dh], k/v [K,Hkv,dh] (same dtype).
    If `lse` ([Hq, K] f32) is given, each row's log-sum-exp is written there."""
    K, hq, dh = q.shape
    hkv = k.shape[1]
    if k.shape != (K, hkv, dh) or v.shape != k.shape or not (q.dtype == k.dtype == v.dtype):
        raise TokenGateError("gated_attention: q [K,Hq,dh], k/v [K,Hkv,dh] with one dtype")
    if q.dtype not in _DT:
        raise TokenGateError(f"gated_attention: unsupported dtype {q.dtype}")
    _numel(s_kept, K, "s_kept")
    _numel(gain, hq, "gain")
    _numel(tau, hq, "tau")
    if cu_kept.numel() < 1:
        raise TokenGateError("cu_kept must have batch+1 >= 1 elements")
    if out is None:
        out = torch.empty_like(q)
    _shape(out, q.shape, "out", q.dtype)
    if lse is not None:
        _shape(lse, (hq, K), "lse", torch.float32)
    B = cu_kept.numel() - 1
    st = _lib.load().tg_gated_attention(
        _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _DT[q.dtype],
        _cuda(s_kept, "s_kept", torch.float32), _cuda(gain, "gain", torch.float32),
        _cuda(tau, "tau", torch.float32), _cuda(cu_kept, "cu_kept", torch.int32), B, K,
        int(max_kept), hq, hkv, dh, _cuda(out, "out"),
        _cuda(lse, "lse") if lse is not None else None, _stream(stream))
    check(st, "tg_gated_attention")
    return out


def gated_attention_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                        dout: torch.Tensor, lse: torch.Tensor, s_kept: torch.Tensor,
                        gain: torch.Tensor, tau: torch.Tensor, cu_kept: torch.Tensor,
                        max_kept: int, grads=None, workspace: Optional[torch.Tensor] = None,
                        stream=None):
    """Gradients of gated_attention: returns (dq, dk, dv, ds, dgain, dtau) for upstream
    dout, from the forward's out and lse ([Hq, K] f32)."""
    K, hq, dh = q.shape
    hkv = k.shape[1]
    if k.shape != (K, hkv, dh) or v.shape != k.shape or not (q.dtype == k.dtype == v.dtype):
        raise TokenGateError("gated_attention_bwd: q [K,Hq,dh], k/v [K,Hkv,dh] with one dtype")
    if q.dtype not in _DT:
        raise TokenGateError(f"gated_attention_bwd: unsupported dtype {q.dtype}")
    _shape(out, q.shape, "out", q.dtype)
    _shape(dout, q.shape, "dout", q.dtype)
    _shape(lse, (hq, K), "lse", torch.float32)
    _numel(s_kept, K, "s_kept")
    _numel(gain, hq, "gain")
    _numel(tau, hq, "tau")
    B = cu_kept.numel() - 1
    if grads is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty(K, **f32), torch.empty(hq, **f32), torch.empty(hq, **f32))
    dq, dk, dv, ds, dg, dt = grads
    _shape(dq, q.shape, "dq", q.dtype)
    _shape(dk, k.shape, "dk", q.dtype)
    _shape(dv, k.shape, "dv", q.dtype)
    _shape(ds, (K,), "ds", torch.float32)
    _shape(dg, (hq,), "dgain", torch.float32)
    _shape(dt, (hq,), "dtau", torch.float32)
    lib = _lib.load()
    need = int(lib.tg_gated_attention_bwd_workspace_size(_DT[q.dtype], B, K, int(max_kept), hq,
                                                           hkv, dh))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    nb = workspace.numel() * workspace.element_size()
    st = lib.tg_gated_attention_bwd(
        _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(out, "out"), _cuda(dout, "dout"),
        _DT[q.dtype], _cuda(lse, "lse"), _cuda(s_kept, "s_kept", torch.float32),
        _cuda(gain, "gain", torch.float32), _cuda(tau, "tau", torch.float32),
        _cuda(cu_kept, "cu_kept", torch.int32), B, K, int(max_kept), hq, hkv, dh, _cuda(dq, "dq"),
        _cuda(dk, "dk"), _cuda(dv, "dv"), _cuda(ds, "ds"), _cuda(dg, "dgain"), _cuda(dt, "dtau"),
        _cuda(workspace, "workspace"), nb, _stream(stream))
    check(st, "tg_gated_attention_bwd")
    return dq, dk, dv, ds, dg, dt


def gated_delta_rule_workspace_size(batch: int, total: int, n_heads: int, head_dim_v: int) -> int:
    return int(_lib.load().tg_gated_delta_rule_workspace_size(batch, total, n_heads, head_dim_v))


def gated_delta_rule(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                     beta: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: Optional[int] = None,
                     out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Gated delta rule per sequence and head over packed rows: q, k [T,H,dk], v [T,H,dv]
    bf16, alpha/beta [T,H] f32 -> out [T,H,dv] bf16 (state reset per sequence).
    max_seqlen bounds every sequence's length; when None it is read from cu_seqlens
    (a device-to-host copy). workspace: uint8 of at least gated_delta_rule_workspace_size
    bytes, allocated here when None."""
    T, H, dk = q.shape
    dv = v.shape[2]
    _shape(k, q.shape, "k", q.dtype)
    _shape(v, (T, H, dv), "v", q.dtype)
    _shape(alpha, (T, H), "alpha", torch.float32)
    _shape(beta, (T, H), "beta", torch.float32)
    if cu_seqlens.numel() < 1:
        raise TokenGateError("cu_seqlens must have batch+1 >= 1 elements")
    if q.dtype not in _DT:
        raise TokenGateError(f"gated_delta_rule: unsupported dtype {q.dtype}")
    B = cu_seqlens.numel() - 1
    if max_seqlen is None:
        cu_h = cu_seqlens.detach().to("cpu", torch.int64)
        max_seqlen = int((cu_h[1:] - cu_h[:-1]).max()) if B > 0 else 0
    if out is None:
        out = torch.empty_like(v)
    _shape(out, v.shape, "out", v.dtype)
    need = gated_delta_rule_workspace_size(B, T, H, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if workspace.dtype != torch.uint8 or workspace.numel() < need:
        raise TokenGateError(f"gated_delta_rule: workspace needs {need} bytes (uint8)")
    st = _lib.load().tg_gated_delta_rule(
        _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _DT[q.dtype], _cuda(alpha, "alpha"),
        _cuda(beta, "beta"), _cuda(cu_seqlens, "cu_seqlens", torch.int32),
        B, T, int(max_seqlen), H, dk, dv, _cuda(out, "out"), _cuda(workspace, "workspace"),
        workspace.numel(), _stream(stream))
    check(st, "tg_gated_delta_rule")
    return out


def qkv_rope(xc: torch.Tensor, w_qkv: torch.Tensor, n_hq: int, n_hkv: int, pos: torch.Tensor,
             rope_base: float = 1e6, out=None, stream=None):
    """The kept rows' projections: (q [K,Hq,dh], k [K,Hkv,dh], v [K,Hkv,dh]) bf16 from
    xc [K,d] bf16 and w_qkv [(Hq+2Hkv)*dh, d] bf16, q/k rotated at pos [K] int32."""
    K, d = xc.shape
    n_out = w_qkv.shape[0]
    if (n_out % (n_hq + 2 * n_hkv)) or w_qkv.shape[1] != d or xc.dtype != w_qkv.dtype:
        raise TokenGateError("qkv_rope: w_qkv [(Hq+2Hkv)*dh, d] with the dtype of xc")
    dh = n_out // (n_hq + 2 * n_hkv)
    _numel(pos, K, "pos")
    if out is None:
        out = (torch.empty(K, n_hq, dh, dtype=xc.dtype, device=xc.device),
               torch.empty(K, n_hkv, dh, dtype=xc.dtype, device=xc.device),
               torch.empty(K, n_hkv, dh, dtype=xc.dtype, device=xc.device))
    q, k, v = out
    _shape(q, (K, n_hq, dh), "q", xc.dtype)
    _shape(k, (K, n_hkv, dh), "k", xc.dtype)
    _shape(v, (K, n_hkv, dh), "v", xc.dtype)
    st = _lib.load().tg_qkv_rope(_cuda(xc, "xc", torch.bfloat16), K, d,
                                 _cuda(w_qkv, "w_qkv", torch.bfloat16), n_hq, n_hkv, dh,
                                 float(rope_base), _cuda(pos, "pos", torch.int32), _cuda(q, "q"),
                                 _cuda(k, "k"), _cuda(v, "v"), _stream(stream))
    check(st, "tg_qkv_rope")
    return q, k, v


def compact_qkv_rope(x: torch.Tensor, kept_idx: torch.Tensor, w_qkv: torch.Tensor, n_hq: int,
                     n_hkv: int, pos: torch.Tensor, rope_base: float = 1e6, xc=None, out=None,
                     write_xc: bool = True, stream=None):
    """The compaction fused into the projections: xc = x[kept_idx] (written when
    write_xc, into `xc` if given) and (q, k, v) of those rows, as qkv_rope(xc, ...)
    would give them, in one kernel that gathers the rows from x itself. x [N,d] bf16,
    kept_idx [K] int32. Returns (xc or None, q, k, v)."""
    N, d = x.shape
    K = kept_idx.numel()
    n_out = w_qkv.shape[0]
    if (n_out % (n_hq + 2 * n_hkv)) or w_qkv.shape[1] != d or x.dtype != w_qkv.dtype:
        raise TokenGateError("compact_qkv_rope: w_qkv [(Hq+2Hkv)*dh, d] with the dtype of x")
    dh = n_out // (n_hq + 2 * n_hkv)
    _numel(pos, K, "pos")
    if write_xc:
        if xc is None:
            xc = torch.empty(K, d, dtype=x.dtype, device=x.device)
        _shape(xc, (K, d), "xc", x.dtype)
    elif xc is not None:
        raise TokenGateError("compact_qkv_rope: xc given with write_xc=False")
    if out is None:
        out = (torch.empty(K, n_hq, dh, dtype=x.dtype, device=x.device),
               torch.empty(K, n_hkv, dh, dtype=x.dtype, device=x.device),
               torch.empty(K, n_hkv, dh, dtype=x.dtype, device=x.device))
    q, k, v = out
    _shape(q, (K, n_hq, dh), "q", x.dtype)
    _shape(k, (K, n_hkv, dh), "k", x.dtype)
    _shape(v, (K, n_hkv, dh), "v", x.dtype)
    st = _lib.load().tg_compact_qkv_rope(
        _cuda(x, "x", torch.bfloat16), N, d, _cuda(kept_idx, "kept_idx", torch.int32), K,
        _cuda(xc, "xc") if xc is not None else None, _cuda(w_qkv, "w_qkv", torch.bfloat16),
        n_hq, n_hkv, dh, float(rope_base), _cuda(pos, "pos", torch.int32), _cuda(q, "q"),
        _cuda(k, "k"), _cuda(v, "v"), _stream(stream))
    check(st, "tg_compact_qkv_rope")
    return xc, q, k, v


def cache_append(k_new: torch.Tensor, v_new: torch.Tensor, s_new: torch.Tensor,
                 k_cache: torch.Tensor, v_cache: torch.Tensor, s_cache: torch.Tensor,
                 cache_len: torch.Tensor, stream=None) -> None:
    """Row cache_len[b] of sequence b's cache gets k_new[b], v_new[b], s_new[b];
    cache_len[b] += 1. Caches [B, cap, Hkv, dh] bf16 and [B, cap] f32."""
    B, cap, hkv, dh = k_cache.shape
    _shape(v_cache, k_cache.shape, "v_cache", k_cache.dtype)
    _shape(k_new, (B, hkv, dh), "k_new", k_cache.dtype)
    _shape(v_new, (B, hkv, dh), "v_new", k_cache.dtype)
    _shape(s_new, (B,), "s_new", torch.float32)
    _shape(s_cache, (B, cap), "s_cache", torch.float32)
    _shape(cache_len, (B,), "cache_len", torch.int32)
    st = _lib.load().tg_cache_append(
        _cuda(k_new, "k_new", torch.bfloat16), _cuda(v_new, "v_new", torch.bfloat16),
        _cuda(s_new, "s_new"), B, cap, hkv, dh, _cuda(k_cache, "k_cache", torch.bfloat16),
        _cuda(v_cache, "v_cache", torch.bfloat16), _cuda(s_cache, "s_cache"),
        _cuda(cache_len, "cache_len"), _stream(stream))
    check(st, "tg_cache_append")


def decode_workspace_size(batch: int, n_hq: int, head_dim: int, max_len: int) -> int:
    return int(_lib.load().tg_gated_decode_workspace_size(batch, n_hq, head_dim, max_len))


def gated_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 s_cache: torch.Tensor, cache_len: torch.Tensor, gain: torch.Tensor,
                 tau: torch.Tensor, max_len: int, out: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One query row per sequence (q [B, Hq, dh] bf16) over its cache rows
    j < cache_len[b]; returns out [B, Hq, dh] bf16."""
    B, hq, dh = q.shape
    Bc, cap, hkv, dh2 = k_cache.shape
    if Bc != B or dh2 != dh:
        raise TokenGateError("gated_decode: q [B,Hq,dh] and caches [B,cap,Hkv,dh]")
    _shape(v_cache, k_cache.shape, "v_cache", k_cache.dtype)
    _shape(s_cache, (B, cap), "s_cache", torch.float32)
    _shape(cache_len, (B,), "cache_len", torch.int32)
    _numel(gain, hq, "gain")
    _numel(tau, hq, "tau")
    if out is None:
        out = torch.empty_like(q)
    _shape(out, q.shape, "out", q.dtype)
    need = decode_workspace_size(B, hq, dh, max(int(max_len), 1))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < need:
        raise TokenGateError(f"gated_decode: workspace needs {need} bytes")
    st = _lib.load().tg_gated_decode(
        _cuda(q, "q", torch.bfloat16), _cuda(k_cache, "k_cache", torch.bfloat16),
        _cuda(v_cache, "v_cache", torch.bfloat16), _cuda(s_cache, "s_cache"),
        _cuda(cache_len, "cache_len"), B, cap, int(max_len), hq, hkv, dh,
        _cuda(gain, "gain", torch.float32), _cuda(tau, "tau", torch.float32), _cuda(out, "out"),
        _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    check(st, "tg_gated_decode")
    return out


def device_status(reset: bool = True, stream=None) -> int:
    """Synchronise the stream and return (then clear) the device status word."""
    return _lib.load().tg_device_status(_stream(stream), 1 if reset else 0)


def selftest_bounded_wait(timeout_ns: int, stream=None) -> None:
    check(_lib.load().tg_selftest_bounded_wait(int(timeout_ns), _stream(stream)),
          "tg_selftest_bounded_wait")
