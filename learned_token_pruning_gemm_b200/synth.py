"""Seeded synthetic workloads for the gated-prefill path.

This module only draws numbers. It holds none of the path's arithmetic (no gate
MLP, no selection, no attention): both the CUDA path and the CPU oracle read
the arrays it returns. Every tensor is drawn from its own counter-based stream,
numpy's Philox keyed by (workload seed, tensor id), so a tensor's values do not
depend on which other tensors were drawn or in which order.

The shapes follow the pages' workloads: a Qwen3-1.7B-shaped layer (hidden 2048,
16 query / 8 KV heads, head dim 128) with a small gate MLP, one A100 at batch 1,
contexts of 16k to 128k tokens (MarkTechPost page, "TL;DR" and "Comment TokenGate
se performe sur les benchmarks"). The public tasks timed on the pages (RepoBench-P,
2WikiMultihopQA, MultiNews, BioDEX, NIAH) are not available here; these synthetic
inputs of the same shapes stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

# tensor ids: one Philox key per tensor so every tensor is an independent stream
_TID = {
    "x": 1, "w1": 2, "b1": 3, "w2": 4, "b2": 5, "gain": 6, "tau": 7,
    "q": 8, "k": 9, "v": 10, "plant": 11, "dup": 12, "tscore": 13, "lens": 14,
    "dn_q": 15, "dn_k": 16, "dn_v": 17, "dn_a": 18, "dn_b": 19,
}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, _TID[name]]))


def _as_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def kept_total(seqlens, doc_begin, doc_end, k_doc) -> List[int]:
    """Per-sequence kept count, the output size rule of the select boundary:
    every token outside the droppable span plus min(k_doc, span length)."""
    out = []
    for n, b, e, k in zip(seqlens, doc_begin, doc_end, k_doc):
        nd = e - b
        out.append((n - nd) + min(max(k, 0), nd))
    return out


@dataclasses.dataclass
class Workload:
    name: str
    dtype: str                      # "f32" or "bf16": the type of x, w1, q, k, v, out
    seed: int
    seqlens: List[int]
    doc_begin: List[int]            # per sequence, positions local to the sequence
    doc_end: List[int]
    k_doc: List[int]
    d: int
    h: int
    hq: int
    hkv: int
    dh: int
    x: torch.Tensor                 # [N, d]
    w1: torch.Tensor                # [h, d]  (nn.Linear weight layout: out x in)
    b1: torch.Tensor                # [h] f32
    w2: torch.Tensor                # [h] f32
    b2: float
    gain: torch.Tensor              # [hq] f32
    tau: torch.Tensor               # [hq] f32
    q: torch.Tensor                 # [K, hq, dh]
    k: torch.Tensor                 # [K, hkv, dh]
    v: torch.Tensor                 # [K, hkv, dh]
    score_override: Optional[torch.Tensor] = None   # [N] f32 (heavy-tailed logits)
    planted: Optional[np.ndarray] = None            # global rows of planted clusters
    duplicates: Optional[np.ndarray] = None         # [n,2] (copied-from, copied-to)
    keep_ratio: Optional[float] = None
    v_dist: str = "normal"

    @property
    def n_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def kept_counts(self) -> List[int]:
        return kept_total(self.seqlens, self.doc_begin, self.doc_end, self.k_doc)

    @property
    def total_kept(self) -> int:
        return int(sum(self.kept_counts))

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)


def _weights(seed, dtype, d, h, hq):
    # weights and biases N(0,1)/sqrt(fan_in): W1, b1 fan_in d; w2, b2 fan_in h
    w1 = _rng(seed, "w1").standard_normal((h, d)) / math.sqrt(d)
    b1 = (_rng(seed, "b1").standard_normal(h) / math.sqrt(d)).astype(np.float32)
    w2 = (_rng(seed, "w2").standard_normal(h) / math.sqrt(h)).astype(np.float32)
    b2 = float(np.float32(_rng(seed, "b2").standard_normal() / math.sqrt(h)))
    gain = _rng(seed, "gain").uniform(0.0, 1.0, hq).astype(np.float32)
    tau = _rng(seed, "tau").uniform(0.8, 1.5, hq).astype(np.float32)
    return (_as_dtype(w1, dtype), torch.from_numpy(b1), torch.from_numpy(w2), b2,
            torch.from_numpy(gain), torch.from_numpy(tau))


def _qkv(seed, dtype, K, hq, hkv, dh, v_dist="normal"):
    # Q, K, V ~ N(0,1): what a projection with N(0,1)/sqrt(fan_in) weights makes of a
    # unit-variance residual. v_dist="uniform" draws V from U(-sqrt3, sqrt3) instead
    # (unit variance, bounded by 1.74), for extra cases that keep |O| below 2.
    q = _rng(seed, "q").standard_normal((K, hq, dh))
    k = _rng(seed, "k").standard_normal((K, hkv, dh))
    if v_dist == "uniform":
        v = _rng(seed, "v").uniform(-math.sqrt(3.0), math.sqrt(3.0), (K, hkv, dh))
    else:
        v = _rng(seed, "v").standard_normal((K, hkv, dh))
    return _as_dtype(q, dtype), _as_dtype(k, dtype), _as_dtype(v, dtype)


def make_workload(name: str, dtype: str, seed: int, seqlens, q_lens, keep_ratio=None,
                  k_doc=None, d=2048, h=256, hq=16, hkv=8, dh=128,
                  v_dist="normal") -> Workload:
    """Generic builder: per sequence the droppable span is [0, n - q_len) and the
    protected question is the last q_len tokens."""
    seqlens = [int(n) for n in seqlens]
    doc_begin = [0] * len(seqlens)
    doc_end = [n - ql for n, ql in zip(seqlens, q_lens)]
    if k_doc is None:
        k_doc = [int(math.floor(keep_ratio * (e - b))) for b, e in zip(doc_begin, doc_end)]
    N = sum(seqlens)
    x = _as_dtype(_rng(seed, "x").standard_normal((N, d)), dtype)
    w1, b1, w2, b2, gain, tau = _weights(seed, dtype, d, h, hq)
    K = sum(kept_total(seqlens, doc_begin, doc_end, k_doc))
    q, k, v = _qkv(seed, dtype, K, hq, hkv, dh, v_dist)
    return Workload(name, dtype, seed, seqlens, doc_begin, doc_end, list(k_doc), d, h, hq,
                    hkv, dh, x, w1, b1, w2, b2, gain, tau, q, k, v, keep_ratio=keep_ratio,
                    v_dist=v_dist)


# --------------------------------------------------------------------------- #
# the five workloads                                                           #
# --------------------------------------------------------------------------- #

PLANT_SCALE = 10.0  # c in x += c * r: the smallest integer that lifts every planted score above
                    # the unplanted document maximum at seed 2 (checked by a test)


def tiny_f32(seed: int = 1) -> Workload:
    """Batch 1, N=512, d=256, h=64, 4/2 heads, dh=64, question = last 32, K=128
    total kept (k_doc=96), fp32."""
    return make_workload("tiny_f32", "f32", seed, [512], [32], k_doc=[96],
                         d=256, h=64, hq=4, hkv=2, dh=64)


def qwen16k(seed: int = 2, plant: bool = True) -> Workload:
    """Batch 1, N=16384, bf16, question = last 256, keep 10% of the document
    (k_doc = 1612, K = 1868). Three random non-overlapping 64-token document
    clusters get x += c*r with r = W1^T max(w2, 0) / |.|, the input direction that
    raises the gate units that w2 weights positively."""
    wl = make_workload("qwen16k", "bf16", seed, [16384], [256], keep_ratio=0.10)
    if plant:
        g = _rng(seed, "plant")
        n_doc = wl.doc_end[0]
        slots = g.choice(n_doc // 64, size=3, replace=False)
        rows = np.concatenate([np.arange(s * 64, s * 64 + 64) for s in sorted(slots)])
        w1 = wl.w1.double().numpy()                       # [h, d]
        r = w1.T @ np.maximum(wl.w2.double().numpy(), 0.0)
        r /= np.linalg.norm(r)
        x = wl.x.float().numpy().copy()
        x[rows] += PLANT_SCALE * r.astype(np.float32)
        wl.x = _as_dtype(x, wl.dtype)
        wl.planted = rows
    return wl


def sweep32k(ratio: float, seed: int = 3) -> Workload:
    """Batch 1, N=32768, bf16, question = last 512, keep ratio in {5,10,25,50}%.
    2% of the document rows are exact copies of another document row, so their
    gate scores tie bit for bit."""
    wl = make_workload(f"sweep32k_{int(round(ratio * 100))}", "bf16", seed, [32768], [512],
                       keep_ratio=ratio)
    g = _rng(seed, "dup")
    n_doc = wl.doc_end[0]
    n_dup = int(0.02 * n_doc)
    perm = g.permutation(n_doc)
    src, dst = perm[:n_dup], perm[n_dup:2 * n_dup]
    x = wl.x.clone()
    x[torch.from_numpy(dst)] = x[torch.from_numpy(src)]
    wl.x = x
    wl.duplicates = np.stack([src, dst], 1)
    return wl


def long128k(seed: int = 4) -> Workload:
    """Batch 1, N=131072, bf16, question = last 256, keep 8% of the document
    (k_doc = 10465). The scores fed to select and attention are Student-t(3)
    draws (heavy-tailed gate logits); the gate itself is still run on x."""
    wl = make_workload("long128k", "bf16", seed, [131072], [256], keep_ratio=0.08)
    t = _rng(seed, "tscore").standard_t(3.0, wl.n_tokens).astype(np.float32)
    wl.score_override = torch.from_numpy(t)
    return wl


def ragged8(seed: int = 5) -> Workload:
    """8 sequences, lengths ~ U[4096, 16384], question spans ~ U[64, 512], keep
    20% of each document; one varlen launch per stage."""
    g = _rng(seed, "lens")
    lens = g.integers(4096, 16384, size=8, endpoint=True)
    qls = g.integers(64, 512, size=8, endpoint=True)
    return make_workload("ragged8", "bf16", seed, lens.tolist(), qls.tolist(), keep_ratio=0.20)


WORKLOADS = {
    "tiny_f32": tiny_f32,
    "qwen16k": qwen16k,
    "sweep32k_5": lambda: sweep32k(0.05),
    "sweep32k_10": lambda: sweep32k(0.10),
    "sweep32k_25": lambda: sweep32k(0.25),
    "sweep32k_50": lambda: sweep32k(0.50),
    "long128k": long128k,
    "ragged8": ragged8,
}


def small_case(seed: int, seqlens, q_lens, k_doc, dtype="bf16", d=128, h=64, hq=4, hkv=2,
               dh=128, doc_begin=None, v_dist="normal") -> Workload:
    """A small workload for parity tests, with an arbitrary droppable span."""
    wl = make_workload(f"small_{seed}", dtype, seed, seqlens, q_lens, k_doc=k_doc, d=d, h=h,
                       hq=hq, hkv=hkv, dh=dh, v_dist=v_dist)
    if doc_begin is not None:
        wl.doc_begin = list(doc_begin)
        K = sum(kept_total(wl.seqlens, wl.doc_begin, wl.doc_end, wl.k_doc))
        wl.q, wl.k, wl.v = _qkv(seed, dtype, K, hq, hkv, dh, v_dist)
    return wl


def uniform_v(wl: Workload) -> Workload:
    """The same workload with V redrawn from U(-sqrt3, sqrt3) (the other arrays unchanged)."""
    K = wl.total_kept
    _, _, wl.v = _qkv(wl.seed, wl.dtype, K, wl.hq, wl.hkv, wl.dh, "uniform")
    wl.v_dist = "uniform"
    return wl


def qkv_weights(wl: Workload, seed: int = 11) -> torch.Tensor:
    """W = [Wq; Wk; Wv] [(hq + 2 hkv) dh, d] ~ N(0,1)/sqrt(d), in the workload's dtype: the
    projection weights of the layer above the gate layer, for the kept rows' q/k/v."""
    g = np.random.Generator(np.random.Philox(key=[wl.seed, 100 + seed]))
    n = (wl.hq + 2 * wl.hkv) * wl.dh
    return _as_dtype(g.standard_normal((n, wl.d)) / math.sqrt(wl.d), wl.dtype)


def deltanet_inputs(wl: Workload):
    """Inputs of a Gated DeltaNet layer over the workload's kept rows (one row per
    kept token, the workload's query-head count and head size): q, k drawn N(0,1)
    and scaled to unit length per head (the layer normalises them before the rule),
    v ~ N(0,1), decay alpha ~ U(0.9, 1), write strength beta ~ U(0, 1)."""
    K, H, d = wl.total_kept, wl.hq, wl.dh
    def unit(name):
        a = _rng(wl.seed, name).standard_normal((K, H, d))
        return a / np.linalg.norm(a, axis=-1, keepdims=True)
    q, k = unit("dn_q"), unit("dn_k")
    v = _rng(wl.seed, "dn_v").standard_normal((K, H, d))
    alpha = _rng(wl.seed, "dn_a").uniform(0.9, 1.0, (K, H)).astype(np.float32)
    beta = _rng(wl.seed, "dn_b").uniform(0.0, 1.0, (K, H)).astype(np.float32)
    return (_as_dtype(q, "bf16"), _as_dtype(k, "bf16"), _as_dtype(v, "bf16"),
            torch.from_numpy(alpha), torch.from_numpy(beta))
