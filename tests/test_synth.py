"""The seeded workloads: shapes, budgets and planted structure."""
import math

import numpy as np
import torch

from learned_token_pruning_gemm_b200 import synth


def test_budgets_follow_keep_ratios():
    # k_doc = floor(ratio * document length); K = k_doc + protected tokens
    assert synth.kept_total([512], [0], [480], [96]) == [128]
    assert synth.kept_total([16384], [0], [16128], [math.floor(0.10 * 16128)]) == [1868]
    for r, K in [(0.05, 2124), (0.10, 3737), (0.25, 8576), (0.50, 16640)]:
        assert synth.kept_total([32768], [0], [32256], [math.floor(r * 32256)]) == [K]
    assert synth.kept_total([131072], [0], [130816], [math.floor(0.08 * 130816)]) == [10721]
    # budget above the document keeps everything; empty document keeps everything
    assert synth.kept_total([10], [2], [6], [99]) == [10]
    assert synth.kept_total([10], [4], [4], [3]) == [10]


def test_tiny_workload_shapes_and_determinism():
    a, b = synth.tiny_f32(), synth.tiny_f32()
    assert a.x.shape == (512, 256) and a.x.dtype == torch.float32
    assert a.w1.shape == (64, 256) and a.q.shape == (128, 4, 64) and a.k.shape == (128, 2, 64)
    assert torch.equal(a.x, b.x) and torch.equal(a.v, b.v) and a.b2 == b.b2
    assert float(a.gain.min()) >= 0 and float(a.gain.max()) <= 1
    assert float(a.tau.min()) >= 0.8 and float(a.tau.max()) <= 1.5
    # Q/K/V ~ N(0,1) as the tiny configuration states: moments and a heavy-ish tail
    for t in (a.q, a.k, a.v):
        assert abs(float(t.mean())) < 0.05 and abs(float(t.std()) - 1.0) < 0.05
    assert float(a.v.abs().max()) > math.sqrt(3.0)      # not the bounded uniform draw
    u = synth.uniform_v(synth.tiny_f32())
    assert float(u.v.abs().max()) <= math.sqrt(3.0) and torch.equal(u.q, a.q)


def test_ragged_workload():
    wl = synth.ragged8()
    assert wl.batch == 8
    assert all(4096 <= n <= 16384 for n in wl.seqlens)
    q = [n - e for n, e in zip(wl.seqlens, wl.doc_end)]
    assert all(64 <= x <= 512 for x in q)
    assert wl.k_doc == [math.floor(0.2 * e) for e in wl.doc_end]
    assert wl.q.shape[0] == wl.total_kept


def test_sweep_duplicates_are_exact_copies():
    wl = synth.sweep32k(0.05)
    src, dst = wl.duplicates[:, 0], wl.duplicates[:, 1]
    assert len(src) == int(0.02 * 32256)
    assert torch.equal(wl.x[torch.from_numpy(src)], wl.x[torch.from_numpy(dst)])
    assert dst.max() < 32256 and src.max() < 32256


def test_planted_clusters_outrank_the_rest(orc):
    wl = synth.qwen16k()
    s64, s32 = orc.gate_score(wl.x, wl.w1, wl.b1, wl.w2, wl.b2)
    n_doc = wl.doc_end[0]
    mask = np.zeros(n_doc, bool)
    mask[wl.planted] = True
    assert mask.sum() == 192
    assert s64[:n_doc][mask].min() > s64[:n_doc][~mask].max()
    idx, _ = orc.select_topk(s32, wl.cu_seqlens, wl.doc_begin, wl.doc_end, wl.k_doc)
    assert len(idx) == 1868 and np.isin(wl.planted, idx).all()


def test_qkv_weights_are_seeded_and_scaled():
    wl = synth.tiny_f32()
    w = synth.qkv_weights(wl)
    assert w.shape == ((wl.hq + 2 * wl.hkv) * wl.dh, wl.d) and w.dtype == wl.x.dtype
    assert torch.equal(w, synth.qkv_weights(synth.tiny_f32()))
    assert abs(float(w.std()) * math.sqrt(wl.d) - 1.0) < 0.05
