"""End-to-end parity of one gated layer (gate -> select -> compact -> attention)
on every workload, in the launch configuration the benchmark times, against the
fp64 oracle. Full-size workloads compare sampled rows for the stages whose
oracle cost grows with N (gate at 128k, attention), all rows otherwise."""
import numpy as np
import pytest
import torch

from helpers import GATE_ATOL, assert_attn_close, sample_rows, to_np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mods():
    from learned_token_pruning_gemm_b200 import api, build, pipeline, synth
    build.build()
    api.device_status(reset=True)
    return api, pipeline, synth


WORKLOADS = ["tiny_f32", "qwen16k", "sweep32k_5", "sweep32k_25", "sweep32k_50", "long128k",
             "ragged8"]


@pytest.mark.parametrize("name", WORKLOADS)
def test_gated_layer_matches_oracle(mods, orc, name):
    api, pipeline, synth = mods
    wl = synth.WORKLOADS[name]()
    gp = pipeline.GatedPrefill(wl)
    gp.step()
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0

    # --- gate: GPU scores vs fp64 oracle (sampled rows at 128k) ---
    scores = gp.scores.cpu().numpy()
    N = wl.n_tokens
    if N > 40000:
        rng = np.random.default_rng(0)
        rows = np.unique(np.r_[0, 127, 128, N - 1, rng.integers(0, N, 4096)])
    else:
        rows = np.arange(N)
    s64, s32 = orc.gate_score(wl.x[torch.from_numpy(rows)], wl.w1, wl.b1, wl.w2, wl.b2)
    gerr = np.abs(scores[rows].astype(np.float64) - s64).max()
    assert gerr <= GATE_ATOL, f"gate max abs err {gerr:.3e}"

    # --- select: oracle on the GPU's fp32 scores -> bit-exact kept set ---
    sel_in = (wl.score_override.numpy() if wl.score_override is not None else scores)
    want_idx, want_cu = orc.select_topk(sel_in, wl.cu_seqlens, wl.doc_begin, wl.doc_end, wl.k_doc)
    idx = gp.kept_idx.cpu().numpy()
    np.testing.assert_array_equal(idx, want_idx)
    np.testing.assert_array_equal(gp.cu_kept.cpu().numpy(), want_cu)
    np.testing.assert_array_equal(gp.kept_scores.cpu().numpy().view(np.int32),
                                  sel_in[want_idx].view(np.int32))
    assert len(idx) == wl.total_kept

    # --- boundary consistency: the oracle's own scores select the same set up to
    #     tokens whose scores lie within 2e-4 of the K-th document score ---
    if wl.score_override is None and N <= 40000:
        o_idx, _ = orc.select_topk(s32, wl.cu_seqlens, wl.doc_begin, wl.doc_end, wl.k_doc)
        diff = np.setxor1d(o_idx, idx)
        if len(diff):
            for b in range(wl.batch):
                base = wl.cu_seqlens[b]
                doc = s64[base + wl.doc_begin[b]: base + wl.doc_end[b]]
                kth = np.sort(doc)[::-1][wl.k_doc[b] - 1]
                mine = diff[(diff >= base) & (diff < wl.cu_seqlens[b + 1])]
                assert np.all(np.abs(s64[mine] - kth) <= 2e-4), (mine, kth)

    # --- workload structure ---
    if wl.planted is not None:
        assert np.isin(wl.planted, idx).all(), "planted clusters must be kept"
    if wl.duplicates is not None:
        src, dst = wl.duplicates[:, 0], wl.duplicates[:, 1]
        assert np.array_equal(scores[src].view(np.int32), scores[dst].view(np.int32))

    # --- compact: bit-exact gather of the residual rows ---
    assert torch.equal(gp.xc.cpu(), wl.x[torch.from_numpy(idx).long()])

    # --- attention on the GPU's kept scores ---
    cu_kept = gp.cu_kept.cpu().numpy()
    arows = None if wl.total_kept <= 2048 else sample_rows(cu_kept, 48)
    ref = orc.gated_attention(wl.q, wl.k, wl.v, gp.kept_scores.cpu(), wl.gain, wl.tau, cu_kept,
                              rows=arows)
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    assert_attn_close(gp.out, ref, dt, arows, what=name)


def test_graph_replay_matches_eager(mods):
    api, pipeline, synth = mods
    wl = synth.ragged8()
    gp = pipeline.GatedPrefill(wl)
    gp.step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in (gp.scores, gp.kept_idx, gp.kept_scores, gp.cu_kept, gp.xc, gp.out)]
    for t in (gp.scores, gp.kept_scores, gp.out):
        t.zero_()
    gp.capture()
    for t in (gp.scores, gp.kept_scores, gp.out):
        t.zero_()
    gp.replay_step()
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0
    got1 = [t.clone() for t in (gp.scores, gp.kept_idx, gp.kept_scores, gp.cu_kept, gp.xc, gp.out)]
    for t in (gp.scores, gp.kept_scores, gp.out):
        t.zero_()
    gp.replay_timed()
    torch.cuda.synchronize()
    st = gp.stage_times_ms()
    assert all(v > 0 for v in st.values()), st
    got = (gp.scores, gp.kept_idx, gp.kept_scores, gp.cu_kept, gp.xc, gp.out)
    for a, b, c in zip(eager, got, got1):
        assert torch.equal(a, b) and torch.equal(a, c)
