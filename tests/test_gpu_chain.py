"""The kept rows' path above the gate layer, end to end on the GPU against the
fp64 oracle: select -> compaction of the residual rows -> q/k/v projections with
the rotary embedding at each kept token's position within its own sequence ->
token-gated attention over the projected rows (MarkTechPost page on TokenGate,
section "Comment TokenGate a-t-il appris le fonctionnement de la réduction des
tokens ?": only the kept tokens get KV entries in the layers above the gate).

Also: a sequence that select rejects leaves defined outputs, and the kernels that
read them next run with no out-of-range access (the status word reports it)."""
import numpy as np
import pytest
import torch

from helpers import assert_attn_close, assert_chain_close, sample_rows

pytestmark = pytest.mark.gpu

# the projection's bar (bf16 outputs rounded from fp32): |gpu - oracle| <= 2^-8 |oracle| + 1e-4
QKV_REL, QKV_ABS = 2.0 ** -8, 1e-4


@pytest.fixture(scope="module")
def mods():
    from learned_token_pruning_gemm_b200 import api, build, pipeline, synth
    build.build()
    api.device_status(reset=True)
    return api, pipeline, synth


def _qkv_close(got, want, rows, what):
    g = got.float().cpu().numpy().astype(np.float64)[rows]
    w = want[rows]
    excess = np.abs(g - w) - (QKV_REL * np.abs(w) + QKV_ABS)
    assert excess.max() <= 0, f"{what}: worst excess {excess.max():.3e}"


def _positions(wl, kept_idx, cu_kept):
    """Each kept row's position within its own sequence, from the host-side offsets."""
    starts = np.repeat(np.asarray(wl.cu_seqlens[:-1], np.int64), np.diff(cu_kept))
    return (kept_idx.astype(np.int64) - starts).astype(np.int32)


@pytest.mark.parametrize("name", ["qwen16k", "ragged8"])
def test_projected_layer_matches_oracle_chain(mods, orc, name):
    api, pipeline, synth = mods
    wl = synth.WORKLOADS[name]()
    gp = pipeline.GatedPrefill(wl, project=True)
    gp.step()
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0

    idx = gp.kept_idx.cpu().numpy()
    cu_kept = gp.cu_kept.cpu().numpy()
    # positions within each sequence (select's own output) equal the host's
    pos = _positions(wl, idx, cu_kept)
    np.testing.assert_array_equal(gp.kept_pos.cpu().numpy(), pos)
    if wl.batch > 1:
        assert (pos != idx).any()          # ragged: positions differ from global row ids
    assert torch.equal(gp.xc.cpu(), wl.x[torch.from_numpy(idx).long()])

    # the projections of the kept rows at their positions (sampled rows)
    K = gp.total_kept
    rows = sample_rows(cu_kept, 24)
    w = gp.w_qkv.cpu()
    q64, k64, v64 = orc.qkv_rope(gp.xc.cpu(), w, wl.hq, wl.hkv, wl.dh, gp.rope_base, pos,
                                 rows=None if K <= 2048 else rows)
    prow = np.arange(K) if K <= 2048 else rows
    for got, ref, nm in zip((gp.q, gp.k, gp.v), (q64, k64, v64), "qkv"):
        _qkv_close(got, ref, prow, f"{name} {nm}")

    # attention on the GPU's projected rows, against the oracle on the same rows
    arows = None if K <= 2048 else sample_rows(cu_kept, 32)
    ref = orc.gated_attention(gp.q.cpu(), gp.k.cpu(), gp.v.cpu(), gp.kept_scores.cpu(), wl.gain,
                              wl.tau, cu_kept, rows=arows)
    assert_attn_close(gp.out, ref, torch.bfloat16, arows, what=f"{name} attention")

    # the whole chain against the oracle's chain: the oracle's projection, rounded to
    # the cache's format (bf16, nearest) as the interface value both sides store,
    # then the oracle's attention
    if K <= 2048:
        to_bf16 = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
        ref_chain = orc.gated_attention(to_bf16(q64), to_bf16(k64), to_bf16(v64),
                                        gp.kept_scores.cpu(), wl.gain, wl.tau, cu_kept)
        max_abs, rl2 = assert_chain_close(gp.out, ref_chain, what=f"{name} oracle chain")
        print(f"{name} chain vs oracle chain: max_abs {max_abs:.2e} rel_l2 {rl2:.2e}")


def test_rejected_sequence_leaves_defined_outputs(mods, orc):
    api, _, _ = mods
    d = lambda a: torch.tensor(a, dtype=torch.int32, device="cuda")
    lens = [1000, 800, 600]
    db, de, kd = [0, 0, 0], [900, 900, 500], [300, 200, 100]   # sequence 1's span passes its end
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    rng = np.random.default_rng(7)
    s = rng.standard_normal(sum(lens)).astype(np.float32)
    # clamped counts: the rejected sequence keeps its clamped extent (span cut at 800)
    counts = [1000 - 900 + 300, 800 - 800 + 200, 600 - 500 + 100]
    total = sum(counts)
    idx, ks, cuk, kpos = api.select_topk(torch.tensor(s, device="cuda"), d(cu), d(db), d(de), d(kd),
                                         total, max(lens), want_pos=True)
    assert api.device_status(reset=True) == 7
    cuk_h = cuk.cpu().numpy()
    np.testing.assert_array_equal(cuk_h, np.r_[0, np.cumsum(counts)])
    idx_h, pos_h = idx.cpu().numpy(), kpos.cpu().numpy()
    assert (idx_h[cuk_h[1]:cuk_h[2]] == -1).all() and (pos_h[cuk_h[1]:cuk_h[2]] == -1).all()
    assert (ks.cpu().numpy()[cuk_h[1]:cuk_h[2]] == 0).all()
    # the valid sequences are unaffected
    for b in (0, 2):
        want, _ = orc.select_topk(s[cu[b]:cu[b + 1]], [0, lens[b]], [db[b]], [de[b]], [kd[b]])
        np.testing.assert_array_equal(idx_h[cuk_h[b]:cuk_h[b + 1]], want + cu[b])
        np.testing.assert_array_equal(pos_h[cuk_h[b]:cuk_h[b + 1]], want)

    # the compaction skips the -1 rows (and records it); the others are copied
    x = torch.randn(sum(lens), 256, device="cuda").to(torch.bfloat16)
    xc = torch.zeros(total, 256, dtype=torch.bfloat16, device="cuda")
    api.compact_rows([x], idx, outs=[xc])
    assert api.device_status(reset=True) == 7
    ok = idx >= 0
    assert torch.equal(xc[ok], x[idx[ok].long()]) and (xc[~ok] == 0).all()

    # attention over select's offsets runs (all in range); with offsets that leave
    # the kept rows it skips the sequence instead of reading or writing outside
    q = torch.randn(total, 4, 128, device="cuda").to(torch.bfloat16)
    kv = torch.randn(total, 2, 128, device="cuda").to(torch.bfloat16)
    g, t = torch.rand(4, device="cuda"), torch.ones(4, device="cuda")
    out = api.gated_attention(q, kv, kv, ks, g, t, cuk, int(np.diff(cuk_h).max()))
    assert api.device_status(reset=True) == 0
    assert torch.isfinite(out.float()).all()
    sentinel = torch.full_like(q, 3.0)
    bad_cu = d([0, total + 500])
    api.gated_attention(q, kv, kv, ks, g, t, bad_cu, total, out=sentinel)
    assert api.device_status(reset=True) == 7
    assert (sentinel.float() == 3.0).all()
    api.gated_attention(q.float(), kv.float(), kv.float(), ks, g, t, d([0, -40, total]), total,
                        out=sentinel.float())
    assert api.device_status(reset=True) == 7


@pytest.mark.parametrize("name", ["qwen16k", "ragged8"])
def test_fused_compaction_matches_separate_kernels(mods, name):
    # the projection gathering the kept rows itself (and writing the compacted rows)
    # against tg_compact_kv then tg_qkv_rope: the same rows, k-blocks and order, so
    # every output is bit-identical
    api, pipeline, synth = mods
    wl = synth.WORKLOADS[name]()
    fused = pipeline.GatedPrefill(wl, project=True, fuse=True)
    sep = pipeline.GatedPrefill(wl, project=True)
    assert fused.STAGES == ("gate", "select", "compact+project", "attention")
    fused.step()
    sep.step()
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0
    for attr in ("kept_idx", "xc", "q", "k", "v", "out"):
        assert torch.equal(getattr(fused, attr), getattr(sep, attr)), attr


def test_fused_compaction_odd_shapes_and_bad_index(mods):
    # 300 of 700 rows (a ragged last row tile), d = 192 (three k-blocks, fewer than the
    # four column tiles that share the compacted rows' writes), 6 q heads and 1 KV head
    # (a column tile holding a k head and a v head)
    api, _, _ = mods
    g = torch.Generator().manual_seed(5)
    N, d, hq, hkv = 700, 192, 6, 1
    x = torch.randn(N, d, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn((hq + 2 * hkv) * 128, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    idx = torch.sort(torch.randperm(N, generator=g)[:300])[0].to(torch.int32).cuda()
    pos = torch.randint(0, 100000, (300,), generator=g, dtype=torch.int32).cuda()
    xc, q, k, v = api.compact_qkv_rope(x, idx, w, hq, hkv, pos)
    assert api.device_status(reset=True) == 0
    xc2 = x[idx.long()]
    q2, k2, v2 = api.qkv_rope(xc2, w, hq, hkv, pos)
    assert torch.equal(xc, xc2)
    for a, b in ((q, q2), (k, k2), (v, v2)):
        assert torch.equal(a, b)
    # without the compacted rows written
    xn, q3, _, _ = api.compact_qkv_rope(x, idx, w, hq, hkv, pos, write_xc=False)
    assert xn is None and torch.equal(q3, q2)
    # an id outside x: recorded, that row projects as zeros, its xc row is left alone
    bad = idx.clone()
    bad[5] = N + 3
    xcb = torch.full((300, d), 7.0, dtype=torch.bfloat16, device="cuda")
    _, qb, kb, vb = api.compact_qkv_rope(x, bad, w, hq, hkv, pos, xc=xcb)
    assert api.device_status(reset=True) == 7
    assert (xcb[5] == 7.0).all()
    for t in (qb, kb, vb):
        assert (t[5] == 0).all()
    keep = torch.ones(300, dtype=torch.bool, device="cuda")
    keep[5] = False
    assert torch.equal(xcb[keep], xc2[keep]) and torch.equal(qb[keep], q2[keep])
