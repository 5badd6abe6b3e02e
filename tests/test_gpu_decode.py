"""GPU parity of decode over the compacted cache (tg_cache_append, tg_gated_decode)
against the fp64 oracle, through the C ABI (MarkTechPost page on TokenGate, section
"Comment déployer TokenGate ?": generation runs on the cache that the pruned
prefill leaves). Tolerances: the bf16 bar of tests/helpers.py."""
import math

import numpy as np
import pytest
import torch

from helpers import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from learned_token_pruning_gemm_b200 import api, build
    build.build()
    api.device_status(reset=True)
    return api


@pytest.fixture(autouse=True)
def _no_device_errors(api):
    yield
    assert api.device_status(reset=True) == 0, "a kernel recorded a device-side error"


def _case(seed, B, cap, lens, hq, hkv, dh=128, garbage=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, hq, dh, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cap, hkv, dh, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, hkv, dh, generator=g).to(torch.bfloat16)
    sc = torch.randn(B, cap, generator=g) * 2
    if garbage:   # rows past the cache's end hold anything, NaN included
        for b, n in enumerate(lens):
            kc[b, n:] = float("nan")
            vc[b, n:] = float("inf")
            sc[b, n:] = float("nan")
    gain = torch.rand(hq, generator=g)
    tau = 0.8 + 0.7 * torch.rand(hq, generator=g)
    return q, kc, vc, sc, torch.tensor(lens, dtype=torch.int32), gain, tau


def _run(api, q, kc, vc, sc, lens, gain, tau, max_len=None, out=None):
    cuda = lambda t: t.cuda()
    return api.gated_decode(cuda(q), cuda(kc), cuda(vc), cuda(sc), cuda(lens), cuda(gain),
                            cuda(tau), int(lens.max()) if max_len is None else max_len, out=out)


@pytest.mark.parametrize("B,cap,lens,hq,hkv", [
    (3, 700, [700, 129, 1], 16, 8),       # several chunks, a ragged last chunk, one row
    (2, 200, [64, 65], 8, 8),             # group of one, chunk edge
    (2, 300, [300, 190], 16, 2),          # group of eight
    (1, 2000, [1868], 16, 8),             # the 16k layer's kept count
])
def test_decode_vs_oracle(api, orc, B, cap, lens, hq, hkv):
    q, kc, vc, sc, ln, gain, tau = _case(B + cap, B, cap, lens, hq, hkv)
    out = _run(api, q, kc, vc, sc, ln, gain, tau)
    ref = orc.gated_decode(q, kc, vc, sc, ln.numpy(), gain, tau)
    max_abs, rl2 = assert_attn_close(out, ref, torch.bfloat16, what=f"decode lens={lens}")
    print(f"decode lens={lens} G={hq // hkv}: max_abs {max_abs:.2e} rel_l2 {rl2:.2e}")


def test_decode_plain_when_gain0_tau1(api):
    q, kc, vc, sc, ln, gain, tau = _case(5, 1, 400, [333], 4, 2, garbage=False)
    gain.zero_()
    tau.fill_(1.0)
    out = _run(api, q, kc, vc, sc, ln, gain, tau).float().cpu()
    for h in range(4):
        want = torch.nn.functional.scaled_dot_product_attention(
            q[0, h].double()[None, None], kc[0, :333, h // 2].double()[None],
            vc[0, :333, h // 2].double()[None])[0, 0]
        assert (out[0, h].double() - want).abs().max() <= 1e-2


def test_append_then_decode(api, orc):
    B, cap, hq, hkv = 2, 130, 4, 2
    q, kc, vc, sc, ln, gain, tau = _case(6, B, cap, [128, 5], hq, hkv, garbage=False)
    g = torch.Generator().manual_seed(8)
    kn = torch.randn(B, hkv, 128, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, hkv, 128, generator=g).to(torch.bfloat16)
    sn = torch.randn(B, generator=g)
    kcd, vcd, scd, lnd = kc.cuda(), vc.cuda(), sc.cuda(), ln.cuda()
    api.cache_append(kn.cuda(), vn.cuda(), sn.cuda(), kcd, vcd, scd, lnd)
    assert lnd.cpu().tolist() == [129, 6]
    for b, r in enumerate([128, 5]):
        assert torch.equal(kcd[b, r].cpu(), kn[b]) and torch.equal(vcd[b, r].cpu(), vn[b])
        assert scd[b, r].item() == sn[b].item()
    out = api.gated_decode(q.cuda(), kcd, vcd, scd, lnd, gain.cuda(), tau.cuda(), 129)
    ref = orc.gated_decode(q, kcd.cpu(), vcd.cpu(), scd.cpu(), lnd.cpu().numpy(), gain, tau)
    assert_attn_close(out, ref, torch.bfloat16, what="append then decode")
    # a full cache is left alone and the error recorded
    api.cache_append(kn.cuda(), vn.cuda(), sn.cuda(), kcd, vcd, scd, lnd)   # 130, 7
    api.cache_append(kn.cuda(), vn.cuda(), sn.cuda(), kcd, vcd, scd, lnd)   # full, 8
    assert api.device_status(reset=True) == 7
    assert lnd.cpu().tolist() == [130, 8]


def test_decode_edges(api):
    q, kc, vc, sc, ln, gain, tau = _case(9, 3, 100, [0, 100, 3], 4, 2)
    out = _run(api, q, kc, vc, sc, ln, gain, tau).float().cpu()
    assert (out[0] == 0).all() and torch.isfinite(out).all()
    # a length beyond max_len leaves the row unchanged and records the error
    sentinel = torch.full((3, 4, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    _run(api, q, kc, vc, sc, ln, gain, tau, max_len=50, out=sentinel)
    assert api.device_status(reset=True) == 7
    assert (sentinel[1].float() == 7.0).all() and (sentinel[0].float() == 0).all()
    from learned_token_pruning_gemm_b200._lib import TokenGateError
    with pytest.raises(TokenGateError, match="workspace"):
        api.gated_decode(q.cuda(), kc.cuda(), vc.cuda(), sc.cuda(), ln.cuda(), gain.cuda(),
                         tau.cuda(), 100, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))


def test_decode_of_last_kept_token_matches_prefill_row(api, orc):
    # the 16k layer: the prefill's last kept row attends over all kept rows; decoding
    # that token over the compacted cache (kept k, v and scores) gives the same row
    from learned_token_pruning_gemm_b200 import pipeline, synth
    wl = synth.qwen16k()
    gp = pipeline.GatedPrefill(wl)
    gp.step()
    torch.cuda.synchronize()
    K = gp.total_kept
    cap = K + 64
    kc = torch.zeros(1, cap, wl.hkv, wl.dh, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    sc = torch.zeros(1, cap, device="cuda")
    kc[0, :K] = gp.k
    vc[0, :K] = gp.v
    sc[0, :K] = gp.kept_scores
    ln = torch.tensor([K], dtype=torch.int32, device="cuda")
    out = api.gated_decode(gp.q[K - 1:K].contiguous(), kc, vc, sc, ln, gp.gain, gp.tau, K)
    ref = orc.gated_decode(gp.q[K - 1:K].cpu(), kc.cpu(), vc.cpu(), sc.cpu(), [K], wl.gain, wl.tau)
    assert_attn_close(out, ref, torch.bfloat16, what="decode of the last kept token")
    diff = (out[0].float() - gp.out[K - 1].float()).abs().max().item()
    assert diff <= 2e-2, diff    # two bf16 results of the same row, each within 1e-2


@pytest.mark.parametrize("name", ["long128k", "ragged8"])
def test_decode_step_on_the_benchmark_caches(api, orc, name):
    # the decode step the benchmark times on its other layers: each sequence's kept
    # rows (k, v, scores of the measured prefill) are its cache, capacity K_b + 64;
    # one new token per sequence is appended and attends over the grown cache
    from learned_token_pruning_gemm_b200 import pipeline, synth
    wl = synth.WORKLOADS[name]()
    gp = pipeline.GatedPrefill(wl)
    gp.step()
    torch.cuda.synchronize()
    counts = wl.kept_counts
    B, cap = wl.batch, max(counts) + 64
    kc = torch.zeros(B, cap, wl.hkv, wl.dh, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    sc = torch.zeros(B, cap, device="cuda")
    cu = gp.cu_kept.cpu().tolist()
    for b in range(B):
        kc[b, :counts[b]] = gp.k[cu[b]:cu[b + 1]]
        vc[b, :counts[b]] = gp.v[cu[b]:cu[b + 1]]
        sc[b, :counts[b]] = gp.kept_scores[cu[b]:cu[b + 1]]
    g = torch.Generator().manual_seed(3)
    qn = torch.randn(B, wl.hq, wl.dh, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, wl.hkv, wl.dh, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, wl.hkv, wl.dh, generator=g).to(torch.bfloat16)
    sn = torch.randn(B, generator=g)
    ln = torch.tensor(counts, dtype=torch.int32, device="cuda")
    api.cache_append(kn.cuda(), vn.cuda(), sn.cuda(), kc, vc, sc, ln)
    out = api.gated_decode(qn.cuda(), kc, vc, sc, ln, gp.gain, gp.tau, cap)
    torch.cuda.synchronize()
    assert ln.cpu().tolist() == [c + 1 for c in counts]
    ref = orc.gated_decode(qn, kc.cpu(), vc.cpu(), sc.cpu(), [c + 1 for c in counts], wl.gain, wl.tau)
    assert_attn_close(out, ref, torch.bfloat16, what=f"decode step on {name}")
