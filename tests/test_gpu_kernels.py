"""GPU parity of each kernel against the fp64 CPU oracle, through the C ABI.

Sizes span several tiles and a ragged tail; edge cases cover empty and degenerate
inputs. See tests/helpers.py for the tolerances."""
import math

import numpy as np
import pytest
import torch

from helpers import (ATTN_BF16_ATOL, GATE_ATOL, assert_attn_close, attn_errors, sample_rows,
                     to_np64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from learned_token_pruning_gemm_b200 import api, build
    build.build()
    assert torch.cuda.is_available()
    api.device_status(reset=True)
    return api


@pytest.fixture(autouse=True)
def _no_device_errors(api):
    yield
    assert api.device_status(reset=True) == 0, "a kernel recorded a device-side error"


def _gen(seed):
    return torch.Generator().manual_seed(seed)


# ------------------------------------------------------------------ gate ----

# the last three have more 128-token tiles than the GPU has SMs (148 on B200), so
# they run the 256-token kernel (two row tiles per CTA), ragged tails included
@pytest.mark.parametrize("n,d,h", [(300, 128, 64), (129, 256, 128), (1000, 2048, 256),
                                   (128, 64, 256), (255, 192, 64), (19100, 256, 256),
                                   (40001, 128, 128), (18945, 192, 64)])
def test_gate_bf16_vs_oracle(api, orc, n, d, h):
    g = _gen(n + d + h)
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    w1 = (torch.randn(h, d, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    b1 = torch.randn(h, generator=g) / math.sqrt(d)
    w2 = torch.randn(h, generator=g) / math.sqrt(h)
    b2 = 0.123
    s = api.gate_score(x.cuda(), w1.cuda(), b1.cuda(), w2.cuda(), b2)
    s64, _ = orc.gate_score(x, w1, b1, w2, b2)
    err = np.abs(s.cpu().double().numpy() - s64).max()
    assert err <= GATE_ATOL, err


def test_gate_f32_vs_oracle(api, orc):
    g = _gen(3)
    n, d, h = 517, 256, 64
    x = torch.randn(n, d, generator=g)
    w1 = torch.randn(h, d, generator=g) / 16
    b1, w2 = torch.randn(h, generator=g) / 16, torch.randn(h, generator=g) / 8
    s = api.gate_score(x.cuda(), w1.cuda(), b1.cuda(), w2.cuda(), -0.5)
    s64, _ = orc.gate_score(x, w1, b1, w2, -0.5)
    assert np.abs(s.cpu().double().numpy() - s64).max() <= GATE_ATOL


@pytest.mark.parametrize("n", [1024, 20000])
def test_gate_duplicate_rows_bit_identical(api, n):
    # copies in other tiles, in the other row tile of the same CTA, and across CTAs
    g = _gen(4)
    d, h = 512, 256
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    src = torch.tensor([3, 200, 511, 900, 10, n - 3])    # disjoint from dst
    dst = torch.tensor([700, 5, 1023, 128, 130, n // 2 + 7])
    x[dst] = x[src]
    w1 = (torch.randn(h, d, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    b1, w2 = torch.randn(h, generator=g) * 0.05, torch.randn(h, generator=g) * 0.06
    s = api.gate_score(x.cuda(), w1.cuda(), b1.cuda(), w2.cuda(), 0.0).cpu()
    assert torch.equal(s[src].view(torch.int32), s[dst].view(torch.int32))


# ---------------------------------------------------------------- select ----

def _select_both(api, orc, scores, lens, db, de, kd):
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    want_idx, want_cu = orc.select_topk(scores, cu, db, de, kd)
    dev = lambda a: torch.tensor(np.asarray(a, np.int32), device="cuda")
    st = torch.tensor(scores, device="cuda")
    idx, ks, cuk, pos = api.select_topk(st, dev(cu), dev(db), dev(de), dev(kd), len(want_idx),
                                        max(lens) if lens else 0, want_pos=True)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    np.testing.assert_array_equal(cuk.cpu().numpy(), want_cu)
    np.testing.assert_array_equal(ks.cpu().numpy().view(np.int32),
                                  scores[want_idx].view(np.int32))
    # a kept row's position is its offset from its sequence's first row
    seq = np.searchsorted(cu, want_idx, side="right") - 1
    np.testing.assert_array_equal(pos.cpu().numpy(), want_idx - cu[seq])
    return want_idx


# a sequence's cluster has one CTA per 4096 tokens: one CTA, then 4 CTAs with
# every slice full, then 5 CTAs with a one-token last slice
@pytest.mark.parametrize("n", [5000, 16384, 16385])
def test_select_ties_and_specials(api, orc, n):
    rng = np.random.default_rng(0)
    s = (rng.integers(-40, 40, n) / 4).astype(np.float32)          # heavy exact ties
    s[rng.integers(0, n, 50)] = np.nan
    s[rng.integers(0, n, 20)] = np.inf
    s[rng.integers(0, n, 20)] = -np.inf
    s[rng.integers(0, n, 30)] = -0.0
    s[rng.integers(0, n, 30)] = 0.0
    nd = n - 256
    for k in [0, 1, 7, nd // 5, nd // 2, nd - 44, nd - 1, nd, 10 ** 6]:
        _select_both(api, orc, s, [n], [0], [nd], [k])


def test_select_ragged_up_to_16384(api, orc):
    # a batch whose longest sequence fills a 4-CTA cluster exactly
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 16384, 11).tolist() + [16384]
    s = rng.standard_normal(sum(lens)).astype(np.float32)
    db = [int(rng.integers(0, 50)) for _ in lens]
    db = [min(d, l) for d, l in zip(db, lens)]
    de = [max(d, l - int(rng.integers(0, 300))) for d, l in zip(db, lens)]
    kd = [int(rng.integers(0, e - d + 2)) for d, e in zip(db, de)]
    _select_both(api, orc, s, lens, db, de, kd)


def test_select_doc_in_middle_and_degenerate_spans(api, orc):
    rng = np.random.default_rng(1)
    lens = [3000, 1, 0, 700, 129, 4096]
    s = rng.standard_normal(sum(lens)).astype(np.float32)
    db = [100, 0, 0, 0, 0, 4096]
    de = [2500, 1, 0, 700, 129, 4096]
    kd = [300, 0, 5, 700, 64, 10]
    _select_both(api, orc, s, lens, db, de, kd)


def test_select_ragged_many_sequences(api, orc):
    rng = np.random.default_rng(2)
    lens = rng.integers(1, 3000, 40).tolist()
    s = rng.standard_normal(sum(lens)).astype(np.float32)
    qs = [int(min(l, rng.integers(0, 300))) for l in lens]
    db = [0] * len(lens)
    de = [l - q for l, q in zip(lens, qs)]
    kd = [int(rng.integers(-5, max(e, 1) + 5)) for e in de]
    _select_both(api, orc, s, lens, db, de, kd)


def test_select_max_seqlen(api, orc):
    n = 196608    # the documented maximum sequence length
    rng = np.random.default_rng(3)
    s = rng.standard_t(3.0, n).astype(np.float32)
    s[rng.integers(0, n, 2000)] = s[17]                             # ties at one value
    kth = np.sort(s[: n - 512])[::-1][15000]
    s[rng.integers(0, n - 512, 40)] = kth                           # ties at the threshold
    _select_both(api, orc, s, [n], [0], [n - 512], [15000])


@pytest.mark.parametrize("n", [16384, 32768])
def test_select_threshold_ties_straddle(api, orc, n):
    # many copies of the K-th value on both sides of the cut
    rng = np.random.default_rng(4)
    s = rng.standard_normal(n).astype(np.float32)
    k = 3225
    kth = np.sort(s[: n - 512])[::-1][k - 1]
    pos = rng.choice(n - 512, 600, replace=False)
    s[pos] = kth
    idx = _select_both(api, orc, s, [n], [0], [n - 512], [k])
    kept_ties = np.intersect1d(idx, pos)
    dropped_ties = np.setdiff1d(pos, idx)
    assert len(kept_ties) > 0 and len(dropped_ties) > 0
    assert kept_ties.max() < dropped_ties.min()


# --------------------------------------------------------------- compact ----

def test_compact_bit_exact(api):
    g = _gen(5)
    n = 3001
    x = torch.randn(n, 2048, generator=g).to(torch.bfloat16).cuda()
    kv = torch.randn(n, 8, 128, generator=g).to(torch.bfloat16).cuda()
    tiny = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, 4), generator=g, dtype=torch.int32).cuda()
    odd = torch.randn(n, 12, generator=g).cuda()                    # 48-byte rows
    idx = torch.sort(torch.randperm(n, generator=g)[:777]).values.to(torch.int32).cuda()
    outs = api.compact_rows([x, kv, tiny, odd], idx)
    for src, o in zip([x, kv, tiny, odd], outs):
        assert torch.equal(o, src.index_select(0, idx.long()))


def test_compact_empty_and_errors(api):
    x = torch.zeros(10, 8, device="cuda")
    idx = torch.zeros(0, dtype=torch.int32, device="cuda")
    (o,) = api.compact_rows([x], idx)
    assert o.shape == (0, 8)
    from learned_token_pruning_gemm_b200._lib import TokenGateError
    with pytest.raises(TokenGateError, match="MISALIGNED"):
        api.compact_rows([torch.zeros(10, 3, device="cuda")],
                         torch.zeros(2, dtype=torch.int32, device="cuda"))


# ------------------------------------------------------------- attention ----

def _attn_case(seed, lens, hq, hkv, dh, dtype, s_scale=1.0, zero_gain=False, v_dist="normal"):
    g = _gen(seed)
    K = sum(lens)
    q = torch.randn(K, hq, dh, generator=g).to(dtype)
    k = torch.randn(K, hkv, dh, generator=g).to(dtype)
    if v_dist == "uniform":     # unit variance, |v| <= 1.74
        v = ((torch.rand(K, hkv, dh, generator=g) * 2 - 1) * math.sqrt(3)).to(dtype)
    else:                       # N(0,1), the configurations' distribution
        v = torch.randn(K, hkv, dh, generator=g).to(dtype)
    s = torch.randn(K, generator=g) * s_scale
    gain = torch.zeros(hq) if zero_gain else torch.rand(hq, generator=g)
    tau = 0.8 + 0.7 * torch.rand(hq, generator=g)
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    return q, k, v, s, gain, tau, cu


def _run_attn(api, q, k, v, s, gain, tau, cu):
    cu_d = torch.tensor(cu, device="cuda")
    max_kept = int(np.diff(cu).max())
    return api.gated_attention(q.cuda(), k.cuda(), v.cuda(), s.cuda(), gain.cuda(), tau.cuda(),
                               cu_d, max_kept)


@pytest.mark.parametrize("v_dist", ["normal", "uniform"])
@pytest.mark.parametrize("lens", [[128], [300], [1000], [1868], [513, 1, 129, 700],
                                  [4000, 260]])
def test_attention_bf16_vs_oracle(api, orc, lens, v_dist):
    q, k, v, s, gain, tau, cu = _attn_case(sum(lens), lens, 16, 8, 128, torch.bfloat16,
                                           v_dist=v_dist)
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    rows = sample_rows(cu, 96) if sum(lens) > 1000 else None
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu, rows=rows)
    max_abs, rl2 = assert_attn_close(out, ref, torch.bfloat16, rows,
                                     what=f"lens={lens} v={v_dist}")
    print(f"lens={lens} v={v_dist}: max|O| {np.abs(ref[rows] if rows is not None else ref).max():.3f}"
          f" max_abs {max_abs:.2e} rel_l2 {rl2:.2e}")


@pytest.mark.parametrize("hq,hkv,lens", [
    (16, 8, [700, 1, 300]),      # groups of two: two heads per CTA
    (16, 2, [513]),              # groups of eight: four head pairs per KV head
    (8, 8, [700, 300]),          # groups of one: one head per CTA
    (12, 4, [257, 640]),         # groups of three: one head per CTA
])
def test_attention_bf16_head_groups(api, orc, hq, hkv, lens):
    q, k, v, s, gain, tau, cu = _attn_case(hq * 100 + hkv, lens, hq, hkv, 128, torch.bfloat16)
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu)
    assert_attn_close(out, ref, torch.bfloat16, what=f"heads {hq}/{hkv} lens={lens}")


def test_attention_bf16_schedule_fallback_matches_walk(api, orc):
    # Up to 256 sequences the CTAs walk lists of query tiles; beyond, one CTA takes
    # one tile. 300 ragged sequences (some of one row) take the second path; their
    # first 200 alone take the first. A row's arithmetic does not depend on which
    # CTA runs it, so the shared rows must agree bit for bit, and the oracle checks
    # a sample of the 300-sequence run. V is drawn uniform (|v| <= 1.74): rows of a
    # few keys carry single values of v, and with N(0,1) values near 4 the bf16
    # rounding of the output alone reaches 2^-7.
    lens = [int(x) for x in np.random.default_rng(7).integers(1, 400, 300)]
    lens[5] = 1
    q, k, v, s, gain, tau, cu = _attn_case(300, lens, 16, 8, 128, torch.bfloat16,
                                           v_dist="uniform")
    out_all = _run_attn(api, q, k, v, s, gain, tau, cu)
    n200 = int(cu[200])
    out_200 = _run_attn(api, q[:n200], k[:n200], v[:n200], s[:n200], gain, tau, cu[:201])
    assert torch.equal(out_all[:n200], out_200)
    rows = sample_rows(cu, 96)
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu, rows=rows)
    assert_attn_close(out_all, ref, torch.bfloat16, rows, what="300 sequences")


def test_attention_bf16_16k_shape_all_rows_normal_v(api, orc):
    # the 16k layer's attention shape (K = 1868, 16/8 heads) with V ~ N(0,1), every row
    q, k, v, s, gain, tau, cu = _attn_case(1868, [1868], 16, 8, 128, torch.bfloat16)
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu)
    max_abs, rl2 = assert_attn_close(out, ref, torch.bfloat16, what="16k shape, V~N(0,1)")
    print(f"16k shape V~N(0,1): max|O| {np.abs(ref).max():.3f} max_abs {max_abs:.2e} "
          f"rel_l2 {rl2:.2e}")


def test_attention_bf16_plain_causal_when_gain0_tau1(api, orc):
    q, k, v, s, gain, tau, cu = _attn_case(9, [640], 4, 2, 128, torch.bfloat16, zero_gain=True)
    tau[:] = 1.0
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().transpose(0, 1), k.double().repeat_interleave(2, 1).transpose(0, 1),
        v.double().repeat_interleave(2, 1).transpose(0, 1), is_causal=True).transpose(0, 1)
    assert_attn_close(out, ref.numpy(), torch.bfloat16, what="gain0 tau1")


def test_attention_bf16_large_bias_rescale(api, orc):
    # strongly varying scores force running-max moves (O rescaled in TMEM)
    q, k, v, s, gain, tau, cu = _attn_case(10, [1500], 8, 2, 128, torch.bfloat16, s_scale=12.0,
                                           v_dist="uniform")
    s[::97] += 40.0
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    rows = sample_rows(cu, 128)
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu, rows=rows)
    assert_attn_close(out, ref, torch.bfloat16, rows, what="rescale")


def test_attention_bf16_v_ones(api):
    q, k, v, s, gain, tau, cu = _attn_case(11, [700, 300], 16, 8, 128, torch.bfloat16)
    v = torch.ones_like(v)
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    assert torch.all(out.float().cpu() == 1.0)


@pytest.mark.parametrize("lens,hq,hkv,dh", [([512], 4, 2, 64), ([37, 1, 90], 4, 1, 32),
                                            ([128], 2, 2, 256)])
def test_attention_f32_vs_oracle(api, orc, lens, hq, hkv, dh):
    q, k, v, s, gain, tau, cu = _attn_case(12, lens, hq, hkv, dh, torch.float32)
    out = _run_attn(api, q, k, v, s, gain, tau, cu)
    ref = orc.gated_attention(q, k, v, s, gain, tau, cu)
    assert_attn_close(out, ref, torch.float32, what="f32")


# ------------------------------------------------------- failure detection ----

def test_bounded_wait_times_out_and_reports(api):
    api.device_status(reset=True)
    api.selftest_bounded_wait(2_000_000)          # 2 ms wait on a flag nothing sets
    assert api.device_status(reset=True) == 6     # TG_ERR_TIMEOUT
    # the context is still usable afterwards
    x = torch.arange(64, dtype=torch.float32, device="cuda").reshape(16, 4)
    idx = torch.tensor([3, 5], dtype=torch.int32, device="cuda")
    (o,) = api.compact_rows([x], idx)
    assert torch.equal(o, x[[3, 5]])


def test_device_check_on_inconsistent_total(api, orc):
    # total_kept that disagrees with the spans: no out-of-range write, status set
    s = torch.randn(1000, device="cuda")
    d = lambda a: torch.tensor(a, dtype=torch.int32, device="cuda")
    idx = torch.full((500,), -7, dtype=torch.int32, device="cuda")
    _, _, cuk = api.select_topk(s, d([0, 1000]), d([0]), d([900]), d([450]), 500, 1000,
                                kept_idx=idx)
    assert api.device_status(reset=True) == 7     # TG_ERR_DEVICE_CHECK
    # the sequence's rows are marked -1 (none left unwritten), cu_kept stays in range
    assert int((idx == -1).sum()) == 500
    assert cuk.cpu().tolist() == [0, 500]
