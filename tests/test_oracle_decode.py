"""Pins for the oracle's decode over the compacted cache (MarkTechPost page, section
"Comment déployer TokenGate ?": generation runs on the cache that the pruned
prefill leaves, bounded by max_kept_prefill_tokens; section "Qu'est-ce que
l'attention gérée par des tokens ?": each kept token's score is a logit bias with
a per-head gain, and a per-head temperature scales the logits).

Reading pinned: one new query row per sequence attends over its cache rows
j < cache_len[b] (its own row included, since the new token is appended first):
z_j = q.k_j / (sqrt(dh) tau_h) + g_h s_j, O = sum_j softmax_j(z) v_j; cache layout
[B, cap, Hkv, dh], query head h reads KV head h / (Hq/Hkv)."""
import math

import numpy as np
import torch
import torch.nn.functional as F


def _case(seed, B, cap, lens, hq, hkv, dh, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, hq, dh, generator=g).to(dtype)
    kc = torch.randn(B, cap, hkv, dh, generator=g).to(dtype)
    vc = torch.randn(B, cap, hkv, dh, generator=g).to(dtype)
    sc = torch.randn(B, cap, generator=g) * 2
    gain = torch.rand(hq, generator=g)
    tau = 0.8 + 0.7 * torch.rand(hq, generator=g)
    return q, kc, vc, sc, np.asarray(lens, np.int32), gain, tau


def _sdpa_witness(q, kc, vc, sc, lens, gain, tau):
    """torch fp64 SDPA, one query per (sequence, head): float mask g_h s_j over the
    cached rows and a per-head scale 1/(sqrt(dh) tau_h)."""
    B, hq, dh = q.shape
    hkv = kc.shape[2]
    out = torch.zeros(B, hq, dh, dtype=torch.float64)
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        for h in range(hq):
            kv = h // (hq // hkv)
            mask = float(gain[h]) * sc[b, :n].double()[None, None, :]
            o = F.scaled_dot_product_attention(
                q[b, h].double()[None, None, :], kc[b, :n, kv].double()[None], vc[b, :n, kv].double()[None],
                attn_mask=mask[0], scale=1.0 / (math.sqrt(dh) * float(tau[h])))
            out[b, h] = o[0, 0]
    return out.numpy()


def test_matches_sdpa_witness(orc):
    q, kc, vc, sc, lens, gain, tau = _case(1, 3, 40, [40, 17, 1], 4, 2, 16)
    got = orc.gated_decode(q, kc, vc, sc, lens, gain, tau)
    np.testing.assert_allclose(got, _sdpa_witness(q, kc, vc, sc, lens, gain, tau), atol=1e-12)


def test_bf16_inputs_read_exactly(orc):
    q, kc, vc, sc, lens, gain, tau = _case(2, 2, 33, [33, 20], 8, 2, 32, torch.bfloat16)
    got = orc.gated_decode(q, kc, vc, sc, lens, gain, tau)
    np.testing.assert_allclose(got, _sdpa_witness(q, kc, vc, sc, lens, gain, tau), atol=1e-12)


def test_plain_attention_when_gain0_tau1(orc):
    q, kc, vc, sc, lens, gain, tau = _case(3, 2, 25, [25, 9], 2, 1, 8)
    gain[:] = 0.0
    tau[:] = 1.0
    got = orc.gated_decode(q, kc, vc, sc, lens, gain, tau)
    for b in range(2):
        n = int(lens[b])
        for h in range(2):
            want = F.scaled_dot_product_attention(q[b, h].double()[None, None], kc[b, :n, 0].double()[None],
                                                  vc[b, :n, 0].double()[None])[0, 0]
            np.testing.assert_allclose(got[b, h], want.numpy(), atol=1e-12)


def test_last_row_of_prefill(orc):
    # decoding token L-1 over rows 0..L-1 is the prefill's causal attention at row L-1
    q, kc, vc, sc, lens, gain, tau = _case(4, 1, 50, [50], 4, 2, 16)
    qs = torch.randn(50, 4, 16, generator=torch.Generator().manual_seed(9))
    qs[49] = q[0]
    pre = orc.gated_attention(qs, kc[0], vc[0], sc[0], gain, tau, [0, 50], rows=[49])
    got = orc.gated_decode(q, kc, vc, sc, lens, gain, tau)
    np.testing.assert_allclose(got[0], pre[49], atol=1e-13)


def test_invariants(orc):
    q, kc, vc, sc, lens, gain, tau = _case(5, 2, 30, [30, 12], 4, 4, 8)
    sc = torch.round(sc * 1024) / 1024          # so that adding 3.5 is exact in fp32
    base = orc.gated_decode(q, kc, vc, sc, lens, gain, tau)
    # a constant added to every score shifts every logit of a row equally
    np.testing.assert_allclose(orc.gated_decode(q, kc, vc, sc + 3.5, lens, gain, tau), base,
                               atol=1e-12)
    # V = 1 gives 1; a single cached row gives that row's v; an empty cache gives 0
    ones = orc.gated_decode(q, kc, torch.ones_like(vc), sc, lens, gain, tau)
    np.testing.assert_allclose(ones, 1.0, atol=1e-14)
    one = orc.gated_decode(q, kc, vc, sc, np.array([1, 0], np.int32), gain, tau)
    np.testing.assert_array_equal(one[0], vc[0, 0].double().numpy())
    assert (one[1] == 0).all()
    # rows at or past cache_len do not matter
    kc2, vc2 = kc.clone(), vc.clone()
    kc2[1, 12:] = 1e3
    vc2[1, 12:] = -1e3
    np.testing.assert_array_equal(orc.gated_decode(q, kc2, vc2, sc, lens, gain, tau), base)


def test_hand_worked_bias_case(orc):
    # dh = 1, q.k = 0 for both keys, s = (0, ln 3), g = 1: weights 1 : 3, so
    # O = (v0 + 3 v1) / 4 = (2 + 3 * 6) / 4 = 5 (up to the fp32 rounding of ln 3)
    q = torch.zeros(1, 1, 1)
    kc = torch.ones(1, 2, 1, 1)
    vc = torch.tensor([2.0, 6.0]).reshape(1, 2, 1, 1)
    sc = torch.tensor([[0.0, math.log(3.0)]])
    got = orc.gated_decode(q, kc, vc, sc, [2], torch.ones(1), torch.ones(1))
    assert abs(got[0, 0, 0] - 5.0) < 1e-6
