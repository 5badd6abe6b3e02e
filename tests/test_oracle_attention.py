"""Pins for the oracle's token-gated causal GQA attention (MarkTechPost page, section
"Qu'est-ce que l'attention gérée par des tokens ?": each kept token's score becomes
a bias on the attention logits; a learnable per-head gain and a learnable per-head
temperature correct for each query seeing fewer keys).

Reading pinned: z_ij = q_i.k_j / (sqrt(dh) tau_h) + g_h s_j over kept keys j <= i,
O_i = sum_j softmax_j(z_ij) v_j, query head h reads KV head h / (Hq/Hkv)."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_worked_cases(orc):
    cases = json.load(open(os.path.join(GOLDEN, "attention_cases.json")))["cases"]
    for c in cases:
        q = torch.tensor(c["q"], dtype=torch.float32)
        k = torch.tensor(c["k"], dtype=torch.float32)
        v = torch.tensor(c["v"], dtype=torch.float32)
        out = orc.gated_attention(q, k, v, c["s"], c["gain"], c["tau"], [0, q.shape[0]])
        np.testing.assert_allclose(out, np.array(c["expect"], np.float64), rtol=0,
                                   atol=c.get("atol", 1e-14),
                                   err_msg=c["what"])


def _rand_case(seed, lens, hq, hkv, dh, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    K = sum(lens)
    q = torch.randn(K, hq, dh, generator=g).to(dtype)
    k = torch.randn(K, hkv, dh, generator=g).to(dtype)
    v = torch.randn(K, hkv, dh, generator=g).to(dtype)
    s = torch.randn(K, generator=g) * 2
    gain = torch.rand(hq, generator=g)
    tau = 0.8 + 0.7 * torch.rand(hq, generator=g)
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    return q, k, v, s, gain, tau, cu


def _sdpa_witness(q, k, v, s, gain, tau, cu):
    """torch fp64 SDPA per sequence: a float mask g_h s_j plus -inf above the
    diagonal, and a per-head softmax scale 1/(sqrt(dh) tau_h)."""
    K, hq, dh = q.shape
    hkv = k.shape[1]
    out = torch.empty(K, hq, dh, dtype=torch.float64)
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        n = e - a
        causal = torch.ones(n, n, dtype=torch.bool).tril()
        for h in range(hq):
            kv = h // (hq // hkv)
            mask = torch.where(causal, float(gain[h]) * s[a:e].double()[None, :],
                               torch.tensor(-math.inf, dtype=torch.float64))
            o = F.scaled_dot_product_attention(
                q[a:e, h].double()[None], k[a:e, kv].double()[None], v[a:e, kv].double()[None],
                attn_mask=mask[None], scale=1.0 / (math.sqrt(dh) * float(tau[h])))
            out[a:e, h] = o[0]
    return out.numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_vs_sdpa_witness_varlen_gqa(orc, dtype):
    q, k, v, s, gain, tau, cu = _rand_case(1, [37, 1, 90], 4, 2, 16, dtype)
    got = orc.gated_attention(q, k, v, s, gain, tau, cu)
    np.testing.assert_allclose(got, _sdpa_witness(q, k, v, s, gain, tau, cu), atol=1e-12, rtol=0)


def test_plain_causal_attention_when_gain0_tau1(orc):
    # g_h = 0 and tau_h = 1: ordinary causal softmax attention (torch SDPA is_causal)
    q, k, v, s, gain, tau, cu = _rand_case(2, [64], 2, 2, 32)
    gain[:] = 0.0
    tau[:] = 1.0
    got = orc.gated_attention(q, k, v, s, gain, tau, cu)
    ref = F.scaled_dot_product_attention(q.double().transpose(0, 1), k.double().transpose(0, 1),
                                         v.double().transpose(0, 1), is_causal=True)
    np.testing.assert_allclose(got, ref.transpose(0, 1).numpy(), atol=1e-12, rtol=0)


def test_constant_score_shift_invariance(orc):
    q, k, v, s, gain, tau, cu = _rand_case(3, [50, 20], 4, 1, 8)
    s = torch.round(s * 256) / 256          # on a grid, so s + 3.75 is exact in fp32
    a = orc.gated_attention(q, k, v, s, gain, tau, cu)
    b = orc.gated_attention(q, k, v, s + 3.75, gain, tau, cu)
    np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def test_v_ones_gives_ones(orc):
    q, k, v, s, gain, tau, cu = _rand_case(4, [33, 7], 4, 2, 8)
    v = torch.ones_like(v)
    got = orc.gated_attention(q, k, v, s, gain, tau, cu)
    np.testing.assert_allclose(got, 1.0, atol=1e-14, rtol=0)


def test_sequences_do_not_leak(orc):
    q, k, v, s, gain, tau, cu = _rand_case(5, [20, 30], 2, 1, 8)
    whole = orc.gated_attention(q, k, v, s, gain, tau, cu)
    second = orc.gated_attention(q[20:], k[20:], v[20:], s[20:], gain, tau, [0, 30])
    np.testing.assert_allclose(whole[20:], second, atol=0, rtol=0)


def test_row_subset_matches_full(orc):
    q, k, v, s, gain, tau, cu = _rand_case(6, [40, 25], 4, 2, 8)
    full = orc.gated_attention(q, k, v, s, gain, tau, cu)
    rows = [0, 5, 39, 40, 64]
    sub = orc.gated_attention(q, k, v, s, gain, tau, cu, rows=rows)
    np.testing.assert_array_equal(sub[rows], full[rows])
    others = np.setdiff1d(np.arange(65), rows)
    assert np.isnan(sub[others]).all()


def test_gather_matches_numpy_indexing(orc):
    rng = np.random.default_rng(0)
    src = rng.standard_normal((100, 3, 8)).astype(np.float32)
    idx = np.sort(rng.choice(100, 37, replace=False)).astype(np.int32)
    np.testing.assert_array_equal(orc.gather_rows(src, idx), src[idx])
