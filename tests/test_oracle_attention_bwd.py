"""Pins for the oracle's backward of the token-gated attention (MarkTechPost page,
section "Qu'est-ce que l'attention gérée par des tokens ?": the key score enters
the logits as a bias so that gradients reach the scorer; gain and temperature are
learned per head).

Three independent witnesses: torch fp64 autograd through SDPA with the bias as a
float mask and the temperature folded into q; central finite differences of the
oracle's own forward; and exact consequences of the formula (a constant added to
every score changes nothing, so the score gradients of a sequence sum to zero; with
all values equal the output is that value, so only dv is non-zero)."""
import math

import numpy as np
import torch
import torch.nn.functional as F


def _case(seed, lens, hq, hkv, dh, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    K = sum(lens)
    q = torch.randn(K, hq, dh, generator=g).to(dtype)
    k = torch.randn(K, hkv, dh, generator=g).to(dtype)
    v = torch.randn(K, hkv, dh, generator=g).to(dtype)
    do = torch.randn(K, hq, dh, generator=g).to(dtype)
    s = torch.randn(K, generator=g) * 2
    gain = torch.rand(hq, generator=g)
    tau = 0.8 + 0.7 * torch.rand(hq, generator=g)
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    return q, k, v, do, s, gain, tau, cu


def _autograd_witness(q, k, v, do, s, gain, tau, cu):
    """dL/d(q, k, v, s, gain, tau) for L = sum(O * dO), O from torch fp64 SDPA per
    sequence and head (causal float mask with gain * s; q scaled by 1/(sqrt(dh) tau))."""
    K, hq, dh = q.shape
    hkv = k.shape[1]
    qd, kd, vd = (t.double().clone().requires_grad_() for t in (q, k, v))
    sd, gd, td = (t.double().clone().requires_grad_() for t in (s, gain, tau))
    loss = 0.0
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        n = e - a
        causal = torch.ones(n, n, dtype=torch.bool).tril()
        for h in range(hq):
            kv = h // (hq // hkv)
            bias = gd[h] * sd[a:e][None, :].expand(n, n)
            mask = torch.where(causal, bias, torch.tensor(-math.inf, dtype=torch.float64))
            qs = qd[a:e, h] / (math.sqrt(dh) * td[h])
            o = F.scaled_dot_product_attention(qs[None], kd[a:e, kv][None], vd[a:e, kv][None],
                                               attn_mask=mask[None], scale=1.0)[0]
            loss = loss + (o * do[a:e, h].double()).sum()
    loss.backward()
    return [t.grad.numpy() for t in (qd, kd, vd, sd, gd, td)]


def test_matches_autograd_witness(orc):
    q, k, v, do, s, gain, tau, cu = _case(1, [9, 1, 14], 4, 2, 8)
    got = orc.gated_attention_bwd(q, k, v, do, s, gain, tau, cu)
    want = _autograd_witness(q, k, v, do, s, gain, tau, cu)
    for name, a, b in zip(["dq", "dk", "dv", "ds", "dgain", "dtau"], got, want):
        np.testing.assert_allclose(a, b, atol=1e-11, rtol=1e-9, err_msg=name)


def test_bf16_inputs_match_autograd_witness(orc):
    q, k, v, do, s, gain, tau, cu = _case(2, [17, 6], 4, 1, 16, torch.bfloat16)
    got = orc.gated_attention_bwd(q, k, v, do, s, gain, tau, cu)
    want = _autograd_witness(q, k, v, do, s, gain, tau, cu)
    for name, a, b in zip(["dq", "dk", "dv", "ds", "dgain", "dtau"], got, want):
        np.testing.assert_allclose(a, b, atol=1e-10, rtol=1e-9, err_msg=name)


def test_central_differences_of_the_forward(orc):
    # L = sum(O * W) with the oracle's own forward; each gradient entry against
    # (L(x + e) - L(x - e)) / 2e. The forward reads fp32 inputs, so the step must be
    # exact in fp32: e = 2^-12 on values of order one is (24-bit significands); the
    # fp64 forward then leaves only the O(e^2) truncation, about 1e-7 here.
    q, k, v, do, s, gain, tau, cu = _case(3, [5, 4], 2, 1, 3)
    W = do.double().numpy()

    def loss(q_, k_, v_, s_, g_, t_):
        return float((orc.gated_attention(q_, k_, v_, s_, g_, t_, cu) * W).sum())

    got = orc.gated_attention_bwd(q, k, v, do, s, gain, tau, cu)
    base = [q, k, v, s, gain, tau]
    eps = 2.0 ** -12
    for idx, g_ in enumerate(got):
        flat = base[idx].reshape(-1)
        for pos in range(flat.numel()):
            up = [t.clone() for t in base]
            dn = [t.clone() for t in base]
            up[idx].reshape(-1)[pos] += eps
            dn[idx].reshape(-1)[pos] -= eps
            fd = (loss(*up) - loss(*dn)) / (2 * eps)
            assert abs(fd - g_.reshape(-1)[pos]) <= 1e-5 + 1e-4 * abs(fd), (idx, pos, fd, g_.reshape(-1)[pos])


def test_score_gradients_of_a_sequence_sum_to_zero(orc):
    q, k, v, do, s, gain, tau, cu = _case(4, [30, 12, 1], 4, 2, 8)
    _, _, _, ds, _, _ = orc.gated_attention_bwd(q, k, v, do, s, gain, tau, cu)
    for b in range(3):
        seg = ds[cu[b]:cu[b + 1]]
        assert abs(seg.sum()) <= 1e-12 * max(1.0, np.abs(seg).sum())


def test_equal_values_leave_only_dv(orc):
    q, k, v, do, s, gain, tau, cu = _case(5, [20, 7], 4, 2, 8)
    v = torch.ones_like(v) * 0.75
    dq, dk, dv, ds, dg, dt = orc.gated_attention_bwd(q, k, v, do, s, gain, tau, cu)
    for a in (dq, dk, ds, dg, dt):
        assert np.abs(a).max() <= 1e-12
    # dv_j = sum over query heads of the group and rows i >= j of P_ij dO_i: with
    # the softmax rows summing to one, the dv rows of a sequence sum to sum_i dO_i
    # over the group's heads
    for b in range(2):
        a, e = cu[b], cu[b + 1]
        for kvh in range(2):
            heads = [kvh * 2, kvh * 2 + 1]
            want = do[a:e][:, heads].double().sum(dim=(0, 1)).numpy()
            np.testing.assert_allclose(dv[a:e, kvh].sum(0), want, atol=1e-12)
