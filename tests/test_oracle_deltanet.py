"""Pins for the oracle's gated delta rule over the kept tokens (MarkTechPost page,
section "Est-ce que cela fonctionne avec les modèles d'attention hybrides ?" and the
comparison table: the hybrid model's Gated DeltaNet layers are pruned as well).

Reading pinned: per sequence and head, S_0 = 0 and for the tokens in order
S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t.
The witnesses are closed forms of the rule, not the rule retyped: with orthonormal
keys and beta = 1 the delta correction vanishes and the rule is decayed linear
attention; a key written twice with beta = 1 is overwritten, so reading it returns
the last value; beta = 0 writes nothing; the map is linear in v; sequences do not
see one another."""
import numpy as np
import torch


def _basis_keys(T, dk, seed):
    """T orthonormal keys (a random rotation of the first T basis vectors)."""
    g = np.random.default_rng(seed)
    Qm, _ = np.linalg.qr(g.standard_normal((dk, dk)))
    return Qm[:, :T].T.copy()


def test_orthonormal_keys_give_decayed_linear_attention(orc):
    T, H, dk, dv = 12, 2, 16, 8
    g = np.random.default_rng(0)
    k = np.stack([_basis_keys(T, dk, 1 + h) for h in range(H)], 1)       # [T, H, dk]
    q = g.standard_normal((T, H, dk))
    v = g.standard_normal((T, H, dv))
    alpha = g.uniform(0.6, 1.0, (T, H))
    beta = np.ones((T, H))
    f = lambda a: torch.tensor(a, dtype=torch.float32)
    # the oracle reads fp32 inputs: compare against the closed form on those values
    q32, k32, v32 = f(q).double().numpy(), f(k).double().numpy(), f(v).double().numpy()
    a32 = f(alpha).double().numpy()
    got = orc.gated_delta_rule(f(q), f(k), f(v), f(alpha), f(beta), [0, T])
    for h in range(H):
        for t in range(T):
            want = np.zeros(dv)
            for s in range(t + 1):
                decay = np.prod(a32[s + 1:t + 1, h])
                want += decay * (k32[s, h] @ q32[t, h]) * v32[s, h]
            np.testing.assert_allclose(got[t, h], want, atol=2e-6)


def test_a_key_written_twice_is_overwritten(orc):
    dk, dv = 8, 4
    g = np.random.default_rng(2)
    key = g.standard_normal(dk)
    key /= np.linalg.norm(key)
    T = 5
    k = np.tile(key, (T, 1))[:, None, :]
    v = g.standard_normal((T, 1, dv))
    q = k.copy()                                     # read back the written slot
    ones = np.ones((T, 1))
    f = lambda a: torch.tensor(a, dtype=torch.float32)
    got = orc.gated_delta_rule(f(q), f(k), f(v), f(ones), f(ones), [0, T])
    kk = float(f(key).double() @ f(key).double())    # |k|^2 of the fp32 key (1 up to rounding)
    for t in range(T):
        np.testing.assert_allclose(got[t, 0], f(v[t, 0]).double().numpy() * kk, atol=1e-5)


def test_beta_zero_writes_nothing_and_linearity_in_v(orc):
    g = torch.Generator().manual_seed(3)
    T, H, dk, dv = 20, 3, 16, 16
    q = torch.randn(T, H, dk, generator=g)
    k = torch.nn.functional.normalize(torch.randn(T, H, dk, generator=g), dim=-1)
    v1 = torch.randn(T, H, dv, generator=g)
    v2 = torch.randn(T, H, dv, generator=g)
    a = torch.rand(T, H, generator=g) * 0.5 + 0.5
    b = torch.rand(T, H, generator=g)
    assert np.abs(orc.gated_delta_rule(q, k, v1, a, torch.zeros(T, H), [0, T])).max() == 0
    o1 = orc.gated_delta_rule(q, k, v1, a, b, [0, T])
    o2 = orc.gated_delta_rule(q, k, v2, a, b, [0, T])
    # 2 v1 - 3 v2 is rounded to fp32 on the way in: equal up to that rounding
    o3 = orc.gated_delta_rule(q, k, 2 * v1 - 3 * v2, a, b, [0, T])
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, atol=1e-5)


def test_sequences_are_independent(orc):
    g = torch.Generator().manual_seed(4)
    lens = [7, 1, 13]
    T, H, dk, dv = sum(lens), 2, 8, 8
    q = torch.randn(T, H, dk, generator=g)
    k = torch.nn.functional.normalize(torch.randn(T, H, dk, generator=g), dim=-1)
    v = torch.randn(T, H, dv, generator=g)
    a = torch.rand(T, H, generator=g)
    b = torch.rand(T, H, generator=g)
    cu = np.r_[0, np.cumsum(lens)]
    whole = orc.gated_delta_rule(q, k, v, a, b, cu)
    for i in range(3):
        s, e = cu[i], cu[i + 1]
        part = orc.gated_delta_rule(q[s:e], k[s:e], v[s:e], a[s:e], b[s:e], [0, e - s])
        np.testing.assert_array_equal(whole[s:e], part)
