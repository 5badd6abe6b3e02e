"""Pins of the oracle's q/k/v projection with rotary embedding (oracle_qkv_rope).

The projection is checked against numpy's fp64 matmul (a library witness); the
rotation against facts that any mistake in it breaks: v is never rotated, the
rotate-half pairing (a lone component i moves only into i and i + dh/2), the
closed form at the first frequency (theta_0 = 1 for every base, so the pair is
(cos p, sin p): this pins the sign), the geometric ratio base^(-2/dh) between
neighbouring frequencies, norm preservation, and the relative-position property
q_m . k_n = q_{m+t} . k_{n+t} that makes RoPE what it is."""
import math

import numpy as np
import torch

import oracle


def _case(seed, n, d, hq, hkv, dh):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    w = (torch.randn((hq + 2 * hkv) * dh, d, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    return x, w


def _proj(x, w, hq, hkv, dh):
    y = x.double().numpy() @ w.double().numpy().T
    n = y.shape[0]
    q = y[:, :hq * dh].reshape(n, hq, dh)
    k = y[:, hq * dh:(hq + hkv) * dh].reshape(n, hkv, dh)
    v = y[:, (hq + hkv) * dh:].reshape(n, hkv, dh)
    return q, k, v


def test_position_zero_is_the_plain_projection():
    x, w = _case(1, 7, 64, 4, 2, 16)
    q, k, v = oracle.qkv_rope(x, w, 4, 2, 16, 1e6, np.zeros(7, np.int32))
    pq, pk, pv = _proj(x, w, 4, 2, 16)
    for a, b in ((q, pq), (k, pk), (v, pv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_values_are_not_rotated_and_norms_are_kept():
    x, w = _case(2, 9, 64, 4, 2, 16)
    pos = np.array([0, 1, 5, 77, 1000, 4095, 65535, 131071, 3], np.int32)
    q, k, v = oracle.qkv_rope(x, w, 4, 2, 16, 1e6, pos)
    pq, pk, pv = _proj(x, w, 4, 2, 16)
    np.testing.assert_allclose(v, pv, rtol=0, atol=1e-12)
    # a rotation of each (i, i + dh/2) pair keeps every pair's length
    for a, b in ((q, pq), (k, pk)):
        la = a[..., :8] ** 2 + a[..., 8:] ** 2
        lb = b[..., :8] ** 2 + b[..., 8:] ** 2
        np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-12)


def _unit_response(i0, p, dh=16, base=1e4):
    # x = e_0 and W with a single 1 at (head 0, component i0): y = e_i0 in q head 0
    d = 16
    x = torch.zeros(1, d)
    x[0, 0] = 1.0
    w = torch.zeros(3 * dh, d)
    w[i0, 0] = 1.0
    q, _, _ = oracle.qkv_rope(x.to(torch.bfloat16), w.to(torch.bfloat16), 1, 1, dh, base,
                              np.array([p], np.int32))
    return q[0, 0]


def test_rotate_half_pairing_and_first_frequency():
    dh = 16
    for i0 in (0, 3, 7):
        for p in (1, 2, 100):
            o = _unit_response(i0, p, dh)
            support = set(np.nonzero(np.abs(o) > 1e-15)[0].tolist())
            assert support <= {i0, i0 + dh // 2}, (i0, p, support)
    # theta_0 = base^0 = 1 for any base: the pair is (cos p, sin p) exactly
    for p in (1, 2, 3, 100, 131071):
        o = _unit_response(0, p, dh)
        assert abs(o[0] - math.cos(p)) < 1e-12 and abs(o[dh // 2] - math.sin(p)) < 1e-12


def test_frequencies_form_a_geometric_sequence():
    dh, base = 16, 1e4
    # at position 1 the angles are small: atan2 reads theta_i back without wrapping
    th = [math.atan2(_unit_response(i, 1, dh, base)[i + dh // 2], _unit_response(i, 1, dh, base)[i])
          for i in range(dh // 2)]
    ratios = np.array(th[1:]) / np.array(th[:-1])
    np.testing.assert_allclose(ratios, base ** (-2.0 / dh), rtol=1e-9)


def test_relative_position_property():
    hq, hkv, dh = 2, 2, 16
    x, w = _case(3, 2, 64, hq, hkv, dh)
    for m, n, t in ((5, 3, 1000), (0, 17, 65536), (100, 100, 31)):
        q1, k1, _ = oracle.qkv_rope(x, w, hq, hkv, dh, 1e6, np.array([m, n], np.int32))
        q2, k2, _ = oracle.qkv_rope(x, w, hq, hkv, dh, 1e6, np.array([m + t, n + t], np.int32))
        for h in range(hq):
            a = float(np.dot(q1[0, h], k1[1, h]))
            b = float(np.dot(q2[0, h], k2[1, h]))
            assert abs(a - b) <= 1e-9 * (1 + abs(a)), (m, n, t, h, a, b)


def test_selected_rows_only():
    x, w = _case(4, 6, 32, 2, 1, 8)
    pos = np.arange(6, dtype=np.int32) * 11
    q_all, k_all, v_all = oracle.qkv_rope(x, w, 2, 1, 8, 1e6, pos)
    q, k, v = oracle.qkv_rope(x, w, 2, 1, 8, 1e6, pos, rows=[1, 4])
    for a, b in ((q, q_all), (k, k_all), (v, v_all)):
        np.testing.assert_array_equal(a[[1, 4]], b[[1, 4]])
        assert np.isnan(a[[0, 2, 3, 5]]).all()
