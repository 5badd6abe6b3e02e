"""GPU parity of the gated attention's backward (tg_gated_attention_bwd) against the
fp64 oracle, through the C ABI (MarkTechPost page on TokenGate, section "Qu'est-ce
que l'attention gérée par des tokens ?": the score bias is how gradients reach the
scorer; gain and temperature are learned).

Tolerances, from the arithmetic (no bar is stated for gradients):
  fp32 path: every step is fp32 with the oracle's formulas; each gradient is a sum
    of up to K products, so the bar is relative to the tensor's largest entry:
    max |gpu - oracle| <= 1e-4 * max(1, max |oracle|).
  bf16 path: P and dS are rounded to bf16 before their contractions (2^-9 relative
    each) and dq/dk/dv are stored in bf16 (2^-9 again), with fp32 accumulation, so
    each tensor is held to relative L2 <= 1e-2 and max-abs <= 3e-2 of its largest
    entry; ds, dgain and dtau are summed in fp32 from unrounded dZ and held to
    relative L2 <= 1e-2 (dgain, dtau over the heads as one vector)."""
import numpy as np
import pytest
import torch

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


def _case(seed, lens, hq, hkv, dh, dtype):
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


def _run(api, q, k, v, do, s, gain, tau, cu):
    c = lambda t: t.cuda()
    K, hq, _ = q.shape
    cu_d = torch.tensor(cu, device="cuda")
    mk = int(np.diff(cu).max())
    lse = torch.empty(hq, K, device="cuda")
    out = api.gated_attention(c(q), c(k), c(v), c(s), c(gain), c(tau), cu_d, mk, lse=lse)
    grads = api.gated_attention_bwd(c(q), c(k), c(v), out, c(do), lse, c(s), c(gain), c(tau),
                                    cu_d, mk)
    torch.cuda.synchronize()
    return [t.float().cpu().double().numpy() for t in grads]


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


NAMES = ["dq", "dk", "dv", "ds", "dgain", "dtau"]


@pytest.mark.parametrize("lens,hq,hkv,dh", [([128], 4, 2, 64), ([37, 1, 90], 4, 1, 32),
                                            ([200, 56], 6, 3, 128)])
def test_backward_f32_vs_oracle(api, orc, lens, hq, hkv, dh):
    args = _case(sum(lens) + hq, lens, hq, hkv, dh, torch.float32)
    got = _run(api, *args)
    want = orc.gated_attention_bwd(*args)
    for name, g, w in zip(NAMES, got, want):
        err = np.abs(g - w).max()
        assert err <= 1e-4 * max(1.0, np.abs(w).max()), f"{name}: {err:.3e}"


def test_backward_f32_tiny_config(api, orc):
    # the tiny configuration's attention shape: K = 128 kept, 4/2 heads, dh = 64
    from learned_token_pruning_gemm_b200 import synth
    wl = synth.tiny_f32()
    g = torch.Generator().manual_seed(77)
    do = torch.randn(wl.q.shape, generator=g)
    s = torch.randn(wl.total_kept, generator=g)
    cu = np.array([0, wl.total_kept], np.int32)
    args = (wl.q, wl.k, wl.v, do, s, wl.gain, wl.tau, cu)
    got = _run(api, *args)
    want = orc.gated_attention_bwd(*args)
    for name, gg, w in zip(NAMES, got, want):
        err = np.abs(gg - w).max()
        assert err <= 1e-4 * max(1.0, np.abs(w).max()), f"{name}: {err:.3e}"


# up to 128 (key tile, KV head, sequence) units each unit's items are split between
# two CTAs whose fp32 partials are summed afterwards; the last case has 240 units,
# which run whole
@pytest.mark.parametrize("lens,hq,hkv", [([128], 4, 2), ([300], 4, 2), ([513, 1, 129], 4, 2),
                                         ([260], 8, 2), ([250], 3, 3), ([600] * 12, 8, 4)])
def test_backward_bf16_vs_oracle(api, orc, lens, hq, hkv):
    args = _case(sum(lens) * 7 + hq, lens, hq, hkv, 128, torch.bfloat16)
    got = _run(api, *args)
    want = orc.gated_attention_bwd(*args)
    for name, g, w in zip(NAMES, got, want):
        rl2 = _rel_l2(g, w)
        assert rl2 <= 1e-2, f"{name}: rel_l2 {rl2:.3e}"
        if name in ("dq", "dk", "dv"):
            err = np.abs(g - w).max()
            assert err <= 3e-2 * np.abs(w).max(), f"{name}: max_abs {err:.3e} of {np.abs(w).max():.3e}"
        print(f"lens={lens} {name}: rel_l2 {rl2:.2e}")


def test_backward_bf16_16k_shape_properties(api):
    # the 16k layer's attention shape (K = 1868, 16/8 heads): exact properties at
    # full size. A constant added to every score changes nothing, so the score
    # gradients sum to zero; with all values equal, only dv is non-zero.
    args = list(_case(5, [1868], 16, 8, 128, torch.bfloat16))
    dq, dk, dv, ds, dg, dt = _run(api, *args)
    assert abs(ds.sum()) <= 1e-3 * np.abs(ds).sum()
    args[2] = torch.full_like(args[2], 0.5)
    dq, dk, dv, ds, dg, dt = _run(api, *args)
    for name, a in zip(["dq", "dk", "ds", "dgain", "dtau"], (dq, dk, ds, dg, dt)):
        assert np.abs(a).max() <= 2e-3, name
    do = args[3].double().numpy()
    for kvh in range(8):
        want = do[:, [2 * kvh, 2 * kvh + 1]].sum(axis=(0, 1))
        np.testing.assert_allclose(dv[:, kvh].sum(0), want, rtol=2e-2, atol=0.5)


def test_backward_bf16_128k_shape_properties(api):
    # the 128k layer's attention shape (K = 10721, 16/8 heads; 672 units, run whole):
    # the score gradients sum to zero, and with all values equal only dv is non-zero
    args = list(_case(6, [10721], 16, 8, 128, torch.bfloat16))
    dq, dk, dv, ds, dg, dt = _run(api, *args)
    assert abs(ds.sum()) <= 1e-3 * np.abs(ds).sum()
    for a in (dq, dk, dv):
        assert np.isfinite(a).all()
    args[2] = torch.full_like(args[2], 0.5)
    dq, dk, dv, ds, dg, dt = _run(api, *args)
    for name, a in zip(["dq", "dk", "ds", "dgain", "dtau"], (dq, dk, ds, dg, dt)):
        assert np.abs(a).max() <= 2e-3, name
    do = args[3].double().numpy()
    for kvh in range(8):
        want = do[:, [2 * kvh, 2 * kvh + 1]].sum(axis=(0, 1))
        np.testing.assert_allclose(dv[:, kvh].sum(0), want, rtol=2e-2, atol=1.0)
