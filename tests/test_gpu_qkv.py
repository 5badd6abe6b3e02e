"""GPU parity of tg_qkv_rope (the kept rows' q/k/v projections with the rotary
embedding at their original positions) against the fp64 oracle.

Tolerance, from the arithmetic: the outputs are bf16, rounded to nearest from
fp32, so each carries up to 2^-9 of its own magnitude; the fp32 accumulation over
d and the reduced-angle sine/cosine (absolute error ~2^-21) add far less. The bar
is |gpu - oracle| <= 2^-8 |oracle| + 1e-4."""
import math

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


def _check(got, want, rows, what):
    g = got.float().cpu().numpy().astype(np.float64)[rows]
    w = want[rows]
    err = np.abs(g - w) - (2.0 ** -8 * np.abs(w) + 1e-4)
    assert err.max() <= 0, f"{what}: worst excess {err.max():.3e}"


def _case(seed, n, d, hq, hkv, max_pos):
    g = torch.Generator().manual_seed(seed)
    xc = torch.randn(n, d, generator=g).to(torch.bfloat16)
    w = (torch.randn((hq + 2 * hkv) * 128, d, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    pos = torch.randint(0, max_pos, (n,), generator=g, dtype=torch.int32)
    return xc, w, pos


@pytest.mark.parametrize("n,d,hq,hkv,max_pos,sample", [
    (300, 256, 4, 2, 1_000_000, None),        # 3 row tiles (ragged), 4 column tiles
    (129, 128, 2, 1, 16, None),               # one row past a tile
    (1868, 2048, 16, 8, 16384, 96),           # the Qwen3-shaped layer, sampled rows
])
def test_qkv_rope_vs_oracle(api, orc, n, d, hq, hkv, max_pos, sample):
    xc, w, pos = _case(n + d, n, d, hq, hkv, max_pos)
    q, k, v = api.qkv_rope(xc.cuda(), w.cuda(), hq, hkv, pos.cuda(), rope_base=1e6)
    assert api.device_status(reset=True) == 0
    if sample is None:
        rows = np.arange(n)
    else:
        rng = np.random.default_rng(0)
        rows = np.unique(np.r_[0, 127, 128, n - 1, rng.integers(0, n, sample)])
    want = orc.qkv_rope(xc, w, hq, hkv, 128, 1e6, pos.numpy(), rows=rows)
    for got, ref, nm in zip((q, k, v), want, "qkv"):
        _check(got, ref, rows, f"{nm} n={n}")


def test_kept_rows_chain(api, orc):
    # compaction of the 16k layer's residual rows, then their projections at the
    # kept tokens' original positions: the KV cache written for kept tokens only
    from learned_token_pruning_gemm_b200 import pipeline, synth
    wl = synth.qwen16k()
    gp = pipeline.GatedPrefill(wl)
    gp.step()
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(7)
    w = (torch.randn(32 * 128, wl.d, generator=g) / math.sqrt(wl.d)).to(torch.bfloat16)
    q, k, v = api.qkv_rope(gp.xc, w.cuda(), 16, 8, gp.kept_idx, rope_base=1e6)
    assert api.device_status(reset=True) == 0
    rng = np.random.default_rng(1)
    K = gp.xc.shape[0]
    rows = np.unique(np.r_[0, K - 1, rng.integers(0, K, 48)])
    want = orc.qkv_rope(gp.xc.cpu(), w, 16, 8, 128, 1e6, gp.kept_idx.cpu().numpy(), rows=rows)
    for got, ref, nm in zip((q, k, v), want, "qkv"):
        _check(got, ref, rows, f"chain {nm}")
