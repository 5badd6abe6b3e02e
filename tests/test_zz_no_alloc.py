"""tg_gated_decode_noalloc: decode over the compacted cache for callers that cannot
allocate device memory where they decode (a host program whose device memory
belongs to another runtime's pool, or a generation loop that must not call
cudaMalloc/cudaFree because they can synchronise the device). It keeps its
per-chunk partials in a fixed array inside the library instead of a caller
workspace.

Called here through the C ABI (ctypes on libtokengate.so), twice in a row with
different shapes, so the second call runs on whatever the first left in the
shared array; each result is checked against the workspace entry point
(tg_gated_decode) on the same inputs, within the bf16 bar the decode tests use.
This file is collected last, so a run that stops at its first failure has run
every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from helpers import ATTN_BF16_ATOL

pytestmark = pytest.mark.gpu

TG_ERR_WORKSPACE = 4


@pytest.fixture(scope="module")
def libs():
    from learned_token_pruning_gemm_b200 import _lib, api, build
    build.build()
    assert torch.cuda.is_available()
    api.device_status(reset=True)
    return _lib.load(), api


def _case(seed, B, cap, lens, hq, hkv, dh=128):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, hq, dh, generator=g).to(torch.bfloat16).cuda()
    kc = torch.randn(B, cap, hkv, dh, generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn(B, cap, hkv, dh, generator=g).to(torch.bfloat16).cuda()
    sc = (torch.randn(B, cap, generator=g) * 2).cuda()
    ln = torch.tensor(lens, dtype=torch.int32).cuda()
    gain = torch.rand(hq, generator=g).cuda()
    tau = (0.8 + 0.7 * torch.rand(hq, generator=g)).cuda()
    return q, kc, vc, sc, ln, gain, tau


def _noalloc(lib, q, kc, vc, sc, ln, gain, tau, max_len, out):
    B, hq, dh = q.shape
    cap, hkv = kc.shape[1], kc.shape[2]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.tg_gated_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sc.data_ptr(),
                                       ln.data_ptr(), B, cap, max_len, hq, hkv, dh,
                                       gain.data_ptr(), tau.data_ptr(), out.data_ptr(),
                                       ctypes.c_void_p(stream))


def test_noalloc_matches_workspace_decode_on_two_calls(libs):
    lib, api = libs
    cases = [(_case(31, 3, 700, [700, 129, 1], 16, 8), 700),
             (_case(32, 2, 300, [300, 190], 16, 2), 300)]
    for args, max_len in cases:
        q = args[0]
        out = torch.full_like(q, 9.0)
        assert _noalloc(lib, *args, max_len, out) == 0
        want = api.gated_decode(*args, max_len)
        torch.cuda.synchronize()
        assert api.device_status(reset=True) == 0
        diff = (out.float() - want.float()).abs().max().item()
        assert diff <= ATTN_BF16_ATOL, f"max |noalloc - workspace| = {diff:.3e}"
        assert torch.isfinite(out.float()).all()


def test_noalloc_rejects_calls_beyond_its_array(libs):
    lib, api = libs
    q, kc, vc, sc, ln, gain, tau = _case(33, 1, 64, [64], 16, 8)
    limit = lib.tg_gated_decode_workspace_size
    # a length whose partials need more than the fixed array: refused, nothing launched
    big = 1
    while limit(8, 16, 128, big) <= (8 << 20):
        big *= 2
    q8 = torch.zeros(8, 16, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q8)
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.tg_gated_decode_noalloc(q8.data_ptr(), kc.data_ptr(), vc.data_ptr(), sc.data_ptr(),
                                     ln.data_ptr(), 8, big, big, 16, 8, 128, gain.data_ptr(),
                                     tau.data_ptr(), out.data_ptr(), ctypes.c_void_p(stream))
    assert st == TG_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0
    assert (out == 0).all()
