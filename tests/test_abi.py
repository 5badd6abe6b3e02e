"""The C-ABI library builds, loads and exports every symbol include/tg.h declares;
host-side argument validation returns status codes without touching a GPU."""
import ctypes
import os
import re

import pytest

from learned_token_pruning_gemm_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "tg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"tg_gate_score", "tg_select_topk", "tg_compact_kv", "tg_gated_attention"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding signatures cover the header"


def test_debug_library_exports_the_same_abi(lib):
    # the debug twin (device index checks) builds too and exports every declared
    # symbol; each library says which it is
    path = build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(dbg, n), n
    dbg.tg_debug_build.restype = ctypes.c_int
    assert dbg.tg_debug_build() == 1
    assert lib.tg_debug_build() == (1 if os.environ.get("TG_DEBUG") == "1" else 0)
    dbg.tg_status_string.restype = ctypes.c_char_p
    assert dbg.tg_status_string(8).decode() == "TG_ERR_DEBUG_BOUNDS"


def test_status_strings(lib):
    assert lib.tg_abi_version() == 5
    for code, name in [(0, "TG_OK"), (1, "TG_ERR_INVALID_ARG"), (3, "TG_ERR_MISALIGNED"),
                       (6, "TG_ERR_TIMEOUT"), (7, "TG_ERR_DEVICE_CHECK"), (8, "TG_ERR_DEBUG_BOUNDS"),
                       (99, "TG_ERR_UNKNOWN")]:
        assert lib.tg_status_string(code).decode() == name


def test_validation_returns_status_without_gpu(lib):
    INVALID, UNSUP, MIS = 1, 2, 3
    P = ctypes.c_void_p
    fake = P(0x10000)      # never dereferenced: validation fails first
    odd = P(0x10004)       # not 16-byte aligned
    # gate: null pointers / bad sizes / unsupported h / misalignment
    assert lib.tg_gate_score(None, 1, 128, 128, fake, fake, fake, 0.0, 64, fake, None) == INVALID
    assert lib.tg_gate_score(fake, 1, -1, 128, fake, fake, fake, 0.0, 64, fake, None) == INVALID
    assert lib.tg_gate_score(fake, 1, 0, 128, fake, fake, fake, 0.0, 64, fake, None) == 0
    assert lib.tg_gate_score(fake, 1, 128, 100, fake, fake, fake, 0.0, 64, fake, None) == UNSUP
    assert lib.tg_gate_score(fake, 1, 128, 128, fake, fake, fake, 0.0, 96, fake, None) == UNSUP
    assert lib.tg_gate_score(odd, 1, 128, 128, fake, fake, fake, 0.0, 64, fake, None) == MIS
    assert lib.tg_gate_score(fake, 7, 128, 128, fake, fake, fake, 0.0, 64, fake, None) == UNSUP
    # select: K > N, too long, null outputs
    assert lib.tg_select_topk(fake, fake, fake, fake, fake, 1, 10, 11, 10, fake, None, None,
                              fake, None) == INVALID
    assert lib.tg_select_topk(fake, fake, fake, fake, fake, 1, 10, 5, 300000, fake, None, None,
                              fake, None) == UNSUP
    assert lib.tg_select_topk(fake, None, fake, fake, fake, 1, 10, 5, 10, fake, None, None,
                              fake, None) == INVALID
    assert lib.tg_select_topk(None, None, None, None, None, 0, 0, 0, 0, None, None, None,
                              None, None) == 0
    # compact: row bytes must be a positive multiple of 16, pointers aligned
    arr = (P * 1)(fake)
    arr_odd = (P * 1)(odd)
    rb = (ctypes.c_int64 * 1)(4096)
    rb_odd = (ctypes.c_int64 * 1)(40)
    assert lib.tg_compact_kv(arr, arr, rb_odd, 1, fake, 5, 10, None) == MIS
    assert lib.tg_compact_kv(arr_odd, arr, rb, 1, fake, 5, 10, None) == MIS
    assert lib.tg_compact_kv(arr, arr, rb, 0, fake, 5, 10, None) == INVALID
    assert lib.tg_compact_kv(arr, arr, rb, 9, fake, 5, 10, None) == INVALID
    assert lib.tg_compact_kv(arr, arr, rb, 1, fake, 5, -1, None) == INVALID
    assert lib.tg_compact_kv(arr, arr, rb, 1, fake, 0, 10, None) == 0
    # attention: GQA divisibility, head dim, max_kept > total, alignment
    args = [fake, fake, fake, 1, fake, fake, fake, fake, 1, 256, 256]
    assert lib.tg_gated_attention(*args, 16, 6, 128, fake, None, None) == INVALID
    assert lib.tg_gated_attention(*args, 16, 8, 64, fake, None, None) == UNSUP
    assert lib.tg_gated_attention(*args[:-1], 300, 16, 8, 128, fake, None, None) == INVALID
    assert lib.tg_gated_attention(*args, 16, 8, 128, odd, None, None) == MIS
    assert lib.tg_gated_attention(fake, fake, fake, 1, fake, fake, fake, fake, 1, 256, 256, 16, 8,
                                  300, fake, None, None) == UNSUP
    # self test bounds
    assert lib.tg_selftest_bounded_wait(10, None) == INVALID
    # q/k/v projection: head_dim 128 only, even head total, d % 64, rope_base > 1,
    # null pointers, alignment; zero rows is a no-op
    assert lib.tg_qkv_rope(fake, 100, 2048, fake, 16, 8, 64, 1e6, fake, fake, fake, fake,
                           None) == UNSUP
    assert lib.tg_qkv_rope(fake, 100, 2048, fake, 15, 8, 128, 1e6, fake, fake, fake, fake,
                           None) == UNSUP
    assert lib.tg_qkv_rope(fake, 100, 2000, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
                           None) == UNSUP
    assert lib.tg_qkv_rope(fake, 100, 2048, fake, 16, 8, 128, 1.0, fake, fake, fake, fake,
                           None) == INVALID
    assert lib.tg_qkv_rope(fake, 100, 2048, None, 16, 8, 128, 1e6, fake, fake, fake, fake,
                           None) == INVALID
    assert lib.tg_qkv_rope(fake, 100, 2048, fake, 16, 8, 128, 1e6, fake, odd, fake, fake,
                           None) == MIS
    assert lib.tg_qkv_rope(None, 0, 2048, None, 16, 8, 128, 1e6, None, None, None, None,
                           None) == 0
    # the same rules for the fused compaction + projection, plus its own: x, kept_idx
    # and n_src > 0 required, xc optional (and aligned when given)
    cq = lib.tg_compact_qkv_rope
    assert cq(fake, 4096, 2048, fake, 100, fake, fake, 16, 8, 64, 1e6, fake, fake, fake, fake,
              None) == UNSUP
    assert cq(fake, 4096, 2000, fake, 100, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == UNSUP
    assert cq(fake, 0, 2048, fake, 100, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == INVALID
    assert cq(None, 4096, 2048, fake, 100, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == INVALID
    assert cq(fake, 4096, 2048, None, 100, fake, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == INVALID
    assert cq(fake, 4096, 2048, fake, 100, fake, fake, 16, 8, 128, 0.5, fake, fake, fake, fake,
              None) == INVALID
    assert cq(fake, 4096, 2048, fake, 100, odd, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == MIS
    assert cq(odd, 4096, 2048, fake, 100, None, fake, 16, 8, 128, 1e6, fake, fake, fake, fake,
              None) == MIS
    assert cq(None, 0, 2048, None, 0, None, None, 16, 8, 128, 1e6, None, None, None, None,
              None) == 0



def test_decode_validation_without_gpu(lib):
    INVALID, UNSUP, MIS, WS = 1, 2, 3, 4
    P = ctypes.c_void_p
    fake, odd = P(0x10000), P(0x10004)
    ws_size = lib.tg_gated_decode_workspace_size
    # partials of (dh + 2) fp32 per (sequence, query head, 64-key chunk)
    assert ws_size(2, 16, 128, 1868) == 2 * 16 * 30 * 130 * 4
    assert ws_size(1, 16, 64, 100) == 0 and ws_size(0, 16, 128, 100) == 0
    need = ws_size(1, 16, 128, 1000)

    def dec(hq=16, hkv=8, dh=128, cap=1000, max_len=1000, ws=fake, ws_bytes=None, q=fake,
            batch=1):
        return lib.tg_gated_decode(q, fake, fake, fake, fake, batch, cap, max_len, hq, hkv, dh,
                                   fake, fake, fake, ws, need if ws_bytes is None else ws_bytes,
                                   None)
    assert dec(hkv=6) == INVALID
    assert dec(dh=64) == UNSUP
    assert dec(hq=32, hkv=2) == UNSUP            # more than 8 query heads per KV head
    assert dec(max_len=1001) == INVALID
    assert dec(ws_bytes=need - 4) == WS
    assert dec(ws=None) == WS
    assert dec(q=odd) == MIS
    assert dec(ws=odd) == MIS
    assert dec(batch=0) == 0
    assert lib.tg_gated_decode(None, fake, fake, fake, fake, 1, 10, 10, 16, 8, 128, fake, fake,
                               fake, fake, need, None) == INVALID
    # append: null pointers, head_dim, alignment
    assert lib.tg_cache_append(None, fake, fake, 1, 10, 8, 128, fake, fake, fake, fake,
                               None) == INVALID
    assert lib.tg_cache_append(fake, fake, fake, 1, 10, 8, 64, fake, fake, fake, fake,
                               None) == UNSUP
    assert lib.tg_cache_append(fake, odd, fake, 1, 10, 8, 128, fake, fake, fake, fake,
                               None) == MIS
    assert lib.tg_cache_append(None, None, None, 0, 10, 8, 128, None, None, None, None,
                               None) == 0


# ---- the Python binding checks every tensor's size against the sizes it passes
#      to the C ABI, before any call (so a CPU tensor reaches none of them) ----

def _raises(fn, match):
    from learned_token_pruning_gemm_b200._lib import TokenGateError
    with pytest.raises(TokenGateError, match=match):
        fn()


def test_binding_gate_checks_lengths():
    import torch
    from learned_token_pruning_gemm_b200 import api
    x, w1 = torch.zeros(8, 64), torch.zeros(16, 64)
    ok = torch.zeros(16)
    _raises(lambda: api.gate_score(x, w1, torch.zeros(15), ok, 0.0), "b1 must have 16")
    _raises(lambda: api.gate_score(x, w1, ok, torch.zeros(17), 0.0), "w2 must have 16")
    _raises(lambda: api.gate_score(x, w1, ok, ok, 0.0, out=torch.zeros(7)), "scores must have 8")
    _raises(lambda: api.gate_score(x, torch.zeros(16, 32), ok, ok, 0.0), "share a dtype")


def test_binding_select_checks_lengths():
    import torch
    from learned_token_pruning_gemm_b200 import api
    i32 = lambda n: torch.zeros(n, dtype=torch.int32)
    s = torch.zeros(100)
    args = (s, i32(3), i32(2), i32(2), i32(2), 40, 60)
    _raises(lambda: api.select_topk(s, i32(2), i32(2), i32(2), i32(2), 40, 60),
            "cu_seqlens must have 3")
    _raises(lambda: api.select_topk(s, i32(3), i32(2), i32(1), i32(2), 40, 60),
            "doc_end must have 2")
    _raises(lambda: api.select_topk(s, i32(3), i32(2), i32(2), i32(3), 40, 60), "k_doc must have 2")
    _raises(lambda: api.select_topk(*args, kept_idx=i32(39)), "kept_idx must have 40")
    _raises(lambda: api.select_topk(*args, kept_scores=torch.zeros(41)), "kept_scores must have 40")
    _raises(lambda: api.select_topk(*args, kept_pos=i32(1)), "kept_pos must have 40")
    _raises(lambda: api.select_topk(*args, cu_kept=i32(2)), "cu_kept must have 3")


def test_binding_compact_checks_shapes():
    import torch
    from learned_token_pruning_gemm_b200 import api
    idx = torch.zeros(4, dtype=torch.int32)
    x = torch.zeros(10, 8)
    _raises(lambda: api.compact_rows([x], idx, outs=[torch.zeros(5, 8)]), "shape/dtype mismatch")
    _raises(lambda: api.compact_rows([x], idx, outs=[torch.zeros(4, 7)]), "shape/dtype mismatch")
    _raises(lambda: api.compact_rows([x, x], idx, outs=[torch.zeros(4, 8)]), "one output per")
    _raises(lambda: api.compact_rows([], idx), "at least one source")


def test_binding_attention_checks_lengths():
    import torch
    from learned_token_pruning_gemm_b200 import api
    K, hq, hkv, dh = 10, 4, 2, 64
    q, k = torch.zeros(K, hq, dh), torch.zeros(K, hkv, dh)
    cu = torch.tensor([0, K], dtype=torch.int32)
    g = torch.zeros(hq)
    _raises(lambda: api.gated_attention(q, k, k, torch.zeros(K - 1), g, g, cu, K),
            "s_kept must have 10")
    _raises(lambda: api.gated_attention(q, k, k, torch.zeros(K), torch.zeros(3), g, cu, K),
            "gain must have 4")
    _raises(lambda: api.gated_attention(q, k, k, torch.zeros(K), g, torch.zeros(5), cu, K),
            "tau must have 4")
    _raises(lambda: api.gated_attention(q, k, k, torch.zeros(K), g, g, cu, K,
                                        out=torch.zeros(K, hq, dh - 1)), "out must have shape")
    _raises(lambda: api.gated_attention(q, k, torch.zeros(K, hkv, dh + 1), torch.zeros(K), g, g,
                                        cu, K), "q \\[K,Hq,dh\\]")


def test_binding_qkv_rope_checks_lengths():
    import torch
    from learned_token_pruning_gemm_b200 import api
    xc = torch.zeros(6, 64, dtype=torch.bfloat16)
    w = torch.zeros(4 * 128, 64, dtype=torch.bfloat16)
    _raises(lambda: api.qkv_rope(xc, w, 2, 1, torch.zeros(5, dtype=torch.int32)), "pos must have 6")
    bad = (torch.zeros(6, 2, 128, dtype=torch.bfloat16), torch.zeros(6, 1, 128, dtype=torch.bfloat16),
           torch.zeros(6, 2, 128, dtype=torch.bfloat16))
    _raises(lambda: api.qkv_rope(xc, w, 2, 1, torch.zeros(6, dtype=torch.int32), out=bad),
            "v must have shape")


def test_binding_decode_checks_shapes():
    import torch
    from learned_token_pruning_gemm_b200 import api
    q = torch.zeros(2, 4, 128, dtype=torch.bfloat16)
    kc = torch.zeros(2, 50, 2, 128, dtype=torch.bfloat16)
    sc, ln, g = torch.zeros(2, 50), torch.zeros(2, dtype=torch.int32), torch.zeros(4)
    _raises(lambda: api.gated_decode(q, kc, kc, torch.zeros(2, 49), ln, g, g, 50), "s_cache must")
    _raises(lambda: api.gated_decode(q, kc, kc, sc, torch.zeros(3, dtype=torch.int32), g, g, 50),
            "cache_len must")
    _raises(lambda: api.gated_decode(q, kc, kc[:, :, :1].contiguous(), sc, ln, g, g, 50),
            "v_cache must")
    _raises(lambda: api.gated_decode(q, kc, kc, sc, ln, torch.zeros(3), g, 50), "gain must have 4")
    _raises(lambda: api.cache_append(kc[:, 0], kc[:, 0], torch.zeros(3), kc, kc, sc, ln),
            "s_new must")


def test_backward_validation_without_gpu(lib):
    INVALID, UNSUP, MIS, WS = 1, 2, 3, 4
    P = ctypes.c_void_p
    fake, odd = P(0x10000), P(0x10004)
    size = lib.tg_gated_attention_bwd_workspace_size
    assert size(1, 1, 1868, 1868, 16, 8, 128) > 0
    assert size(1, 1, 1868, 1868, 16, 6, 128) == 0
    need = size(1, 1, 1000, 1000, 16, 8, 128)

    def bwd(dtype=1, hq=16, hkv=8, dh=128, ws=fake, nb=None, q=fake, total=1000, mk=1000):
        return lib.tg_gated_attention_bwd(q, fake, fake, fake, fake, dtype, fake, fake, fake, fake,
                                          fake, 1, total, mk, hq, hkv, dh, fake, fake, fake, fake,
                                          fake, fake, ws, need if nb is None else nb, None)
    assert bwd(hkv=6) == INVALID
    assert bwd(mk=1001) == INVALID
    assert bwd(dh=64) == UNSUP
    assert bwd(dtype=0, dh=512) == UNSUP
    assert bwd(dtype=5) == UNSUP
    assert bwd(nb=need - 1) == WS
    assert bwd(ws=None) == WS
    assert bwd(ws=odd) == MIS
    assert bwd(q=odd) == MIS
    assert bwd(q=None) == INVALID
    assert bwd(total=0) == 0


def test_delta_rule_validation_without_gpu(lib):
    INVALID, UNSUP, MIS, WS = 1, 2, 3, 4
    P = ctypes.c_void_p
    fake, odd = P(0x10000), P(0x10004)
    big = 1 << 30

    def dn(dtype=1, dk=128, dv=128, q=fake, a=fake, total=10, batch=1, max_len=10, ws=fake,
           ws_bytes=big):
        return lib.tg_gated_delta_rule(q, fake, fake, dtype, a, fake, fake, batch, total, max_len,
                                       4, dk, dv, fake, ws, ws_bytes, None)
    assert dn(dtype=0) == UNSUP
    assert dn(dk=64) == UNSUP
    assert dn(dv=100) == UNSUP
    assert dn(q=odd) == MIS
    assert dn(a=P(0x10002)) == MIS
    assert dn(q=None) == INVALID
    assert dn(total=0) == 0 and dn(batch=0) == 0 and dn(max_len=0) == 0
    assert dn(total=-1) == INVALID
    assert dn(max_len=-1) == INVALID
    assert dn(ws=None) == WS
    assert dn(ws=odd) == MIS
    # one record per (64-row chunk slot, head): floor(total / 64) + batch slots
    need = lib.tg_gated_delta_rule_workspace_size(3, 1000, 4, 128)
    assert need == (1000 // 64 + 3) * 4 * (53760 + 256 * 128)
    assert dn(total=1000, batch=3, ws_bytes=need - 1) == WS
    assert lib.tg_gated_delta_rule_workspace_size(0, 10, 4, 128) == 0
