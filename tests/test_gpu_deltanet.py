"""GPU parity of the gated delta rule over the kept tokens (tg_gated_delta_rule)
against the fp64 oracle, through the C ABI (MarkTechPost page on TokenGate, section
"Est-ce que cela fonctionne avec les modèles d'attention hybrides ?": the hybrid
model's Gated DeltaNet layers are pruned too).

The GPU runs the rule in chunks of 64 tokens (a per-chunk pass with a triangular
solve, then a pass over each sequence's chunks with the state); the oracle runs it
token by token. Tolerance: the outputs are bf16 like the attention's, so the bf16
bar of tests/helpers.py (1e-2 max-abs, 5e-3 relative L2). The GPU's products carry
16 significant bits per operand with fp32 accumulation; with unit keys and
alpha <= 1 each update is a contraction, so rounding does not grow with the
sequence length (the 16k layer's 1868 rows and a 5000-row sequence check it)."""
import numpy as np
import pytest
import torch

from helpers import assert_attn_close

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


def _case(seed, lens, H, dv=128):
    g = torch.Generator().manual_seed(seed)
    T = sum(lens)
    q = torch.nn.functional.normalize(torch.randn(T, H, 128, generator=g), dim=-1).to(torch.bfloat16)
    k = torch.nn.functional.normalize(torch.randn(T, H, 128, generator=g), dim=-1).to(torch.bfloat16)
    v = torch.randn(T, H, dv, generator=g).to(torch.bfloat16)
    a = 0.9 + 0.1 * torch.rand(T, H, generator=g)
    b = torch.rand(T, H, generator=g)
    cu = np.r_[0, np.cumsum(lens)].astype(np.int32)
    return q, k, v, a, b, cu


@pytest.mark.parametrize("lens,H,dv", [([100], 2, 128), ([33, 1, 70, 0, 200], 3, 128),
                                       ([64], 1, 48), ([1868], 16, 128),
                                       ([63, 64, 65, 127, 128, 129], 2, 128),
                                       ([300, 17], 2, 272), ([5000], 1, 32)])
def test_delta_rule_vs_oracle(api, orc, lens, H, dv):
    q, k, v, a, b, cu = _case(sum(lens) + H, lens, H, dv)
    out = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                               torch.tensor(cu, device="cuda"))
    ref = orc.gated_delta_rule(q, k, v, a, b, cu)
    max_abs, rl2 = assert_attn_close(out, ref, torch.bfloat16, what=f"delta rule lens={lens}")
    print(f"delta rule lens={lens} H={H}: max|O| {np.abs(ref).max():.3f} max_abs {max_abs:.2e} "
          f"rel_l2 {rl2:.2e}")


def test_delta_rule_on_the_16k_layers_kept_rows(api, orc):
    # the workload's own DeltaNet inputs over its 1868 kept rows, sampled heads
    from learned_token_pruning_gemm_b200 import synth
    wl = synth.qwen16k()
    q, k, v, a, b = synth.deltanet_inputs(wl)
    cu = np.array([0, wl.total_kept], np.int32)
    out = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                               torch.tensor(cu, device="cuda"))
    heads = [0, 7, 15]
    ref = orc.gated_delta_rule(q[:, heads], k[:, heads], v[:, heads], a[:, heads], b[:, heads], cu)
    assert_attn_close(out[:, heads].contiguous(), ref, torch.bfloat16, what="16k kept rows")


def test_delta_rule_strong_decay_and_repeated_keys(api, orc):
    # decays down to 0.05 (decay products over a chunk reach 1e-80 and underflow to
    # zero) and every fourth key a copy of the previous one written with beta = 1
    # (the overwrite case: the triangular solve's entries reach +-1)
    q, k, v, a, b, cu = _case(11, [150, 90], 2)
    g = torch.Generator().manual_seed(12)
    a = 0.05 + 0.95 * torch.rand(a.shape, generator=g)
    k[3::4] = k[2::4][: k[3::4].shape[0]]
    b[3::4] = 1.0
    out = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                               torch.tensor(cu, device="cuda"))
    ref = orc.gated_delta_rule(q, k, v, a, b, cu)
    assert_attn_close(out, ref, torch.bfloat16, what="strong decay, repeated keys")


def test_delta_rule_sequence_longer_than_max_seqlen_is_reported(api):
    q, k, v, a, b, cu = _case(13, [70, 40], 1)
    out = torch.full(v.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                         torch.tensor(cu, device="cuda"), max_seqlen=64, out=out)
    assert api.device_status(reset=True) == 7          # TG_ERR_DEVICE_CHECK
    o = out.float().cpu()
    assert torch.all(o[:70] == 7.0)                     # the 70-row sequence is skipped
    assert not torch.all(o[70:] == 7.0)                 # the 40-row one is computed


def test_delta_rule_on_the_128k_layers_kept_rows(api, orc):
    # the 128k layer's 10721 kept rows (168 chunks of 64 in one sequence), sampled heads
    from learned_token_pruning_gemm_b200 import synth
    wl = synth.long128k()
    q, k, v, a, b = synth.deltanet_inputs(wl)
    cu = np.array([0, wl.total_kept], np.int32)
    out = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                               torch.tensor(cu, device="cuda"), wl.total_kept)
    heads = [0, 9]
    ref = orc.gated_delta_rule(q[:, heads], k[:, heads], v[:, heads], a[:, heads], b[:, heads], cu)
    assert_attn_close(out[:, heads].contiguous(), ref, torch.bfloat16, what="128k kept rows")


def test_delta_rule_on_the_ragged_layers_kept_rows(api, orc):
    # the ragged layer's 8 sequences of kept rows (1385 to 3493 each), sampled heads
    from learned_token_pruning_gemm_b200 import synth
    wl = synth.ragged8()
    q, k, v, a, b = synth.deltanet_inputs(wl)
    cu = np.r_[0, np.cumsum(wl.kept_counts)].astype(np.int32)
    out = api.gated_delta_rule(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(),
                               torch.tensor(cu, device="cuda"), max(wl.kept_counts))
    heads = [3, 12]
    ref = orc.gated_delta_rule(q[:, heads], k[:, heads], v[:, heads], a[:, heads], b[:, heads], cu)
    assert_attn_close(out[:, heads].contiguous(), ref, torch.bfloat16, what="ragged kept rows")
