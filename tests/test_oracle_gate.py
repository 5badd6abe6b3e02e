"""Pins for the oracle's gate MLP scorer (MarkTechPost page, section "Comment
TokenGate a-t-il appris le fonctionnement de la réduction des tokens ?": a small
MLP scores every token from its post-attention residual at the gate layer).

Reading pinned here: s = b2 + w2 . GELU(W1 x + b1), GELU(u) = u * Phi(u) (exact
erf form), W1 stored [h, d]."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _phi_table():
    rows = []
    for line in open(os.path.join(GOLDEN, "normal_cdf_table.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            u, p = line.split()
            rows.append((float(u), float(p)))
    return rows


def test_gelu_matches_printed_normal_cdf(orc):
    # d = h = 1, w1 = w2 = 1, b1 = b2 = 0: s = GELU(x) = x * Phi(x)
    for u, phi in _phi_table():
        x = torch.tensor([[u]], dtype=torch.float32)
        w1 = torch.ones(1, 1)
        s64, _ = orc.gate_score(x, w1, [0.0], [1.0], 0.0)
        assert s64[0] == pytest.approx(u * phi, abs=1e-15, rel=1e-14), u
    # the tanh approximation would be off by more than 1e-4 at u = 1
    tanh_gelu = 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * (1 + 0.044715)))
    assert abs(tanh_gelu - 0.8413447460685429) > 1e-4


def test_gate_hand_example(orc):
    # x = (1, 0), W1 = I, b1 = 0, w2 = (1, 1), b2 = 0.25:
    # s = GELU(1) + GELU(0) + 0.25 = Phi(1) + 0.25
    x = torch.tensor([[1.0, 0.0]])
    w1 = torch.eye(2)
    s64, s32 = orc.gate_score(x, w1, [0.0, 0.0], [1.0, 1.0], 0.25)
    assert s64[0] == pytest.approx(0.8413447460685429 + 0.25, abs=1e-15)
    assert s32[0] == np.float32(s64[0])


def test_gate_uses_both_biases_and_layout(orc):
    # b1 shifts the pre-activation, b2 the score; W1 row k feeds hidden unit k
    x = torch.tensor([[2.0, -1.0, 0.5]])
    w1 = torch.tensor([[1.0, 0.0, 0.0], [0.0, 0.0, 2.0]])   # h=2, d=3
    s64, _ = orc.gate_score(x, w1, [-1.0, 0.0], [3.0, -1.0], 0.5)
    # u = (2 - 1, 1) = (1, 1): s = 3 Phi(1) - Phi(1) + 0.5
    assert s64[0] == pytest.approx(2 * 0.8413447460685429 + 0.5, abs=1e-14)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_vs_torch_fp64_witness(orc, dtype):
    g = torch.Generator().manual_seed(7)
    n, d, h = 37, 96, 24
    x = torch.randn(n, d, generator=g).to(dtype)
    w1 = (torch.randn(h, d, generator=g) / d ** 0.5).to(dtype)
    b1 = torch.randn(h, generator=g) / d ** 0.5
    w2 = torch.randn(h, generator=g) / h ** 0.5
    b2 = 0.3125
    ref = F.linear(F.gelu(F.linear(x.double(), w1.double(), b1.double()), approximate="none"),
                   w2.double()[None, :]).squeeze(1) + b2
    s64, s32 = orc.gate_score(x, w1, b1, w2, b2)
    np.testing.assert_allclose(s64, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(s32, s64.astype(np.float32))


def test_bf16_inputs_are_widened_exactly(orc):
    # bf16 bit patterns 0x3F80 = 1.0, 0x3F81 = 1.0078125, 0xC000 = -2.0
    bits = torch.tensor([[0x3F80, 0x3F81, -16384]], dtype=torch.int16)   # 0xC000 as int16
    x = bits.view(torch.bfloat16)
    w1 = torch.eye(3).to(torch.bfloat16)
    # with w2 = e_k and GELU we read back GELU(x_k); use a large h to isolate units
    for kk, val in enumerate([1.0, 1.0078125, -2.0]):
        w2 = [0.0] * 3
        w2[kk] = 1.0
        s64, _ = orc.gate_score(x, w1, [0.0] * 3, w2, 0.0)
        assert s64[0] == pytest.approx(val * 0.5 * (1 + math.erf(val / math.sqrt(2))), abs=1e-15)
