"""Shared helpers for the parity tests: tolerances and comparisons.

Tolerances (fixed by the project's accuracy targets):
  gate scores              |gpu - oracle| <= 1e-4 absolute (fp32 scores)
  kept indices             bit-exact given identical scores
  attention, fp32 path     max-abs <= 1e-4
  attention, bf16 path     max-abs <= 1e-2 and relative L2 <= 5e-3
"""
import numpy as np
import torch

GATE_ATOL = 1e-4
ATTN_F32_ATOL = 1e-4
ATTN_BF16_ATOL = 1e-2
ATTN_BF16_RL2 = 5e-3


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def attn_errors(gpu_out: torch.Tensor, ref: np.ndarray, rows=None):
    g = to_np64(gpu_out)
    if rows is not None:
        g, ref = g[rows], ref[rows]
    diff = g - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rl2 = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rl2


def assert_attn_close(gpu_out, ref, dtype, rows=None, what=""):
    max_abs, rl2 = attn_errors(gpu_out, ref, rows)
    max_o = float(np.abs(ref if rows is None else ref[rows]).max())
    if dtype == torch.float32:
        assert max_abs <= ATTN_F32_ATOL, f"{what}: max_abs {max_abs:.3e} (max|O| {max_o:.3f})"
    else:
        assert max_abs <= ATTN_BF16_ATOL and rl2 <= ATTN_BF16_RL2, (
            f"{what}: max_abs {max_abs:.3e} rel_l2 {rl2:.3e} (max|O| {max_o:.3f})")
    return max_abs, rl2


def sample_rows(cu_kept, n_random=64, seed=0):
    """First, last and tile-edge rows of every sequence, plus random rows."""
    cu = np.asarray(cu_kept, np.int64)
    rows = set()
    rng = np.random.default_rng(seed)
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        if e <= a:
            continue
        for r in (a, a + 1, e - 1, e - 2):
            if a <= r < e:
                rows.add(r)
        for t in range(a + 127, e, 128):
            rows.update(x for x in (t, t + 1) if x < e)
        rows.update(int(x) for x in rng.integers(a, e, min(n_random, e - a)))
    return np.array(sorted(rows), np.int32)
