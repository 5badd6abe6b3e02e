"""The debug library (libtokengate_debug.so, TG_DEBUG) against the release library:
every kernel of the layer, the backward, the delta rule and decode run once through
each, in separate processes (tests/debug_run.py). The debug library checks the index
of every data-dependent global load and store; on these inputs none may fire (the
status word stays TG_OK), and its outputs must equal the release library's bit for
bit, since the checks change no arithmetic."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(tmp_path, debug):
    path = str(tmp_path / ("debug.pt" if debug else "release.pt"))
    env = dict(os.environ)
    env.pop("TG_DEBUG", None)
    if debug:
        env["TG_DEBUG"] = "1"
    subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_run.py"), path],
                   check=True, env=env, cwd=ROOT, timeout=600)
    return torch.load(path)


def _bits(t):
    t = t.contiguous()
    return t.view({1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[t.element_size()])


def test_debug_library_matches_release(tmp_path):
    from learned_token_pruning_gemm_b200 import build
    build.build()
    build.build(debug=True)
    rel = _run(tmp_path, False)
    dbg = _run(tmp_path, True)
    assert rel["debug_build"] == 0 and dbg["debug_build"] == 1
    assert rel["status"] == 0
    assert dbg["status"] == 0, f"a debug index check fired (status {dbg['status']})"
    assert set(rel) == set(dbg)
    for key in rel:
        if isinstance(rel[key], torch.Tensor):
            assert torch.equal(_bits(rel[key]), _bits(dbg[key])), key
