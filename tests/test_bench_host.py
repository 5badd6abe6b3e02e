"""The benchmark's host-side arithmetic, on the CPU: the algorithmic work of a step
(closed forms of the flops and bytes each stage must do), the per-stage report, and
the roofline of the dominant kernel (which stage dominates, achieved / peak, and
that DRAM traffic is reported only while the kernel source it was measured on is
unchanged)."""
import importlib.util
import json
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _wl16k():
    return types.SimpleNamespace(n_tokens=16384, d=2048, h=256, dh=128, hq=16, hkv=8,
                                 dtype="bf16", kept_counts=[1868])


def test_algorithmic_work_closed_forms(bench):
    w = bench._algorithmic_work(_wl16k())
    assert w["gate_flops"] == 2 * 16384 * 2048 * 256                      # 17.18 GFLOP
    assert w["gate_bytes"] == 2 * 16384 * 2048 + 2 * 2048 * 256 + 4 * 16384
    assert w["attn_flops"] == 4 * 128 * 16 * 1868 * 1869 // 2             # 14.30 GFLOP, causal
    assert w["compact_bytes"] == 2 * 1868 * 2048 * 2                       # read + write
    assert w["select_bytes"] == 4 * 16384 + 8 * 1868
    assert w["project_flops"] == 2 * 1868 * 2048 * (16 + 2 * 8) * 128
    # a ragged batch: the causal flops are per sequence, not of the concatenation
    rag = types.SimpleNamespace(**{**vars(_wl16k()), "kept_counts": [1000, 868]})
    assert bench._algorithmic_work(rag)["attn_flops"] == (4 * 128 * 16 * (1000 * 1001 + 868 * 869)) // 2


def test_stage_report_and_roofline(bench):
    w = bench._algorithmic_work(_wl16k())
    ms = {"gate": 0.025, "select": 0.016, "compact": 0.008, "attention": 0.0287}
    st = bench._stages_report(w, ms, 1702.2, 6455.6)
    tf = w["attn_flops"] / 28.7e-6 / 1e12
    assert st["attention"]["tflops"] == pytest.approx(tf)
    assert st["attention"]["frac_tc"] == pytest.approx(tf / 1702.2)
    assert st["compact"]["frac_hbm"] == pytest.approx(w["compact_bytes"] / 8e-6 / 1e9 / 6455.6)
    assert st["select+compact"]["us"] == pytest.approx(24.0)
    r = bench._roofline(w, ms, 1702.2, 6455.6, "measured", "no-such-workload")
    assert r["kernel"] == "attention" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(tf) and r["frac"] == pytest.approx(tf / 1702.2)
    assert r["traffic"] is None   # nothing recorded for that workload
    # the projection stages never count as the dominant kernel of the metric's step
    r2 = bench._roofline(w, {**ms, "compact+project": 0.1}, 1702.2, 6455.6, "measured", "x")
    assert r2["kernel"] == "attention"
    # the gate at 16k sits on the ridge: it is reported against the larger floor (bytes)
    r3 = bench._roofline(w, {**ms, "gate": 0.05}, 1702.2, 6455.6, "measured", "x")
    assert r3["kernel"] == "gate" and r3["bound"] == "hbm" and r3["unit"] == "GB/s"
    assert r3["achieved"] == pytest.approx(w["gate_bytes"] / 50e-6 / 1e9)


def test_traffic_reported_only_for_the_measured_source(bench):
    w = bench._algorithmic_work(_wl16k())
    ms = {"gate": 0.025, "select": 0.016, "compact": 0.008, "attention": 0.0287}
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))["qwen16k"]
    r = bench._roofline(w, ms, 1702.2, 6455.6, "measured", "qwen16k")
    if rec["attention"]["kernel_rev"] == bench._kernel_rev("attention"):
        assert r["traffic"] == rec["attention"]["bytes_per_launch"]
    else:
        assert r["traffic"] is None
    # the record's figure is close to the algorithmic bytes (q, k, v read once)
    qkv = 1868 * (16 + 8 + 8) * 128 * 2
    assert abs(rec["attention"]["bytes_per_launch"] - qkv) / qkv < 0.01
