#!/usr/bin/env python
"""Gated-prefill benchmark: one gated layer (gate MLP -> question-protected top-K
-> compaction -> token-gated causal GQA attention) on synthetic inputs shaped like
the Qwen3-1.7B layer of the TokenGate pages (16k tokens, d=2048, 16/8 heads,
dh=128, keep 10% of the document).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen16k]

Prints ONE JSON line (rank 0). Multi-GPU runs (torchrun) are independent
replicas: every rank runs the whole layer on its own copy (no data-path
collective); the timed region is bracketed by barriers and the slowest rank's
time is reported.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "gated-prefill tokens/s (gate+top-K+attn) at 16k-128k; % of bf16 TC / HBM peak"
L2_FLUSH_BYTES = 512 << 20      # > 126 MB L2
L2_CLEAN_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons, sampled by a background thread through
    NVML (about every 0.5 ms) while the benchmark runs; `window(t0, t1)` keeps
    the samples taken inside a host-time window."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: int):
        self.samples = []
        self._stop = False
        self._thread = None
        self.error = None
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = device
            if hasattr(torch.cuda, "_get_nvml_device_index"):
                idx = torch.cuda._get_nvml_device_index(device)
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # noqa: BLE001
            self.error = f"nvml unavailable: {e}"

    def _run(self):
        while not self._stop:
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self._reasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.0005)

    def start(self):
        import threading
        if self.error is None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        self._stop = True
        if self._thread is not None:
            self._thread.join()

    def window(self, t0, t1):
        if self.error is not None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error]}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        where = "timed region"
        if len(inside) < 3:          # too short a region: widen to the whole loaded run
            inside, where = self.samples, "warm-up + timed region"
        mhz = [s[1] for s in inside]
        reasons = sorted({n for s in inside for bit, n in self.REASONS.items() if s[2] & bit})
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "sampled_over": where}


def _work(wl):
    """Algorithmic work of one step (bytes / flops the method must move / do)."""
    N, d, h, dh, hq = wl.n_tokens, wl.d, wl.h, wl.dh, wl.hq
    esz = 2 if wl.dtype == "bf16" else 4
    Ks = wl.kept_counts
    K = sum(Ks)
    return {
        "gate_bytes": esz * N * d + esz * d * h + 4 * N,
        "gate_flops": 2 * N * d * h,
        "select_bytes": 4 * N + 8 * K,
        "compact_bytes": 2 * K * d * esz,
        "attn_flops": sum(4 * dh * hq * k * (k + 1) // 2 for k in Ks),
    }


def _oracle_sample_time(wl, oracle, n_gate=4096, n_attn_rows=128):
    """Oracle time for one whole step, extrapolated from a bounded sample: gate on
    n_gate rows (scaled by N), select and gather in full, attention on n_attn_rows
    query rows per sequence (scaled by the causal pair count)."""
    rng = np.random.default_rng(0)
    N = wl.n_tokens
    rows = np.sort(rng.choice(N, min(n_gate, N), replace=False))
    t0 = time.perf_counter()
    s64, s32 = oracle.gate_score(wl.x[torch.from_numpy(rows)], wl.w1, wl.b1, wl.w2, wl.b2)
    t_gate = (time.perf_counter() - t0) * N / len(rows)
    scores = np.zeros(N, np.float32)
    scores[rows] = s32
    sel = wl.score_override.numpy() if wl.score_override is not None else scores
    t0 = time.perf_counter()
    idx, cu = oracle.select_topk(sel, wl.cu_seqlens, wl.doc_begin, wl.doc_end, wl.k_doc)
    t_sel = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.gather_rows(wl.x.view(torch.int16).numpy(), idx)
    t_gather = time.perf_counter() - t0
    # attention sample: rows spread over each sequence; cost ~ (row index + 1)
    arows, pairs_sample = [], 0
    for b in range(wl.batch):
        a, e = int(cu[b]), int(cu[b + 1])
        if e <= a:
            continue
        r = np.unique(np.linspace(a, e - 1, min(n_attn_rows, e - a)).astype(np.int32))
        arows.append(r)
        pairs_sample += int(np.sum(r - a + 1))
    arows = np.concatenate(arows)
    pairs_full = sum(k * (k + 1) // 2 for k in wl.kept_counts)
    t0 = time.perf_counter()
    oracle.gated_attention(wl.q, wl.k, wl.v, sel[idx], wl.gain, wl.tau, cu, rows=arows)
    t_attn = (time.perf_counter() - t0) * pairs_full / max(pairs_sample, 1)
    total = t_gate + t_sel + t_gather + t_attn
    sample = (f"oracle fp64 on host cores: gate on {len(rows)} of {N} rows (x{N / len(rows):.0f}), "
              f"select+gather in full, attention on {len(arows)} query rows x {wl.hq} heads "
              f"(scaled by causal pairs x{pairs_full / max(pairs_sample, 1):.0f})")
    return total, {"gate": t_gate, "select": t_sel, "compact": t_gather, "attention": t_attn}, sample


def _threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def run_reference(args, rep):
    """The oracle timed as the reference arm (rank 0 only; other ranks exit)."""
    ws = rep.world
    if rep.rank != 0:
        return
    import oracle
    from learned_token_pruning_gemm_b200 import synth
    oracle.build()
    wl = synth.WORKLOADS[args.workload]()
    for _ in range(args.warmup):
        _oracle_sample_time(wl, oracle, n_gate=64, n_attn_rows=4)
    times = []
    sample = ""
    for _ in range(args.steps):
        t, _, sample = _oracle_sample_time(wl, oracle)
        times.append(t)
    ms = 1e3 * statistics.mean(times)
    value = wl.n_tokens / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "tokens": wl.n_tokens, "kept": wl.total_kept},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rep):
    ws, rank = rep.world, rep.rank
    from learned_token_pruning_gemm_b200 import api, pipeline, synth
    dev_index = torch.cuda.current_device()
    wl = synth.WORKLOADS[args.workload]()
    gp = pipeline.GatedPrefill(wl)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    clean = torch.ones(L2_CLEAN_BYTES // 4, dtype=torch.float32, device="cuda")

    def flush_l2():
        # evict the inputs (write a buffer larger than L2), then read another buffer
        # larger than L2 so the lines left behind are clean: otherwise the first
        # kernel of the step pays for writing back the flush buffer's dirty lines
        flush.zero_()
        clean.sum()
    work = _work(wl)
    peaks, peak_src = _peaks()

    clocks = ClockSampler(dev_index)
    clocks.start()
    gp.capture()                          # the whole layer as one CUDA graph
    for _ in range(args.warmup):
        flush_l2()
        gp.replay_step()
    torch.cuda.synchronize()
    assert api.device_status(reset=True) == 0

    # timed region: exactly `steps` whole-layer steps (one graph each), L2 flushed
    # between them outside the events
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    rep.barrier()
    torch.cuda.synchronize()
    t_host0 = time.perf_counter()
    for a, b in step_ev:
        flush_l2()
        a.record(stream)
        gp.replay_step()
        b.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    rep.barrier()
    clocks.stop()
    clk = clocks.window(t_host0, t_host1)
    status = api.device_status(reset=True)
    if status != 0:
        raise RuntimeError(f"device status {status} during the timed region")
    step_ms = [a.elapsed_time(b) for a, b in step_ev]

    # per-stage breakdown (separate pass): events recorded inside the step graph
    per = []
    for _ in range(args.steps):
        flush_l2()
        gp.replay_timed()
        torch.cuda.synchronize()
        per.append(gp.stage_times_ms())
    stage_ms = {name: statistics.mean(p[name] for p in per) for name in gp.STAGES}
    ms = rep.max(statistics.mean(step_ms))
    value = ws * wl.n_tokens / (ms / 1e3)

    # dominant kernel and its roofline
    dom = max(stage_ms, key=stage_ms.get)
    t = stage_ms[dom] / 1e3
    tf_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    if dom == "attention":
        ach, peak, unit, bound = work["attn_flops"] / t / 1e12, tf_peak, "TFLOP/s", "tensor"
    elif dom == "gate":
        # at the ridge: report against the binding floor (the larger one)
        if work["gate_flops"] / (tf_peak * 1e12) >= work["gate_bytes"] / (hbm_peak * 1e9):
            ach, peak, unit, bound = work["gate_flops"] / t / 1e12, tf_peak, "TFLOP/s", "tensor"
        else:
            ach, peak, unit, bound = work["gate_bytes"] / t / 1e9, hbm_peak, "GB/s", "hbm"
    elif dom == "compact":
        ach, peak, unit, bound = work["compact_bytes"] / t / 1e9, hbm_peak, "GB/s", "hbm"
    else:
        ach, peak, unit, bound = work["select_bytes"] / t / 1e9, hbm_peak, "GB/s", "hbm"
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if os.path.exists(tpath):
        tr = json.load(open(tpath))
        ent = tr.get(args.workload, {}).get(dom)
        if ent and ent.get("kernel_rev") == _kernel_rev(dom):
            traffic = ent["bytes_per_launch"]
    roofline = {"kernel": dom, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
                "frac": ach / peak, "traffic": traffic, "peak_source": peak_src}
    stages = {
        "gate": {"us": stage_ms["gate"] * 1e3,
                 "tflops": work["gate_flops"] / (stage_ms["gate"] / 1e3) / 1e12,
                 "gbs": work["gate_bytes"] / (stage_ms["gate"] / 1e3) / 1e9},
        "select": {"us": stage_ms["select"] * 1e3,
                   "gbs": work["select_bytes"] / (stage_ms["select"] / 1e3) / 1e9},
        "compact": {"us": stage_ms["compact"] * 1e3,
                    "gbs": work["compact_bytes"] / (stage_ms["compact"] / 1e3) / 1e9},
        "attention": {"us": stage_ms["attention"] * 1e3,
                      "tflops": work["attn_flops"] / (stage_ms["attention"] / 1e3) / 1e12},
    }
    for s in stages.values():
        if "tflops" in s:
            s["frac_tc"] = s["tflops"] / tf_peak
        if "gbs" in s:
            s["frac_hbm"] = s["gbs"] / hbm_peak
    sc_bytes = work["select_bytes"] + work["compact_bytes"]
    stages["select+compact"] = {
        "us": (stage_ms["select"] + stage_ms["compact"]) * 1e3,
        "frac_hbm": sc_bytes / ((stage_ms["select"] + stage_ms["compact"]) / 1e3) / 1e9 / hbm_peak}

    # ---- the next step on the path, measured on its own (not part of the metric
    #      above): the kept rows' q/k/v projections with the rotary embedding at
    #      their original positions, from the compacted residual rows ----
    next_step = None
    nh = wl.hq + 2 * wl.hkv
    if wl.dtype == "bf16" and wl.dh == 128 and nh % 2 == 0:
        gw = torch.Generator().manual_seed(11)
        w_qkv = (torch.randn(nh * wl.dh, wl.d, generator=gw) / math.sqrt(wl.d)).to(
            torch.bfloat16).cuda()
        kept = gp.kept_idx.cpu().numpy().astype(np.int64)
        starts = np.repeat(np.asarray(wl.cu_seqlens[:-1], np.int64),
                           np.diff(gp.cu_kept.cpu().numpy()))
        pos = torch.from_numpy((kept - starts).astype(np.int32)).cuda()
        K = gp.xc.shape[0]
        outs = (torch.empty(K, wl.hq, wl.dh, dtype=torch.bfloat16, device="cuda"),
                torch.empty(K, wl.hkv, wl.dh, dtype=torch.bfloat16, device="cuda"),
                torch.empty(K, wl.hkv, wl.dh, dtype=torch.bfloat16, device="cuda"))
        q_ms = []
        for i in range(args.steps + 3):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            api.qkv_rope(gp.xc, w_qkv, wl.hq, wl.hkv, pos, rope_base=1e6, out=outs)
            b.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                q_ms.append(a.elapsed_time(b))
        if api.device_status(reset=True) != 0:
            raise RuntimeError("device status set by the q/k/v projection")
        t_q = statistics.median(q_ms) / 1e3
        flops = 2.0 * K * wl.d * nh * wl.dh
        nbytes = 2.0 * K * wl.d + 2.0 * nh * wl.dh * wl.d + 2.0 * K * nh * wl.dh
        next_step = {"kept_qkv_rope": {
            "us": t_q * 1e6, "tflops": flops / t_q / 1e12, "frac_tc": flops / t_q / 1e12 / tf_peak,
            "gbs": nbytes / t_q / 1e9, "rows": K, "d": wl.d, "heads": f"{wl.hq}/{wl.hkv}",
            "note": "y = W xc, q/k rotated at the kept tokens' original positions (rotate-half, "
                    "base 1e6), v copied; CUDA events around one launch, L2 flushed before each"}}

    # ---- e2e: host buffers in, result out, through the same public calls ----
    e2e = None
    if not args.no_e2e:
        host_in = [t.pin_memory() for t in (wl.x, wl.q, wl.k, wl.v)]
        dev_in = [gp.x, gp.q, gp.k, gp.v]
        host_out = torch.empty(gp.out.shape, dtype=gp.out.dtype).pin_memory()
        host_idx = torch.empty(gp.kept_idx.shape, dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = host_out.numel() * host_out.element_size() + host_idx.numel() * 4

        def e2e_step():
            for hsrc, dst in zip(host_in, dev_in):
                dst.copy_(hsrc, non_blocking=True)
            gp.replay_step()
            host_out.copy_(gp.out, non_blocking=True)
            host_idx.copy_(gp.kept_idx, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        rep.barrier()
        for a, b in e_ev:
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize()
        rep.barrier()
        e_ms = rep.max(statistics.mean(a.elapsed_time(b) for a, b in e_ev))
        e2e = {"value": ws * wl.n_tokens / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        t_cpu, parts, sample = _oracle_sample_time(wl, oracle)
        cpu = {"value": wl.n_tokens / t_cpu, "unit": "tokens/s", "cores": _threads(),
               "kind": "oracle", "sample": sample,
               "stage_s": {k: round(v, 4) for k, v in parts.items()}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": args.workload, "tokens": wl.n_tokens,
                       "kept": wl.total_kept, "d": wl.d, "gate_hidden": wl.h,
                       "heads": f"{wl.hq}/{wl.hkv}", "head_dim": wl.dh,
                       "l2": "flushed between timed steps (512 MB write, then a 256 MB read so that no dirty line is left to write back)",
                       "parallelism": f"replicas x{ws}"},
            "stages": stages,
            "roofline": roofline,
            "gpu_launches": gp.LAUNCHES_PER_STEP * args.steps,
            "stage_sum_us": sum(stage_ms.values()) * 1e3,
            "launch": ("timed steps: the whole layer as one CUDA graph of 4 kernels chained by "
                       "programmatic dependent launch, events around each replay; stage times: "
                       "a second graph with events between the stages"),
            "clocks": clk,
            "e2e": e2e,
            "next_step": next_step,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


_STAGE_SRC = {"gate": "gate.cu", "select": "select.cu", "compact": "compact.cu",
              "attention": "attn.cu", "compact+attention": "attn.cu"}


def _kernel_rev(stage: str) -> str:
    """Hash of one stage's kernel source and the shared header, so DRAM-traffic
    figures are reported only while that kernel is the one they were taken on."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "learned_token_pruning_gemm_b200", "csrc")
    for f in ("common.cuh", _STAGE_SRC[stage]):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen16k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    from learned_token_pruning_gemm_b200.dist import Replicas
    rep = Replicas()
    try:
        if args.impl == "reference":
            run_reference(args, rep)
        else:
            run_ours(args, rep)
    finally:
        rep.close()


if __name__ == "__main__":
    main()
