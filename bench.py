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


def _algorithmic_work(wl):
    """Algorithmic work of one step (bytes / flops the method must move / do)."""
    N, d, h, dh, hq = wl.n_tokens, wl.d, wl.h, wl.dh, wl.hq
    esz = 2 if wl.dtype == "bf16" else 4
    Ks = wl.kept_counts
    K = sum(Ks)
    nh = wl.hq + 2 * wl.hkv
    return {
        "gate_bytes": esz * N * d + esz * d * h + 4 * N,
        "gate_flops": 2 * N * d * h,
        "select_bytes": 4 * N + 8 * K,
        "compact_bytes": 2 * K * d * esz,
        "attn_flops": sum(4 * dh * hq * k * (k + 1) // 2 for k in Ks),
        "project_flops": 2 * K * d * nh * dh,
    }


def _oracle_step(wl, oracle):
    """One whole step of the fp64 oracle on the host cores: gate on every row, select,
    gather, and attention on every kept query row and head. Returns (seconds, per-stage
    seconds)."""
    t0 = time.perf_counter()
    _, s32 = oracle.gate_score(wl.x, wl.w1, wl.b1, wl.w2, wl.b2)
    t1 = time.perf_counter()
    sel = wl.score_override.numpy() if wl.score_override is not None else s32
    idx, cu = oracle.select_topk(sel, wl.cu_seqlens, wl.doc_begin, wl.doc_end, wl.k_doc)
    t2 = time.perf_counter()
    oracle.gather_rows(wl.x.view(torch.int16).numpy(), idx)
    t3 = time.perf_counter()
    oracle.gated_attention(wl.q, wl.k, wl.v, sel[idx], wl.gain, wl.tau, cu)
    t4 = time.perf_counter()
    return t4 - t0, {"gate": t1 - t0, "select": t2 - t1, "compact": t3 - t2, "attention": t4 - t3}


def _oracle_warm(wl, oracle):
    """A small untimed pass over the same code (threads started, pages touched)."""
    rows = torch.arange(min(256, wl.n_tokens))
    oracle.gate_score(wl.x[rows], wl.w1, wl.b1, wl.w2, wl.b2)
    cu = np.array([0, min(64, wl.total_kept)], np.int32)
    oracle.gated_attention(wl.q[:cu[1]], wl.k[:cu[1]], wl.v[:cu[1]], np.zeros(cu[1], np.float32),
                           wl.gain, wl.tau, cu)


def _threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_reference(args, rep):
    """The oracle timed as the reference arm (rank 0 only; other ranks exit): each
    timed step is one whole step of the workload (no sampling, no extrapolation)."""
    ws = rep.world
    if rep.rank != 0:
        return
    import oracle
    from learned_token_pruning_gemm_b200 import synth
    oracle.build()
    wl = synth.WORKLOADS[args.workload]()
    for _ in range(args.warmup):
        _oracle_warm(wl, oracle)
    times = [_oracle_step(wl, oracle)[0] for _ in range(args.steps)]
    ms = 1e3 * statistics.mean(times)
    value = wl.n_tokens / (ms / 1e3)
    sample = (f"the whole {args.workload} step ({wl.n_tokens} tokens, K={wl.total_kept}): gate on "
              f"every row, select, gather, attention on every kept row and head; fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "tokens": wl.n_tokens, "kept": wl.total_kept},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _threads(),
                         "cpu_model": _cpu_model(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class _Flush:
    """Evict the inputs from L2 between timed steps: write a buffer larger than L2,
    then read another one, so the lines left behind are clean (otherwise the first
    kernel of the next step pays for writing back the flush buffer's dirty lines)."""

    def __init__(self):
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
        self.clean = torch.ones(L2_CLEAN_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.flush.zero_()
        self.clean.sum()


def _time_layer(gp, steps, warmup, rep, flush, stream, clocks=None):
    """Capture the layer as a CUDA graph, run `warmup` untimed steps, then time exactly
    `steps` steps (CUDA events on the launching stream around each replay, L2 flushed
    before each, outside the events), bracketed by barriers. Then a second pass with
    events between the stages for the per-stage breakdown. Returns (max over ranks of
    the mean step ms, per-stage ms, clock window)."""
    from learned_token_pruning_gemm_b200 import api
    gp.capture()
    for _ in range(warmup):
        flush()
        gp.replay_step()
    torch.cuda.synchronize()
    if api.device_status(reset=True) != 0:
        raise RuntimeError("device status set during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    rep.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for a, b in ev:
        flush()
        a.record(stream)
        gp.replay_step()
        b.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    rep.barrier()
    clk = clocks.window(t0, t1) if clocks is not None else None
    if api.device_status(reset=True) != 0:
        raise RuntimeError("device status set during the timed region")
    step_ms = rep.max(statistics.mean(a.elapsed_time(b) for a, b in ev))
    per = []
    for _ in range(steps):
        flush()
        gp.replay_timed()
        torch.cuda.synchronize()
        per.append(gp.stage_times_ms())
    stage_ms = {n: statistics.mean(p[n] for p in per) for n in gp.STAGES}
    return step_ms, stage_ms, clk


def _stages_report(work, stage_ms, tf_peak, hbm_peak):
    st = {}
    for name, ms in stage_ms.items():
        t = ms / 1e3
        e = {"us": ms * 1e3}
        if name == "gate":
            e["tflops"] = work["gate_flops"] / t / 1e12
            e["gbs"] = work["gate_bytes"] / t / 1e9
        elif name == "select":
            e["gbs"] = work["select_bytes"] / t / 1e9
        elif name == "compact":
            e["gbs"] = work["compact_bytes"] / t / 1e9
        elif name == "attention":
            e["tflops"] = work["attn_flops"] / t / 1e12
        elif name in ("project", "compact+project"):
            e["tflops"] = work["project_flops"] / t / 1e12
        if "tflops" in e:
            e["frac_tc"] = e["tflops"] / tf_peak
        if "gbs" in e:
            e["frac_hbm"] = e["gbs"] / hbm_peak
        st[name] = e
    if "select" in stage_ms and "compact" in stage_ms:
        t = (stage_ms["select"] + stage_ms["compact"]) / 1e3
        st["select+compact"] = {
            "us": t * 1e6,
            "frac_hbm": (work["select_bytes"] + work["compact_bytes"]) / t / 1e9 / hbm_peak}
    return st


def _roofline(work, stage_ms, tf_peak, hbm_peak, peak_src, workload):
    """The dominant kernel of the step against its bound."""
    dom = max((n for n in stage_ms if "project" not in n), key=stage_ms.get)
    t = stage_ms[dom] / 1e3
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
        ent = json.load(open(tpath)).get(workload, {}).get(dom)
        if ent and ent.get("kernel_rev") == _kernel_rev(dom):
            traffic = ent["bytes_per_launch"]
    return {"kernel": dom, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
            "frac": ach / peak, "traffic": traffic, "peak_source": peak_src}


def _time_decode(gp, wl, steps, warmup, rep, flush, stream, hbm_peak):
    """One decode step per sequence over the compacted cache of the measured prefill:
    the kept rows' k, v and scores are the cache (batch-major, capacity K_b + 64); a
    step appends one new token (tg_cache_append) and attends over the cache
    (tg_gated_decode), captured as one CUDA graph (three launches). The cache
    length is reset before every step (outside the events), so every step reads the
    same number of rows."""
    from learned_token_pruning_gemm_b200 import api
    counts = wl.kept_counts
    B, cap = wl.batch, max(counts) + 64
    dev = gp.q.device
    kc = torch.zeros(B, cap, wl.hkv, wl.dh, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    sc = torch.zeros(B, cap, device=dev)
    cu = gp.cu_kept.cpu().tolist()
    for b in range(B):
        n = cu[b + 1] - cu[b]
        kc[b, :n] = gp.k[cu[b]:cu[b + 1]]
        vc[b, :n] = gp.v[cu[b]:cu[b + 1]]
        sc[b, :n] = gp.kept_scores[cu[b]:cu[b + 1]]
    base_len = torch.tensor(counts, dtype=torch.int32, device=dev)
    ln = base_len.clone()
    g = torch.Generator(device="cpu").manual_seed(3)
    qn = torch.randn(B, wl.hq, wl.dh, generator=g).to(torch.bfloat16).to(dev)
    kn = torch.randn(B, wl.hkv, wl.dh, generator=g).to(torch.bfloat16).to(dev)
    vn = torch.randn(B, wl.hkv, wl.dh, generator=g).to(torch.bfloat16).to(dev)
    sn = torch.randn(B, generator=g).to(dev)
    out = torch.empty(B, wl.hq, wl.dh, dtype=torch.bfloat16, device=dev)
    max_len = cap
    ws = torch.empty(api.decode_workspace_size(B, wl.hq, wl.dh, max_len), dtype=torch.uint8,
                     device=dev)

    def step():
        api.cache_append(kn, vn, sn, kc, vc, sc, ln)
        api.gated_decode(qn, kc, vc, sc, ln, gp.gain, gp.tau, max_len, out=out, workspace=ws)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    ln.copy_(base_len)
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        ln.copy_(base_len)
        flush()
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    rep.barrier()
    for a, b in ev:
        ln.copy_(base_len)
        flush()
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    rep.barrier()
    if api.device_status(reset=True) != 0:
        raise RuntimeError("device status set by the decode step")
    ms = rep.max(statistics.mean(a.elapsed_time(b) for a, b in ev))
    rows = sum(counts) + B
    nbytes = rows * wl.hkv * wl.dh * 2 * 2 + rows * 4 + 2 * B * wl.hq * wl.dh * 2
    return {"us": ms * 1e3, "tokens_per_s": B / (ms / 1e3), "batch": B,
            "cache_rows": rows, "gbs": nbytes / (ms / 1e3) / 1e9,
            "frac_hbm": nbytes / (ms / 1e3) / 1e9 / hbm_peak, "launches_per_step": 3,
            "note": "append + split-KV decode + combine, one CUDA graph; bytes = the cache's "
                    "K, V and scores read once, q and out"}


def _time_backward(gp, wl, steps, warmup, rep, flush, stream, tf_peak):
    """The backward of the gated attention on the measured layer's kept rows: the
    forward once (with its log-sum-exp), then `steps` backward calls for a seeded
    upstream gradient, captured as one CUDA graph (five launches), L2 flushed before
    each. Algorithmic flops: the five causal contractions S, dP, dV, dK, dQ, i.e.
    2.5 times the forward's."""
    from learned_token_pruning_gemm_b200 import api
    K = gp.total_kept
    lse = torch.empty(wl.hq, K, device=gp.q.device)
    out = api.gated_attention(gp.q, gp.k, gp.v, gp.kept_scores, gp.gain, gp.tau, gp.cu_kept,
                              gp.max_kept, lse=lse)
    g = torch.Generator(device="cpu").manual_seed(9)
    dout = torch.randn(out.shape, generator=g).to(out.dtype).to(out.device)
    grads = api.gated_attention_bwd(gp.q, gp.k, gp.v, out, dout, lse, gp.kept_scores, gp.gain,
                                    gp.tau, gp.cu_kept, gp.max_kept)
    need = api._lib.load().tg_gated_attention_bwd_workspace_size(1, wl.batch, K, gp.max_kept,
                                                                  wl.hq, wl.hkv, wl.dh)
    ws = torch.empty(need, dtype=torch.uint8, device=gp.q.device)

    def step():
        api.gated_attention_bwd(gp.q, gp.k, gp.v, out, dout, lse, gp.kept_scores, gp.gain,
                                gp.tau, gp.cu_kept, gp.max_kept, grads=grads, workspace=ws)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    rep.barrier()
    for a, b in ev:
        flush()
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    rep.barrier()
    if api.device_status(reset=True) != 0:
        raise RuntimeError("device status set by the backward")
    ms = rep.max(statistics.mean(a.elapsed_time(b) for a, b in ev))
    flops = 2.5 * _algorithmic_work(wl)["attn_flops"]
    return {"us": ms * 1e3, "tflops": flops / (ms / 1e3) / 1e12,
            "frac_tc": flops / (ms / 1e3) / 1e12 / tf_peak, "launches_per_step": 5,
            "note": "dQ, dK, dV, score, gain and temperature gradients; flops = 2.5 x the "
                    "forward's causal flops (S, dP, dV, dK, dQ)"}


def _time_deltanet(gp, wl, steps, warmup, rep, flush, stream, tf_peak, hbm_peak):
    """A Gated DeltaNet layer's gated delta rule over the layer's kept rows (row f3):
    the workload's seeded DeltaNet inputs, one call (two launches) per step in a CUDA
    graph, L2 flushed before each. The rule is computed in 64-token chunks: a parallel
    per-chunk pass, then each sequence's chunks in order, so its time is set by that
    chain of chunk steps, not by bytes or tensor throughput. Reported: the rule's
    algorithmic flops (6 dk dv per token and head: k.s, the update, q.s) against the
    bf16 tensor peak, its algorithmic bytes (q, k, v, alpha, beta read, out written)
    against the HBM peak, and the time per chunk step."""
    from learned_token_pruning_gemm_b200 import api, synth
    q, k, v, a, b = (t.to(gp.q.device) for t in synth.deltanet_inputs(wl))
    cu = gp.cu_kept
    out = torch.empty_like(v)
    max_len = max(wl.kept_counts)
    ws = torch.empty(api.gated_delta_rule_workspace_size(wl.batch, q.shape[0], q.shape[1],
                                                         v.shape[2]), dtype=torch.uint8,
                     device=q.device)

    def step():
        api.gated_delta_rule(q, k, v, a, b, cu, max_len, out=out, workspace=ws)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    rep.barrier()
    for e0, e1 in ev:
        flush()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    rep.barrier()
    if api.device_status(reset=True) != 0:
        raise RuntimeError("device status set by the delta rule")
    ms = rep.max(statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev))
    K, H, d = q.shape
    dv = v.shape[2]
    flops = 6.0 * K * H * d * dv
    nbytes = K * H * (2 * d + 2 * dv) * 2 + K * H * 8   # q, k, v, out (bf16); alpha, beta
    chunks = max((n + 63) // 64 for n in wl.kept_counts)
    tflops = flops / (ms / 1e3) / 1e12
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"us": ms * 1e3, "tokens_per_s": K / (ms / 1e3), "tflops": tflops,
            "frac_tensor": tflops / tf_peak, "gbs": gbs, "frac_hbm": gbs / hbm_peak,
            "bound": "sequential chunk steps", "chunk_steps": chunks,
            "us_per_chunk_step": ms * 1e3 / chunks, "launches_per_step": 2,
            "note": "chunked gated delta rule: per-chunk pass (T = (I + A)^-1, W, U~, masked "
                    "Q K^T) in parallel, then each sequence's 64-token chunks in order with "
                    "the state; mma.sync with split bf16 operands"}


def run_ours(args, rep):
    ws, rank = rep.world, rep.rank
    from learned_token_pruning_gemm_b200 import pipeline, synth
    dev_index = torch.cuda.current_device()
    stream = torch.cuda.current_stream()
    flush = _Flush()
    peaks, peak_src = _peaks()
    tf_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])

    wl = synth.WORKLOADS[args.workload]()
    gp = pipeline.GatedPrefill(wl)
    work = _algorithmic_work(wl)
    clocks = ClockSampler(dev_index)
    clocks.start()
    ms, stage_ms, clk = _time_layer(gp, args.steps, args.warmup, rep, flush, stream, clocks)
    value = ws * wl.n_tokens / (ms / 1e3)
    stages = _stages_report(work, stage_ms, tf_peak, hbm_peak)
    roofline = _roofline(work, stage_ms, tf_peak, hbm_peak, peak_src, args.workload)

    # ---- the same layer with the kept rows' q/k/v projections computed on the path
    #      (rotary embedding at each kept token's position): the KV entries of the
    #      layer above the gate exist for the kept tokens only ----
    with_proj = None
    if wl.dtype == "bf16" and wl.dh == 128 and (wl.hq + 2 * wl.hkv) % 2 == 0:
        gpp = pipeline.GatedPrefill(wl, project=True)
        pms, pstage, _ = _time_layer(gpp, args.steps, args.warmup, rep, flush, stream)
        with_proj = {"value": ws * wl.n_tokens / (pms / 1e3), "unit": "tokens/s",
                     "ms_per_step": pms, "launches_per_step": gpp.LAUNCHES_PER_STEP,
                     "stages": _stages_report(work, pstage, tf_peak, hbm_peak)}
        del gpp

    # ---- decode over the compacted cache the prefill leaves (one new token per
    #      sequence: append its k/v/score, then attend over the cache) ----
    decode = None
    if wl.dtype == "bf16" and wl.dh == 128 and not args.no_decode:
        decode = _time_decode(gp, wl, args.steps, args.warmup, rep, flush, stream, hbm_peak)

    deltanet = None
    if wl.dtype == "bf16" and wl.dh == 128 and not args.no_deltanet:
        deltanet = _time_deltanet(gp, wl, args.steps, args.warmup, rep, flush, stream, tf_peak,
                                  hbm_peak)

    backward = None
    if wl.dtype == "bf16" and wl.dh == 128 and not args.no_backward:
        backward = _time_backward(gp, wl, args.steps, args.warmup, rep, flush, stream, tf_peak)

    # ---- the other single-GPU workloads of the metric (16k-128k): same measurement ----
    others = {}
    for name in ([] if args.no_extra_workloads else args.extra_workloads.split(",")):
        if not name or name == args.workload:
            continue
        owl = synth.WORKLOADS[name]()
        ogp = pipeline.GatedPrefill(owl)
        owork = _algorithmic_work(owl)
        oms, ostage, _ = _time_layer(ogp, args.steps, args.warmup, rep, flush, stream)
        others[name] = {
            "value": ws * owl.n_tokens / (oms / 1e3), "unit": "tokens/s", "ms_per_step": oms,
            "tokens": owl.n_tokens, "kept": owl.total_kept, "batch": owl.batch,
            "stages": _stages_report(owork, ostage, tf_peak, hbm_peak),
            "roofline": _roofline(owork, ostage, tf_peak, hbm_peak, peak_src, name)}
        if not args.no_decode and owl.dtype == "bf16" and owl.dh == 128:
            others[name]["decode"] = _time_decode(ogp, owl, args.steps, args.warmup, rep, flush,
                                                  stream, hbm_peak)
        if not args.no_backward and owl.dtype == "bf16" and owl.dh == 128:
            others[name]["backward"] = _time_backward(ogp, owl, args.steps, args.warmup, rep, flush,
                                                      stream, tf_peak)
        del ogp, owl
        torch.cuda.empty_cache()
    clocks.stop()

    # ---- e2e: host buffers in, result out, through the same public calls. Steps are
    #      pipelined as a serving loop runs them: two device buffer sets (the layer
    #      captured twice), the upload of step i+1's inputs (pinned host -> device, one
    #      stream) under step i's compute (another), and the read-back of step i's
    #      result (device -> pinned host, a third stream, the other PCIe direction);
    #      every step's copies lie inside the timed region, which spans all K steps ----
    e2e = None
    if not args.no_e2e:
        host_in = [t.pin_memory() for t in (wl.x, wl.q, wl.k, wl.v)]
        gps = [gp, pipeline.GatedPrefill(wl).capture()]
        host_out = [torch.empty(gp.out.shape, dtype=gp.out.dtype).pin_memory() for _ in range(2)]
        host_idx = [torch.empty(gp.kept_idx.shape, dtype=torch.int32).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = host_out[0].numel() * host_out[0].element_size() + host_idx[0].numel() * 4
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        loaded = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        freed = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                j, g = i % 2, gps[i % 2]
                if i >= 2:   # buffer set j: step i-2's read-back (so its compute) is done
                    up.wait_event(freed[j])
                with torch.cuda.stream(up):
                    for hsrc, dst in zip(host_in, (g.x, g.q, g.k, g.v)):
                        dst.copy_(hsrc, non_blocking=True)
                    loaded[j].record(up)
                stream.wait_event(loaded[j])
                with torch.cuda.stream(stream):
                    g.replay_step()
                    computed[j].record(stream)
                down.wait_event(computed[j])
                with torch.cuda.stream(down):
                    host_out[j].copy_(g.out, non_blocking=True)
                    host_idx[j].copy_(g.kept_idx, non_blocking=True)
                    freed[j].record(down)
            stream.wait_stream(down)
            stream.wait_stream(up)

        torch.cuda.synchronize()
        e2e_steps(max(2, args.warmup))
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        rep.barrier()
        t0.record(stream)
        up.wait_stream(stream)
        e2e_steps(args.steps)
        t1.record(stream)
        torch.cuda.synchronize()
        rep.barrier()
        e_ms = rep.max(t0.elapsed_time(t1) / args.steps)
        e2e = {"value": ws * wl.n_tokens / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "pipelined": "two buffer sets; step i+1's upload under step i's compute and "
                            "read-back; all K steps timed as one span"}
        del gps[1]

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        _oracle_warm(wl, oracle)
        t_cpu, parts = _oracle_step(wl, oracle)
        cpu = {"value": wl.n_tokens / t_cpu, "unit": "tokens/s", "cores": _threads(),
               "cpu_model": _cpu_model(), "kind": "oracle",
               "sample": (f"one whole {args.workload} step timed once: gate on all "
                          f"{wl.n_tokens} rows, select, gather, attention on all {wl.total_kept} "
                          f"kept rows x {wl.hq} heads (fp64, OpenMP over the host cores)"),
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
            "launch": (f"timed steps: the whole layer as one CUDA graph of {gp.LAUNCHES_PER_STEP} "
                       "kernels chained by programmatic dependent launch, events around each "
                       "replay; stage times: a second graph with events between the stages"),
            "clocks": clk,
            "e2e": e2e,
            "with_projection": with_proj,
            "decode": decode,
            "backward": backward,
            "deltanet": deltanet,
            "workloads": others,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


_STAGE_SRC = {"gate": "gate.cu", "select": "select.cu", "compact": "compact.cu",
              "attention": "attn.cu", "project": "qkv.cu"}


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
    ap.add_argument("--extra-workloads", default="long128k,ragged8",
                    help="other workloads measured the same way, reported under 'workloads'")
    ap.add_argument("--no-extra-workloads", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-deltanet", action="store_true")
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
