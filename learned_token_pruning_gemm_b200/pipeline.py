"""One gated layer of the prefill path, end to end on the GPU:
gate scores -> question-protected top-K -> compaction of the residual rows ->
token-gated causal GQA attention over the kept tokens (MarkTechPost page on
TokenGate, section "Comment TokenGate a-t-il appris le fonctionnement de la
réduction des tokens ?").

Two modes. By default the attention inputs q/k/v are supplied already compacted
([K, H, dh], drawn for the kept rows), and only the key scores come from the
selection: this is the measured metric (gate + top-K + attention). With
`project=True` the layer above the gate layer computes them itself: the kept
residual rows' q/k/v projections with the rotary embedding at each kept token's
original position, so the KV entries exist for the kept tokens only, and
attention reads those: tg_compact_kv, then tg_qkv_rope on the compacted rows.
`fuse=True` runs the compaction fused into the projection instead
(tg_compact_qkv_rope gathers the kept rows from the residual itself and writes the
compacted rows on the way): the same outputs bit for bit, but slower on a B200,
because its 16-byte row gathers feed the tensor cores less steadily than TMA
loads of rows that the compaction has already made contiguous.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import api
from .synth import Workload


class GatedPrefill:
    """Device-resident buffers for one workload and a `step()` that runs the stages
    (one kernel launch each)."""

    def __init__(self, wl: Workload, device: str = "cuda", use_score_override: bool = True,
                 project: bool = False, w_qkv: Optional[torch.Tensor] = None,
                 rope_base: float = 1e6, fuse: bool = False):
        dev = torch.device(device)
        self.wl = wl
        self.project = project
        self.rope_base = rope_base
        self.x = wl.x.to(dev)
        self.w1 = wl.w1.to(dev)
        self.b1 = wl.b1.to(dev)
        self.w2 = wl.w2.to(dev)
        self.b2 = float(wl.b2)
        self.gain = wl.gain.to(dev)
        self.tau = wl.tau.to(dev)
        self.q = wl.q.to(dev)
        self.k = wl.k.to(dev)
        self.v = wl.v.to(dev)
        i32 = dict(dtype=torch.int32, device=dev)
        self.cu_seqlens = torch.tensor(wl.cu_seqlens, **i32)
        self.doc_begin = torch.tensor(wl.doc_begin, **i32)
        self.doc_end = torch.tensor(wl.doc_end, **i32)
        self.k_doc = torch.tensor(wl.k_doc, **i32)
        self.override = (wl.score_override.to(dev)
                         if (use_score_override and wl.score_override is not None) else None)
        self.n_tokens = wl.n_tokens
        self.total_kept = wl.total_kept
        self.max_seqlen = max(wl.seqlens)
        self.max_kept = max(wl.kept_counts)
        K = self.total_kept
        self.scores = torch.empty(self.n_tokens, dtype=torch.float32, device=dev)
        self.kept_idx = torch.empty(K, dtype=torch.int32, device=dev)
        self.kept_scores = torch.empty(K, dtype=torch.float32, device=dev)
        self.cu_kept = torch.empty(wl.batch + 1, **i32)
        self.xc = torch.empty((K, wl.d), dtype=self.x.dtype, device=dev)
        self.out = torch.empty_like(self.q)
        if project:
            from .synth import qkv_weights
            self.w_qkv = (w_qkv if w_qkv is not None else qkv_weights(wl)).to(dev)
            self.kept_pos = torch.empty(K, **i32)
            # the kept rows' projections replace the supplied q/k/v
            self.q = torch.empty((K, wl.hq, wl.dh), dtype=self.x.dtype, device=dev)
            self.k = torch.empty((K, wl.hkv, wl.dh), dtype=self.x.dtype, device=dev)
            self.v = torch.empty((K, wl.hkv, wl.dh), dtype=self.x.dtype, device=dev)
        else:
            self.w_qkv = None
            self.kept_pos = None
        self.fuse = project and fuse
        self.STAGES = (("gate", "select", "compact+project", "attention") if self.fuse
                       else ("gate", "select", "compact", "project", "attention") if project
                       else ("gate", "select", "compact", "attention"))
        self.LAUNCHES_PER_STEP = len(self.STAGES)

    def stage_gate(self, stream=None):
        api.gate_score(self.x, self.w1, self.b1, self.w2, self.b2, out=self.scores, stream=stream)

    def stage_select(self, stream=None):
        sel = self.override if self.override is not None else self.scores
        api.select_topk(sel, self.cu_seqlens, self.doc_begin, self.doc_end, self.k_doc,
                        self.total_kept, self.max_seqlen, kept_idx=self.kept_idx,
                        kept_scores=self.kept_scores, cu_kept=self.cu_kept,
                        kept_pos=self.kept_pos, stream=stream)

    def stage_compact(self, stream=None):
        api.compact_rows([self.x], self.kept_idx, outs=[self.xc], stream=stream)

    def stage_project(self, stream=None):
        api.qkv_rope(self.xc, self.w_qkv, self.wl.hq, self.wl.hkv, self.kept_pos,
                     rope_base=self.rope_base, out=(self.q, self.k, self.v), stream=stream)

    def stage_compact_project(self, stream=None):
        api.compact_qkv_rope(self.x, self.kept_idx, self.w_qkv, self.wl.hq, self.wl.hkv,
                             self.kept_pos, rope_base=self.rope_base, xc=self.xc,
                             out=(self.q, self.k, self.v), stream=stream)

    def stage_attention(self, stream=None):
        api.gated_attention(self.q, self.k, self.v, self.kept_scores, self.gain, self.tau,
                            self.cu_kept, self.max_kept, out=self.out, stream=stream)

    def step(self, stream=None, events: Optional[list] = None):
        """Run the stages back to back on one stream (each kernel launched with
        programmatic dependent launch, so its prologue overlaps the previous one's
        tail). If `events` is a list of len(STAGES)+1 CUDA events, they are recorded
        on the stream before, between and after the stages."""
        s = stream if stream is not None else torch.cuda.current_stream()
        fns = [getattr(self, "stage_" + n.replace("+", "_")) for n in self.STAGES]
        for i, fn in enumerate(fns):
            if events is not None:
                events[i].record(s)
            fn(stream=s)
        if events is not None:
            events[len(fns)].record(s)

    # ------------------------------------------------------------------ graphs
    def capture(self):
        """Capture the whole layer as CUDA graphs: one as launched in
        production and one with timing events between the stages. One eager
        step runs first (outside capture) so that every lazily initialised piece of
        the library exists before capture."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step(side)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        # the step as launched in production: kernels back to back, each launched with
        # programmatic dependent launch so its prologue overlaps the previous tail
        self.step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.step_graph):
            self.step()
        # the same step with timing events between the stages (the event nodes turn
        # the programmatic edges into full dependencies; used for the breakdown only)
        self.stage_events = [torch.cuda.Event(enable_timing=True, external=True)
                             for _ in range(len(self.STAGES) + 1)]
        self.timed_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.timed_graph):
            self.step(events=self.stage_events)
        torch.cuda.synchronize()
        return self

    def replay_step(self):
        """Replay the whole layer (one graph, one launch per stage) on the current stream."""
        self.step_graph.replay()

    def replay_timed(self):
        """Replay the step with timing events between the stages."""
        self.timed_graph.replay()

    def stage_times_ms(self):
        """Per-stage device times of the last completed `replay_timed` (sync first)."""
        ev = self.stage_events
        return {n: ev[i].elapsed_time(ev[i + 1]) for i, n in enumerate(self.STAGES)}
