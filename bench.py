#!/usr/bin/env python
"""Benchmark of the sink-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one "step" = one call over one batch of synthetic input): SWA sink-attention
prefill at model width, B=2, L=32768, 64 Q / 8 KV heads, d_qk=192, d_v=128, W=128. Metric:
attention TFLOP/s counting only the band-limited (visible) pairs at 640 FLOP per (row, head,
key), with its roofline fraction. The other workloads (GA prefill, GA chunked prefill, the fused
RoPE + value-scale pass over the headline Q/K/V, GA decode with a bf16 and with an FP8 cache,
SWA decode, the hybrid
speculative-verify step) are measured after it and reported under "secondary".

With N > 1 (torchrun) every rank runs the same per-GPU workload on its own GPU (independent
batches, no collective on the data path: weak scaling); time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method has) on a bounded
sample of the same workload, on the host cores; under torchrun only rank 0 runs it.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from global_attention_sink_softmax_b200 import workloads as W  # noqa: E402

METRIC = "prefill attn TFLOP/s and decode KV GB/s on 1 B200, as % of roofline"
FLOP_PER_PAIR = 2 * (W.DQ + W.DV)
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------------------------
# algorithmic counts
# ----------------------------------------------------------------------------------------------

def visible_pairs_prefill(L: int, window: int) -> int:
    """sum over rows i of the number of visible keys (min(i+1, W) or i+1)."""
    if window <= 0 or window >= L:
        return L * (L + 1) // 2
    return window * L - window * (window - 1) // 2


def prefill_counts(w, L=None, B=None):
    L = w.L if L is None else L
    B = w.B if B is None else B
    P = w.prefix
    # a chunk after P cached positions: rows P .. P+L-1 of the whole sequence's pairs
    pairs = B * w.Hq * (visible_pairs_prefill(P + L, w.window) - visible_pairs_prefill(P, w.window))
    flops = pairs * FLOP_PER_PAIR
    nbytes = (B * L * (w.Hq * w.dq + w.Hq * w.dv) * 2 + B * (P + L) * w.Hkv * (w.dq + w.dv) * 2
              + B * w.Hq * L * 4)
    return flops, nbytes


def decode_counts(w, d):
    """FLOPs over visible (query row, key) pairs; bytes = cache KV read once per (seq, KV head),
    new K/V, Q, O, LSE."""
    T, G = w.T, w.Hq // w.Hkv
    if w.kind == W.KV_RING:
        n_cache = d["ring_len"].clamp(max=w.ring_cap).to(torch.int64)
    else:
        n_cache = d["ctx_len"].to(torch.int64)
    if w.window > 0:
        n_used = n_cache.clamp(max=w.window - 1)
    else:
        n_used = n_cache
    pairs = 0
    for t in range(T):
        if w.window > 0:
            vis = n_used.clamp(max=max(0, w.window - 1 - t)) + min(t + 1, w.window)
        else:
            vis = n_used + (t + 1)
        pairs += int(vis.sum()) * w.Hq
    flops = pairs * FLOP_PER_PAIR
    kv_row = w.Hkv * (w.dq + w.dv) * 2
    cache_row = w.Hkv * (w.dq + w.dv) * d["k_cache"].element_size()  # 1 byte for an FP8 cache
    nbytes = int(n_used.sum()) * cache_row
    nbytes += w.B * T * (kv_row + w.Hq * (w.dq + w.dv) * 2 + w.Hq * 4)
    return flops, nbytes


# ----------------------------------------------------------------------------------------------
# runners (ours)
# ----------------------------------------------------------------------------------------------

class PrefillRunner:
    def __init__(self, w, dev, fused_rope=False):
        import global_attention_sink_softmax_b200 as sa
        self.sa, self.w, self.dev = sa, w, dev
        self.fused_rope = fused_rope
        self.d = W.prefill_inputs(w, device=dev, L=w.prefix + w.L)
        if w.prefix:
            self.d["q"] = self.d["q"][:, w.prefix:]  # the chunk's queries (a strided view)
        self.o = torch.empty(w.B, w.L, w.Hq, w.dv, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(w.B, w.Hq, w.L, dtype=torch.float32, device=dev)
        self.flops, self.bytes = prefill_counts(w)
        self.launches = 1
        # the kernel the library dispatches this workload to
        packed = w.window > 0 and w.Hq // w.Hkv == 8 and w.window <= 128 and w.prefix == 0
        self.kernel = ("prefill_swa_packed_kernel" if packed else
                       "prefill_wide_kernel" if w.window == 0 else "prefill_band_kernel")
        self.workload = w.name
        self.config = dict(B=w.B, L=w.L, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.dq, d_v=w.dv,
                           window=w.window, kind="SWA" if w.window else "GA")
        if w.prefix:
            self.config["prefix"] = w.prefix
        if fused_rope:
            # the SWA layers' partial RoPE (64 dims, theta 1e4) and value scale, in the loads
            self.workload = w.name + "_fused_rope"
            self.config.update(rope_dim=sa.ROPE_DIM, theta=sa.ROPE_THETA_SWA, v_scale=sa.V_SCALE)
        self.in_bytes = sum(self.d[k].numel() * self.d[k].element_size() for k in self.d)

    def step(self):
        d, w = self.d, self.w
        if self.fused_rope:
            self.sa.sinkattn_prefill_swa_rope(d["q"], d["k"], d["v"], d["sink"], w.window,
                                              theta=self.sa.ROPE_THETA_SWA, o=self.o, lse=self.lse)
        elif w.prefix:
            self.sa.sinkattn_prefill_chunk(d["q"], d["k"], d["v"], d["sink"], prefix=w.prefix,
                                           window=w.window, o=self.o, lse=self.lse)
        elif w.window:
            self.sa.sinkattn_prefill_swa(d["q"], d["k"], d["v"], d["sink"], w.window, o=self.o,
                                         lse=self.lse)
        else:
            self.sa.sinkattn_prefill_ga(d["q"], d["k"], d["v"], d["sink"], o=self.o, lse=self.lse)

    # end to end through the host-resident call: pinned host Q / K / V in, O / LSE back to
    # pinned host memory, copies in both directions overlapping the kernels chunk by chunk
    def e2e_setup(self):
        self.h_in = {k: self.d[k].cpu().pin_memory() for k in ("q", "k", "v")}
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h_lse = torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()
        h = self.h_in
        need = self.sa.sinkattn_prefill_host_workspace_size(h["q"], h["k"], h["v"])
        self.ws = torch.empty(need, dtype=torch.uint8, device=self.dev)
        self.h2d = sum(v.numel() * v.element_size() for v in self.h_in.values())
        self.d2h = self.h_o.numel() * 2 + self.h_lse.numel() * 4
        self.e2e_api = "sinkattn_prefill_host"

    def e2e_step(self):
        h = self.h_in
        self.sa.sinkattn_prefill_host(h["q"], h["k"], h["v"], self.d["sink"], window=self.w.window,
                                      o=self.h_o, lse=self.h_lse, workspace=self.ws)

    def release(self):
        for k in ("d", "o", "lse", "h_in", "ws", "h_o", "h_lse"):
            if hasattr(self, k):
                delattr(self, k)


class DecodeRunner:
    def __init__(self, w, dev, d=None):
        import global_attention_sink_softmax_b200 as sa
        self.sa, self.w, self.dev = sa, w, dev
        self.d = W.decode_inputs(w, device=dev) if d is None else d
        d = self.d
        self.o = torch.empty(w.B, w.T, w.Hq, w.dv, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(w.B, w.T, w.Hq, dtype=torch.float32, device=dev)
        self.kw = dict(window=w.window)
        if w.kind == W.KV_RING:
            self.kw.update(ring_head=d["ring_head"], ring_len=d["ring_len"])
        else:
            self.kw.update(ctx_len=d["ctx_len"], max_ctx=d["max_ctx"])
        if w.kind == W.KV_PAGED:
            self.kw.update(page_table=d["page_table"])
        fp8 = "k_scale" in d
        need = sa.sinkattn_decode_workspace_size(w.kind, d["q"], d["k_new"], d["v_new"],
                                                 d["k_cache"], d["v_cache"], **self.kw)
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        self.launches = 1 if need == 0 else 2
        # the kernel the library dispatches this workload to
        if fp8:
            self.kw.update(k_scale=d["k_scale"], v_scale=d["v_scale"])
        rows = w.T * (w.Hq // w.Hkv)
        if fp8:
            # whole 64-key tiles of codes by TMA (contiguous, pages of a multiple of 64 tokens
            # without a window, one-span rings of a multiple of 64 slots), else cp.async
            tma = (w.kind == W.KV_CONTIG or (w.kind == W.KV_PAGED and w.window == 0 and
                                             w.page_size % 64 == 0) or
                   (w.kind == W.KV_RING and w.ring_cap % 64 == 0))
            self.kernel = "decode_fp8_tma_kernel" if tma else "decode_fp8_kernel"
        elif w.kind == W.KV_RING:
            if w.ring_cap == 128 and w.Hq // w.Hkv == 8 and w.T <= 4:
                self.kernel = "decode_ring_umma_kernel"
            elif rows <= 16 and w.ring_cap % 32 == 0:
                self.kernel = "decode_ring_kernel"
            else:
                self.kernel = "decode_split_kernel"
        elif w.kind == W.KV_PAGED and w.page_size % 64 != 0:
            self.kernel = "decode_split_kernel"
        else:
            self.kernel = "decode_umma_kernel" if rows > 16 else "decode_tma_kernel"
        self.flops, self.bytes = decode_counts(w, d)
        self.workload = w.name
        self.config = dict(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.dq, d_v=w.dv,
                           window=w.window, cache=["ring", "contiguous", "paged"][w.kind])
        if fp8:
            self.config.update(cache_dtype="fp8_e4m3", k_scale=d["k_scale"], v_scale=d["v_scale"])
            self.workload = w.name + "_fp8"

    def step(self):
        d = self.d
        self.sa.sinkattn_decode(self.w.kind, d["q"], d["k_new"], d["v_new"], d["k_cache"],
                                d["v_cache"], d["sink"], o=self.o, lse=self.lse,
                                workspace=self.ws, **self.kw)

    def release(self):
        for k in ("d", "o", "lse", "ws", "kw"):
            if hasattr(self, k):
                delattr(self, k)


class RopeRunner:
    """The fused partial-RoPE + value-scale pass (in place) over a prefill workload's Q, K, V:
    the step the attention module runs just before the attention core."""

    ROPE_DIM = 64

    def __init__(self, w, dev, theta):
        import global_attention_sink_softmax_b200 as sa
        self.sa, self.w, self.theta = sa, w, theta
        self.d = W.prefill_inputs(w, device=dev)
        ntok = w.B * w.L
        # read + write of the rotary part of every Q / K head and of all of V, bf16
        self.bytes = 2 * ntok * ((w.Hq + w.Hkv) * self.ROPE_DIM * 2 + w.Hkv * w.dv * 2)
        # 6 FLOP per rotated pair, 1 per scaled value
        self.flops = ntok * ((w.Hq + w.Hkv) * (self.ROPE_DIM // 2) * 6 + w.Hkv * w.dv)
        self.launches = 1
        self.kernel = "rope_qkv_kernel"
        self.workload = "rope_vscale_" + w.name
        self.config = dict(B=w.B, L=w.L, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.dq, d_v=w.dv,
                           rope_dim=self.ROPE_DIM, theta=theta, v_scale=sa.V_SCALE,
                           in_place=True)

    def step(self):
        d = self.d
        self.sa.sinkattn_rope_qkv(d["q"], d["k"], d["v"], theta=self.theta)

    def release(self):
        if hasattr(self, "d"):
            del self.d


class BackwardRunner:
    """The prefill backward (the training variant) on a prefill workload: the forward runs once
    to give O and LSE, then each step computes dq, dk, dv and dsink from dout. Algorithmic FLOPs
    per visible (row, head, key) pair: 2 (d_qk + d_qk + d_qk + d_v + d_v) = 1664 (S recomputed
    once, dP, dV, dK, dQ); bytes: q, k, v, o, dout and LSE read once, the fp32 gradients written
    once."""

    FLOP_PER_PAIR = 2 * (3 * W.DQ + 2 * W.DV)

    def __init__(self, w, dev):
        import global_attention_sink_softmax_b200 as sa
        self.sa, self.w = sa, w
        d = W.prefill_inputs(w, device=dev)
        self.q, self.k, self.v, self.sink = d["q"], d["k"], d["v"], d["sink"]
        if w.window:
            self.o, self.lse = sa.sinkattn_prefill_swa(self.q, self.k, self.v, self.sink, w.window)
        else:
            self.o, self.lse = sa.sinkattn_prefill_ga(self.q, self.k, self.v, self.sink)
        g = torch.Generator(device=dev).manual_seed(w.seed + 7)
        self.dout = torch.randn(self.o.shape, generator=g, device=dev).to(torch.bfloat16)
        f32 = dict(dtype=torch.float32, device=dev)
        self.dq = torch.empty(w.B, w.L, w.Hq, w.dq, **f32)
        self.dk = torch.empty(w.B, w.L, w.Hkv, w.dq, **f32)
        self.dv = torch.empty(w.B, w.L, w.Hkv, w.dv, **f32)
        self.dsink = torch.empty(w.Hq, **f32)
        self.ws = torch.empty(w.B * w.Hq * w.L * 4, dtype=torch.uint8, device=dev)
        pairs = w.B * w.Hq * visible_pairs_prefill(w.L, w.window)
        self.flops = pairs * self.FLOP_PER_PAIR
        bf16 = 2 * w.B * w.L * (w.Hq * w.dq + w.Hkv * (w.dq + w.dv) + 2 * w.Hq * w.dv)
        self.bytes = bf16 + 4 * w.B * w.Hq * w.L + 4 * w.B * w.L * (w.Hq * w.dq + w.Hkv * (w.dq + w.dv))
        self.launches = 4  # dsink clear, delta, dK / dV, dQ
        self.kernel = None
        self.workload = w.name + "_backward"
        self.config = dict(B=w.B, L=w.L, Hq=w.Hq, Hkv=w.Hkv, d_qk=w.dq, d_v=w.dv,
                           window=w.window, kind=("SWA" if w.window else "GA") + " backward",
                           grads="fp32")

    def step(self):
        self.sa.sinkattn_prefill_backward(self.q, self.k, self.v, self.o, self.lse, self.dout,
                                          self.sink, window=self.w.window, dq=self.dq, dk=self.dk,
                                          dv=self.dv, dsink=self.dsink, workspace=self.ws)

    def release(self):
        for k in ("q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv", "ws", "sink", "dsink"):
            if hasattr(self, k):
                delattr(self, k)


def graph_of(fn):
    """fn's launches captured once into a CUDA graph (after two plain calls that do the one-time
    setup: function attributes, device queries). A decode step of many short layer calls issued
    one by one from Python is bound by the host's call overhead (~25 us a call against ~15 us of
    GPU time for an SWA layer); a serving loop replays the step as one graph, as here."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


class HybridRunner:
    """One speculative-verify step of the hybrid stack: every layer's decode call in order, the
    49 calls replayed as one CUDA graph."""

    def __init__(self, dev):
        self.layers = [DecodeRunner(W.hybrid_layer_workload(i), dev)
                       for i in range(len(W.HYBRID_LAYERS))]
        self.graph = graph_of(self.eager_step)
        self.flops = sum(r.flops for r in self.layers)
        self.bytes = sum(r.bytes for r in self.layers)
        self.ga_bytes = sum(r.bytes for r in self.layers if r.w.kind != W.KV_RING)
        self.launches = sum(r.launches for r in self.layers)
        self.workload = "hybrid_verify_b64_t4_49layers"
        self.config = dict(B=W.HYBRID_B, T=W.HYBRID_T, layers=len(W.HYBRID_LAYERS),
                           ga_layers=W.HYBRID_LAYERS.count("GA"),
                           swa_layers=W.HYBRID_LAYERS.count("SWA"),
                           ctx_range=[W.HYBRID_CTX_LO, W.HYBRID_CTX_HI], cuda_graph=True)

    def eager_step(self):
        for r in self.layers:
            r.step()

    def step(self):
        self.graph.replay()

    def kind_runner(self, ring):
        """The GA (ring=False) or SWA (ring=True) layers alone, for a per-kind breakdown (also
        one CUDA graph per step)."""
        sel = [r for r in self.layers if (r.w.kind == W.KV_RING) == ring]

        def eager():
            for r in sel:
                r.step()
        graph = graph_of(eager)
        self.sub_graphs = getattr(self, "sub_graphs", []) + [graph]

        class Sub:
            flops = sum(r.flops for r in sel)
            bytes = sum(r.bytes for r in sel)
            launches = sum(r.launches for r in sel)

            @staticmethod
            def step():
                graph.replay()
        return Sub

    def release(self):
        self.graph = None
        self.sub_graphs = []
        for r in self.layers:
            r.release()
        self.layers = []


# ----------------------------------------------------------------------------------------------
# timing
# ----------------------------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.path = index, None, None

    def __enter__(self):
        try:
            self.path = os.path.join("/tmp", f"sinkattn_clocks_{os.getpid()}.csv")
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def flush_l2(buf):
    if buf is not None:
        buf.add_(1)


def time_steps(fn, steps, warmup, flush=None):
    """CUDA-event time of `steps` calls of fn on the current stream (ms total)."""
    for _ in range(warmup):
        flush_l2(flush)
        fn()
    torch.cuda.synchronize()
    if flush is None:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            fn()
        end.record()
        torch.cuda.synchronize()
        return start.elapsed_time(end)
    total = 0.0
    for _ in range(steps):
        flush_l2(flush)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        total += s.elapsed_time(e)
    return total


def max_over_ranks(x: float) -> float:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def measured_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu table, or None when the kernel's
    sources changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    entry = json.load(open(path)).get(kernel)
    if not entry or entry.get("bytes_per_launch") is None:
        return None
    csrc = os.path.join(ROOT, "global_attention_sink_softmax_b200", "csrc")
    files = {"prefill_swa_packed_kernel": ["common.cuh", "swa_kernels.cuh"],
             "prefill_band_kernel": ["common.cuh", "prefill_kernels.cuh"],
             "prefill_wide_kernel": ["common.cuh", "prefill_kernels.cuh",
                                     "prefill_wide_kernels.cuh"],
             "decode_split_kernel": ["common.cuh", "decode_kernels.cuh"],
             "decode_tma_kernel": ["common.cuh", "decode_kernels.cuh",
                                   "decode_tma_kernels.cuh"],
             "decode_umma_kernel": ["common.cuh", "decode_kernels.cuh",
                                    "decode_tma_kernels.cuh", "decode_umma_kernels.cuh"],
             "decode_ring_kernel": ["common.cuh", "decode_kernels.cuh",
                                    "decode_ring_kernels.cuh"],
             "decode_ring_umma_kernel": ["common.cuh", "decode_ring_umma_kernels.cuh"],
             "rope_qkv_kernel": ["common.cuh", "rope_kernels.cuh"],
             "decode_fp8_kernel": ["common.cuh", "decode_kernels.cuh",
                                   "decode_fp8_kernels.cuh"],
             "decode_fp8_tma_kernel": ["common.cuh", "decode_kernels.cuh",
                                       "decode_tma_kernels.cuh", "decode_fp8_kernels.cuh",
                                       "decode_fp8_tma_kernels.cuh"]}.get(kernel)
    if files is None:
        return None
    m = hashlib.sha256()
    for f in files:
        m.update(open(os.path.join(csrc, f), "rb").read())
    return entry["bytes_per_launch"] if m.hexdigest() == entry.get("source_sha256") else None


def roofline(runner, ms_per_launch, peaks, source, bound=None):
    ai = runner.flops / max(1, runner.bytes)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = bound or ("tensor" if ai > ridge else "hbm")
    if bound == "tensor":
        achieved = runner.flops / (ms_per_launch * 1e-3) / 1e12
        peak, unit = peaks["bf16_tflops"], "TFLOP/s"
    else:
        achieved = runner.bytes / (ms_per_launch * 1e-3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    kernel = getattr(runner, "kernel", None)
    traffic = measured_traffic(kernel) if kernel else None
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
            "peak_source": source, "algorithmic_flops": runner.flops,
            "algorithmic_bytes": runner.bytes}


# ----------------------------------------------------------------------------------------------
# CPU baseline (the fp64 oracle on a bounded sample)
# ----------------------------------------------------------------------------------------------

def oracle_prefill_sample(w, d_cpu, n_rows, seed=0):
    import oracle
    g = torch.Generator().manual_seed(seed)
    rows = torch.stack([torch.randint(0, w.B, (n_rows,), generator=g),
                        torch.randint(0, w.L, (n_rows,), generator=g)], 1)
    t0 = time.perf_counter()
    oracle.prefill(d_cpu["q"], d_cpu["k"], d_cpu["v"], d_cpu["sink"], W.SCALE, w.window,
                   rows=rows)
    dt = time.perf_counter() - t0
    pairs = 0
    for i in rows[:, 1].tolist():
        pairs += (min(i + 1, w.window) if w.window else i + 1) * w.Hq
    return pairs * FLOP_PER_PAIR, dt


def omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_prefill(w, d_cpu, target_s=12.0):
    """Times the oracle on a row sample sized for about target_s seconds of CPU work."""
    n = 256
    flops, dt = oracle_prefill_sample(w, d_cpu, n)
    n = max(n, min(1 << 22, int(n * target_s / max(dt, 1e-3))))
    flops, dt = oracle_prefill_sample(w, d_cpu, n, seed=n)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": omp_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"{n} random (batch, position) rows x all {w.Hq} heads of {w.name}",
            "full_workload_s_extrapolated": round(prefill_counts(w)[0] / (flops / dt), 3)}


def _cpu(t):
    return t.cpu() if isinstance(t, torch.Tensor) else t


def cpu_oracle_sample(kind, w, d, n, seed=0):
    """One timed oracle call on a sample of size n of a secondary workload (inputs on any
    device; only the sample is copied to the host). Returns (work, seconds, what) where work is
    FLOPs for prefill and bytes (the job's algorithmic bytes per unit) otherwise."""
    import oracle
    g = torch.Generator().manual_seed(seed)
    if kind == "prefill":
        P = getattr(w, "prefix", 0)
        q = d["q"]
        if P:  # the chunk's queries sit at positions P.. of sequences of P + L positions
            qf = torch.zeros((w.B, P + w.L) + tuple(q.shape[2:]), dtype=q.dtype)
            qf[:, P:] = _cpu(q)
        else:
            qf = _cpu(q)
        rows = torch.stack([torch.randint(0, w.B, (n,), generator=g),
                            P + torch.randint(0, w.L, (n,), generator=g)], 1)
        t0 = time.perf_counter()
        oracle.prefill(qf, _cpu(d["k"]), _cpu(d["v"]), _cpu(d["sink"]), W.SCALE, w.window,
                       rows=rows)
        dt = time.perf_counter() - t0
        pairs = sum((min(i + 1, w.window) if w.window else i + 1) for i in rows[:, 1].tolist())
        return pairs * w.Hq * FLOP_PER_PAIR, dt, f"{n} random (batch, position) rows x {w.Hq} heads"
    if kind == "rope":
        b = torch.randint(0, w.B, (n,), generator=g)
        l = torch.randint(0, w.L, (n,), generator=g)
        qs, ks, vs = _cpu(d["q"][b, l]), _cpu(d["k"][b, l]), _cpu(d["v"][b, l])
        t0 = time.perf_counter()
        oracle.rope(qs, l.numpy(), 1e4)
        oracle.rope(ks, l.numpy(), 1e4)
        oracle.vscale(vs, 0.707)
        dt = time.perf_counter() - t0
        per_tok = 2 * ((w.Hq + w.Hkv) * 64 * 2 + w.Hkv * w.dv * 2)
        return n * per_tok, dt, f"{n} random tokens (all heads)"
    # decode against a contiguous or ring cache, bf16 or FP8: n sampled sequences
    seqs = torch.randperm(w.B, generator=g)[:n]
    per_seq = ("q", "k_new", "v_new", "k_cache", "v_cache", "ring_head", "ring_len", "ctx_len")
    sub = {k: (_cpu(v[seqs.to(v.device)]) if k in per_seq else _cpu(v)) for k, v in d.items()}
    kw = {}
    if w.kind == W.KV_RING:
        kw.update(ring_head=sub["ring_head"], ring_len=sub["ring_len"])
    else:
        kw.update(ctx_len=sub["ctx_len"])
    t0 = time.perf_counter()
    if "k_scale" in d:
        oracle.decode_fp8(w.kind, sub["q"], sub["k_new"], sub["v_new"], sub["k_cache"],
                          sub["v_cache"], d["k_scale"], d["v_scale"], sub["sink"], W.SCALE,
                          w.window, **kw)
    else:
        oracle.decode(w.kind, sub["q"], sub["k_new"], sub["v_new"], sub["k_cache"],
                      sub["v_cache"], sub["sink"], W.SCALE, w.window, **kw)
    dt = time.perf_counter() - t0
    return None, dt, f"{len(seqs)} random sequences of {w.B}"


def cpu_baseline_secondary(kind, r, target_s=2.0):
    """The oracle on the host cores, on a bounded sample of a secondary workload: its rate in
    the job's unit and the whole workload's oracle time extrapolated from that rate (labelled
    so). Never raises: a failure is reported in the entry instead."""
    try:
        w = r.w
        if kind == "decode":
            n = min(w.B, 2 if w.B <= 8 else 16)
            _, dt, what = cpu_oracle_sample(kind, w, r.d, n)
            grown = max(n, min(w.B, int(n * target_s / max(dt, 1e-3))))
            if grown > n:
                n = grown
                _, dt, what = cpu_oracle_sample(kind, w, r.d, n, seed=n)
            work = r.bytes * n / w.B  # every sequence of these workloads holds the same context
            rate, unit, full = work / dt / 1e9, "GB/s", r.bytes / (work / dt)
        else:
            n = 16
            work, dt, what = cpu_oracle_sample(kind, w, r.d, n)
            n = max(n, min(1 << 16, int(n * target_s / max(dt, 1e-3))))
            work, dt, what = cpu_oracle_sample(kind, w, r.d, n, seed=n)
            if kind == "prefill":
                rate, unit, full = work / dt / 1e12, "TFLOP/s", r.flops / (work / dt)
            else:
                rate, unit, full = work / dt / 1e9, "GB/s", r.bytes / (work / dt)
        cores = 1 if kind == "rope" else omp_threads()  # the RoPE oracle is one plain loop
        return {"value": round(rate, 6), "unit": unit, "cores": cores, "kind": "oracle",
                "seconds": round(dt, 2), "sample": f"{what} of {getattr(r, 'workload', w.name)}",
                "full_workload_s_extrapolated": round(full, 3)}
    except Exception as e:  # the baseline is a report; it must not cost the benchmark its line
        return {"kind": "oracle", "error": f"{type(e).__name__}: {e}"[:200]}


# ----------------------------------------------------------------------------------------------
# main
# ----------------------------------------------------------------------------------------------

def init_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def run_reference(args, world, rank):
    """The oracle as the reference arm: fp64 C on the host cores, bounded sample per step."""
    if rank != 0:
        return None
    w = W.SWA_PREFILL
    if args.ref_L:
        import dataclasses
        w = dataclasses.replace(w, L=args.ref_L, name=f"{w.name}_L{args.ref_L}")
    # inputs of the full workload, drawn on the CPU generator
    d_cpu = W.prefill_inputs(w, device="cpu")
    rows_per_step = args.ref_rows
    for i in range(args.warmup):
        oracle_prefill_sample(w, d_cpu, rows_per_step, seed=i)
    tot_f, tot_t = 0, 0.0
    for i in range(args.steps):
        f, t = oracle_prefill_sample(w, d_cpu, rows_per_step, seed=1000 + i)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12
    sample = f"{rows_per_step} random (batch, position) rows x all {w.Hq} heads per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv,
                       "d_qk": w.dq, "d_v": w.dv, "window": w.window},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": omp_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def measure(runner, steps, warmup, flush, world):
    barrier()
    torch.cuda.synchronize()
    ms = time_steps(runner.step, steps, warmup, flush)
    barrier()
    return max_over_ranks(ms)


def compact_summary(result, secondary):
    """{workload key: [ms per step, roofline fraction, bound, achieved, unit]} for the headline
    and every secondary workload, plus the hybrid step's GA and SWA layers apart."""
    def short(ms, rl):
        return [ms, rl.get("frac"), rl.get("bound"), rl.get("achieved"), rl.get("unit")]

    out = {}
    if result.get("roofline"):
        out["headline"] = short(result.get("ms_per_step"), result["roofline"])
    for name, e in secondary.items():
        out[name] = short(e["ms_per_step"], e["roofline"])
        for kind, sub in e.get("by_kind", {}).items():
            out[f"{name}.{kind}"] = short(sub["ms_per_step"], sub["roofline"])
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default=None,
                    help="run one workload only: swa_prefill, ga_prefill, ga_chunk_prefill, "
                         "ga_backward, ga_decode, ga_decode_fp8, swa_decode, hybrid, rope, "
                         "swa_prefill_rope")
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--ref-L", type=int, default=0, help="reference arm: shorter sequences (tests)")
    ap.add_argument("--small", action="store_true",
                    help="profiling case: prefill workloads at B=1 (SWA L=16384, GA L=8192), "
                         "decode at B=2, SWA decode at B=64, hybrid verify as its first GA "
                         "layer alone at B=8 and its first SWA layer alone")
    args = ap.parse_args()
    world, rank, local = init_dist(args)
    args.gpus = max(args.gpus, world)

    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import global_attention_sink_softmax_b200 as sa
    sa.lib()  # fails loudly if the CUDA library is missing
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    flush = None

    swa_w, ga_w, gad_w, swad_w = W.SWA_PREFILL, W.GA_PREFILL, W.GA_DECODE, W.SWA_DECODE
    gac_w = W.GA_CHUNK
    if args.small:
        import dataclasses
        swa_w = dataclasses.replace(swa_w, B=1, L=16384, name=swa_w.name + "_small_B1_L16384")
        ga_w = dataclasses.replace(ga_w, L=8192, name=ga_w.name + "_small_L8192")
        gad_w = dataclasses.replace(gad_w, B=2, name=gad_w.name + "_small_B2")
        swad_w = dataclasses.replace(swad_w, B=64, name=swad_w.name + "_small_B64")
        gac_w = dataclasses.replace(gac_w, L=4096, prefix=4096, name=gac_w.name + "_small_P4096_L4096")

    def head_runner():
        return PrefillRunner(swa_w, dev)

    only = args.only
    result = None
    secondary = {}
    cpu_base = None

    if only in (None, "swa_prefill"):
        r = head_runner()
        # the inputs (3 GB) exceed L2: no flush needed between steps
        with ClockSampler(local) as clk:
            ms = measure(r, args.steps, args.warmup, None, world)
        ms_step = ms / args.steps
        units = r.flops * world
        value = units / (ms_step * 1e-3) / 1e12
        result = {"metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s",
                  "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                  "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
                  "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                  "config": {"workload": r.workload, **r.config,
                             "parallelism": f"independent batches x{world}" if world > 1 else "single GPU",
                             "l2": "inputs (3.0 GB) larger than L2, no flush"},
                  "roofline": roofline(r, ms_step, peaks, peak_src),
                  "clocks": clk.summary(), "gpu_launches": r.launches * args.steps}
        result["roofline"]["tensor_frac_of_bf16_peak"] = round(value / peaks["bf16_tflops"] / world, 4)
        if not args.no_e2e:
            r.e2e_setup()
            barrier()
            ms_e = time_steps(r.e2e_step, max(1, min(args.steps, 5)), 1, None)
            ms_e = max_over_ranks(ms_e) / max(1, min(args.steps, 5))
            result["e2e"] = {"value": round(units / (ms_e * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
                             "h2d_bytes_per_step": r.h2d, "d2h_bytes_per_step": r.d2h,
                             "ms_per_step": round(ms_e, 3), "api": r.e2e_api}
        if rank == 0 and not args.no_cpu_baseline:
            d_cpu = {k: v.cpu() for k, v in r.d.items()}
            r.release()
            torch.cuda.empty_cache()
            cpu_base = cpu_baseline_prefill(swa_w, d_cpu)
            del d_cpu
        r.release()
        del r
        torch.cuda.empty_cache()

    if not args.no_secondary:
        jobs = []
        if only in (None, "ga_prefill"):
            jobs.append(("ga_prefill", lambda: PrefillRunner(ga_w, dev), None))
        if only in (None, "ga_chunk_prefill"):
            jobs.append(("ga_chunk_prefill", lambda: PrefillRunner(gac_w, dev), None))
        if only in (None, "rope"):
            jobs.append(("rope_qkv", lambda: RopeRunner(swa_w, dev, 1e4), None))
        if only in (None, "swa_prefill_rope"):
            # the headline workload with the RoPE pass fused into the prefill's loads
            jobs.append(("swa_prefill_fused_rope", lambda: PrefillRunner(swa_w, dev, True), None))
        if only in (None, "ga_backward"):
            jobs.append(("ga_prefill_backward", lambda: BackwardRunner(ga_w, dev), None))
        if only in (None, "ga_decode"):
            jobs.append(("ga_decode", lambda: DecodeRunner(gad_w, dev), None))
        if only in (None, "ga_decode_fp8"):
            jobs.append(("ga_decode_fp8",
                         lambda: DecodeRunner(gad_w, dev, W.decode_inputs(gad_w, device=dev, fp8=True)),
                         None))
        if only in (None, "swa_decode"):
            # inputs (178 MB) larger than L2: no flush (a flush by writing a 252 MB buffer leaves
            # L2 full of dirty lines whose write-back would land in the timed kernel)
            jobs.append(("swa_decode", lambda: DecodeRunner(swad_w, dev), None))
        if only in (None, "hybrid") and not args.small:
            jobs.append(("hybrid", lambda: HybridRunner(dev), None))
        if only == "hybrid" and args.small:
            import dataclasses
            hyb0 = W.hybrid_layer_workload(0)
            hyb0 = dataclasses.replace(hyb0, B=8, name=hyb0.name + "_small_B8")
            jobs.append(("hybrid_ga_layer", lambda: DecodeRunner(hyb0, dev), None))
            # one SWA layer of the step at its full size (B=64; 43 MB, flushed between steps)
            jobs.append(("hybrid_swa_layer",
                         lambda: DecodeRunner(W.hybrid_layer_workload(1), dev), "flush"))
        for name, make, fl in jobs:
            r = make()
            flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if fl else None
            steps = max(3, args.steps)
            with ClockSampler(local) as clk:
                ms = measure(r, steps, max(3, args.warmup), flush, world)
            ms_step = ms / steps
            rl = roofline(r, ms_step, peaks, peak_src,
                          bound="hbm" if isinstance(r, RopeRunner) else
                          ("tensor" if isinstance(r, BackwardRunner) else None))
            entry = {"workload": r.workload, "config": r.config, "ms_per_step": round(ms_step, 4),
                     "tflops": round(r.flops / (ms_step * 1e-3) / 1e12, 3),
                     "gbs": round(r.bytes / (ms_step * 1e-3) / 1e9, 2), "roofline": rl,
                     "gpu_launches_per_step": r.launches, "clocks": clk.summary(),
                     "l2": "flushed between steps" if fl else "working set larger than L2"}
            cb_kind = {"ga_prefill": "prefill", "ga_chunk_prefill": "prefill", "rope_qkv": "rope",
                       "ga_decode": "decode", "ga_decode_fp8": "decode",
                       "swa_decode": "decode"}.get(name)
            if cb_kind and rank == 0 and world == 1 and not args.no_cpu_baseline:
                entry["cpu_baseline"] = cpu_baseline_secondary(cb_kind, r)
            if name == "hybrid":
                entry["note"] = ("layer list taken literally: 49 layer calls (9 GA, 40 SWA); "
                                 "GB/s over all layers' algorithmic bytes")
                # the GA and the SWA layers timed on their own (the GA layers carry the target)
                # the SWA layers first, after a pause: right after the GA layers' power draw the
                # SM clock sits lower (sw_power_cap) for a while, and the short SWA kernels
                # follow it; each kind carries its own clock samples
                by_kind = {}
                for kind, ring in (("swa_layers", True), ("ga_layers", False)):
                    sub = r.kind_runner(ring)
                    if ring:
                        time.sleep(2.0)
                    with ClockSampler(local) as clk_k:
                        ms_k = measure(sub, steps, max(3, args.warmup), None, world) / steps
                    by_kind[kind] = {"ms_per_step": round(ms_k, 4),
                                     "gbs": round(sub.bytes / (ms_k * 1e-3) / 1e9, 2),
                                     "roofline": roofline(sub, ms_k, peaks, peak_src, bound="hbm"),
                                     "clocks": clk_k.summary()}
                entry["by_kind"] = by_kind
            secondary[name] = entry
            r.release()
            del r, flush
            torch.cuda.empty_cache()

    if rank == 0:
        if result is None:
            result = {"metric": METRIC, "n_gpus": world, "steps": args.steps,
                      "warmup": args.warmup, "value": None, "unit": None}
        if cpu_base is not None:
            result["cpu_baseline"] = cpu_base
        if secondary:
            result["secondary"] = secondary
            # the same figures in short, as the line's last key: a reader that keeps only the
            # end of the output still sees every workload's time and roofline fraction
            result["summary"] = compact_summary(result, secondary)
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
