"""Seeded synthetic workloads for sink-softmax attention.

This module only draws random inputs and describes the workload shapes; it holds none of the
attention arithmetic. Both the CUDA path (tests, benchmark) and the fp64 oracle take their
inputs from here, so the two sides see identical bits.

Recipe (the same for every workload):
  * Q, K, V ~ N(0, 1), drawn in fp32 by a seeded torch generator and rounded to bf16
    (round-to-nearest-even);
  * per-query-head sink ~ U[0, 6] fp32; some workloads set chosen heads to -inf (plain
    softmax for that head);
  * softmax scale 1/sqrt(192) (the qk head dim);
  * ring-buffer heads ~ U{0..127}, context lengths ~ U{lo..hi}, all from the same generator.
Small workloads are drawn on the CPU generator; large ones on a CUDA generator on the device
(the draws are still seeded and reproducible; the oracle reads the slices it needs back).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

DQ, DV = 192, 128
SCALE = 1.0 / math.sqrt(DQ)
KV_RING, KV_CONTIG, KV_PAGED = 0, 1, 2


@dataclass
class PrefillWorkload:
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    window: int  # > 0: sliding window, 0: global causal
    seed: int
    neg_inf_heads: List[int] = field(default_factory=list)
    dq: int = DQ
    dv: int = DV
    prefix: int = 0  # chunked prefill: L query tokens after `prefix` cached positions


@dataclass
class DecodeWorkload:
    name: str
    kind: int
    B: int
    T: int
    Hq: int
    Hkv: int
    window: int
    seed: int
    ctx: int = 0               # fixed context (CONTIG) or 0
    ctx_lo: int = 0            # context range for PAGED workloads
    ctx_hi: int = 0
    ring_cap: int = 128
    page_size: int = 128
    dq: int = DQ
    dv: int = DV


# The five workloads of the hot path (sizes as stated by the benchmark specification).
SWA_PREFILL_SMALL = PrefillWorkload("swa_prefill_b1_l1024_8q1kv", B=1, L=1024, Hq=8, Hkv=1,
                                    window=128, seed=1235)
SWA_PREFILL = PrefillWorkload("swa_prefill_b2_l32768_64q8kv", B=2, L=32768, Hq=64, Hkv=8,
                              window=128, seed=1236)
GA_PREFILL = PrefillWorkload("ga_prefill_b1_l32768_64q4kv", B=1, L=32768, Hq=64, Hkv=4, window=0,
                             seed=1237, neg_inf_heads=[h for h in range(64) if h % 8 == 7])
# Chunked prefill (the serving command's --chunked-prefill-size 16384): the second 16384-token
# chunk of a 32768-token GA prompt, against the first chunk's cached keys.
GA_CHUNK = PrefillWorkload("ga_chunk_prefill_b1_p16384_l16384_64q4kv", B=1, L=16384, Hq=64, Hkv=4,
                           window=0, seed=1300, neg_inf_heads=[h for h in range(64) if h % 8 == 7],
                           prefix=16384)
GA_DECODE = DecodeWorkload("ga_decode_b8_ctx262144_64q4kv", kind=KV_CONTIG, B=8, T=1, Hq=64,
                           Hkv=4, window=0, seed=1238, ctx=262144)
SWA_DECODE = DecodeWorkload("swa_decode_b256_ring128_64q8kv", kind=KV_RING, B=256, T=1, Hq=64,
                            Hkv=8, window=128, seed=1239)
# Hybrid speculative-verify step: layer pattern [GA] + ([SWA] x 5 + [GA]) x 8, taken literally
# (49 layer calls: 9 GA, 40 SWA), B=64 sequences, 4 query tokens each.
HYBRID_LAYERS = ["GA"] + (["SWA"] * 5 + ["GA"]) * 8
HYBRID_B, HYBRID_T, HYBRID_CTX_LO, HYBRID_CTX_HI = 64, 4, 4096, 65536


def hybrid_layer_workload(layer: int) -> DecodeWorkload:
    kind = HYBRID_LAYERS[layer]
    seed = 1240 + 1000 * layer
    if kind == "GA":
        return DecodeWorkload(f"hybrid_L{layer}_ga", kind=KV_PAGED, B=HYBRID_B, T=HYBRID_T,
                              Hq=64, Hkv=4, window=0, seed=seed, ctx_lo=HYBRID_CTX_LO,
                              ctx_hi=HYBRID_CTX_HI)
    return DecodeWorkload(f"hybrid_L{layer}_swa", kind=KV_RING, B=HYBRID_B, T=HYBRID_T, Hq=64,
                          Hkv=8, window=128, seed=seed)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


# Per-tensor scales of the synthetic FP8 caches: N(0, 1) values up to ~6 fill the E4M3 range.
FP8_K_SCALE, FP8_V_SCALE = 6.0 / 448.0, 5.0 / 448.0


def fp8_codes(shape, g: torch.Generator, device, scale: float) -> torch.Tensor:
    """One-byte E4M3 codes of N(0, 1) draws divided by `scale`, made with torch's float8 cast
    (a library conversion, as torch.randn is a library draw), clamped to the finite range."""
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32) / scale
    return x.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def sinks(Hq: int, g: torch.Generator, device, neg_inf_heads=()) -> torch.Tensor:
    s = torch.rand(Hq, generator=g, device=device, dtype=torch.float32) * 6.0
    for h in neg_inf_heads:
        s[h] = float("-inf")
    return s


def prefill_inputs(w: PrefillWorkload, device="cpu", L: Optional[int] = None,
                   B: Optional[int] = None, seed: Optional[int] = None):
    """Returns dict(q [B,L,Hq,dq], k [B,L,Hkv,dq], v [B,L,Hkv,dv], sink [Hq]) on `device`."""
    L = w.L if L is None else L
    B = w.B if B is None else B
    g = _gen(w.seed if seed is None else seed, device)
    q = normal_bf16((B, L, w.Hq, w.dq), g, device)
    k = normal_bf16((B, L, w.Hkv, w.dq), g, device)
    v = normal_bf16((B, L, w.Hkv, w.dv), g, device)
    s = sinks(w.Hq, g, device, w.neg_inf_heads)
    return dict(q=q, k=k, v=v, sink=s)


def decode_inputs(w: DecodeWorkload, device="cpu", B: Optional[int] = None,
                  ctx: Optional[int] = None, ctx_hi: Optional[int] = None,
                  seed: Optional[int] = None, fp8: bool = False):
    """Seeded decode inputs. Returns a dict with q/k_new/v_new [B,T,H,d], the cache tensors and
    the cache metadata of the workload's kind (ring_head/ring_len, ctx_len, page_table).
    fp8=True: the caches are uint8 E4M3 codes (fp8_codes, scales FP8_K_SCALE / FP8_V_SCALE,
    also returned as k_scale / v_scale)."""
    B = w.B if B is None else B
    g = _gen(w.seed if seed is None else seed, device)

    def cache(shape, which):
        if not fp8:
            return normal_bf16(shape, g, device)
        return fp8_codes(shape, g, device, FP8_K_SCALE if which == "k" else FP8_V_SCALE)
    d = dict(q=normal_bf16((B, w.T, w.Hq, w.dq), g, device),
             k_new=normal_bf16((B, w.T, w.Hkv, w.dq), g, device),
             v_new=normal_bf16((B, w.T, w.Hkv, w.dv), g, device),
             sink=sinks(w.Hq, g, device))
    if w.kind == KV_RING:
        d["k_cache"] = cache((B, w.ring_cap, w.Hkv, w.dq), "k")
        d["v_cache"] = cache((B, w.ring_cap, w.Hkv, w.dv), "v")
        d["ring_head"] = torch.randint(0, w.ring_cap, (B,), generator=g, device=device,
                                       dtype=torch.int32)
        d["ring_len"] = torch.full((B,), w.ring_cap, dtype=torch.int32, device=device)
    elif w.kind == KV_CONTIG:
        c = w.ctx if ctx is None else ctx
        d["k_cache"] = cache((B, c, w.Hkv, w.dq), "k")
        d["v_cache"] = cache((B, c, w.Hkv, w.dv), "v")
        d["ctx_len"] = torch.full((B,), c, dtype=torch.int32, device=device)
        d["max_ctx"] = c
    else:
        hi = w.ctx_hi if ctx_hi is None else ctx_hi
        lo = min(w.ctx_lo, hi)
        ctx_len = torch.randint(lo, hi + 1, (B,), generator=g, device=device, dtype=torch.int32)
        P = w.page_size
        pages_per = [(int(c) + P - 1) // P for c in ctx_len.tolist()]
        max_pages = max(1, (hi + P - 1) // P)
        total = max(1, sum(pages_per))
        # pages of all sequences are handed out in a seeded random order
        perm = torch.randperm(total, generator=g, device=device).to(torch.int32)
        table = torch.zeros((B, max_pages), dtype=torch.int32, device=device)
        off = 0
        for b, n in enumerate(pages_per):
            table[b, :n] = perm[off:off + n]
            off += n
        d["k_cache"] = cache((total, P, w.Hkv, w.dq), "k")
        d["v_cache"] = cache((total, P, w.Hkv, w.dv), "v")
        d["ctx_len"] = ctx_len
        d["page_table"] = table
        d["max_ctx"] = max_pages * P
        d["page_size"] = P
    if fp8:
        d["k_scale"], d["v_scale"] = FP8_K_SCALE, FP8_V_SCALE
    return d
