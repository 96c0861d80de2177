"""The no-allocation decode entry point, sinkattn_decode_noalloc.

It exists for callers that cannot allocate device memory and have no workspace to lend: a plugin
host that hands the library only its input and output buffers, or a serving loop whose device
memory is all reserved up front. It must give the same result as sinkattn_decode with a caller
workspace, call after call, although every call reuses the library's one fixed array.

This file is collected last on purpose, so a run that stops at the first failure has run every
other test before it.
"""
import ctypes
import math

import pytest
import torch

import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import build as sa_build
from parity import LSE_TOL, O_TOL


def rnd(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def contig_case(seed, B, T, ctx):
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv, maxc = 64, 4, max(ctx)
    return dict(kind=sa.KV_CONTIG, window=0,
                q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
                v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, maxc, Hkv, 192), g),
                v_cache=rnd((B, maxc, Hkv, 128), g), sink=torch.rand(Hq, generator=g) * 6,
                meta=dict(ctx_len=torch.tensor(ctx, dtype=torch.int32)))


def ring_case(seed, B, T):
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv = 64, 8
    return dict(kind=sa.KV_RING, window=128,
                q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
                v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, 128, Hkv, 192), g),
                v_cache=rnd((B, 128, Hkv, 128), g), sink=torch.rand(Hq, generator=g) * 6,
                meta=dict(ring_head=torch.randint(0, 128, (B,), generator=g, dtype=torch.int32),
                          ring_len=torch.full((B,), 128, dtype=torch.int32)))


def on_gpu(c):
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in c.items() if k != "meta"}
    d["meta"] = {k: v.cuda() for k, v in c["meta"].items()}
    return d


def with_workspace(d):
    return sa.sinkattn_decode(d["kind"], d["q"], d["k_new"], d["v_new"], d["k_cache"],
                              d["v_cache"], d["sink"], window=d["window"], **d["meta"])


def without_workspace(d):
    B, T, Hq = d["q"].shape[:3]
    o = torch.full((B, T, Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, T, Hq), float("nan"), dtype=torch.float32, device="cuda")
    return sa.sinkattn_decode_noalloc(d["kind"], d["q"], d["k_new"], d["v_new"], d["k_cache"],
                                      d["v_cache"], d["sink"], window=d["window"], o=o, lse=lse,
                                      **d["meta"])


def assert_same(a, b, what):
    """Both calls take the same split plan and run the same deterministic kernels, so their
    results must agree bit for bit: a stale partial left in the shared array, however small its
    effect, shows up here. (Agreement with the oracle, within O_TOL and LSE_TOL, is the parity
    tests' job; the workspace path checked here is one of those they cover.)"""
    (oa, la), (ob, lb) = a, b
    assert torch.isfinite(ob.float()).all() and torch.isfinite(lb).all(), what
    eo = (oa.float() - ob.float()).abs().max().item()
    el = (la - lb).abs().max().item()
    assert torch.equal(oa, ob) and torch.equal(la, lb), (what, eo, el, O_TOL, LSE_TOL)


@pytest.mark.gpu
def test_noalloc_decode_matches_decode_with_workspace_on_consecutive_calls():
    first = on_gpu(contig_case(1, B=2, T=4, ctx=[5000, 3001]))   # split-KV: uses the array
    second = on_gpu(contig_case(2, B=3, T=1, ctx=[1, 4096, 2500]))
    ring = on_gpu(ring_case(3, B=16, T=2))                       # one span: no array needed
    need1 = sa.sinkattn_decode_workspace_size(first["kind"], first["q"], first["k_new"],
                                              first["v_new"], first["k_cache"],
                                              first["v_cache"], **first["meta"])
    assert 0 < need1 <= sa.NOALLOC_WORKSPACE_BYTES
    ref1, ref2, ref3 = with_workspace(first), with_workspace(second), with_workspace(ring)
    got1 = without_workspace(first)
    got2 = without_workspace(second)      # reuses the array right after the first call
    got3 = without_workspace(ring)
    again = without_workspace(first)
    torch.cuda.synchronize()
    assert_same(ref1, got1, "first call")
    assert_same(ref2, got2, "second call")
    assert_same(ref3, got3, "ring")
    assert_same(ref1, again, "first inputs again")
    assert sa.sinkattn_take_device_error() == 0


def test_noalloc_rejects_problems_larger_than_its_array():
    """Rejected on the host, before any CUDA call: runs without a GPU as well."""
    sa_build.build()
    L = sa.lib()
    a = sa.DecodeArgs()
    a.kind, a.B, a.T, a.Hq, a.Hkv, a.dq, a.dv, a.window = 1, 64, 4, 64, 4, 192, 128, 0
    a.scale = 1 / math.sqrt(192)
    a.q = a.k_new = a.v_new = a.k_cache = a.v_cache = a.o = 0x20000
    a.ctx_len, a.max_ctx = 0x30000, 65536
    for pre, d in (("q", 192), ("kn", 192), ("vn", 128), ("kc", 192), ("vc", 128), ("o", 128)):
        mid = "ss" if pre in ("kc", "vc") else "st"
        setattr(a, f"{pre}_sb", d * 65536 * 4)
        setattr(a, f"{pre}_{mid}", d * 4)
        setattr(a, f"{pre}_sh", d)
    need = L.sinkattn_decode_workspace_size(ctypes.byref(a))
    assert need > sa.NOALLOC_WORKSPACE_BYTES
    assert L.sinkattn_decode_noalloc(ctypes.byref(a), None) == 4   # workspace too small
    a.T = 5
    assert L.sinkattn_decode_noalloc(ctypes.byref(a), None) == 2   # same validation as decode
