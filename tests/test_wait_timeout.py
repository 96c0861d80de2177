"""The failure path of the kernels' bounded waits, exercised without a fault.

Every wait of a kernel on an internal barrier gives up after a limit (1 s by default), records
bit 0 (prefill) or bit 1 (decode) in a device flag and lets the kernel return, so a stuck copy or
MMA ends the call instead of hanging the GPU. Here the limit is set to 0, which makes a wait give
up as soon as its first (blocking, briefly suspending) try fails, as it does for the waits that
span a load and an MMA step: the call must still return, the flag must report it, and with the
limit restored the same process must compute correct results again.
"""
import math

import pytest
import torch

import oracle
from parity import LSE_TOL, O_TOL

pytestmark = pytest.mark.gpu


def sa():
    import global_attention_sink_softmax_b200 as m
    return m


def rnd(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


@pytest.fixture
def limit_zero():
    m = sa()
    assert m.sinkattn_take_device_error() == 0
    m.sinkattn_set_wait_limit_ns(0)
    try:
        yield m
    finally:
        m.sinkattn_set_wait_limit_ns(10 ** 9)


def test_prefill_wait_gives_up_then_next_call_is_correct(limit_zero):
    m = limit_zero
    g = torch.Generator().manual_seed(5)
    # 4 query tiles: the last one has 4 key tiles, so its producer waits for a free stage
    B, L, Hq, Hkv = 1, 512, 4, 1
    q, k, v = rnd((B, L, Hq, 192), g), rnd((B, L, Hkv, 192), g), rnd((B, L, Hkv, 128), g)
    sink = torch.rand(Hq, generator=g) * 6
    args = (q.cuda(), k.cuda(), v.cuda(), sink.cuda())
    m.sinkattn_prefill_ga(*args)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() & 1
    m.sinkattn_set_wait_limit_ns(10 ** 9)
    o, lse = m.sinkattn_prefill_ga(*args)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() == 0
    ro, rl, _ = oracle.prefill(q, k, v, sink, 1 / math.sqrt(192), 0)
    assert (o.double().cpu() - ro).abs().max().item() <= O_TOL
    assert (lse.permute(0, 2, 1).double().cpu() - rl).abs().max().item() <= LSE_TOL


def test_decode_wait_gives_up_then_next_call_is_correct(limit_zero):
    m = limit_zero
    g = torch.Generator().manual_seed(6)
    # a 4-token verify on a contiguous GA cache, 16 heads per KV head (64 query rows per KV
    # head): the tcgen05 verify kernel, whose first waits span a Q and K load and an S step
    B, T, Hq, Hkv, maxc = 2, 4, 64, 4, 3000
    q, kn, vn = rnd((B, T, Hq, 192), g), rnd((B, T, Hkv, 192), g), rnd((B, T, Hkv, 128), g)
    kc, vc = rnd((B, maxc, Hkv, 192), g), rnd((B, maxc, Hkv, 128), g)
    sink = torch.rand(Hq, generator=g) * 6
    ctx = torch.tensor([1500, 2999], dtype=torch.int32)
    args = [x.cuda() for x in (q, kn, vn, kc, vc, sink)]
    kw = dict(ctx_len=ctx.cuda())
    m.sinkattn_decode(m.KV_CONTIG, *args, **kw)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() & 2
    m.sinkattn_set_wait_limit_ns(10 ** 9)
    o, lse = m.sinkattn_decode(m.KV_CONTIG, *args, **kw)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() == 0
    ro, rl, _ = oracle.decode(oracle.KV_CONTIG, q, kn, vn, kc, vc, sink, 1 / math.sqrt(192), 0,
                              ctx_len=ctx)
    assert (o.double().cpu() - ro).abs().max().item() <= O_TOL
    assert (lse.double().cpu() - rl).abs().max().item() <= LSE_TOL


def test_ring_decode_wait_gives_up_then_next_call_is_correct(limit_zero):
    m = limit_zero
    g = torch.Generator().manual_seed(7)
    # a 4-token verify on 128-slot rings, 8 heads per KV head: the tcgen05 ring kernel, whose
    # first waits span the Q / K / V loads and an S step
    B, T, Hq, Hkv, cap = 3, 4, 16, 2, 128
    q, kn, vn = rnd((B, T, Hq, 192), g), rnd((B, T, Hkv, 192), g), rnd((B, T, Hkv, 128), g)
    kc, vc = rnd((B, cap, Hkv, 192), g), rnd((B, cap, Hkv, 128), g)
    sink = torch.rand(Hq, generator=g) * 6
    head = torch.tensor([0, 77, 127], dtype=torch.int32)
    ln = torch.tensor([128, 128, 50], dtype=torch.int32)
    args = [x.cuda() for x in (q, kn, vn, kc, vc, sink)]
    kw = dict(window=128, ring_head=head.cuda(), ring_len=ln.cuda())
    m.sinkattn_decode(m.KV_RING, *args, **kw)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() & 2
    m.sinkattn_set_wait_limit_ns(10 ** 9)
    o, lse = m.sinkattn_decode(m.KV_RING, *args, **kw)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() == 0
    ro, rl, _ = oracle.decode(oracle.KV_RING, q, kn, vn, kc, vc, sink, 1 / math.sqrt(192), 128,
                              ring_head=head, ring_len=ln)
    assert (o.double().cpu() - ro).abs().max().item() <= O_TOL
    assert (lse.double().cpu() - rl).abs().max().item() <= LSE_TOL
