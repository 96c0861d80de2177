"""Parity of the prefill backward (sinkattn_prefill_backward) with the fp64 oracle.

The GPU forward's O (bf16) and LSE feed the GPU backward; the oracle computes dq, dk, dv and
dsink of sum(O * dout) from scratch in fp64 ("MiMo-V2-Flash 模型架构深度拆解" CH10.1: the sink is
a softmax column with no value, so its gradient is -sum_i p_sink,i delta_i). The backward rounds P
and dS to bf16 for the tensor cores and reads O rounded to bf16 (about 2^-9 relative per term),
so each gradient tensor must match within GRAD_TOL of its own largest magnitude: the same 1e-2
the forward allows on O, whose magnitude is of order one, taken relative here because gradient
magnitudes scale with L and the group size.
"""
import math

import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-2


def sa():
    import global_attention_sink_softmax_b200 as m
    return m


def rnd(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def check(name, got, ref):
    got = got.double().cpu()
    scale = max(ref.abs().max().item(), 1e-3)
    err = (got - ref).abs().max().item()
    assert torch.isfinite(got).all(), f"{name}: non-finite"
    assert err <= GRAD_TOL * scale, f"{name}: max err {err:.3e} > {GRAD_TOL} x {scale:.3e}"


def run_case(B, L, Hq, Hkv, window, sink_kind, seed):
    m = sa()
    g = torch.Generator().manual_seed(seed)
    q, k, v = rnd((B, L, Hq, 192), g), rnd((B, L, Hkv, 192), g), rnd((B, L, Hkv, 128), g)
    dout = rnd((B, L, Hq, 128), g)
    if sink_kind == "none":
        sink = None
    else:
        sink = torch.rand(Hq, generator=g) * 6
        if sink_kind == "mixed":
            sink[::3] = -math.inf
    scale = 1 / math.sqrt(192)
    dev = [x.cuda() for x in (q, k, v, dout)]
    s_dev = None if sink is None else sink.cuda()
    if window:
        o, lse = m.sinkattn_prefill_swa(dev[0], dev[1], dev[2], s_dev, window)
    else:
        o, lse = m.sinkattn_prefill_ga(dev[0], dev[1], dev[2], s_dev)
    gq, gk, gv, gs = m.sinkattn_prefill_backward(dev[0], dev[1], dev[2], o, lse, dev[3], s_dev,
                                                 window=window)
    torch.cuda.synchronize()
    assert m.sinkattn_take_device_error() == 0
    rq, rk, rv, rs = oracle.prefill_backward(q, k, v, sink, dout, scale, window)
    check("dq", gq, rq)
    check("dk", gk, rk)
    check("dv", gv, rv)
    if sink is None:
        assert torch.equal(gs.cpu(), torch.zeros(Hq))
    else:
        err = (gs.double().cpu() - rs).abs().max().item()
        assert err <= GRAD_TOL * max(rs.abs().max().item(), 1e-3) + 1e-4, ("dsink", err)


@pytest.mark.parametrize("L", [1, 64, 127, 129, 300])
def test_backward_ga(L):
    run_case(1, L, 4, 1, 0, "mixed", seed=L)


@pytest.mark.parametrize("window", [1, 7, 128, 200])
def test_backward_swa(window):
    run_case(1, 300, 8, 1, window, "sink", seed=window)


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (8, 4), (16, 1)])
def test_backward_gqa_groups(Hq, Hkv):
    run_case(2, 200, Hq, Hkv, 0, "sink", seed=Hq * 10 + Hkv)


def test_backward_without_sink():
    run_case(1, 150, 4, 2, 0, "none", seed=3)


def test_backward_model_heads_swa():
    """The SWA layer's heads (64 Q / 8 KV, W = 128) on a short sequence."""
    run_case(1, 256, 64, 8, 128, "sink", seed=11)
