"""GPU parity of the SWA prefill with the partial RoPE and the value scale fused into its loads
(sinkattn_prefill_swa_rope) against the oracle and against the separate pass followed by the
plain prefill.

The fused kernel rotates each Q tile and K chunk in shared memory with the pass's own arithmetic,
so Q K^T, the softmax and hence LSE come out bit for bit as after the pass. The value scale
multiplies O instead of V, so O matches the oracle (V exact, O scaled) within the prefill
tolerances, and the pass-then-prefill result within one bf16 step (their V roundings differ)."""
import math

import numpy as np
import pytest
import torch

import oracle
import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import workloads as W
from parity import assert_close
from test_parity_prefill import sample_rows

pytestmark = pytest.mark.gpu


def rand_qkv(B, L, Hq, Hkv, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, 192, generator=g).to(torch.bfloat16)
    k = torch.randn(B, L, Hkv, 192, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, 128, generator=g).to(torch.bfloat16)
    s = torch.rand(Hq, generator=g) * 6.0
    s[::5] = float("-inf")
    return q, k, v, s


def positions(B, L, pos0, pos_base):
    base = np.zeros(B, np.int64) if pos_base is None else pos_base.cpu().numpy().astype(np.int64)
    return pos0 + base[:, None] + np.arange(L)[None, :]


def pass_then_prefill(q, k, v, s, window, theta, pos0, pos_base):
    qd, kd, vd = q.clone(), k.clone(), v.clone()
    sa.sinkattn_rope_qkv(qd, kd, vd, theta=theta, pos0=pos0, pos_base=pos_base)
    return sa.sinkattn_prefill_swa(qd, kd, vd, s, window)


@pytest.mark.parametrize("B,L,Hq,Hkv,window,pos0,base_hi", [
    (1, 300, 8, 1, 128, 0, 0),          # one KV head, ragged length
    (2, 700, 64, 8, 128, 0, 0),         # the model's SWA heads
    (2, 257, 16, 2, 128, 16384, 0),     # positions after a 16384-token offset
    (3, 160, 8, 1, 120, 5, 262000),     # per-sequence offsets up to the longest context
    (1, 16, 8, 1, 128, 0, 0),           # a single item
])
def test_fused_rope_prefill(B, L, Hq, Hkv, window, pos0, base_hi):
    q, k, v, s = rand_qkv(B, L, Hq, Hkv, seed=L + window + pos0)
    dev = "cuda"
    qd, kd, vd, sd = q.to(dev), k.to(dev), v.to(dev), s.to(dev)
    pos_base = None
    if base_hi:
        g = torch.Generator().manual_seed(B + L)
        pos_base = torch.randint(0, base_hi + 1, (B,), generator=g, dtype=torch.int32)
        pos_base[0] = base_hi
        pos_base = pos_base.to(dev)
    theta = sa.ROPE_THETA_SWA
    q0, k0, v0 = qd.clone(), kd.clone(), vd.clone()
    o, lse = sa.sinkattn_prefill_swa_rope(qd, kd, vd, sd, window, theta=theta, pos0=pos0,
                                          pos_base=pos_base)
    o2, lse2 = pass_then_prefill(qd, kd, vd, sd, window, theta, pos0, pos_base)
    torch.cuda.synchronize()
    # the inputs are not modified
    assert torch.equal(qd, q0) and torch.equal(kd, k0) and torch.equal(vd, v0)
    # Q and K rotated exactly as the pass rotates them: the softmax, hence LSE, bit for bit
    assert torch.equal(lse, lse2)
    # the oracle of the fused definition: Q, K rotated and rounded to bf16 like the pass, V as
    # given, O times the value scale
    pos = positions(B, L, pos0, pos_base)
    rq = oracle.rope(q, pos, theta).to(torch.bfloat16)
    rk = oracle.rope(k, pos, theta).to(torch.bfloat16)
    ro, rl, _ = oracle.prefill(rq, rk, v, s, 1 / math.sqrt(192), window)
    assert_close(o, ro * sa.V_SCALE, lse.permute(0, 2, 1), rl, f"fused rope B{B} L{L} W{window}")
    # and the pass-then-prefill result: both outputs are bf16 values of nearly the same number
    # (their V rounding differs), so they may differ by one bf16 step, 2^-7 of the value
    a, b2 = o.double().cpu(), o2.double().cpu()
    excess = (a - b2).abs() - torch.clamp(2.0 ** -7 * b2.abs(), min=1e-2)
    assert excess.max().item() <= 0, f"fused vs pass + prefill: max excess {excess.max().item():.3e}"
    assert sa.sinkattn_take_device_error() == 0


@pytest.mark.parametrize("rope_dim", [16, 32, 48])
def test_fused_rope_prefill_rope_widths(rope_dim):
    """Narrower rotary widths (one to three of the four 8-pair chunks a rotator lane holds) and
    the GA theta: LSE bit for bit against the pass then the prefill, O against the oracle."""
    B, L, Hq, Hkv, window, pos0 = 2, 333, 16, 2, 128, 1000
    q, k, v, s = rand_qkv(B, L, Hq, Hkv, seed=7 * rope_dim)
    qd, kd, vd, sd = q.cuda(), k.cuda(), v.cuda(), s.cuda()
    theta = sa.ROPE_THETA_GA
    o, lse = sa.sinkattn_prefill_swa_rope(qd, kd, vd, sd, window, theta=theta, rope_dim=rope_dim,
                                          pos0=pos0)
    q2, k2, v2 = qd.clone(), kd.clone(), vd.clone()
    sa.sinkattn_rope_qkv(q2, k2, v2, theta=theta, rope_dim=rope_dim, pos0=pos0)
    o2, lse2 = sa.sinkattn_prefill_swa(q2, k2, v2, sd, window)
    torch.cuda.synchronize()
    assert torch.equal(lse, lse2)
    pos = positions(B, L, pos0, None)
    rq = oracle.rope(q, pos, theta, rope_dim).to(torch.bfloat16)
    rk = oracle.rope(k, pos, theta, rope_dim).to(torch.bfloat16)
    ro, rl, _ = oracle.prefill(rq, rk, v, s, 1 / math.sqrt(192), window)
    assert_close(o, ro * sa.V_SCALE, lse.permute(0, 2, 1), rl, f"fused rope width {rope_dim}")
    assert sa.sinkattn_take_device_error() == 0


def test_fused_rope_prefill_full_size_sampled():
    """The headline workload (B=2, L=32768, 64 Q / 8 KV, W=128) with the SWA layers' RoPE:
    LSE bit for bit against the pass then the prefill; O against the oracle on sampled rows."""
    w = W.SWA_PREFILL
    d = W.prefill_inputs(w, device="cuda")
    o, lse = sa.sinkattn_prefill_swa_rope(d["q"], d["k"], d["v"], d["sink"], w.window,
                                          theta=sa.ROPE_THETA_SWA)
    o2, lse2 = pass_then_prefill(d["q"], d["k"], d["v"], d["sink"], w.window, sa.ROPE_THETA_SWA,
                                 0, None)
    torch.cuda.synchronize()
    assert torch.equal(lse, lse2)
    rows = sample_rows(w.B, w.L, seed=w.seed + 2, extra=8)
    idx_b = torch.tensor([r[0] for r in rows])
    idx_i = torch.tensor([r[1] for r in rows])
    # the oracle on the sampled rows: those rows' Q and every key they see, rotated at their
    # positions and rounded to bf16 like the pass; the other rows are not read
    qc, kc, vc = d["q"].cpu(), d["k"].cpu(), d["v"].cpu()
    rq, rk = qc.clone(), kc.clone()
    for b in range(w.B):
        qi = sorted({r[1] for r in rows if r[0] == b})
        ki = sorted({j for i in qi for j in range(max(0, i - w.window + 1), i + 1)})
        rq[b, qi] = oracle.rope(qc[b, qi], np.array(qi), sa.ROPE_THETA_SWA).to(torch.bfloat16)
        rk[b, ki] = oracle.rope(kc[b, ki], np.array(ki), sa.ROPE_THETA_SWA).to(torch.bfloat16)
    ro, rl, _ = oracle.prefill(rq, rk, vc, d["sink"].cpu(), W.SCALE, w.window, rows=rows)
    assert_close(o.cpu()[idx_b, idx_i], ro * sa.V_SCALE, lse.cpu().permute(0, 2, 1)[idx_b, idx_i],
                 rl, w.name + " fused rope")
    assert sa.sinkattn_take_device_error() == 0


def test_fused_rope_prefill_other_shapes_are_unsupported():
    q, k, v, s = rand_qkv(1, 64, 8, 2, seed=1)  # 4 query heads per KV head: not the packed path
    with pytest.raises(sa.SinkAttnError):
        sa.sinkattn_prefill_swa_rope(q.cuda(), k.cuda(), v.cuda(), s.cuda(), 128)
    q, k, v, s = rand_qkv(1, 64, 8, 1, seed=2)  # a window the packed span does not take
    with pytest.raises(sa.SinkAttnError):
        sa.sinkattn_prefill_swa_rope(q.cuda(), k.cuda(), v.cuda(), s.cuda(), 64)
