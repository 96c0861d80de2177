"""Parity of the fused partial-RoPE + value-scale pass (sinkattn_rope_qkv) with the fp64 oracle.

The rotated dims must match the oracle within the rounding the kernel is allowed: one fp32
evaluation rounded once to bf16 (at most 2^-8 of the value, since half an ulp of bf16 is at most
2^-8 of the number it rounds), plus 1e-6 of the row's scale for the fp32 sine / cosine and
products. The dims past rope_dim must come back bit for bit; V must be v_scale * v within the
same bf16 rounding. Positions run up to 262143, the longest context of the pages' model.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from global_attention_sink_softmax_b200 import workloads as W

pytestmark = pytest.mark.gpu

ROPE_TOL_REL = 2.0 ** -8
ROPE_TOL_ROW = 1e-6


def sa():
    import global_attention_sink_softmax_b200 as m
    return m


def inputs(B, L, Hq, Hkv, dq=192, dv=128, seed=0):
    w = dataclasses.replace(W.SWA_PREFILL, B=B, L=L, Hq=Hq, Hkv=Hkv, dq=dq, dv=dv)
    d = W.prefill_inputs(w, device="cuda", seed=seed)
    return d["q"], d["k"], d["v"]


def positions(B, L, pos0, pos_base):
    base = np.zeros(B, np.int64) if pos_base is None else pos_base.cpu().numpy().astype(np.int64)
    return pos0 + base[:, None] + np.arange(L)[None, :]


def check_rotated(got, x_in, pos, theta, rope_dim):
    ref = oracle.rope(x_in.cpu(), pos, theta, rope_dim)
    g = got.cpu().double()
    row = x_in.cpu().double().abs().amax(-1, keepdim=True)
    err = (g[..., :rope_dim] - ref[..., :rope_dim]).abs()
    tol = ROPE_TOL_REL * ref[..., :rope_dim].abs() + ROPE_TOL_ROW * row
    assert torch.all(err <= tol), f"max excess {(err - tol).max().item():.3e}"
    # the rest of every head row is not touched
    assert torch.equal(got[..., rope_dim:].cpu(), x_in[..., rope_dim:].cpu())


def check_scaled(got, v_in, v_scale):
    ref = oracle.vscale(v_in.cpu(), v_scale)
    err = (got.cpu().double() - ref).abs()
    tol = ROPE_TOL_REL * ref.abs() + 1e-7 * v_in.cpu().double().abs()
    assert torch.all(err <= tol), f"max excess {(err - tol).max().item():.3e}"


@pytest.mark.parametrize("B,L,Hq,Hkv,theta,pos0,base_hi", [
    (1, 1, 64, 8, 1e4, 0, 0),            # one token
    (2, 37, 64, 8, 1e4, 0, 0),           # SWA heads, ragged token count (not a multiple of 8)
    (1, 300, 64, 4, 5e6, 0, 0),          # GA heads
    (3, 19, 64, 4, 5e6, 16384, 0),       # a chunk after a 16384-token prefix
    (4, 4, 64, 4, 5e6, 0, 262140),       # decode-like: T = 4 new tokens at per-sequence offsets
    (5, 1, 64, 8, 1e4, 0, 262143),       # SWA decode at the longest context
    (2, 64, 8, 1, 1e4, 7, 1000),         # a small GQA group
])
def test_rope_qkv_matches_oracle(B, L, Hq, Hkv, theta, pos0, base_hi):
    m = sa()
    q, k, v = inputs(B, L, Hq, Hkv, seed=B * 1000 + L)
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    pos_base = None
    if base_hi:
        g = torch.Generator().manual_seed(L)
        pos_base = torch.randint(0, base_hi + 1, (B,), generator=g, dtype=torch.int32)
        pos_base[0] = base_hi  # the largest offset always present
        pos_base = pos_base.cuda()
    m.sinkattn_rope_qkv(q, k, v, theta=theta, pos0=pos0, pos_base=pos_base)
    torch.cuda.synchronize()
    pos = positions(B, L, pos0, pos_base)
    check_rotated(q, q0, pos, theta, 64)
    check_rotated(k, k0, pos, theta, 64)
    check_scaled(v, v0, 0.707)


@pytest.mark.parametrize("rope_dim", [16, 32, 128])
def test_rope_other_widths(rope_dim):
    m = sa()
    q, k, v = inputs(2, 21, 16, 2, seed=rope_dim)
    q0, k0 = q.clone(), k.clone()
    m.sinkattn_rope_qkv(q, k, None, theta=1e4, rope_dim=rope_dim, pos0=5)
    torch.cuda.synchronize()
    pos = positions(2, 21, 5, None)
    check_rotated(q, q0, pos, 1e4, rope_dim)
    check_rotated(k, k0, pos, 1e4, rope_dim)


def test_rope_subsets_touch_only_what_is_given():
    m = sa()
    q, k, v = inputs(2, 33, 64, 8, seed=5)
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    m.sinkattn_rope_qkv(None, None, v, theta=1e4, v_scale=0.5)
    torch.cuda.synchronize()
    assert torch.equal(q, q0) and torch.equal(k, k0)
    check_scaled(v, v0, 0.5)
    v1 = v.clone()
    m.sinkattn_rope_qkv(q, None, None, theta=5e6, pos0=100)
    torch.cuda.synchronize()
    assert torch.equal(k, k0) and torch.equal(v, v1)
    check_rotated(q, q0, positions(2, 33, 100, None), 5e6, 64)


def test_rope_on_views_of_a_fused_projection():
    """Q, K and V as strided views of one [B, L, Hq*192 + Hkv*192 + Hkv*128] projection output:
    every view is rotated / scaled and nothing between or around them changes."""
    m = sa()
    B, L, Hq, Hkv = 2, 45, 16, 2
    width = Hq * 192 + Hkv * 192 + Hkv * 128
    g = torch.Generator(device="cuda").manual_seed(9)
    buf = torch.randn(B, L, width + 8, generator=g, device="cuda").to(torch.bfloat16)
    buf0 = buf.clone()
    q = buf[..., :Hq * 192].view(B, L, Hq, 192)
    k = buf[..., Hq * 192:(Hq + Hkv) * 192].view(B, L, Hkv, 192)
    v = buf[..., (Hq + Hkv) * 192:width].view(B, L, Hkv, 128)
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    m.sinkattn_rope_qkv(q, k, v, theta=1e4, pos0=3)
    torch.cuda.synchronize()
    pos = positions(B, L, 3, None)
    check_rotated(q, q0, pos, 1e4, 64)
    check_rotated(k, k0, pos, 1e4, 64)
    check_scaled(v, v0, 0.707)
    assert torch.equal(buf[..., width:], buf0[..., width:])


def test_rope_empty_is_a_no_op():
    m = sa()
    q, k, v = inputs(2, 8, 64, 8)
    m.sinkattn_rope_qkv(q[:, :0], k[:, :0], v[:, :0], theta=1e4)
    m.sinkattn_rope_qkv(q[:0], k[:0], v[:0], theta=1e4)
    torch.cuda.synchronize()


def test_rope_full_size_sampled():
    """The benchmark's launch: the SWA prefill workload (B=2, L=32768, 64 Q / 8 KV heads), SWA
    theta. Sampled (sequence, token) rows are checked against the oracle; the no-pe dims of
    every row must come back unchanged."""
    m = sa()
    w = W.SWA_PREFILL
    d = W.prefill_inputs(w, device="cuda")
    q, k, v = d["q"], d["k"], d["v"]
    g = torch.Generator().manual_seed(77)
    rows = torch.stack([torch.randint(0, w.B, (96,), generator=g),
                        torch.randint(0, w.L, (96,), generator=g)], 1)
    rows[0] = torch.tensor([w.B - 1, w.L - 1])
    bi, li = rows[:, 0].cuda(), rows[:, 1].cuda()
    qs, ks, vs = q[bi, li].clone(), k[bi, li].clone(), v[bi, li].clone()
    q_nope = q[..., 64:].clone()
    m.sinkattn_rope_qkv(q, k, v, theta=m.ROPE_THETA_SWA)
    torch.cuda.synchronize()
    pos = rows[:, 1].numpy().astype(np.int64)
    check_rotated(q[bi, li], qs, pos, 1e4, 64)
    check_rotated(k[bi, li], ks, pos, 1e4, 64)
    check_scaled(v[bi, li], vs, 0.707)
    assert torch.equal(q[..., 64:], q_nope)
