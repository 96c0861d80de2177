"""Parity of the fused partial-RoPE + value-scale pass (sinkattn_rope_qkv) with the fp64 oracle.

The rotated dims must match the oracle within the rounding the kernel is allowed: one fp32
evaluation rounded once to bf16 (at most 2^-8 of the value, since half an ulp of bf16 is at most
2^-8 of the number it rounds), plus 2e-6 of the row's scale for the fp32 parts before that
rounding: the hardware sine and cosine (absolute error at most 2^-21.19 on [-pi, pi], on both
terms of a rotated pair: 8e-7), the reduced angle rounded to fp32 (at most 2^-24 pi rad, on the
pair's norm: 2.7e-7) and the fp32 products (1.2e-7); 1.2e-6 in all, doubled for margin. The dims past rope_dim must come back bit for bit; V must be v_scale * v within the
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
ROPE_TOL_ROW = 2e-6


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


# ----------------------------------------------------------------------------------------------
# RoPE + value scale fused into the cache commit ("MiMo-V2-Flash 模型架构深度拆解" CH10.3: the
# value scale and the rotation precede attention, and the KV-cache update stores their result)
# ----------------------------------------------------------------------------------------------

def _commit_case(kind, fp8, seed):
    """Seeded new tokens, a cache of the given kind and its metadata, on the GPU."""
    g = torch.Generator().manual_seed(seed)
    B, T = 5, 4
    Hkv = 8 if kind == "ring" else 4
    kn = torch.randn(B, T, Hkv, 192, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, T, Hkv, 128, generator=g).to(torch.bfloat16)
    acc = torch.tensor([0, 1, 4, 3, 2], dtype=torch.int32)
    meta, rows = {}, None
    if kind == "ring":
        rows, lead = 128, (B,)
        meta["ring_head"] = torch.randint(0, 128, (B,), generator=g, dtype=torch.int32)
        meta["ring_len"] = torch.tensor([128, 0, 5, 127, 128], dtype=torch.int32)
        pos = torch.randint(0, 262140, (B,), generator=g, dtype=torch.int32)
        pos[0] = 262140  # the longest context's last tokens
    elif kind == "contig":
        rows, lead = 300, (B,)
        meta["ctx_len"] = torch.tensor([0, 17, 296, 64, 298], dtype=torch.int32)
        pos = None  # the cache's own count
    else:
        P, max_pages = 64, 5
        rows, lead = P, (B * max_pages + 2,)
        perm = torch.randperm(B * max_pages + 2, generator=g).to(torch.int32)
        meta["page_table"] = perm[:B * max_pages].reshape(B, max_pages).contiguous()
        meta["ctx_len"] = torch.tensor([63, 0, 128, 300, 200], dtype=torch.int32)
        pos = None
    shape_k, shape_v = lead + (rows, Hkv, 192), lead + (rows, Hkv, 128)
    if fp8:
        kc = torch.randint(0, 256, shape_k, generator=g, dtype=torch.uint8)
        vc = torch.randint(0, 256, shape_v, generator=g, dtype=torch.uint8)
        kc[(kc & 0x7f) == 0x7f] = 0  # no NaN codes in the untouched rows
        vc[(vc & 0x7f) == 0x7f] = 0
    else:
        kc = torch.randn(shape_k, generator=g).to(torch.bfloat16)
        vc = torch.randn(shape_v, generator=g).to(torch.bfloat16)
    return dict(kn=kn, vn=vn, acc=acc, kc=kc, vc=vc, meta=meta, pos=pos, T=T,
                theta=1e4 if kind == "ring" else 5e6)


def _slots(kind, c):
    """Where the oracle's commit puts accepted token u of sequence b: found by committing
    marker tokens (the value b * T + u + 1 everywhere) into an empty bf16 cache of the same
    geometry. Returns {(b, u): (leading index, row)} and the oracle's new metadata."""
    B, T = c["kn"].shape[:2]
    mk = (torch.arange(B * T, dtype=torch.float32) + 1).reshape(B, T, 1, 1)
    mk_k = mk.expand(B, T, c["kn"].shape[2], 192).to(torch.bfloat16).contiguous()
    mk_v = mk.expand(B, T, c["kn"].shape[2], 128).to(torch.bfloat16).contiguous()
    zk = torch.zeros(c["kc"].shape, dtype=torch.bfloat16)
    zv = torch.zeros(c["vc"].shape, dtype=torch.bfloat16)
    okind = {"ring": oracle.KV_RING, "contig": oracle.KV_CONTIG, "paged": oracle.KV_PAGED}[kind]
    extra = dict(page_table=c["meta"]["page_table"], page_size=zk.shape[1]) if kind == "paged" else {}
    mkc, _, h2, l2, c2 = oracle.commit(okind, mk_k, mk_v, c["acc"], zk, zv,
                                       ring_head=c["meta"].get("ring_head"),
                                       ring_len=c["meta"].get("ring_len"),
                                       ctx_len=c["meta"].get("ctx_len"), **extra)
    where = {}
    tag = mkc[..., 0, 0].float()
    for b in range(B):
        for u in range(int(c["acc"][b])):
            idx = (tag == b * T + u + 1).nonzero()
            assert idx.shape[0] == 1
            where[(b, u)] = tuple(int(x) for x in idx[0])
    return where, (h2, l2, c2)


@pytest.mark.parametrize("kind", ["ring", "contig", "paged"])
@pytest.mark.parametrize("fp8", [False, True])
def test_commit_with_rope_and_value_scale(kind, fp8):
    m = sa()
    c = _commit_case(kind, fp8, seed={"ring": 1, "contig": 2, "paged": 3}[kind] + 10 * fp8)
    B, T = c["kn"].shape[:2]
    kvk = {"ring": m.KV_RING, "contig": m.KV_CONTIG, "paged": m.KV_PAGED}[kind]
    scales = dict(k_scale=6 / 448, v_scale=5 / 448) if fp8 else {}
    kn, vn = c["kn"].cuda(), c["vn"].cuda()
    kn0, vn0 = kn.clone(), vn.clone()
    pos = None if c["pos"] is None else c["pos"].cuda()

    def run(fused):
        meta = {k: v.cuda().clone() for k, v in c["meta"].items()}
        kc, vc = c["kc"].cuda().clone(), c["vc"].cuda().clone()
        k_in, v_in = kn.clone(), vn.clone()
        base = pos if pos is not None else meta.get("ctx_len").clone()
        if fused:
            m.sinkattn_kv_commit(kvk, k_in, v_in, c["acc"].cuda(), kc, vc, rope_theta=c["theta"],
                                 pos=pos, **meta, **scales)
        else:  # the RoPE pass on the new tokens, then a plain commit
            m.sinkattn_rope_qkv(None, k_in, v_in, theta=c["theta"], pos_base=base)
            m.sinkattn_kv_commit(kvk, k_in, v_in, c["acc"].cuda(), kc, vc, **meta, **scales)
        torch.cuda.synchronize()
        return kc.cpu(), vc.cpu(), {k: v.cpu() for k, v in meta.items()}, k_in.cpu(), v_in.cpu()

    kc_f, vc_f, meta_f, _, _ = run(True)
    kc_p, vc_p, meta_p, k_rot, v_sc = run(False)
    # the caller's new tokens are not modified by the fused commit
    assert torch.equal(kn, kn0) and torch.equal(vn, vn0)
    # one code path: the fused commit stores exactly what the pass + commit store
    assert torch.equal(kc_f, kc_p) and torch.equal(vc_f, vc_p)
    # metadata as the oracle's commit leaves it
    where, (h2, l2, c2) = _slots(kind, c)
    for key, ref in (("ring_head", h2), ("ring_len", l2), ("ctx_len", c2)):
        if key in meta_f:
            assert torch.equal(meta_f[key], ref), key
    # every accepted token's stored K / V against the oracle's rotation and value scale; every
    # other row unchanged
    touched = torch.zeros(c["kc"].shape[:2], dtype=torch.bool)
    base = c["pos"] if c["pos"] is not None else c["meta"]["ctx_len"]
    for (b, u), (i0, r) in where.items():
        touched[i0, r] = True
        p_ = np.full((1,), int(base[b]) + u, np.int64)
        v_ref = oracle.vscale(c["vn"][b, u], 0.707)
        if fp8:
            # the codes are the E4M3 encoding of the rotated / scaled bf16 values (the decision
            # taken in the kernel's precision); those values are checked against the oracle
            assert torch.equal(kc_f[i0, r], oracle.fp8_encode(k_rot[b, u], 6 / 448))
            assert torch.equal(vc_f[i0, r], oracle.fp8_encode(v_sc[b, u], 5 / 448))
            got_k, got_v = k_rot[b, u], v_sc[b, u]
        else:
            got_k, got_v = kc_f[i0, r], vc_f[i0, r]
        check_rotated(got_k[None], c["kn"][b, u][None], p_, c["theta"], 64)
        err = (got_v.double() - v_ref).abs()
        assert torch.all(err <= ROPE_TOL_REL * v_ref.abs() + 1e-7 * c["vn"][b, u].double().abs())
    assert torch.equal(kc_f[~touched], c["kc"][~touched])
    assert torch.equal(vc_f[~touched], c["vc"][~touched])


def test_commit_with_rope_rejects_bad_arguments():
    m = sa()
    c = _commit_case("ring", False, seed=4)
    meta = {k: v.cuda() for k, v in c["meta"].items()}
    kc, vc = c["kc"].cuda(), c["vc"].cuda()
    args = (m.KV_RING, c["kn"].cuda(), c["vn"].cuda(), c["acc"].cuda(), kc, vc)
    with pytest.raises(m.SinkAttnError) as e:  # a ring needs the tokens' positions
        m.sinkattn_kv_commit(*args, rope_theta=1e4, **meta)
    assert e.value.status == 1
    pos = torch.zeros(5, dtype=torch.int32, device="cuda")
    with pytest.raises(m.SinkAttnError) as e:
        m.sinkattn_kv_commit(*args, rope_theta=1e4, rope_dim=24, pos=pos, **meta)
    assert e.value.status == 2
    with pytest.raises(m.SinkAttnError) as e:
        m.sinkattn_kv_commit(*args, rope_theta=-1.0, pos=pos, **meta)
    assert e.value.status == 1
