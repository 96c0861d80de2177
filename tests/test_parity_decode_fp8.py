"""GPU parity of decode against an FP8 (E4M3) KV cache, and of the commit into one, with the
fp64 oracle (oracle.decode_fp8 / oracle.fp8_encode).

The decode bar is the bf16 path's (max |O - oracle| <= 1e-2, |LSE - oracle| <= 1e-3): the
kernel multiplies the exact E4M3 values, so the only new rounding is Q and P in fp16. The commit
stores integer codes and must match the oracle's encoding bit for bit; the decode's own
quantisation of the new tokens is checked through the oracle, which encodes them the same way.
"""
import math

import pytest
import torch

import oracle
import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(192)
KS, VS = 0.0213, 0.0171


def rnd(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def codes(shape, g, scale):
    x = torch.randn(shape, generator=g) / scale
    return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)


def to_dev(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def meta(kind, d, dev=True):
    src = to_dev(d) if dev else d
    kw = {}
    if kind == sa.KV_RING:
        kw.update(ring_head=src["ring_head"], ring_len=src["ring_len"])
    else:
        kw.update(ctx_len=src["ctx_len"])
    if kind == sa.KV_PAGED:
        kw.update(page_table=src["page_table"])
    return kw


def check(kind, d, window, what, ks=KS, vs=VS, seqs=None):
    dd = to_dev(d)
    kw = meta(kind, d)
    if kind != sa.KV_RING:
        kw["max_ctx"] = d.get("max_ctx")
    o, lse = sa.sinkattn_decode(kind, dd["q"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                dd["v_cache"], dd["sink"], window=window, k_scale=ks, v_scale=vs,
                                **kw)
    torch.cuda.synchronize()
    okw = meta(kind, d, dev=False)
    if kind == sa.KV_PAGED:
        okw["page_size"] = d["k_cache"].shape[1]
    ro, rl, _ = oracle.decode_fp8(kind, d["q"], d["k_new"], d["v_new"], d["k_cache"],
                                  d["v_cache"], ks, vs, d["sink"], SCALE, window, seqs=seqs, **okw)
    if seqs is not None:
        o, lse = o[seqs], lse[seqs]
    assert_close(o, ro, lse, rl, what)
    assert sa.sinkattn_take_device_error() == 0


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("Hq,Hkv,ctx", [(64, 4, [0, 1, 63, 64, 65, 1000]), (16, 2, [5, 300]),
                                        (64, 8, [129, 7])])
def test_fp8_contiguous(T, Hq, Hkv, ctx):
    g = torch.Generator().manual_seed(7 * T + Hq + len(ctx))
    B, max_ctx = len(ctx), max(ctx) + 3
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=codes((B, max_ctx, Hkv, 192), g, KS),
             v_cache=codes((B, max_ctx, Hkv, 128), g, VS),
             sink=torch.rand(Hq, generator=g) * 6,
             ctx_len=torch.tensor(ctx, dtype=torch.int32), max_ctx=max_ctx)
    d["sink"][::5] = float("-inf")
    check(sa.KV_CONTIG, d, 0, f"fp8 contig T{T} {Hq}/{Hkv}")


@pytest.mark.parametrize("T,window", [(1, 128), (3, 128), (4, 64)])
def test_fp8_ring(T, window):
    g = torch.Generator().manual_seed(40 + T)
    B, cap, Hq, Hkv = 5, 128, 64, 8
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=codes((B, cap, Hkv, 192), g, KS),
             v_cache=codes((B, cap, Hkv, 128), g, VS), sink=torch.rand(Hq, generator=g) * 6,
             ring_head=torch.tensor([0, 5, 127, 64, 90], dtype=torch.int32),
             ring_len=torch.tensor([128, 0, 1, 127, 40], dtype=torch.int32))
    check(sa.KV_RING, d, window, f"fp8 ring T{T} W{window}")


@pytest.mark.parametrize("page", [16, 64, 128])
def test_fp8_paged_with_a_missing_page(page):
    g = torch.Generator().manual_seed(page)
    B, T, Hq, Hkv, max_pages = 3, 2, 64, 4, 6
    ctx = torch.tensor([page * 5 + 3, 17, page * 2], dtype=torch.int32)
    total = 24
    perm = torch.randperm(total, generator=g).to(torch.int32)
    table = perm[:B * max_pages].view(B, max_pages).clone()
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=codes((total, page, Hkv, 192), g, KS),
             v_cache=codes((total, page, Hkv, 128), g, VS), sink=torch.rand(Hq, generator=g) * 6,
             ctx_len=ctx, page_table=table, max_ctx=max_pages * page)
    check(sa.KV_PAGED, d, 0, f"fp8 paged {page}")
    # a page the table does not map hides its keys: equal to a cache without those tokens
    table2 = table.clone()
    table2[0, 1] = -1
    d2 = dict(d, page_table=table2)
    dd = to_dev(d2)
    o, lse = sa.sinkattn_decode(sa.KV_PAGED, dd["q"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                dd["v_cache"], dd["sink"], ctx_len=dd["ctx_len"],
                                page_table=dd["page_table"], max_ctx=d["max_ctx"], k_scale=KS,
                                v_scale=VS)
    torch.cuda.synchronize()
    # the oracle view: sequence 0's tokens without page 1, as a contiguous cache
    keep = [c for c in range(int(ctx[0])) if c // page != 1]
    rows = [(int(table[0, c // page]), c % page) for c in keep]
    kc = torch.stack([d["k_cache"][p_, r_] for p_, r_ in rows])[None]
    vc = torch.stack([d["v_cache"][p_, r_] for p_, r_ in rows])[None]
    ro, rl, _ = oracle.decode_fp8(oracle.KV_CONTIG, d["q"][:1], d["k_new"][:1], d["v_new"][:1],
                                  kc, vc, KS, VS, d["sink"], SCALE, 0,
                                  ctx_len=torch.tensor([len(keep)], dtype=torch.int32))
    assert_close(o[:1], ro, lse[:1], rl, "fp8 paged, missing page")


def test_fp8_commit_is_bit_exact_and_round_trips():
    """Commit quantises exactly as the oracle encodes; a decode of the next tokens over the grown
    cache then equals the oracle. (Decode quantises its new tokens on load by the same rule: the
    oracle's decode uses the same encoding, so decode and commit agree through it.)"""
    g = torch.Generator().manual_seed(55)
    B, T, Hq, Hkv, max_ctx = 4, 4, 64, 4, 300
    kc = codes((B, max_ctx, Hkv, 192), g, KS)
    vc = codes((B, max_ctx, Hkv, 128), g, VS)
    ctx = torch.tensor([0, 10, 200, 296], dtype=torch.int32)
    k_new, v_new = rnd((B, T, Hkv, 192), g), rnd((B, T, Hkv, 128), g)
    n_acc = torch.tensor([4, 1, 0, 4], dtype=torch.int32)
    kd, vd, cd, nd = kc.cuda(), vc.cuda(), ctx.cuda(), n_acc.cuda()
    sa.sinkattn_kv_commit(sa.KV_CONTIG, k_new.cuda(), v_new.cuda(), nd, kd, vd, ctx_len=cd,
                          k_scale=KS, v_scale=VS)
    torch.cuda.synchronize()
    ek, ev = oracle.fp8_encode(k_new, KS), oracle.fp8_encode(v_new, VS)
    want_k, want_v = kc.clone(), vc.clone()
    for b in range(B):
        for u in range(int(n_acc[b])):
            pos = int(ctx[b]) + u
            if pos < max_ctx:
                want_k[b, pos], want_v[b, pos] = ek[b, u], ev[b, u]
    assert torch.equal(kd.cpu(), want_k) and torch.equal(vd.cpu(), want_v)
    assert cd.cpu().tolist() == [4, 11, 200, 300]
    # the next step over the committed cache
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=kd.cpu(), v_cache=vd.cpu(),
             sink=torch.rand(Hq, generator=g) * 6, ctx_len=cd.cpu(), max_ctx=max_ctx)
    check(sa.KV_CONTIG, d, 0, "fp8 after commit")


def test_fp8_commit_ring_and_paged():
    g = torch.Generator().manual_seed(56)
    B, T, Hkv, cap = 3, 2, 8, 128
    kc, vc = codes((B, cap, Hkv, 192), g, KS), codes((B, cap, Hkv, 128), g, VS)
    head = torch.tensor([0, 127, 5], dtype=torch.int32)
    ln = torch.tensor([128, 3, 127], dtype=torch.int32)
    k_new, v_new = rnd((B, T, Hkv, 192), g), rnd((B, T, Hkv, 128), g)
    n_acc = torch.tensor([2, 2, 1], dtype=torch.int32)
    kd, vd, hd, ld = kc.cuda(), vc.cuda(), head.cuda(), ln.cuda()
    sa.sinkattn_kv_commit(sa.KV_RING, k_new.cuda(), v_new.cuda(), n_acc.cuda(), kd, vd,
                          ring_head=hd, ring_len=ld, k_scale=KS, v_scale=VS)
    torch.cuda.synchronize()
    ek, ev = oracle.fp8_encode(k_new, KS), oracle.fp8_encode(v_new, VS)
    # the oracle's commit moves bf16 rows, so the oracle's codes are placed here by the ring's
    # slot rule (the same rule the bf16 commit tests check against the oracle)
    want_k, want_v = kc.clone(), vc.clone()
    for b in range(B):
        h_, l_ = int(head[b]), int(ln[b])
        for u in range(int(n_acc[b])):
            if l_ < cap:
                slot = (h_ + l_) % cap
                l_ += 1
            else:
                slot = h_
                h_ = (h_ + 1) % cap
            want_k[b, slot], want_v[b, slot] = ek[b, u], ev[b, u]
    assert torch.equal(kd.cpu(), want_k) and torch.equal(vd.cpu(), want_v)
    assert hd.cpu().tolist() == [2, 127, 5] and ld.cpu().tolist() == [128, 5, 128]
    # paged: 32-token pages
    P, max_pages, total = 32, 4, 12
    kc, vc = codes((total, P, Hkv, 192), g, KS), codes((total, P, Hkv, 128), g, VS)
    table = torch.randperm(total, generator=g).to(torch.int32)[:B * max_pages].view(B, max_pages).clone()
    ctx = torch.tensor([31, 0, 64], dtype=torch.int32)
    kd, vd, cd = kc.cuda(), vc.cuda(), ctx.cuda()
    sa.sinkattn_kv_commit(sa.KV_PAGED, k_new.cuda(), v_new.cuda(), n_acc.cuda(), kd, vd,
                          ctx_len=cd, page_table=table.cuda(), k_scale=KS, v_scale=VS)
    torch.cuda.synchronize()
    want_k, want_v = kc.clone(), vc.clone()
    for b in range(B):
        for u in range(int(n_acc[b])):
            c = int(ctx[b]) + u
            pg, r = int(table[b, c // P]), c % P
            want_k[pg, r], want_v[pg, r] = ek[b, u], ev[b, u]
    assert torch.equal(kd.cpu(), want_k) and torch.equal(vd.cpu(), want_v)
    assert cd.cpu().tolist() == [33, 2, 65]


def test_fp8_scales_are_applied_separately():
    """k_scale enters the logits and v_scale the output: doubling v_scale doubles O and leaves
    LSE unchanged; changing k_scale changes the logits (checked against the oracle)."""
    g = torch.Generator().manual_seed(57)
    B, T, Hq, Hkv, n = 2, 1, 16, 2, 90
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=codes((B, n, Hkv, 192), g, KS),
             v_cache=codes((B, n, Hkv, 128), g, VS), sink=torch.rand(Hq, generator=g) * 6,
             ctx_len=torch.tensor([n, 33], dtype=torch.int32), max_ctx=n)
    for ks, vs in ((KS, VS), (0.05, VS), (KS, 2 * VS)):
        check(sa.KV_CONTIG, d, 0, f"fp8 scales {ks}/{vs}", ks=ks, vs=vs)


def test_fp8_full_size_sampled():
    """The benchmark's launch: GA decode, B = 8 sequences of 262144 cached tokens, 64 Q / 4 KV
    heads, FP8 cache (split-KV with merge); four sequences checked against the oracle."""
    w = W.GA_DECODE
    d = W.decode_inputs(w, device="cuda", fp8=True)
    o, lse = sa.sinkattn_decode(w.kind, d["q"], d["k_new"], d["v_new"], d["k_cache"],
                                d["v_cache"], d["sink"], ctx_len=d["ctx_len"],
                                max_ctx=d["max_ctx"], k_scale=d["k_scale"], v_scale=d["v_scale"])
    torch.cuda.synchronize()
    seqs = [0, 3, 5, 7]
    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    sub = lambda t: t[seqs]
    ro, rl, _ = oracle.decode_fp8(oracle.KV_CONTIG, sub(cpu["q"]), sub(cpu["k_new"]),
                                  sub(cpu["v_new"]), sub(cpu["k_cache"]), sub(cpu["v_cache"]),
                                  d["k_scale"], d["v_scale"], cpu["sink"], SCALE, 0,
                                  ctx_len=sub(cpu["ctx_len"]))
    assert_close(o[seqs], ro, lse[seqs], rl, "fp8 GA decode full size")
    assert sa.sinkattn_take_device_error() == 0
