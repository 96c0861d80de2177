"""GPU parity of sink-attention decode / speculative verify (ring, contiguous and paged
caches, split-KV with the sink merged once) and of the cache commit, against the fp64 oracle."""
import math

import pytest
import torch

import oracle
import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(192)


def rnd(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def to_dev(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def gpu_decode(kind, d, window):
    dd = to_dev(d)
    kw = dict(window=window)
    if kind == sa.KV_RING:
        kw.update(ring_head=dd["ring_head"], ring_len=dd["ring_len"])
    else:
        kw.update(ctx_len=dd["ctx_len"], max_ctx=d.get("max_ctx"))
    if kind == sa.KV_PAGED:
        kw.update(page_table=dd["page_table"])
    o, lse = sa.sinkattn_decode(kind, dd["q"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                dd["v_cache"], dd["sink"], **kw)
    torch.cuda.synchronize()
    return o, lse


def oracle_decode(kind, d, window, seqs=None):
    kw = {}
    if kind == sa.KV_RING:
        kw.update(ring_head=d["ring_head"], ring_len=d["ring_len"])
    else:
        kw.update(ctx_len=d["ctx_len"])
    if kind == sa.KV_PAGED:
        kw.update(page_table=d["page_table"], page_size=d["k_cache"].shape[1])
    return oracle.decode(kind, d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                         d["sink"], SCALE, window, seqs=seqs, **kw)


def check(kind, d, window, what, seqs=None):
    o, lse = gpu_decode(kind, d, window)
    ro, rl, _ = oracle_decode(kind, d, window, seqs)
    if seqs is not None:
        o, lse = o[seqs], lse[seqs]
    assert_close(o, ro, lse, rl, what)
    assert sa.sinkattn_take_device_error() == 0


def make_sink(Hq, g, mode="rand"):
    if mode == "none":
        return None
    s = torch.rand(Hq, generator=g) * 6
    if mode == "mixed":
        s[::5] = float("-inf")
    return s


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("Hq,Hkv", [(64, 8), (8, 1), (16, 2)])
def test_ring_decode(T, Hq, Hkv):
    g = torch.Generator().manual_seed(100 * T + Hq)
    B, cap = 6, 128
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, cap, Hkv, 192), g),
             v_cache=rnd((B, cap, Hkv, 128), g), sink=make_sink(Hq, g, "mixed"),
             ring_head=torch.tensor([0, 5, 127, 64, 3, 90], dtype=torch.int32),
             ring_len=torch.tensor([128, 0, 1, 127, 128, 40], dtype=torch.int32))
    check(sa.KV_RING, d, 128, f"ring T{T} {Hq}/{Hkv}")


@pytest.mark.parametrize("cap,window", [(32, 128), (96, 64), (256, 128), (256, 0)])
@pytest.mark.parametrize("T", [1, 3])
def test_ring_decode_other_capacities(cap, window, T):
    """Rings of other sizes (the one-warp-per-item ring kernel takes any multiple of 32 slots),
    a window shorter than the ring, and a ring without a window."""
    g = torch.Generator().manual_seed(cap + 7 * T + window)
    B, Hq, Hkv = 5, 16, 2
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, cap, Hkv, 192), g),
             v_cache=rnd((B, cap, Hkv, 128), g), sink=make_sink(Hq, g, "mixed"),
             ring_head=torch.tensor([0, 1, cap - 1, cap // 2, 3], dtype=torch.int32),
             ring_len=torch.tensor([cap, cap - 1, 1, 0, cap // 3], dtype=torch.int32))
    check(sa.KV_RING, d, window, f"ring cap {cap} W{window} T{T}")


@pytest.mark.parametrize("window", [0, 1, 3, 64, 127, 200])
@pytest.mark.parametrize("T", [3, 4])
def test_ring_verify_windows(window, T):
    """128-slot rings with a 3- or 4-token verify on 8-head groups (the tensor-core ring kernel):
    windows shorter than the ring (down to one key), equal to it, longer, and none; empty,
    partial and full rings with wrapped heads; a sink of -inf on some heads."""
    g = torch.Generator().manual_seed(31 * window + T)
    B, Hq, Hkv, cap = 7, 16, 2, 128
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, cap, Hkv, 192), g),
             v_cache=rnd((B, cap, Hkv, 128), g), sink=make_sink(Hq, g, "mixed"),
             ring_head=torch.tensor([0, 17, 127, 64, 125, 90, 1], dtype=torch.int32),
             ring_len=torch.tensor([128, 0, 1, 127, 128, 40, 2], dtype=torch.int32))
    check(sa.KV_RING, d, window, f"ring verify W{window} T{T}")


@pytest.mark.parametrize("T", [1, 4])
def test_ring_decode_strided_views(T):
    """The tensor-core ring kernel on views: Q, K_new and V_new sliced out of one fused
    projection buffer per token (strided heads and tokens), the ring caches slices of wider
    per-slot buffers; results must equal the oracle on the same values."""
    g = torch.Generator().manual_seed(41 + T)
    B, Hq, Hkv, cap = 3, 16, 2, 128
    width = Hq * 192 + Hkv * 192 + Hkv * 128 + 64
    qkv = torch.randn(B, T, width, generator=g).to(torch.bfloat16).cuda()
    o1, o2 = Hq * 192, (Hq + Hkv) * 192
    q = qkv[:, :, :o1].view(B, T, Hq, 192)
    kn = qkv[:, :, o1:o2].view(B, T, Hkv, 192)
    vn = qkv[:, :, o2:o2 + Hkv * 128].view(B, T, Hkv, 128)
    kwide = torch.randn(B, cap, Hkv, 256, generator=g).to(torch.bfloat16).cuda()
    vwide = torch.randn(B, cap, Hkv, 192, generator=g).to(torch.bfloat16).cuda()
    kc, vc = kwide[..., :192], vwide[..., :128]
    assert not q.is_contiguous() and not kc.is_contiguous()
    sink = make_sink(Hq, g, "mixed")
    head = torch.tensor([3, 127, 64], dtype=torch.int32)
    ln = torch.tensor([128, 100, 128], dtype=torch.int32)
    o, lse = sa.sinkattn_decode(sa.KV_RING, q, kn, vn, kc, vc, sink.cuda(), window=128,
                                ring_head=head.cuda(), ring_len=ln.cuda())
    torch.cuda.synchronize()
    d = dict(q=q.cpu(), k_new=kn.cpu(), v_new=vn.cpu(), k_cache=kc.cpu(), v_cache=vc.cpu(),
             sink=sink, ring_head=head, ring_len=ln)
    ro, rl, _ = oracle_decode(sa.KV_RING, d, 128)
    assert_close(o, ro, lse, rl, f"ring views T{T}")
    assert sa.sinkattn_take_device_error() == 0


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("ctx", [[0, 1, 63, 64], [65, 127, 128, 129], [1000, 5000, 3, 4093]])
def test_contig_decode(T, ctx):
    g = torch.Generator().manual_seed(sum(ctx) + T)
    B, Hq, Hkv = len(ctx), 64, 4
    maxc = max(max(ctx), 1)
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, maxc, Hkv, 192), g),
             v_cache=rnd((B, maxc, Hkv, 128), g), sink=make_sink(Hq, g, "mixed"),
             ctx_len=torch.tensor(ctx, dtype=torch.int32), max_ctx=maxc)
    check(sa.KV_CONTIG, d, 0, f"contig T{T} ctx{ctx}")


def test_contig_decode_sink_none_and_window():
    g = torch.Generator().manual_seed(77)
    B, T, Hq, Hkv, maxc = 3, 3, 16, 2, 700
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((B, maxc, Hkv, 192), g),
             v_cache=rnd((B, maxc, Hkv, 128), g), sink=None,
             ctx_len=torch.tensor([700, 100, 2], dtype=torch.int32), max_ctx=maxc)
    check(sa.KV_CONTIG, d, 0, "contig no sink")
    d["sink"] = make_sink(Hq, g)
    check(sa.KV_CONTIG, d, 128, "contig with a 128 window")
    check(sa.KV_CONTIG, d, 5, "contig with a 5 window")


@pytest.mark.parametrize("P", [256, 192, 128, 64, 16])
@pytest.mark.parametrize("T", [1, 4])
def test_paged_decode(P, T):
    g = torch.Generator().manual_seed(P + T)
    B, Hq, Hkv = 4, 64, 4
    ctx = torch.tensor([1, 300, 2049, 4000], dtype=torch.int32)
    max_pages = (4000 + P - 1) // P
    pages = [(int(c) + P - 1) // P for c in ctx]
    total = sum(pages)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    table = torch.zeros(B, max_pages, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        table[b, :n] = perm[off:off + n]
        off += n
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=rnd((total, P, Hkv, 192), g),
             v_cache=rnd((total, P, Hkv, 128), g), sink=make_sink(Hq, g, "mixed"),
             ctx_len=ctx, page_table=table, max_ctx=max_pages * P)
    check(sa.KV_PAGED, d, 0, f"paged P{P} T{T}")


@pytest.mark.parametrize("P", [128, 16])
@pytest.mark.parametrize("T", [1, 2])
def test_paged_decode_missing_pages(P, T):
    """Page ids outside the pool hide that page's keys (the library's contract for a sparse
    page table). Without a window every cached key is visible whatever its position, so the
    answer is the oracle on a contiguous cache holding only the present pages' rows."""
    g = torch.Generator().manual_seed(900 + P + T)
    B, Hq, Hkv = 3, 64, 4
    ctx = [5 * P + 7, 3 * P, 2 * P - 1]
    max_pages = max((c + P - 1) // P for c in ctx)
    npg = [(c + P - 1) // P for c in ctx]
    total = sum(npg)
    perm = torch.randperm(total, generator=g).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[off:off + n]
        off += n
    table[0, 1] = -1         # a hole in the middle
    table[0, 4] = total + 3  # an id past the pool
    table[1, 0] = -7         # the first page
    table[2, 1] = total      # the last, partial page
    kc, vc = rnd((total, P, Hkv, 192), g), rnd((total, P, Hkv, 128), g)
    d = dict(q=rnd((B, T, Hq, 192), g), k_new=rnd((B, T, Hkv, 192), g),
             v_new=rnd((B, T, Hkv, 128), g), k_cache=kc, v_cache=vc,
             sink=make_sink(Hq, g, "mixed"), ctx_len=torch.tensor(ctx, dtype=torch.int32),
             page_table=table, max_ctx=max_pages * P)
    o, lse = gpu_decode(sa.KV_PAGED, d, 0)
    assert sa.sinkattn_take_device_error() == 0
    # the keys that stay: rows c < ctx of pages whose id is in the pool, in position order
    rows_k, rows_v, kept = [], [], []
    for b in range(B):
        ks, vs = [], []
        for c in range(ctx[b]):
            pid = int(table[b, c // P])
            if 0 <= pid < total:
                ks.append(kc[pid, c % P])
                vs.append(vc[pid, c % P])
        kept.append(len(ks))
        rows_k.append(ks)
        rows_v.append(vs)
    assert kept[0] == ctx[0] - 2 * P and kept[1] == ctx[1] - P and kept[2] == P
    maxc = max(kept)
    kcc = torch.zeros(B, maxc, Hkv, 192, dtype=torch.bfloat16)
    vcc = torch.zeros(B, maxc, Hkv, 128, dtype=torch.bfloat16)
    for b in range(B):
        if kept[b]:
            kcc[b, :kept[b]] = torch.stack(rows_k[b])
            vcc[b, :kept[b]] = torch.stack(rows_v[b])
    dc = dict(d, k_cache=kcc, v_cache=vcc, ctx_len=torch.tensor(kept, dtype=torch.int32))
    ro, rl, _ = oracle_decode(sa.KV_CONTIG, dc, 0)
    assert_close(o, ro, lse, rl, f"paged P{P} T{T} with missing pages")


def test_full_size_swa_ring_decode():
    """B=256 sequences, 128-slot ring, 64 Q / 8 KV heads: every output."""
    w = W.SWA_DECODE
    d = W.decode_inputs(w)
    check(w.kind, d, w.window, w.name)


def test_full_size_ga_decode_sampled_sequences():
    """B=8, context 262144 (split-KV path), all heads of two sequences."""
    w = W.GA_DECODE
    dd = W.decode_inputs(w, device="cuda")
    o, lse = sa.sinkattn_decode(w.kind, dd["q"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                dd["v_cache"], dd["sink"], ctx_len=dd["ctx_len"])
    torch.cuda.synchronize()
    seqs = [0, 5]
    sub = {k: (v[seqs].cpu() if k not in ("sink",) and isinstance(v, torch.Tensor) else v)
           for k, v in dd.items()}
    sub["sink"] = dd["sink"].cpu()
    ro, rl, _ = oracle.decode(w.kind, sub["q"], sub["k_new"], sub["v_new"], sub["k_cache"],
                              sub["v_cache"], sub["sink"], SCALE, 0, ctx_len=sub["ctx_len"])
    assert_close(o[seqs], ro, lse[seqs], rl, w.name)
    assert sa.sinkattn_take_device_error() == 0


@pytest.mark.parametrize("layer", [0, 1])
def test_hybrid_verify_layers_sampled(layer):
    """Hybrid speculative-verify step, B=64, T=4, context ~U[4096, 65536]: one GA layer (paged
    cache, sampled sequences) and one SWA layer (ring, every sequence)."""
    w = W.hybrid_layer_workload(layer)
    d = W.decode_inputs(w, device="cuda")
    dc = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    if w.kind == sa.KV_RING:
        check(w.kind, dc, w.window, w.name)
        return
    o, lse = sa.sinkattn_decode(w.kind, d["q"], d["k_new"], d["v_new"], d["k_cache"],
                                d["v_cache"], d["sink"], ctx_len=d["ctx_len"],
                                page_table=d["page_table"], max_ctx=d["max_ctx"])
    torch.cuda.synchronize()
    seqs = [0, 17, 63]
    ro, rl, _ = oracle_decode(w.kind, dc, w.window, seqs=seqs)
    assert_close(o[seqs], ro, lse[seqs], rl, w.name)


# ----------------------------------------------------------------------------------------------
# commit
# ----------------------------------------------------------------------------------------------

def test_commit_ring_contig_paged():
    g = torch.Generator().manual_seed(5)
    B, T, Hkv = 4, 4, 2
    kn, vn = rnd((B, T, Hkv, 192), g), rnd((B, T, Hkv, 128), g)
    acc = torch.tensor([0, 1, 3, 4], dtype=torch.int32)
    # ring
    kc, vc = rnd((B, 128, Hkv, 192), g), rnd((B, 128, Hkv, 128), g)
    head = torch.tensor([0, 127, 5, 60], dtype=torch.int32)
    ln = torch.tensor([128, 128, 10, 126], dtype=torch.int32)
    want = oracle.commit(oracle.KV_RING, kn, vn, acc, kc, vc, ring_head=head, ring_len=ln)
    kcd, vcd, hd, ld = kc.cuda(), vc.cuda(), head.cuda(), ln.cuda()
    sa.sinkattn_kv_commit(sa.KV_RING, kn.cuda(), vn.cuda(), acc.cuda(), kcd, vcd,
                          ring_head=hd, ring_len=ld)
    torch.cuda.synchronize()
    assert torch.equal(kcd.cpu(), want[0]) and torch.equal(vcd.cpu(), want[1])
    assert torch.equal(hd.cpu(), want[2]) and torch.equal(ld.cpu(), want[3])
    # contiguous
    kc, vc = rnd((B, 64, Hkv, 192), g), rnd((B, 64, Hkv, 128), g)
    ctx = torch.tensor([0, 10, 62, 63], dtype=torch.int32)
    want = oracle.commit(oracle.KV_CONTIG, kn[:, :, :], vn, torch.tensor([0, 1, 2, 1], dtype=torch.int32),
                         kc, vc, ctx_len=ctx)
    kcd, vcd, cd = kc.cuda(), vc.cuda(), ctx.cuda()
    sa.sinkattn_kv_commit(sa.KV_CONTIG, kn.cuda(), vn.cuda(),
                          torch.tensor([0, 1, 2, 1], dtype=torch.int32, device="cuda"), kcd, vcd,
                          ctx_len=cd)
    torch.cuda.synchronize()
    assert torch.equal(kcd.cpu(), want[0]) and torch.equal(vcd.cpu(), want[1])
    assert torch.equal(cd.cpu(), want[4])
    # paged
    P, max_pages = 16, 4
    table = torch.randperm(B * max_pages, generator=g).to(torch.int32).reshape(B, max_pages)
    kp, vp = rnd((B * max_pages, P, Hkv, 192), g), rnd((B * max_pages, P, Hkv, 128), g)
    ctx = torch.tensor([0, 15, 30, 60], dtype=torch.int32)
    want = oracle.commit(oracle.KV_PAGED, kn, vn, acc, kp, vp, ctx_len=ctx, page_table=table,
                         page_size=P)
    kpd, vpd, cd = kp.cuda(), vp.cuda(), ctx.cuda()
    sa.sinkattn_kv_commit(sa.KV_PAGED, kn.cuda(), vn.cuda(), acc.cuda(), kpd, vpd, ctx_len=cd,
                          page_table=table.cuda())
    torch.cuda.synchronize()
    assert torch.equal(kpd.cpu(), want[0]) and torch.equal(vpd.cpu(), want[1])
    assert torch.equal(cd.cpu(), want[4])


def test_decode_then_commit_matches_prefill():
    """Speculative step: verify T=4 drafts, accept some, commit, decode the next token; the
    result equals prefill of the whole sequence at that row (SWA ring and GA contiguous)."""
    g = torch.Generator().manual_seed(9)
    Hq, Hkv, T = 16, 2, 4
    L0 = 200
    seq_k, seq_v = rnd((1, L0 + 8, Hkv, 192), g), rnd((1, L0 + 8, Hkv, 128), g)
    seq_q = rnd((1, L0 + 8, Hq, 192), g)
    sink = torch.rand(Hq, generator=g) * 6
    for window in (128, 0):
        if window:
            cap = 128
            kc = torch.zeros(1, cap, Hkv, 192, dtype=torch.bfloat16)
            vc = torch.zeros(1, cap, Hkv, 128, dtype=torch.bfloat16)
            for p in range(L0 - cap, L0):
                kc[0, p % cap], vc[0, p % cap] = seq_k[0, p], seq_v[0, p]
            meta = dict(ring_head=torch.tensor([L0 % cap], dtype=torch.int32).cuda(),
                        ring_len=torch.tensor([cap], dtype=torch.int32).cuda())
            kind = sa.KV_RING
        else:
            kc = torch.zeros(1, L0 + 8, Hkv, 192, dtype=torch.bfloat16)
            vc = torch.zeros(1, L0 + 8, Hkv, 128, dtype=torch.bfloat16)
            kc[0, :L0], vc[0, :L0] = seq_k[0, :L0], seq_v[0, :L0]
            meta = dict(ctx_len=torch.tensor([L0], dtype=torch.int32).cuda())
            kind = sa.KV_CONTIG
        kcd, vcd = kc.cuda(), vc.cuda()
        sl = slice(L0, L0 + T)
        o, lse = sa.sinkattn_decode(kind, seq_q[:, sl].cuda(), seq_k[:, sl].cuda(),
                                    seq_v[:, sl].cuda(), kcd, vcd, sink.cuda(), window=window,
                                    **meta)
        sa.sinkattn_kv_commit(kind, seq_k[:, sl].cuda(), seq_v[:, sl].cuda(),
                              torch.tensor([3], dtype=torch.int32).cuda(), kcd, vcd, **meta)
        sl2 = slice(L0 + 3, L0 + 4)
        o2, lse2 = sa.sinkattn_decode(kind, seq_q[:, sl2].cuda(), seq_k[:, sl2].cuda(),
                                      seq_v[:, sl2].cuda(), kcd, vcd, sink.cuda(), window=window,
                                      **meta)
        torch.cuda.synchronize()
        ro, rl, _ = oracle.prefill(seq_q[:, :L0 + 4], seq_k[:, :L0 + 4], seq_v[:, :L0 + 4], sink,
                                   SCALE, window, rows=[[0, L0 + t] for t in range(4)])
        assert_close(o[0], ro, lse[0], rl, f"verify W{window}")
        assert_close(o2[0, 0], ro[3], lse2[0, 0], rl[3], f"after commit W{window}")
