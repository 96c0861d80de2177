"""Pins for the fp64 oracle: it is checked against things other than itself.

* the worked example printed on the page "MiMo-V2-Flash Technical Report" (paper notes), §4.3
  (tests/golden/worked_example.json), plus its closed form;
* a library attention routine (torch scaled_dot_product_attention, fp64, CPU) when the sink is
  -inf, which the pages say reduces to standard softmax ("MiMo-V2-Flash 架构 QA", Q3.7);
* the eager concat -> softmax -> drop formulation ("MiMo-V2-Flash 模型架构深度拆解", CH10.1 and
  "MiMo-V2-Flash 架构 QA", Q3.8) built from library softmax / logsumexp;
* invariants the mathematics fixes: weights + sink share = 1, shift invariance, SWA == GA when
  the window covers the sequence, GQA == MHA with repeated K/V, decode == prefill of the
  concatenated sequence, ring / paged caches == the contiguous cache, split + merge == direct.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from global_attention_sink_softmax_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")
pytestmark = pytest.mark.filterwarnings("ignore")


def bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def rand_bf16(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16)


# ----------------------------------------------------------------------------------------------
# the worked example (paper notes §4.3)
# ----------------------------------------------------------------------------------------------

def worked_example_inputs(L, n_keys_logit, window):
    """All logits equal 2 (scale 1: q = 2 e0, k_j = e0), sink 4, v_j = e_(j mod 128)."""
    dq, dv = 192, 128
    q = torch.zeros(1, L, 1, dq)
    q[..., 0] = n_keys_logit
    k = torch.zeros(1, L, 1, dq)
    k[..., 0] = 1.0
    v = torch.zeros(1, L, 1, dv)
    for j in range(L):
        v[0, j, 0, j % dv] = 1.0
    return bf(q), bf(k), bf(v), torch.tensor([4.0])


@pytest.mark.parametrize("L,row,window", [(128, 127, 128), (128, 127, 0), (256, 200, 128),
                                          (300, 299, 128)])
def test_worked_example_printed_numbers(L, row, window):
    gold = json.load(open(GOLDEN))
    p, tol = gold["printed"], gold["printed_half_ulp"]
    q, k, v, sink = worked_example_inputs(L, gold["inputs"]["logit"], window)
    o, lse, ws = oracle.prefill(q, k, v, sink, scale=1.0, window=window,
                                rows=[[0, row]], want_wsink=True)
    weights = o[0, 0]                     # v is one-hot, so O is the weight vector
    lse = float(lse[0, 0])
    m = 4.0                               # the page: m = max(max(0..2), 4) = 4
    D = math.exp(lse - m)                 # LSE = m + ln D
    nz = weights[weights > 0]
    # exactly 128 keys are visible: the window holds 128 keys including the query
    assert nz.numel() == gold["inputs"]["n_keys"]
    checks = {
        "denominator": D,
        "per_key_weight": float(nz.max()),
        "weights_sum": float(weights.sum()),
        "sink_share": float(ws[0, 0]),
        "per_key_numerator": float(nz.max()) * D,
        "sink_numerator": float(ws[0, 0]) * D,
        "m": m,
    }
    for key, val in checks.items():
        assert abs(val - p[key]) <= tol[key] + 1e-12, (key, val, p[key])
    # closed form: D = 1 + 128 e^-2, w_j = e^-2 / D, w_s = 1 / D
    Dx = 1.0 + 128.0 * math.exp(-2.0)
    assert abs(D - Dx) < 1e-12
    assert torch.allclose(nz, torch.full_like(nz, math.exp(-2.0) / Dx), rtol=0, atol=1e-15)
    assert abs(float(ws[0, 0]) - 1.0 / Dx) < 1e-15


def test_worked_example_bound_for_logits_in_0_2():
    """Logits anywhere in [0, 2] with sink 4: 1 + 128 e^-4 <= D <= 1 + 128 e^-2 (paper notes
    §4.3 bounds each numerator term by exp(-2))."""
    g = torch.Generator().manual_seed(7)
    L, dq, dv = 128, 192, 128
    u = torch.rand(L, generator=g) * 2.0
    q = torch.zeros(1, L, 1, dq)
    q[..., 0] = 1.0
    k = torch.zeros(1, L, 1, dq)
    k[0, :, 0, 0] = u
    v = rand_bf16((1, L, 1, dv), g)
    o, lse, ws = oracle.prefill(bf(q), bf(k), v, torch.tensor([4.0]), scale=1.0, window=128,
                                rows=[[0, L - 1]], want_wsink=True)
    D = math.exp(float(lse[0, 0]) - 4.0)
    assert 1 + 128 * math.exp(-4) - 1e-12 <= D <= 1 + 128 * math.exp(-2) + 1e-12
    # and it is exact for the drawn logits (they are bf16-rounded)
    a = bf(u).double()
    assert abs(D - (1 + torch.exp(a - 4).sum().item())) < 1e-12


# ----------------------------------------------------------------------------------------------
# library routines
# ----------------------------------------------------------------------------------------------

def band_mask(L, window):
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    keep = j <= i
    if window > 0:
        keep &= j > i - window
    return keep


def to_bhld(x):
    return x.double().permute(0, 2, 1, 3)


@pytest.mark.parametrize("B,L,Hq,Hkv,window", [(2, 37, 4, 2, 0), (1, 70, 8, 1, 16),
                                               (2, 33, 6, 3, 5), (1, 129, 4, 4, 128)])
def test_no_sink_equals_library_attention(B, L, Hq, Hkv, window):
    """sink = -inf (and sink = NULL) reduce to standard softmax (QA Q3.7): compare with torch
    scaled_dot_product_attention in fp64 (GQA via enable_gqa, head h -> KV head h // G)."""
    g = torch.Generator().manual_seed(11)
    dq, dv = 192, 128
    q, k, v = rand_bf16((B, L, Hq, dq), g), rand_bf16((B, L, Hkv, dq), g), rand_bf16((B, L, Hkv, dv), g)
    scale = 1.0 / math.sqrt(dq)
    mask = band_mask(L, window)
    ref = F.scaled_dot_product_attention(to_bhld(q), to_bhld(k), to_bhld(v), attn_mask=mask,
                                         scale=scale, enable_gqa=True).permute(0, 2, 1, 3)
    scores = torch.matmul(to_bhld(q), to_bhld(k).repeat_interleave(Hq // Hkv, 1).transpose(-1, -2))
    scores = (scores * scale).masked_fill(~mask, float("-inf"))
    ref_lse = torch.logsumexp(scores, dim=-1).permute(0, 2, 1)
    for sink in (None, torch.full((Hq,), float("-inf"))):
        o, lse, _ = oracle.prefill(q, k, v, sink, scale, window)
        assert torch.allclose(o, ref, rtol=0, atol=1e-12)
        assert torch.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def eager_sink_attention(q, k, v, sink, scale, window):
    """The pages' eager formulation: scaled, masked scores; append the per-head sink as one
    more column; softmax over S+1; drop the sink column; multiply by V."""
    B, L, Hq, _ = q.shape
    G = Hq // k.shape[2]
    qq, kk, vv = to_bhld(q), to_bhld(k).repeat_interleave(G, 1), to_bhld(v).repeat_interleave(G, 1)
    scores = torch.matmul(qq, kk.transpose(-1, -2)) * scale
    scores = scores.masked_fill(~band_mask(L, window), float("-inf"))
    s = sink.double().reshape(1, Hq, 1, 1).expand(B, Hq, L, 1)
    cat = torch.cat([scores, s], dim=-1)
    probs = torch.softmax(cat, dim=-1)[..., :-1]
    out = torch.matmul(probs, vv).permute(0, 2, 1, 3)
    lse = torch.logsumexp(cat, dim=-1).permute(0, 2, 1)
    wsink = torch.softmax(cat, dim=-1)[..., -1].permute(0, 2, 1)
    return out, lse, wsink


@pytest.mark.parametrize("B,L,Hq,Hkv,window,scale", [
    (1, 64, 8, 1, 128, 1 / math.sqrt(192)),
    (2, 50, 4, 2, 0, 1 / math.sqrt(192)),
    (1, 200, 4, 1, 128, 1 / math.sqrt(192)),
    (1, 40, 2, 1, 7, 0.37),           # scale != 1 separates "sink in post-scale units"
])
def test_equals_eager_concat_softmax_drop(B, L, Hq, Hkv, window, scale):
    g = torch.Generator().manual_seed(13)
    dq, dv = 192, 128
    q, k, v = rand_bf16((B, L, Hq, dq), g), rand_bf16((B, L, Hkv, dq), g), rand_bf16((B, L, Hkv, dv), g)
    sink = torch.rand(Hq, generator=g) * 6.0
    sink[0] = float("-inf")
    o, lse, ws = oracle.prefill(q, k, v, sink, scale, window, want_wsink=True)
    ro, rl, rw = eager_sink_attention(q, k, v, sink, scale, window)
    assert torch.allclose(o, ro, rtol=0, atol=1e-12)
    assert torch.allclose(lse, rl, rtol=0, atol=1e-12)
    assert torch.allclose(ws, rw, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------------------------

def test_weights_plus_sink_share_is_one():
    """The kept weights sum to 1 - (sink share) (QA Q3.8: the sink's mass is dropped)."""
    g = torch.Generator().manual_seed(17)
    L, dq, dv = 128, 192, 128
    q, k = rand_bf16((1, L, 4, dq), g), rand_bf16((1, L, 2, dq), g)
    v = torch.eye(L, dv).reshape(1, L, 1, dv).repeat(1, 1, 2, 1).to(torch.bfloat16)
    sink = torch.tensor([0.0, 3.0, 6.0, float("-inf")])
    for window in (0, 128, 31):
        o, lse, ws = oracle.prefill(q, k, v, sink, 1 / math.sqrt(dq), window, want_wsink=True)
        total = o.sum(-1) + ws
        assert torch.allclose(total, torch.ones_like(total), rtol=0, atol=1e-12)
        assert (ws[..., 3] == 0).all()          # -inf sink takes no mass
        assert (ws[..., :3] > 0).all()


def test_shift_invariance():
    """Adding c to every logit and to the sink leaves O unchanged and adds c to LSE."""
    g = torch.Generator().manual_seed(19)
    L, dq, dv, c = 40, 16, 128, 3.0
    q, k, v = rand_bf16((1, L, 2, dq), g), rand_bf16((1, L, 1, dq), g), rand_bf16((1, L, 1, dv), g)
    sink = torch.tensor([1.5, 5.0])
    o, lse, _ = oracle.prefill(q, k, v, sink, 1.0, 0)
    q2 = torch.cat([q, torch.ones(1, L, 2, 1, dtype=torch.bfloat16)], -1)
    k2 = torch.cat([k, torch.full((1, L, 1, 1), c, dtype=torch.bfloat16)], -1)
    o2, lse2, _ = oracle.prefill(q2, k2, v, sink + c, 1.0, 0)
    assert torch.allclose(o2, o, rtol=0, atol=1e-12)
    assert torch.allclose(lse2, lse + c, rtol=0, atol=1e-12)


def test_swa_equals_ga_when_window_covers_sequence():
    g = torch.Generator().manual_seed(23)
    L = 100
    q, k, v = rand_bf16((2, L, 4, 192), g), rand_bf16((2, L, 2, 192), g), rand_bf16((2, L, 2, 128), g)
    sink = torch.rand(4, generator=g) * 6
    a = oracle.prefill(q, k, v, sink, 0.07, 0)
    for window in (L, L + 1, 4096):
        b = oracle.prefill(q, k, v, sink, 0.07, window)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    c = oracle.prefill(q, k, v, sink, 0.07, L - 1)
    assert not torch.equal(a[0], c[0])


def test_gqa_equals_mha_with_repeated_kv():
    g = torch.Generator().manual_seed(29)
    L, Hq, Hkv = 30, 8, 2
    q, k, v = rand_bf16((1, L, Hq, 192), g), rand_bf16((1, L, Hkv, 192), g), rand_bf16((1, L, Hkv, 128), g)
    sink = torch.rand(Hq, generator=g) * 6
    a = oracle.prefill(q, k, v, sink, 0.07, 9)
    G = Hq // Hkv
    b = oracle.prefill(q, k.repeat_interleave(G, 2), v.repeat_interleave(G, 2), sink, 0.07, 9)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_row_sampling_matches_full():
    g = torch.Generator().manual_seed(31)
    q, k, v = rand_bf16((2, 50, 4, 192), g), rand_bf16((2, 50, 1, 192), g), rand_bf16((2, 50, 1, 128), g)
    sink = torch.rand(4, generator=g) * 6
    full = oracle.prefill(q, k, v, sink, 0.07, 16)
    rows = [[1, 0], [0, 49], [1, 17]]
    part = oracle.prefill(q, k, v, sink, 0.07, 16, rows=rows)
    for n, (b, i) in enumerate(rows):
        assert torch.equal(part[0][n], full[0][b, i]) and torch.equal(part[1][n], full[1][b, i])


# ----------------------------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------------------------

def concat_prefill_rows(k_cache_seq, v_cache_seq, q, k_new, v_new, sink, scale, window):
    """Prefill of [cached tokens ++ new tokens]; returns the rows of the new tokens."""
    n = k_cache_seq.shape[0]
    T, Hq, dq = q.shape
    Hkv = k_new.shape[1]
    L = n + T
    qq = torch.zeros(1, L, Hq, dq, dtype=torch.bfloat16)
    qq[0, n:] = q
    kk = torch.cat([k_cache_seq, k_new], 0)[None]
    vv = torch.cat([v_cache_seq, v_new], 0)[None]
    rows = [[0, n + t] for t in range(T)]
    o, lse, _ = oracle.prefill(qq, kk, vv, sink, scale, window, rows=rows)
    return o, lse


@pytest.mark.parametrize("T,window", [(1, 0), (4, 0), (1, 128), (4, 128), (3, 7)])
def test_decode_contig_equals_prefill_of_concatenation(T, window):
    g = torch.Generator().manual_seed(37)
    B, Hq, Hkv, maxc = 3, 4, 2, 300
    q = rand_bf16((B, T, Hq, 192), g)
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    kc, vc = rand_bf16((B, maxc, Hkv, 192), g), rand_bf16((B, maxc, Hkv, 128), g)
    ctx = torch.tensor([0, 129, 300], dtype=torch.int32)
    sink = torch.rand(Hq, generator=g) * 6
    o, lse, _ = oracle.decode(oracle.KV_CONTIG, q, kn, vn, kc, vc, sink, 0.07, window, ctx_len=ctx)
    for b in range(B):
        n = int(ctx[b])
        ro, rl = concat_prefill_rows(kc[b, :n], vc[b, :n], q[b], kn[b], vn[b], sink, 0.07, window)
        assert torch.equal(o[b], ro) and torch.equal(lse[b], rl)


@pytest.mark.parametrize("T", [1, 2, 4])
def test_decode_ring_equals_contig_tail(T):
    """A 128-slot ring with head h holds the last ring_len tokens, oldest at slot h."""
    g = torch.Generator().manual_seed(41)
    B, Hq, Hkv, cap, W = 4, 8, 2, 128, 128
    q = rand_bf16((B, T, Hq, 192), g)
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    ring_len = torch.tensor([128, 5, 128, 0], dtype=torch.int32)
    ring_head = torch.tensor([77, 3, 0, 9], dtype=torch.int32)
    hist = [rand_bf16((int(n), Hkv, 192), g) for n in ring_len]   # tokens oldest first
    histv = [rand_bf16((int(n), Hkv, 128), g) for n in ring_len]
    kc = torch.zeros(B, cap, Hkv, 192, dtype=torch.bfloat16)
    vc = torch.zeros(B, cap, Hkv, 128, dtype=torch.bfloat16)
    for b in range(B):
        for c in range(int(ring_len[b])):
            kc[b, (int(ring_head[b]) + c) % cap] = hist[b][c]
            vc[b, (int(ring_head[b]) + c) % cap] = histv[b][c]
    sink = torch.rand(Hq, generator=g) * 6
    o, lse, _ = oracle.decode(oracle.KV_RING, q, kn, vn, kc, vc, sink, 0.07, W,
                              ring_head=ring_head, ring_len=ring_len)
    for b in range(B):
        ro, rl = concat_prefill_rows(hist[b], histv[b], q[b], kn[b], vn[b], sink, 0.07, W)
        assert torch.equal(o[b], ro) and torch.equal(lse[b], rl)


def test_decode_paged_equals_contig():
    g = torch.Generator().manual_seed(43)
    B, T, Hq, Hkv, P = 3, 2, 4, 1, 16
    ctx = torch.tensor([1, 40, 64], dtype=torch.int32)
    maxc = 64
    q = rand_bf16((B, T, Hq, 192), g)
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    kc, vc = rand_bf16((B, maxc, Hkv, 192), g), rand_bf16((B, maxc, Hkv, 128), g)
    max_pages = maxc // P
    perm = torch.randperm(B * max_pages, generator=g).to(torch.int32)
    table = perm.reshape(B, max_pages)
    kp = torch.zeros(B * max_pages, P, Hkv, 192, dtype=torch.bfloat16)
    vp = torch.zeros(B * max_pages, P, Hkv, 128, dtype=torch.bfloat16)
    for b in range(B):
        for c in range(maxc):
            kp[table[b, c // P], c % P] = kc[b, c]
            vp[table[b, c // P], c % P] = vc[b, c]
    sink = torch.rand(Hq, generator=g) * 6
    a = oracle.decode(oracle.KV_CONTIG, q, kn, vn, kc, vc, sink, 0.07, 0, ctx_len=ctx)
    b_ = oracle.decode(oracle.KV_PAGED, q, kn, vn, kp, vp, sink, 0.07, 0, ctx_len=ctx,
                       page_table=table, page_size=P)
    assert torch.equal(a[0], b_[0]) and torch.equal(a[1], b_[1])


def test_decode_seq_sampling():
    w = W.SWA_DECODE
    d = W.decode_inputs(w, B=6)
    full = oracle.decode(w.kind, d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                         d["sink"], W.SCALE, w.window, ring_head=d["ring_head"], ring_len=d["ring_len"])
    part = oracle.decode(w.kind, d["q"], d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                         d["sink"], W.SCALE, w.window, ring_head=d["ring_head"],
                         ring_len=d["ring_len"], seqs=[4, 1])
    assert torch.equal(part[0][0], full[0][4]) and torch.equal(part[0][1], full[0][1])


# ----------------------------------------------------------------------------------------------
# split-KV algebra and the cache commit
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("cuts", [[0, 200], [0, 1, 200], [0, 64, 64, 128, 199, 200],
                                  [0, 13, 50, 77, 140, 200]])
def test_split_merge_equals_direct_and_counts_sink_once(cuts):
    g = torch.Generator().manual_seed(47)
    n = cuts[-1]
    q = rand_bf16((1, n, 1, 192), g)
    k, v = rand_bf16((1, n, 1, 192), g), rand_bf16((1, n, 1, 128), g)
    sink = torch.tensor([4.5])
    o, lse, _ = oracle.prefill(q, k, v, sink, 0.07, 0, rows=[[0, n - 1]])
    parts = [oracle.partial(q[0, n - 1, 0], k[0, :, 0], v[0, :, 0], a, b, 0.07)
             for a, b in zip(cuts[:-1], cuts[1:])]
    mo, ml = oracle.merge([p[0].numpy() for p in parts], [p[1] for p in parts],
                          [p[2] for p in parts], 4.5)
    assert torch.allclose(mo, o[0, 0], rtol=0, atol=1e-12)
    assert abs(ml - float(lse[0, 0])) < 1e-12
    # counting the sink once per span would be wrong: check the merge is not that
    wrong = math.log(math.exp(ml) + (len(parts) - 1) * math.exp(4.5))
    assert len(parts) == 1 or abs(wrong - ml) > 1e-6


def test_commit_ring_and_contig_semantics():
    g = torch.Generator().manual_seed(53)
    B, T, Hkv, cap = 3, 4, 2, 8
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    kc, vc = rand_bf16((B, cap, Hkv, 192), g), rand_bf16((B, cap, Hkv, 128), g)
    head = torch.tensor([6, 0, 2], dtype=torch.int32)
    ln = torch.tensor([8, 5, 7], dtype=torch.int32)
    acc = torch.tensor([3, 4, 0], dtype=torch.int32)
    k2, v2, h2, l2, _ = oracle.commit(oracle.KV_RING, kn, vn, acc, kc, vc, ring_head=head, ring_len=ln)
    for b in range(B):
        before = [kc[b, (int(head[b]) + c) % cap] for c in range(int(ln[b]))]
        seq = before + [kn[b, u] for u in range(int(acc[b]))]
        want = seq[-cap:]
        assert int(l2[b]) == len(want)
        got = [k2[b, (int(h2[b]) + c) % cap] for c in range(int(l2[b]))]
        assert all(torch.equal(x, y) for x, y in zip(got, want))
    ctx = torch.tensor([0, 3, 10], dtype=torch.int32)
    kc3, vc3 = rand_bf16((B, 16, Hkv, 192), g), rand_bf16((B, 16, Hkv, 128), g)
    k3, v3, _, _, c3 = oracle.commit(oracle.KV_CONTIG, kn, vn, acc, kc3, vc3, ctx_len=ctx)
    for b in range(B):
        assert int(c3[b]) == int(ctx[b]) + int(acc[b])
        assert torch.equal(k3[b, :int(ctx[b])], kc3[b, :int(ctx[b])])
        assert torch.equal(k3[b, int(ctx[b]):int(c3[b])], kn[b, :int(acc[b])])
        assert torch.equal(v3[b, int(ctx[b]):int(c3[b])], vn[b, :int(acc[b])])
        assert torch.equal(k3[b, int(c3[b]):], kc3[b, int(c3[b]):])


@pytest.mark.parametrize("accept", ["none", "one", "all"])
def test_commit_paged_equals_contig(accept):
    """The paged commit stores what the contiguous commit stores, through the page table.

    ("MiMo-V2-Flash 模型架构深度拆解" CH10.3, the "KV cache update" step; the page table of the
    serving stack, "MiMo-V2-Flash" model card.) Pages are handed out in a random permutation;
    contexts start just before, on and after page boundaries so the accepted tokens cross one.
    Checked two ways: the pool read back row by row through the table equals the contiguous
    cache (and pages no sequence owns are untouched), and the oracle's decode over the grown
    paged cache (its paged addressing pinned against prefill above) equals the decode over the
    grown contiguous cache."""
    g = torch.Generator().manual_seed(59)
    B, T, Hq, Hkv, P, maxc = 4, 4, 4, 2, 8, 32
    n = {"none": 0, "one": 1, "all": T}[accept]
    acc = torch.full((B,), n, dtype=torch.int32)
    ctx = torch.tensor([6, 8, 15, 0], dtype=torch.int32)
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    kc, vc = rand_bf16((B, maxc, Hkv, 192), g), rand_bf16((B, maxc, Hkv, 128), g)
    max_pages = maxc // P
    spare = 3  # pages in the pool that no sequence owns
    perm = torch.randperm(B * max_pages + spare, generator=g).to(torch.int32)
    table = perm[:B * max_pages].reshape(B, max_pages).contiguous()
    kp = rand_bf16((B * max_pages + spare, P, Hkv, 192), g)
    vp = rand_bf16((B * max_pages + spare, P, Hkv, 128), g)
    for b in range(B):
        for c in range(maxc):
            kp[table[b, c // P], c % P] = kc[b, c]
            vp[table[b, c // P], c % P] = vc[b, c]
    k1, v1, _, _, c1 = oracle.commit(oracle.KV_CONTIG, kn, vn, acc, kc, vc, ctx_len=ctx)
    k2, v2, _, _, c2 = oracle.commit(oracle.KV_PAGED, kn, vn, acc, kp, vp, ctx_len=ctx,
                                     page_table=table, page_size=P)
    assert torch.equal(c1, c2) and torch.equal(c1, ctx + acc)
    for b in range(B):
        for c in range(maxc):
            assert torch.equal(k2[table[b, c // P], c % P], k1[b, c]), (b, c)
            assert torch.equal(v2[table[b, c // P], c % P], v1[b, c]), (b, c)
    for pg in perm[B * max_pages:].tolist():
        assert torch.equal(k2[pg], kp[pg]) and torch.equal(v2[pg], vp[pg])
    q = rand_bf16((B, T, Hq, 192), g)
    kn2, vn2 = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    sink = torch.rand(Hq, generator=g) * 6
    a = oracle.decode(oracle.KV_CONTIG, q, kn2, vn2, k1, v1, sink, 0.07, 0, ctx_len=c1)
    b_ = oracle.decode(oracle.KV_PAGED, q, kn2, vn2, k2, v2, sink, 0.07, 0, ctx_len=c2,
                       page_table=table, page_size=P)
    assert torch.equal(a[0], b_[0]) and torch.equal(a[1], b_[1])


def test_workload_generators_are_seeded():
    a = W.prefill_inputs(W.SWA_PREFILL_SMALL, L=64)
    b = W.prefill_inputs(W.SWA_PREFILL_SMALL, L=64)
    assert all(torch.equal(a[x], b[x]) for x in a)
    s = W.prefill_inputs(W.GA_PREFILL, L=8)["sink"]
    assert torch.isinf(s[7::8]).all() and torch.isfinite(s[0::8]).all()
    assert float(s[torch.isfinite(s)].min()) >= 0 and float(s[torch.isfinite(s)].max()) <= 6


# ----------------------------------------------------------------------------------------------
# partial rotary embedding and the value scale ("MiMo-V2-Flash 模型架构深度拆解" CH3.5, CH10.3,
# CH10.5; "MiMo-V2-Flash 架构 QA" Q2.7)
# ----------------------------------------------------------------------------------------------

COS1, SIN1 = 0.5403023058681398, 0.8414709848078965  # cos(1 rad), sin(1 rad)


def unit_rows(d, dims):
    """One bf16 row of d dims per entry of dims, 1.0 in that dim."""
    x = torch.zeros(len(dims), 1, d, dtype=torch.bfloat16)
    for r, c in enumerate(dims):
        x[r, 0, c] = 1.0
    return x


def test_rope_position_zero_is_identity():
    g = torch.Generator().manual_seed(11)
    x = rand_bf16((5, 3, 192), g)
    for theta in (1e4, 5e6):
        y = oracle.rope(x, np.zeros(5, np.int64), theta)
        assert torch.equal(y, x.double())


def test_rope_closed_form_angles():
    # pair 0 turns at frequency 1: position 1 -> 1 rad; e_0 -> (cos, sin), e_32 -> (-sin, cos)
    y = oracle.rope(unit_rows(192, [0, 32]), np.array([1, 1]), 1e4)[:, 0]
    assert abs(y[0, 0] - COS1) < 1e-15 and abs(y[0, 32] - SIN1) < 1e-15
    assert abs(y[1, 0] + SIN1) < 1e-15 and abs(y[1, 32] - COS1) < 1e-15
    # pair 16 of 32 turns at theta^(-1/2): 0.01 for theta 1e4, so position 100 -> 1 rad
    y = oracle.rope(unit_rows(192, [16]), np.array([100]), 1e4)[0, 0]
    assert abs(y[16] - COS1) < 1e-13 and abs(y[48] - SIN1) < 1e-13
    # GA theta 5e6: pair 16 turns at 1/sqrt(5e6) = 1/2236.0679774997896
    y = oracle.rope(unit_rows(192, [16]), np.array([2236]), 5e6)[0, 0]
    a = 2236 / 2236.0679774997896
    assert abs(y[16] - math.cos(a)) < 1e-13 and abs(y[48] - math.sin(a)) < 1e-13
    # last pair (31) at 1e4^(-62/64) = 10^(-3.875)
    y = oracle.rope(unit_rows(192, [31]), np.array([7499]), 1e4)[0, 0]
    a = 7499 * 10 ** -3.875
    assert abs(y[31] - math.cos(a)) < 1e-12 and abs(y[63] - math.sin(a)) < 1e-12
    # nothing else moves
    mask = torch.ones(192, dtype=torch.bool)
    mask[[31, 63]] = False
    assert torch.all(y[mask] == 0)


@pytest.mark.parametrize("theta", [1e4, 5e6])
def test_rope_rotation_invariants(theta):
    g = torch.Generator().manual_seed(12)
    n = 64
    q = rand_bf16((n, 4, 192), g)
    k = rand_bf16((n, 4, 192), g)
    m = torch.randint(0, 262144, (n,), generator=g).numpy()
    s = torch.randint(0, 4096, (n,), generator=g).numpy()
    yq = oracle.rope(q, m, theta)
    # the no-pe dims pass unchanged
    assert torch.equal(yq[..., 64:], q.double()[..., 64:])
    # each pair (i, i + 32) keeps its length
    xd = q.double()
    n_in = xd[..., :32] ** 2 + xd[..., 32:64] ** 2
    n_out = yq[..., :32] ** 2 + yq[..., 32:64] ** 2
    assert torch.allclose(n_out, n_in, rtol=1e-12, atol=1e-12)
    # relative position: <R(m) q, R(n) k> depends on m - n only
    nk = torch.randint(0, 262144, (n,), generator=g).numpy()
    d1 = (yq[..., :64] * oracle.rope(k, nk, theta)[..., :64]).sum(-1)
    d2 = (oracle.rope(q, m + s, theta)[..., :64] * oracle.rope(k, nk + s, theta)[..., :64]).sum(-1)
    assert torch.allclose(d1, d2, rtol=1e-9, atol=1e-9)
    # and it is not position-free: a shifted query alone changes the score
    d3 = (oracle.rope(q, m + 1, theta)[..., :64] * oracle.rope(k, nk, theta)[..., :64]).sum(-1)
    assert (d3 - d1).abs().max() > 1e-3


def test_vscale_multiplies_every_element():
    g = torch.Generator().manual_seed(13)
    v = rand_bf16((3, 7, 2, 128), g)
    y = oracle.vscale(v, 0.707)
    assert y.shape == v.shape
    assert torch.equal(y, v.double() * 0.707)


# ----------------------------------------------------------------------------------------------
# FP8 (E4M3) cache codes and decode against an FP8 cache
# ----------------------------------------------------------------------------------------------

def test_e4m3_values_equal_the_library_for_every_code():
    codes = torch.arange(256, dtype=torch.uint8)
    ours = oracle.fp8_decode(codes)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64)
    nan = torch.isnan(lib)
    assert torch.equal(torch.isnan(ours), nan) and nan.sum() == 2  # 0x7f and 0xff
    assert torch.equal(ours[~nan], lib[~nan])


def test_e4m3_closed_forms():
    v = oracle.fp8_decode(torch.tensor([0x00, 0x01, 0x07, 0x08, 0x38, 0xb8, 0x7e, 0xfe, 0x57, 0x58],
                                       dtype=torch.uint8)).tolist()
    assert v == [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, -1.0, 448.0, -448.0, 15.0, 16.0]


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    enc = lambda xs: oracle.e4m3_encode_f32(np.array(xs, np.float32)).tolist()
    # ties go to the even code: 1.0625 between 1 (0x38) and 1.125 (0x39); 1.1875 between 1.125
    # and 1.25 (0x3a); 2^-10 between 0 and 2^-9; 3 * 2^-10 between 2^-9 and 2^-8 (0x02);
    # 15.5 between 15 (0x57) and 16 (0x58), across a binade
    assert enc([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 15.5]) == [0x38, 0x3a, 0x00, 0x02, 0x58]
    assert enc([1.0626, 1.1874, -1.0626]) == [0x39, 0x39, 0xb9]
    # beyond the largest finite value: +-448 (satfinite), NaN stays NaN
    assert enc([448.0, 449.0, 464.0, 1e30, float("inf"), -500.0, float("-inf")]) == \
        [0x7e, 0x7e, 0x7e, 0x7e, 0x7e, 0xfe, 0xfe]
    assert enc([float("nan")]) == [0x7f]
    # every finite code round-trips
    finite = [c for c in range(256) if c not in (0x7f, 0xff)]
    vals = oracle.fp8_decode(torch.tensor(finite, dtype=torch.uint8)).numpy().astype(np.float32)
    assert oracle.e4m3_encode_f32(vals).tolist() == finite


def test_e4m3_encode_equals_the_library_cast_in_range():
    g = torch.Generator().manual_seed(21)
    mag = torch.exp2(torch.rand(20000, generator=g) * 20 - 12)  # 2^-12 .. 2^8
    y = (mag * torch.where(torch.rand(20000, generator=g) < 0.5, -1.0, 1.0)).float()
    y = y.clamp(-448.0, 448.0)
    lib = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode_f32(y), lib)


def test_fp8_encode_divides_in_fp32():
    g = torch.Generator().manual_seed(22)
    x = rand_bf16((3, 5, 64), g)
    for s in (0.013, 0.5, 1 / 3):
        codes = oracle.fp8_encode(x, s)
        y = x.float().numpy() / np.float32(s)  # IEEE fp32 division
        assert np.array_equal(codes.numpy().reshape(-1), oracle.e4m3_encode_f32(y))


def eager_fp8_decode(q, k_new, v_new, kc_codes, vc_codes, ks, vs, ctx, sink, scale, window):
    """Contiguous-cache FP8 decode written out directly: dequantise (library cast for the new
    tokens), concatenate, softmax with the sink column (library), drop it."""
    B, T, Hq, _ = q.shape
    Hkv = k_new.shape[2]
    G = Hq // Hkv
    f32 = lambda s: float(np.float32(s))
    deq = lambda c, s: c.view(torch.float8_e4m3fn).to(torch.float64) * f32(s)
    quant = lambda x, s: (x.float() / torch.tensor(s, dtype=torch.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    kn, vn = deq(quant(k_new, ks), ks), deq(quant(v_new, vs), vs)
    kc, vc = deq(kc_codes, ks), deq(vc_codes, vs)
    o = torch.zeros(B, T, Hq, v_new.shape[3], dtype=torch.float64)
    lse = torch.zeros(B, T, Hq, dtype=torch.float64)
    for b in range(B):
        n = int(ctx[b])
        K = torch.cat([kc[b, :n], kn[b]], 0)      # [n + T, Hkv, dq], positions -n .. T-1
        V = torch.cat([vc[b, :n], vn[b]], 0)
        pos = torch.arange(-n, T)
        for t in range(T):
            vis = (pos <= t) & ((pos > t - window) if window > 0 else True)
            for h in range(Hq):
                a = scale * (K[vis, h // G] @ q[b, t, h].double())
                logits = torch.cat([a, torch.tensor([float(sink[h])], dtype=torch.float64)])
                w = torch.softmax(logits, 0)[:-1]
                o[b, t, h] = w @ V[vis, h // G]
                lse[b, t, h] = torch.logsumexp(logits, 0)
    return o, lse


@pytest.mark.parametrize("window", [0, 7])
def test_decode_fp8_equals_eager_dequantised(window):
    g = torch.Generator().manual_seed(23)
    B, T, Hq, Hkv, max_ctx = 2, 3, 4, 2, 24
    ks, vs = 0.021, 0.017
    q = rand_bf16((B, T, Hq, 192), g)
    k_new, v_new = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    lib_codes = lambda x, s: (x.float() / s).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    kc = lib_codes(torch.randn(B, max_ctx, Hkv, 192, generator=g), ks)
    vc = lib_codes(torch.randn(B, max_ctx, Hkv, 128, generator=g), vs)
    ctx = torch.tensor([17, 0], dtype=torch.int32)
    sink = torch.tensor([0.5, -1.0, float("-inf"), 2.0])
    scale = 1.0 / math.sqrt(192)
    o, lse, _ = oracle.decode_fp8(oracle.KV_CONTIG, q, k_new, v_new, kc, vc, ks, vs, sink, scale,
                                  window, ctx_len=ctx)
    eo, el = eager_fp8_decode(q, k_new, v_new, kc, vc, ks, vs, ctx, sink, scale, window)
    assert torch.allclose(o, eo, rtol=0, atol=1e-12)
    assert torch.allclose(lse, el, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# brute force: a second, naive fp64 double loop over tiny inputs
# ----------------------------------------------------------------------------------------------

def naive_row(qv, keys, vals, sink, scale):
    """One query row by hand: plain Python floats, math.exp / math.log, nothing shared."""
    a = [scale * sum(x * y for x, y in zip(qv, kv)) for kv in keys]
    m = max([sink] + a)
    ws = math.exp(sink - m) if sink != -math.inf else 0.0
    es = [math.exp(x - m) for x in a]
    D = ws + sum(es)
    o = [sum(e * vv[c] for e, vv in zip(es, vals)) / D for c in range(len(vals[0]))]
    return o, m + math.log(D)


@pytest.mark.parametrize("L,window", [(1, 0), (2, 0), (5, 0), (8, 0), (8, 3), (7, 1), (6, 128)])
def test_brute_force_tiny_prefill(L, window):
    g = torch.Generator().manual_seed(31 + L + window)
    B, Hq, Hkv = 2, 4, 2
    q, k, v = rand_bf16((B, L, Hq, 192), g), rand_bf16((B, L, Hkv, 192), g), rand_bf16((B, L, Hkv, 128), g)
    sink = torch.tensor([1.5, float("-inf"), -2.0, 4.0])
    scale = 1.0 / math.sqrt(192)
    o, lse, _ = oracle.prefill(q, k, v, sink, scale, window)
    qd, kd, vd = q.double().tolist(), k.double().tolist(), v.double().tolist()
    for b in range(B):
        for i in range(L):
            lo = max(0, i - window + 1) if window > 0 else 0
            for h in range(Hq):
                gk = h // (Hq // Hkv)
                keys = [kd[b][j][gk] for j in range(lo, i + 1)]
                vals = [vd[b][j][gk] for j in range(lo, i + 1)]
                ro, rl = naive_row(qd[b][i][h], keys, vals, float(sink[h]), scale)
                assert max(abs(x - y) for x, y in zip(o[b, i, h].tolist(), ro)) < 1e-12
                assert abs(lse[b, i, h].item() - rl) < 1e-12


def test_brute_force_tiny_decode():
    """Decode over a 5-token contiguous cache + T = 3 new tokens, window 4, by hand."""
    g = torch.Generator().manual_seed(37)
    B, T, Hq, Hkv, n = 1, 3, 2, 1, 5
    q = rand_bf16((B, T, Hq, 192), g)
    kn, vn = rand_bf16((B, T, Hkv, 192), g), rand_bf16((B, T, Hkv, 128), g)
    kc, vc = rand_bf16((B, n + 2, Hkv, 192), g), rand_bf16((B, n + 2, Hkv, 128), g)
    sink = torch.tensor([0.7, -1.0])
    scale = 1.0 / math.sqrt(192)
    for window in (0, 4):
        o, lse, _ = oracle.decode(oracle.KV_CONTIG, q, kn, vn, kc, vc, sink, scale, window,
                                  ctx_len=torch.tensor([n], dtype=torch.int32))
        # positions: cached token c at c - n, new token u at u
        K = [(c - n, kc[0, c, 0].double().tolist(), vc[0, c, 0].double().tolist()) for c in range(n)]
        K += [(u, kn[0, u, 0].double().tolist(), vn[0, u, 0].double().tolist()) for u in range(T)]
        for t in range(T):
            vis = [(kk, vv) for p, kk, vv in K if p <= t and (window == 0 or p > t - window)]
            for h in range(Hq):
                ro, rl = naive_row(q[0, t, h].double().tolist(), [x[0] for x in vis],
                                   [x[1] for x in vis], float(sink[h]), scale)
                assert max(abs(x - y) for x, y in zip(o[0, t, h].tolist(), ro)) < 1e-12
                assert abs(lse[0, t, h].item() - rl) < 1e-12


# ----------------------------------------------------------------------------------------------
# backward (the training variant): gradients of sum(O * dO)
# ----------------------------------------------------------------------------------------------

def eager_grads(q, k, v, sink, dout, scale, window):
    """Library autograd (fp64) through the eager concat -> softmax -> drop formulation."""
    B, L, Hq, _ = q.shape
    G = Hq // k.shape[2]
    qd, kd, vd = (x.double().clone().requires_grad_(True) for x in (q, k, v))
    sd = sink.double().clone().requires_grad_(True)
    kr = kd.repeat_interleave(G, 2).permute(0, 2, 1, 3)          # [B, Hq, L, dq]
    vr = vd.repeat_interleave(G, 2).permute(0, 2, 1, 3)
    a = scale * qd.permute(0, 2, 1, 3) @ kr.transpose(-1, -2)     # [B, Hq, L, L]
    a = a.masked_fill(~band_mask(L, window), float("-inf"))
    col = sd.view(1, Hq, 1, 1).expand(B, Hq, L, 1)
    w = torch.softmax(torch.cat([a, col], -1), -1)[..., :-1]
    o = (w @ vr).permute(0, 2, 1, 3)
    (o * dout.double()).sum().backward()
    return qd.grad, kd.grad, vd.grad, sd.grad


@pytest.mark.parametrize("L,window,Hq,Hkv", [(9, 0, 4, 2), (9, 3, 4, 2), (6, 1, 2, 2), (7, 0, 8, 1)])
def test_backward_equals_library_autograd(L, window, Hq, Hkv):
    g = torch.Generator().manual_seed(41 + L + window)
    B = 2
    q, k, v = rand_bf16((B, L, Hq, 192), g), rand_bf16((B, L, Hkv, 192), g), rand_bf16((B, L, Hkv, 128), g)
    dout = rand_bf16((B, L, Hq, 128), g)
    sink = torch.rand(Hq, generator=g) * 4 - 1
    scale = 1.0 / math.sqrt(192)
    ours = oracle.prefill_backward(q, k, v, sink, dout, scale, window)
    ref = eager_grads(q, k, v, sink, dout, scale, window)
    for name, x, y in zip(("dq", "dk", "dv", "dsink"), ours, ref):
        assert torch.allclose(x, y, rtol=1e-10, atol=1e-11), name


def test_backward_sink_by_central_differences():
    """d/ds_h of sum(O * dO) against central differences of the (separately pinned) forward."""
    g = torch.Generator().manual_seed(47)
    B, L, Hq, Hkv = 1, 6, 2, 1
    q, k, v = rand_bf16((B, L, Hq, 192), g), rand_bf16((B, L, Hkv, 192), g), rand_bf16((B, L, Hkv, 128), g)
    dout = rand_bf16((B, L, Hq, 128), g)
    sink = torch.tensor([0.3, 1.7], dtype=torch.float64)
    scale = 1.0 / math.sqrt(192)
    ds = oracle.prefill_backward(q, k, v, sink.float(), dout, scale, 0)[3]

    def f(s):  # the forward oracle takes fp32 sinks: step in fp32-exact increments
        o, _, _ = oracle.prefill(q, k, v, s.float(), scale, 0)
        return (o * dout.double()).sum().item()
    h = 2.0 ** -12
    for hh in range(Hq):
        e = torch.zeros(Hq, dtype=torch.float64)
        e[hh] = h
        num = (f(sink + e) - f(sink - e)) / (2 * h)
        assert abs(num - ds[hh].item()) < 1e-5 * max(1.0, abs(num)), (hh, num, ds[hh].item())


def test_backward_without_sink_equals_library_attention_backward():
    """sink = -inf: no sink gradient, and dq / dk / dv equal the library's fp64 attention
    backward (scaled_dot_product_attention, GQA)."""
    g = torch.Generator().manual_seed(43)
    B, L, Hq, Hkv = 2, 8, 4, 2
    q, k, v = rand_bf16((B, L, Hq, 192), g), rand_bf16((B, L, Hkv, 192), g), rand_bf16((B, L, Hkv, 128), g)
    dout = rand_bf16((B, L, Hq, 128), g)
    scale = 1.0 / math.sqrt(192)
    ours = oracle.prefill_backward(q, k, v, torch.full((Hq,), float("-inf")), dout, scale, 0)
    qd, kd, vd = (to_bhld(x).clone().requires_grad_(True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=band_mask(L, 0), scale=scale,
                                       enable_gqa=True)
    (o * to_bhld(dout)).sum().backward()
    for x, y in zip(ours[:3], (qd.grad, kd.grad, vd.grad)):
        assert torch.allclose(x, y.permute(0, 2, 1, 3), rtol=1e-10, atol=1e-11)
    assert torch.all(ours[3] == 0)
