"""GPU parity of sink-attention prefill (SWA and GA) against the fp64 oracle."""
import math

import pytest
import torch

import oracle
import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu


def rand_inputs(B, L, Hq, Hkv, seed, sink_mode="rand"):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, 192, generator=g).to(torch.bfloat16)
    k = torch.randn(B, L, Hkv, 192, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, Hkv, 128, generator=g).to(torch.bfloat16)
    if sink_mode == "none":
        s = None
    elif sink_mode == "neginf":
        s = torch.full((Hq,), float("-inf"))
    else:
        s = torch.rand(Hq, generator=g) * 6.0
        s[::3] = float("-inf")
    return q, k, v, s


def run_gpu(q, k, v, s, window):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    sd = None if s is None else s.to(dev)
    if window > 0:
        o, lse = sa.sinkattn_prefill_swa(qd, kd, vd, sd, window)
    else:
        o, lse = sa.sinkattn_prefill_ga(qd, kd, vd, sd)
    torch.cuda.synchronize()
    return o, lse


def check_full(q, k, v, s, window, what):
    o, lse = run_gpu(q, k, v, s, window)
    ro, rl, _ = oracle.prefill(q, k, v, s, 1 / math.sqrt(192), window)
    assert_close(o, ro, lse.permute(0, 2, 1), rl, what)
    assert sa.sinkattn_take_device_error() == 0


def test_swa_prefill_small_workload_full():
    """B=1, L=1024, 8 Q heads / 1 KV head, W=128: every output element."""
    w = W.SWA_PREFILL_SMALL
    d = W.prefill_inputs(w)
    check_full(d["q"], d["k"], d["v"], d["sink"], w.window, w.name)


@pytest.mark.parametrize("B,L,Hq,Hkv,window", [
    (2, 1, 8, 8, 128), (1, 2, 4, 1, 128), (1, 127, 8, 1, 128), (1, 128, 8, 1, 128),
    (1, 129, 8, 8, 128), (2, 257, 16, 2, 128), (1, 300, 4, 1, 1), (1, 300, 4, 1, 7),
    (1, 500, 4, 2, 200), (1, 400, 2, 1, 1000), (1, 384, 16, 1, 129), (3, 200, 2, 2, 64),
])
def test_swa_prefill_shapes(B, L, Hq, Hkv, window):
    q, k, v, s = rand_inputs(B, L, Hq, Hkv, seed=B * 1000 + L + window)
    check_full(q, k, v, s, window, f"swa B{B} L{L} {Hq}/{Hkv} W{window}")


@pytest.mark.parametrize("B,L,Hq,Hkv", [
    (1, 1, 4, 4), (1, 128, 16, 1), (2, 255, 8, 4), (1, 513, 16, 1), (1, 700, 64, 4),
    (2, 129, 2, 1),
])
def test_ga_prefill_shapes(B, L, Hq, Hkv):
    q, k, v, s = rand_inputs(B, L, Hq, Hkv, seed=7 * L + Hq)
    check_full(q, k, v, s, 0, f"ga B{B} L{L} {Hq}/{Hkv}")


@pytest.mark.parametrize("B,L,Hq,Hkv,growth", [
    (1, 1000, 8, 1, 1 / 32), (2, 777, 4, 2, 1 / 16), (1, 1500, 16, 1, -1 / 32),
])
def test_ga_prefill_growing_scores(B, L, Hq, Hkv, growth):
    """Scores that rise (or fall) steadily with the key position: one query dim is 8 and the
    same key dim is growth x position, so a row's maximum climbs by tens of log2 units across its
    keys and the kernel's running maximum is raised (and O rescaled) many times over."""
    q, k, v, s = rand_inputs(B, L, Hq, Hkv, seed=int(L / abs(growth)))
    q[..., 0] = 8.0
    k[..., 0] = (torch.arange(L, dtype=torch.float32) * growth).view(1, L, 1).to(torch.bfloat16)
    check_full(q, k, v, s, 0, f"ga growing B{B} L{L} {Hq}/{Hkv} x{growth}")


@pytest.mark.parametrize("mode", ["none", "neginf", "rand"])
@pytest.mark.parametrize("window", [0, 128])
def test_sink_modes(mode, window):
    q, k, v, s = rand_inputs(1, 300, 8, 2, seed=99, sink_mode=mode)
    check_full(q, k, v, s, window, f"sink {mode} W{window}")


def test_large_sink_dominates_and_small_sink_vanishes():
    q, k, v, _ = rand_inputs(1, 256, 4, 1, seed=5)
    for val in (40.0, -40.0):
        s = torch.full((4,), val)
        check_full(q, k, v, s, 128, f"sink={val}")


def test_strided_inputs():
    """q is a head slice of a wider tensor; k and v are views into one fused KV tensor."""
    g = torch.Generator().manual_seed(3)
    B, L, Hq, Hkv = 2, 333, 8, 2
    big_q = torch.randn(B, L, Hq + 4, 192, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, L, Hkv, 192 + 128, generator=g).to(torch.bfloat16)
    s = torch.rand(Hq, generator=g) * 6
    qd, kvd = big_q.cuda(), kv.cuda()
    q_d = qd[:, :, 2:2 + Hq]
    k_d, v_d = kvd[..., :192], kvd[..., 192:]
    o_full = torch.zeros(B, L, Hq, 256, dtype=torch.bfloat16, device="cuda")
    o_d = o_full[..., 64:192]
    for window in (0, 128):
        fn = sa.sinkattn_prefill_swa if window else sa.sinkattn_prefill_ga
        args = (window,) if window else ()
        o, lse = fn(q_d, k_d, v_d, s.cuda(), *args, o=o_d)
        torch.cuda.synchronize()
        ro, rl, _ = oracle.prefill(big_q[:, :, 2:2 + Hq], kv[..., :192], kv[..., 192:], s,
                                   1 / math.sqrt(192), window)
        assert_close(o_d, ro, lse.permute(0, 2, 1), rl, f"strided W{window}")
        assert (o_full[..., :64] == 0).all() and (o_full[..., 192:] == 0).all()


def test_deterministic():
    q, k, v, s = rand_inputs(1, 640, 16, 2, seed=11)
    a = run_gpu(q, k, v, s, 0)
    b = run_gpu(q, k, v, s, 0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_lse_optional():
    q, k, v, s = rand_inputs(1, 200, 4, 1, seed=12)
    o, lse = sa.sinkattn_prefill_ga(q.cuda(), k.cuda(), v.cuda(), s.cuda(), want_lse=False)
    assert lse is None
    ro, _, _ = oracle.prefill(q, k, v, s, 1 / math.sqrt(192), 0)
    assert_close(o, ro, what="no lse")


def sample_rows(B, L, seed, extra=8):
    g = torch.Generator().manual_seed(seed)
    fixed = [0, 1, 126, 127, 128, 129, 255, 256, L // 2, L - 129, L - 128, L - 1]
    rows = []
    for b in range(B):
        rs = set(r for r in fixed if 0 <= r < L)
        rs.update(torch.randint(0, L, (extra,), generator=g).tolist())
        rows += [[b, r] for r in sorted(rs)]
    return rows


@pytest.mark.parametrize("w", [W.SWA_PREFILL, W.GA_PREFILL], ids=lambda w: w.name)
def test_full_size_workloads_sampled_rows(w):
    """The full-size workloads in the launch configuration the benchmark times; every head of
    a seeded sample of rows (tile edges, window edges, the last row, random rows)."""
    d = W.prefill_inputs(w, device="cuda")
    if w.window:
        o, lse = sa.sinkattn_prefill_swa(d["q"], d["k"], d["v"], d["sink"], w.window)
    else:
        o, lse = sa.sinkattn_prefill_ga(d["q"], d["k"], d["v"], d["sink"])
    torch.cuda.synchronize()
    rows = sample_rows(w.B, w.L, seed=w.seed, extra=6 if w.window == 0 else 24)
    qc, kc, vc, sc = d["q"].cpu(), d["k"].cpu(), d["v"].cpu(), d["sink"].cpu()
    ro, rl, _ = oracle.prefill(qc, kc, vc, sc, W.SCALE, w.window, rows=rows)
    idx_b = torch.tensor([r[0] for r in rows])
    idx_i = torch.tensor([r[1] for r in rows])
    og = o.cpu()[idx_b, idx_i]
    lg = lse.cpu().permute(0, 2, 1)[idx_b, idx_i]
    assert_close(og, ro, lg, rl, w.name)
    assert sa.sinkattn_take_device_error() == 0


@pytest.mark.parametrize("B,P,L,Hq,Hkv,window", [
    (1, 0, 200, 16, 1, 0), (2, 1, 129, 16, 1, 0), (1, 127, 1, 8, 1, 0), (1, 128, 128, 16, 4, 0),
    (1, 300, 257, 16, 1, 0), (2, 1000, 300, 8, 2, 0), (1, 200, 300, 8, 1, 128),
    (1, 50, 77, 4, 1, 7), (1, 129, 64, 8, 8, 200),
])
@pytest.mark.parametrize("sink_mode", ["rand", "none"])
def test_chunked_prefill(B, P, L, Hq, Hkv, window, sink_mode):
    """A chunk of L tokens after a P-token prefix equals rows P .. P+L-1 of the whole-sequence
    prefill of the concatenated sequence (the oracle, restricted to those rows)."""
    q, k, v, s = rand_inputs(B, P + L, Hq, Hkv, 31 * P + L + window, sink_mode)
    dev = "cuda"
    o, lse = sa.sinkattn_prefill_chunk(q[:, P:].to(dev), k.to(dev), v.to(dev),
                                       None if s is None else s.to(dev), prefix=P, window=window)
    torch.cuda.synchronize()
    rows = [[b, P + i] for b in range(B) for i in range(L)]
    ro, rl, _ = oracle.prefill(q, k, v, s, 1 / math.sqrt(192), window, rows=rows)
    assert_close(o.reshape(B * L, Hq, 128), ro, lse.permute(0, 2, 1).reshape(B * L, Hq), rl,
                 f"chunk P{P} L{L} W{window}")
    assert sa.sinkattn_take_device_error() == 0


def test_chunked_prefill_full_size_sampled():
    """The chunk workload of the benchmark (GA, B=1, a 16384-token chunk after a 16384-token
    prefix, 64 Q / 4 KV), on sampled rows."""
    w = W.GA_CHUNK
    d = W.prefill_inputs(w, device="cuda", L=w.prefix + w.L)
    o, lse = sa.sinkattn_prefill_chunk(d["q"][:, w.prefix:], d["k"], d["v"], d["sink"],
                                       prefix=w.prefix)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(5)
    sample = sorted(set([0, 1, 127, 128, 129, w.L - 1] + torch.randint(0, w.L, (26,), generator=g).tolist()))
    rows = [[0, w.prefix + i] for i in sample]
    ro, rl, _ = oracle.prefill(d["q"].cpu(), d["k"].cpu(), d["v"].cpu(), d["sink"].cpu(),
                               1 / math.sqrt(192), 0, rows=rows)
    idx = torch.tensor(sample)
    assert_close(o[0, idx].cpu(), ro, lse[0][:, idx].permute(1, 0).cpu(), rl, w.name)
    assert sa.sinkattn_take_device_error() == 0


def paged_prefix(k, v, P, page, seed):
    """The first P positions of k / v in a page pool: each sequence's pages handed out in a
    seeded random order, plus two spare pages no sequence owns. Returns (k_pages, v_pages,
    page_table [B, max_pages])."""
    B, _, Hkv, _ = k.shape
    max_pages = max(1, (P + page - 1) // page)
    g = torch.Generator().manual_seed(seed)
    n = B * max_pages + 2
    perm = torch.randperm(n, generator=g).to(torch.int32)
    table = perm[:B * max_pages].reshape(B, max_pages).contiguous()
    kp = torch.randn(n, page, Hkv, 192, generator=g).to(torch.bfloat16)
    vp = torch.randn(n, page, Hkv, 128, generator=g).to(torch.bfloat16)
    for b in range(B):
        for c in range(P):
            kp[table[b, c // page], c % page] = k[b, c]
            vp[table[b, c // page], c % page] = v[b, c]
    return kp, vp, table


@pytest.mark.parametrize("B,P,L,Hq,Hkv,window,page", [
    (1, 128, 77, 8, 1, 0, 128),     # one prefix page, a ragged chunk
    (2, 256, 300, 16, 1, 0, 256),   # GA group of 16, 256-token pages
    (1, 384, 129, 8, 1, 128, 128),  # the SWA window reaching back into the pages
    (2, 1024, 200, 8, 2, 200, 128), # a window wider than a tile, two KV heads
    (1, 0, 64, 4, 1, 0, 128),       # no prefix at all
])
def test_chunked_prefill_paged_prefix(B, P, L, Hq, Hkv, window, page):
    """The same chunked prefill with the prefix in a paged pool (the serving stack's paged KV
    cache) instead of one contiguous tensor: rows P .. P+L-1 of the whole-sequence prefill."""
    q, k, v, s = rand_inputs(B, P + L, Hq, Hkv, 7 * P + L + window, "mixed")
    kp, vp, table = paged_prefix(k, v, P, page, seed=P + L)
    dev = "cuda"
    o, lse = sa.sinkattn_prefill_chunk_paged(q[:, P:].to(dev), k[:, P:].to(dev), v[:, P:].to(dev),
                                             kp.to(dev), vp.to(dev), table.to(dev), s.to(dev),
                                             prefix=P, window=window)
    torch.cuda.synchronize()
    rows = [[b, P + i] for b in range(B) for i in range(L)]
    ro, rl, _ = oracle.prefill(q, k, v, s, 1 / math.sqrt(192), window, rows=rows)
    assert_close(o.reshape(B * L, Hq, 128), ro, lse.permute(0, 2, 1).reshape(B * L, Hq), rl,
                 f"paged chunk P{P} L{L} W{window} page{page}")
    assert sa.sinkattn_take_device_error() == 0
