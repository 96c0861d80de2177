"""The oracle: a plain fp64 CPU restatement of sink-softmax attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never reaches it, and it imports nothing
from the CUDA library: the two share no code. The arithmetic lives in ``sinkattn_oracle.c``
(plain C, fp64); this module only compiles it with gcc and marshals arrays.

Every function takes bf16 tensors (CPU, any layout; they are made contiguous here) and returns
float64 tensors.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sinkattn_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libsinkattn_oracle.so")
_lock = threading.Lock()
_lib = None

# KV-cache kinds (same numbering as the library header; restated, not shared).
KV_RING, KV_CONTIG, KV_PAGED = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, IEEE semantics, no fast-math, no FMA contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
             "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SINKATTN_ORACLE_LIB points the oracle at another build of the same source; the
            # mutation test uses it to load deliberately broken copies of the oracle.
            path = os.environ.get("SINKATTN_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.sinkattn_oracle_prefill.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                                    f64, P, i64, P, P, P]
            lib.sinkattn_oracle_prefill.restype = i32
            lib.sinkattn_oracle_decode.argtypes = [i32, P, P, P, P, P, P, P, i32, P, i32, P, i32,
                                                   i32, P, i32, i32, i32, i32, i32, i32, i32, f64,
                                                   P, i32, P, P, P]
            lib.sinkattn_oracle_decode.restype = i32
            lib.sinkattn_oracle_partial.argtypes = [P, P, P, i32, i32, i32, i32, f64, P, P, P]
            lib.sinkattn_oracle_partial.restype = None
            lib.sinkattn_oracle_merge.argtypes = [P, P, P, i32, i32, f64, P, P]
            lib.sinkattn_oracle_merge.restype = None
            lib.sinkattn_oracle_commit.argtypes = [i32, P, P, P, P, P, P, P, i32, P, i32, P, i32,
                                                   i32, i32, i32, i32, i32, i32]
            lib.sinkattn_oracle_commit.restype = i32
            lib.sinkattn_oracle_rope.argtypes = [P, P, i64, i32, i32, i32, f64, P]
            lib.sinkattn_oracle_rope.restype = i32
            lib.sinkattn_oracle_vscale.argtypes = [P, i64, f64, P]
            lib.sinkattn_oracle_vscale.restype = None
            lib.sinkattn_oracle_fp8_encode.argtypes = [P, i64, ctypes.c_float, P]
            lib.sinkattn_oracle_fp8_encode.restype = None
            lib.sinkattn_oracle_fp8_decode.argtypes = [P, i64, P]
            lib.sinkattn_oracle_fp8_decode.restype = None
            lib.sinkattn_oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.sinkattn_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.sinkattn_oracle_prefill_backward.argtypes = [P, P, P, P, P, i32, i32, i32, i32,
                                                             i32, i32, i32, f64, P, P, P, P]
            lib.sinkattn_oracle_prefill_backward.restype = i32
            _lib = lib
    return _lib


def _bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> contiguous uint16 numpy array of its bit patterns."""
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()).view(np.uint16)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _i32(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.int32))


def _f32(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.float32))


def prefill(q, k, v, sink, scale, window=0, rows=None, want_wsink=False):
    """Sink attention over a whole sequence (prefill).

    q [B,L,Hq,dq], k [B,L,Hkv,dq], v [B,L,Hkv,dv] bf16; sink [Hq] fp32 or None (no sink);
    window > 0 selects the sliding window (keys i-window < j <= i), 0 the full causal mask.
    rows: optional [n, 2] int array of (b, i) pairs; then outputs are [n, Hq, ...].
    Returns (o [B,L,Hq,dv] or [n,Hq,dv], lse [B,L,Hq] or [n,Hq], wsink or None), float64.
    """
    lib = _load()
    B, L, Hq, dq = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    s = _f32(sink)
    r = _i32(rows)
    n = B * L if r is None else r.shape[0]
    o = np.zeros((n, Hq, dv), np.float64)
    lse = np.zeros((n, Hq), np.float64)
    ws = np.zeros((n, Hq), np.float64) if want_wsink else None
    rc = lib.sinkattn_oracle_prefill(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(s), B, L, Hq, Hkv, dq, dv,
                                     int(window), float(scale), _ptr(r), 0 if r is None else n,
                                     _ptr(o), _ptr(lse), _ptr(ws))
    if rc != 0:
        raise ValueError("oracle prefill: bad arguments")
    if r is None:
        o, lse = o.reshape(B, L, Hq, dv), lse.reshape(B, L, Hq)
        ws = None if ws is None else ws.reshape(B, L, Hq)
    return (torch.from_numpy(o), torch.from_numpy(lse),
            None if ws is None else torch.from_numpy(ws))


def decode(kind, q, k_new, v_new, k_cache, v_cache, sink, scale, window=0, *, ring_head=None,
           ring_len=None, ctx_len=None, page_table=None, page_size=0, seqs=None,
           want_wsink=False):
    """Sink attention for T new tokens per sequence against a KV cache (decode / verify).

    kind: KV_RING (k_cache [B,cap,Hkv,dq] + ring_head/ring_len), KV_CONTIG (k_cache
    [B,max_ctx,Hkv,dq] + ctx_len) or KV_PAGED (k_cache [pages,page_size,Hkv,dq] + page_table
    [B,max_pages] + ctx_len). seqs: optional list of sequence indices to evaluate.
    Returns (o [n,T,Hq,dv], lse [n,T,Hq], wsink or None), float64.
    """
    lib = _load()
    B, T, Hq, dq = q.shape
    Hkv, dv = k_new.shape[2], v_new.shape[3]
    qb, knb, vnb = _bits(q), _bits(k_new), _bits(v_new)
    kcb, vcb = _bits(k_cache), _bits(v_cache)
    s = _f32(sink)
    rh, rl, cl, pt = _i32(ring_head), _i32(ring_len), _i32(ctx_len), _i32(page_table)
    sq = _i32(seqs)
    ring_cap = k_cache.shape[1] if kind == KV_RING else 0
    max_ctx = k_cache.shape[1] if kind == KV_CONTIG else 0
    max_pages = pt.shape[1] if pt is not None else 0
    n = B if sq is None else sq.shape[0]
    o = np.zeros((n, T, Hq, dv), np.float64)
    lse = np.zeros((n, T, Hq), np.float64)
    ws = np.zeros((n, T, Hq), np.float64) if want_wsink else None
    rc = lib.sinkattn_oracle_decode(int(kind), _ptr(qb), _ptr(knb), _ptr(vnb), _ptr(kcb), _ptr(vcb),
                                    _ptr(rh), _ptr(rl), ring_cap, _ptr(cl), max_ctx, _ptr(pt),
                                    int(page_size), max_pages, _ptr(s), B, T, Hq, Hkv, dq, dv,
                                    int(window), float(scale), _ptr(sq), n, _ptr(o), _ptr(lse),
                                    _ptr(ws))
    if rc != 0:
        raise ValueError("oracle decode: bad arguments")
    return (torch.from_numpy(o), torch.from_numpy(lse),
            None if ws is None else torch.from_numpy(ws))


def partial(q_row, k_rows, v_rows, j0, j1, scale):
    """(O_P, m_P, l_P) of one query row over keys [j0, j1) without the sink.

    q_row [dq], k_rows [n,dq], v_rows [n,dv] bf16."""
    lib = _load()
    qb, kb, vb = _bits(q_row), _bits(k_rows), _bits(v_rows)
    dq, dv = q_row.shape[0], v_rows.shape[1]
    o = np.zeros(dv, np.float64)
    m = np.zeros(1, np.float64)
    l = np.zeros(1, np.float64)
    lib.sinkattn_oracle_partial(_ptr(qb), _ptr(kb), _ptr(vb), int(j0), int(j1), dq, dv,
                                float(scale), _ptr(o), _ptr(m), _ptr(l))
    return torch.from_numpy(o), float(m[0]), float(l[0])


def merge(o_parts, m_parts, l_parts, sink):
    """Merge span partials, counting the sink once. Returns (o [dv], lse)."""
    lib = _load()
    op = np.ascontiguousarray(np.asarray(o_parts, np.float64))
    mp = np.ascontiguousarray(np.asarray(m_parts, np.float64))
    lp = np.ascontiguousarray(np.asarray(l_parts, np.float64))
    nparts, dv = op.shape
    o = np.zeros(dv, np.float64)
    lse = np.zeros(1, np.float64)
    lib.sinkattn_oracle_merge(_ptr(op), _ptr(mp), _ptr(lp), nparts, dv, float(sink), _ptr(o),
                              _ptr(lse))
    return torch.from_numpy(o), float(lse[0])


def commit(kind, k_new, v_new, n_accept, k_cache, v_cache, *, ring_head=None, ring_len=None,
           ctx_len=None, page_table=None, page_size=0):
    """Append the first n_accept[b] new tokens of each sequence to the cache.

    Returns new (k_cache, v_cache, ring_head, ring_len, ctx_len); inputs are not modified."""
    lib = _load()
    B, T, Hkv, dq = k_new.shape
    dv = v_new.shape[3]
    knb, vnb = _bits(k_new), _bits(v_new)
    kcb, vcb = _bits(k_cache).copy(), _bits(v_cache).copy()
    na = _i32(n_accept)
    rh = None if ring_head is None else _i32(ring_head).copy()
    rl = None if ring_len is None else _i32(ring_len).copy()
    cl = None if ctx_len is None else _i32(ctx_len).copy()
    pt = _i32(page_table)
    ring_cap = k_cache.shape[1] if kind == KV_RING else 0
    max_ctx = k_cache.shape[1] if kind == KV_CONTIG else 0
    max_pages = pt.shape[1] if pt is not None else 0
    rc = lib.sinkattn_oracle_commit(int(kind), _ptr(knb), _ptr(vnb), _ptr(na), _ptr(kcb), _ptr(vcb),
                                    _ptr(rh), _ptr(rl), ring_cap, _ptr(cl), max_ctx, _ptr(pt),
                                    int(page_size), max_pages, B, T, Hkv, dq, dv)
    if rc != 0:
        raise ValueError("oracle commit: bad arguments")

    def back(a, like):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).reshape(like.shape)

    to_t = (lambda a: None if a is None else torch.from_numpy(a))
    return back(kcb, k_cache), back(vcb, v_cache), to_t(rh), to_t(rl), to_t(cl)


def rope(x, pos, theta, rope_dim=64):
    """Partial rotary embedding of the first rope_dim dims of every head.

    x [..., H, d] bf16 (any leading dims); pos: positions with x's leading shape (one per row
    of H heads). Returns float64 [..., H, d]."""
    lib = _load()
    *lead, H, d = x.shape
    n = int(np.prod(lead)) if lead else 1
    xb = _bits(x)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos.cpu() if isinstance(pos, torch.Tensor)
                                                        else pos, dtype=np.int64), lead)).reshape(-1)
    out = np.zeros((n, H, d), np.float64)
    rc = lib.sinkattn_oracle_rope(_ptr(xb), _ptr(p), n, H, d, int(rope_dim), float(theta),
                                  _ptr(out))
    if rc != 0:
        raise ValueError("oracle rope: bad arguments")
    return torch.from_numpy(out.reshape(x.shape))


def vscale(v, v_scale):
    """Every element of v (bf16) times v_scale, float64."""
    lib = _load()
    vb = _bits(v)
    out = np.zeros(vb.size, np.float64)
    lib.sinkattn_oracle_vscale(_ptr(vb), vb.size, float(v_scale), _ptr(out))
    return torch.from_numpy(out.reshape(v.shape))


def fp8_encode(x, scale):
    """FP8 (E4M3) cache codes of a bf16 tensor: encode(x / scale), the division in fp32.
    Returns a torch.uint8 tensor of x's shape."""
    lib = _load()
    xb = _bits(x)
    codes = np.zeros(xb.size, np.uint8)
    lib.sinkattn_oracle_fp8_encode(_ptr(xb), xb.size, float(np.float32(scale)), _ptr(codes))
    return torch.from_numpy(codes.reshape(x.shape))


def e4m3_encode_f32(y):
    """E4M3 code of each fp32 value in y (numpy or torch), as a uint8 numpy array."""
    lib = _load()
    ya = np.asarray(y.cpu() if isinstance(y, torch.Tensor) else y, dtype=np.float32).reshape(-1)
    return np.array([lib.sinkattn_oracle_e4m3_encode(float(v)) for v in ya], np.uint8)


def fp8_decode(codes):
    """E4M3 values (without the scale) of a uint8 code tensor, float64."""
    lib = _load()
    c = np.ascontiguousarray(np.asarray(codes.cpu() if isinstance(codes, torch.Tensor) else codes,
                                        dtype=np.uint8))
    out = np.zeros(c.size, np.float64)
    lib.sinkattn_oracle_fp8_decode(_ptr(c), c.size, _ptr(out))
    return torch.from_numpy(out.reshape(c.shape))


def decode_fp8(kind, q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, sink, scale, window=0,
               **kw):
    """Decode against an FP8 (E4M3) cache: cached token values are e(code) * scale.

    The T new tokens are quantised as the cache will store them (fp8_encode), so every key is
    e(c_k) * k_scale and every value e(c_v) * v_scale. By linearity
        a_j = scale * <q, k_scale e(c_j)> = (scale * k_scale) * <q, e(c_j)>,
        O   = sum_j w_j v_scale e(c_vj) = v_scale * sum_j w_j e(c_vj),
    and e(c) is exact in bf16 (4 significant bits, exponents -9..8), so this is the bf16 decode
    above on the E4M3 values with the scale scale * k_scale, and O times v_scale. LSE is the
    one of those logits. Returns (o, lse, wsink) as decode()."""
    lut = fp8_decode(torch.arange(256, dtype=torch.uint8)).to(torch.bfloat16)

    def values_bf16(codes):  # e(c), exact in bf16; one leading index at a time bounds memory
        return torch.stack([lut[c.long()] for c in codes.cpu()]) if codes.shape[0] else \
            torch.empty(codes.shape, dtype=torch.bfloat16)

    kn = values_bf16(fp8_encode(k_new, k_scale))
    vn = values_bf16(fp8_encode(v_new, v_scale))
    kc, vc = values_bf16(k_codes), values_bf16(v_codes)
    f32 = lambda s: float(np.float32(s))
    o, lse, ws = decode(kind, q, kn, vn, kc, vc, sink, scale * f32(k_scale), window, **kw)
    return o * f32(v_scale), lse, ws


def prefill_backward(q, k, v, sink, dout, scale, window=0):
    """Gradients of sum(O * dout) of the prefill (serial; small cases).

    q [B,L,Hq,dq], k [B,L,Hkv,dq], v [B,L,Hkv,dv], dout [B,L,Hq,dv] bf16; sink [Hq] or None.
    Returns (dq, dk, dv, dsink [Hq]) float64."""
    lib = _load()
    B, L, Hq, dq = q.shape
    Hkv, dv = k.shape[2], v.shape[3]
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    s = _f32(sink)
    gq = np.zeros((B, L, Hq, dq), np.float64)
    gk = np.zeros((B, L, Hkv, dq), np.float64)
    gv = np.zeros((B, L, Hkv, dv), np.float64)
    gs = np.zeros(Hq, np.float64)
    rc = lib.sinkattn_oracle_prefill_backward(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(s), _ptr(db), B,
                                              L, Hq, Hkv, dq, dv, int(window), float(scale),
                                              _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gs))
    if rc != 0:
        raise ValueError("oracle prefill_backward: bad arguments")
    return tuple(torch.from_numpy(x) for x in (gq, gk, gv, gs))
