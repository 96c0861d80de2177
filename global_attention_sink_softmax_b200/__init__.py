"""Sink-softmax GQA attention for NVIDIA B200: a thin ctypes binding over ``libsinkattn.so``.

The functions carry the names of the C entry points declared in ``include/sinkattn.h`` and only
marshal arguments: torch tensors supply device memory and the current CUDA stream, and every
step of the computation runs in the library's CUDA kernels. There is no fallback: if the
library is missing or cannot be loaded, every call raises.

    o, lse = sinkattn_prefill_swa(q, k, v, sink, window=128)
    o, lse = sinkattn_prefill_ga(q, k, v, sink)
    o, lse = sinkattn_prefill_chunk(q_chunk, k_all, v_all, sink, prefix=P)
    o, lse = sinkattn_decode(KV_CONTIG, q, k_new, v_new, k_cache, v_cache, sink, ctx_len=...)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from . import workloads  # noqa: F401  (seeded inputs; no attention arithmetic)

__all__ = [
    "KV_RING", "KV_CONTIG", "KV_PAGED", "SinkAttnError", "lib", "library_path",
    "sinkattn_prefill_swa", "sinkattn_prefill_ga", "sinkattn_prefill_chunk", "sinkattn_decode",
    "sinkattn_decode_workspace_size", "sinkattn_kv_commit", "sinkattn_take_device_error",
    "sinkattn_status_string", "sinkattn_version", "EXPORTED_SYMBOLS",
    "sinkattn_decode_noalloc", "NOALLOC_WORKSPACE_BYTES", "sinkattn_rope_qkv",
    "ROPE_THETA_GA", "ROPE_THETA_SWA", "V_SCALE", "KV_BF16", "KV_FP8_E4M3",
    "sinkattn_set_wait_limit_ns", "sinkattn_prefill_backward", "sinkattn_prefill_chunk_paged",
    "sinkattn_prefill_host", "sinkattn_prefill_host_workspace_size", "HOST_CHUNK",
    "sinkattn_prefill_swa_rope",
]

KV_RING, KV_CONTIG, KV_PAGED = 0, 1, 2
KV_BF16, KV_FP8_E4M3 = 0, 1  # cache element types; an FP8 cache is a uint8 / float8_e4m3fn tensor
DQ, DV = 192, 128
# The model's rotary thetas (GA / SWA layers), rotated width and value scale.
ROPE_THETA_GA, ROPE_THETA_SWA, ROPE_DIM, V_SCALE = 5_000_000.0, 10_000.0, 64, 0.707
_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libsinkattn.so")
EXPORTED_SYMBOLS = [
    "sinkattn_prefill_swa", "sinkattn_prefill_ga", "sinkattn_prefill_chunk",
    "sinkattn_decode_workspace_size", "sinkattn_decode", "sinkattn_kv_commit", "sinkattn_status_string", "sinkattn_version",
    "sinkattn_take_device_error", "sinkattn_decode_noalloc", "sinkattn_rope_qkv",
    "sinkattn_set_wait_limit_ns", "sinkattn_prefill_backward_workspace_size",
    "sinkattn_prefill_backward", "sinkattn_prefill_chunk_paged",
    "sinkattn_prefill_host_workspace_size", "sinkattn_prefill_host", "sinkattn_prefill_swa_rope",
]
# Positions per chunk of the host-resident prefill (its copies in and out overlap chunk by chunk).
HOST_CHUNK = 1024
# Size of the library's own split-KV workspace used by sinkattn_decode_noalloc.
NOALLOC_WORKSPACE_BYTES = 16 << 20


class SinkAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {sinkattn_status_string(status)} (status {status})")


_P, _I32, _I64, _F32, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)


class PrefillArgs(ctypes.Structure):
    _fields_ = [("q", _P), ("k", _P), ("v", _P), ("sink", _P), ("o", _P), ("lse", _P),
                ("B", _I32), ("L", _I32), ("Hq", _I32), ("Hkv", _I32), ("dq", _I32),
                ("dv", _I32), ("scale", _F32),
                ("q_sb", _I64), ("q_sl", _I64), ("q_sh", _I64),
                ("k_sb", _I64), ("k_sl", _I64), ("k_sh", _I64),
                ("v_sb", _I64), ("v_sl", _I64), ("v_sh", _I64),
                ("o_sb", _I64), ("o_sl", _I64), ("o_sh", _I64)]


class RopeSpec(ctypes.Structure):
    _fields_ = [("pos_base", _P), ("pos0", _I64), ("rope_dim", _I32), ("theta", ctypes.c_double),
                ("v_scale", _F32)]


class RopeArgs(ctypes.Structure):
    _fields_ = [("q", _P), ("k", _P), ("v", _P), ("pos_base", _P), ("pos0", _I64),
                ("B", _I32), ("L", _I32), ("Hq", _I32), ("Hkv", _I32), ("dq", _I32),
                ("dv", _I32), ("rope_dim", _I32), ("theta", ctypes.c_double),
                ("v_scale", _F32),
                ("q_sb", _I64), ("q_sl", _I64), ("q_sh", _I64),
                ("k_sb", _I64), ("k_sl", _I64), ("k_sh", _I64),
                ("v_sb", _I64), ("v_sl", _I64), ("v_sh", _I64)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("q", _P), ("k", _P), ("v", _P), ("o", _P), ("dout", _P), ("lse", _P),
                ("sink", _P), ("dq", _P), ("dk", _P), ("dv", _P), ("dsink", _P),
                ("B", _I32), ("L", _I32), ("Hq", _I32), ("Hkv", _I32), ("d_qk", _I32),
                ("d_v", _I32), ("scale", _F32)] + [
                (f"{t}_{s}", _I64) for t in ("q", "k", "v", "o", "do", "dq", "dk", "dv")
                for s in ("sb", "sl", "sh")]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("kind", _I32), ("B", _I32), ("T", _I32), ("Hq", _I32), ("Hkv", _I32),
                ("dq", _I32), ("dv", _I32), ("window", _I32), ("scale", _F32), ("sink", _P),
                ("q", _P), ("q_sb", _I64), ("q_st", _I64), ("q_sh", _I64),
                ("k_new", _P), ("kn_sb", _I64), ("kn_st", _I64), ("kn_sh", _I64),
                ("v_new", _P), ("vn_sb", _I64), ("vn_st", _I64), ("vn_sh", _I64),
                ("k_cache", _P), ("kc_sb", _I64), ("kc_ss", _I64), ("kc_sh", _I64),
                ("v_cache", _P), ("vc_sb", _I64), ("vc_ss", _I64), ("vc_sh", _I64),
                ("ring_head", _P), ("ring_len", _P), ("ring_cap", _I32),
                ("ctx_len", _P), ("max_ctx", _I32),
                ("page_table", _P), ("page_size", _I32), ("max_pages", _I32),
                ("num_pages", _I32),
                ("o", _P), ("o_sb", _I64), ("o_st", _I64), ("o_sh", _I64), ("lse", _P),
                ("kv_dtype", _I32), ("k_scale", _F32), ("v_scale", _F32),
                ("commit_rope", _I32), ("rope_dim", _I32), ("rope_theta", ctypes.c_double),
                ("commit_v_scale", _F32), ("commit_pos", _P)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library. Raises if it has not been built or cannot be loaded."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise RuntimeError(
                    f"{library_path} is missing: build it with "
                    "`python -m global_attention_sink_softmax_b200.build` (needs nvcc)")
            L = ctypes.CDLL(library_path)
            L.sinkattn_prefill_swa.argtypes = [ctypes.POINTER(PrefillArgs), _I32, _P]
            L.sinkattn_prefill_swa.restype = ctypes.c_int
            L.sinkattn_prefill_ga.argtypes = [ctypes.POINTER(PrefillArgs), _P]
            L.sinkattn_prefill_chunk.restype = ctypes.c_int
            L.sinkattn_prefill_chunk.argtypes = [ctypes.POINTER(PrefillArgs), _I32, _I32, _P]
            L.sinkattn_prefill_chunk_paged.restype = ctypes.c_int
            L.sinkattn_prefill_chunk_paged.argtypes = [ctypes.POINTER(PrefillArgs),
                                                       ctypes.POINTER(PagedKV), _I32, _I32, _P]
            L.sinkattn_prefill_ga.restype = ctypes.c_int
            L.sinkattn_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
            L.sinkattn_decode_workspace_size.restype = _SZ
            L.sinkattn_decode.argtypes = [ctypes.POINTER(DecodeArgs), _P, _SZ, _P]
            L.sinkattn_decode.restype = ctypes.c_int
            L.sinkattn_decode_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), _P]
            L.sinkattn_decode_noalloc.restype = ctypes.c_int
            L.sinkattn_kv_commit.argtypes = [ctypes.POINTER(DecodeArgs), _P, _P]
            L.sinkattn_kv_commit.restype = ctypes.c_int
            L.sinkattn_status_string.argtypes = [ctypes.c_int]
            L.sinkattn_status_string.restype = ctypes.c_char_p
            L.sinkattn_version.argtypes = []
            L.sinkattn_version.restype = ctypes.c_int
            L.sinkattn_take_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
            L.sinkattn_take_device_error.restype = ctypes.c_int
            L.sinkattn_rope_qkv.argtypes = [ctypes.POINTER(RopeArgs), _P]
            L.sinkattn_rope_qkv.restype = ctypes.c_int
            L.sinkattn_prefill_backward_workspace_size.argtypes = [ctypes.POINTER(BackwardArgs)]
            L.sinkattn_prefill_backward_workspace_size.restype = _SZ
            L.sinkattn_prefill_backward.argtypes = [ctypes.POINTER(BackwardArgs), _I32, _P, _SZ, _P]
            L.sinkattn_prefill_backward.restype = ctypes.c_int
            L.sinkattn_prefill_host_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs), _I32]
            L.sinkattn_prefill_host_workspace_size.restype = _SZ
            L.sinkattn_prefill_host.argtypes = [ctypes.POINTER(PrefillArgs), _I32, _I32, _P, _SZ, _P]
            L.sinkattn_prefill_host.restype = ctypes.c_int
            L.sinkattn_prefill_swa_rope.argtypes = [ctypes.POINTER(PrefillArgs), _I32,
                                                    ctypes.POINTER(RopeSpec), _P]
            L.sinkattn_prefill_swa_rope.restype = ctypes.c_int
            L.sinkattn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.sinkattn_set_wait_limit_ns.restype = ctypes.c_int
            _lib = L
    return _lib


def sinkattn_status_string(status: int) -> str:
    return lib().sinkattn_status_string(int(status)).decode()


def sinkattn_version() -> int:
    return int(lib().sinkattn_version())


# ----------------------------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------------------------

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream))


def _check_bf16(name, t, ndim=4):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim or t.stride(-1) != 1:
        raise ValueError(f"{name} must be {ndim}-D with a contiguous last dim")


def _check_vec(name, t, dtype):
    if t is None:
        return
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


def _raise(status, where):
    if status != 0:
        raise SinkAttnError(status, where)


# ----------------------------------------------------------------------------------------------
# prefill
# ----------------------------------------------------------------------------------------------

def _prefill_args(q, k, v, sink, o, lse, scale):
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check_bf16(n, t)
    _check_vec("sink", sink, torch.float32)
    _check_vec("lse", lse, torch.float32)
    B, L, Hq, dq = q.shape
    a = PrefillArgs()
    a.q, a.k, a.v, a.sink, a.o, a.lse = (_ptr(q), _ptr(k), _ptr(v), _ptr(sink), _ptr(o),
                                         _ptr(lse))
    a.B, a.L, a.Hq, a.Hkv, a.dq, a.dv = B, L, Hq, k.shape[2], dq, v.shape[3]
    a.scale = scale
    a.q_sb, a.q_sl, a.q_sh = q.stride(0), q.stride(1), q.stride(2)
    a.k_sb, a.k_sl, a.k_sh = k.stride(0), k.stride(1), k.stride(2)
    a.v_sb, a.v_sl, a.v_sh = v.stride(0), v.stride(1), v.stride(2)
    a.o_sb, a.o_sl, a.o_sh = o.stride(0), o.stride(1), o.stride(2)
    return a


class PagedKV(ctypes.Structure):
    _fields_ = [("k_pages", _P), ("v_pages", _P),
                ("kp_sb", _I64), ("kp_ss", _I64), ("kp_sh", _I64),
                ("vp_sb", _I64), ("vp_ss", _I64), ("vp_sh", _I64),
                ("page_table", _P), ("page_size", _I32), ("max_pages", _I32), ("num_pages", _I32)]


def _prefill(fn, q, k, v, sink, window, o, lse, scale, stream, want_lse, prefix=0, paged=None):
    B, L, Hq, dq = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    if o is None:
        o = torch.empty(B, L, Hq, v.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device)
    a = _prefill_args(q, k, v, sink, o, lse, scale)
    L_ = lib()
    if fn == "swa":
        st = L_.sinkattn_prefill_swa(ctypes.byref(a), int(window), _stream(stream))
    elif fn == "chunk":
        st = L_.sinkattn_prefill_chunk(ctypes.byref(a), int(prefix), int(window), _stream(stream))
    elif fn == "chunk_paged":
        st = L_.sinkattn_prefill_chunk_paged(ctypes.byref(a), ctypes.byref(paged), int(prefix),
                                             int(window), _stream(stream))
    else:
        st = L_.sinkattn_prefill_ga(ctypes.byref(a), _stream(stream))
    _raise(st, f"sinkattn_prefill_{fn}")
    return o, lse


def sinkattn_prefill_swa(q, k, v, sink=None, window=128, *, o=None, lse=None, scale=None,
                         stream=None, want_lse=True):
    """Sliding-window sink attention over whole sequences.

    q [B,L,Hq,192], k [B,L,Hkv,192], v [B,L,Hkv,128] bf16 CUDA tensors (token-major, any
    strides with a contiguous last dim); sink fp32 [Hq] or None. Returns (o [B,L,Hq,128] bf16,
    lse [B,Hq,L] fp32 or None)."""
    return _prefill("swa", q, k, v, sink, window, o, lse, scale, stream, want_lse)


def sinkattn_prefill_swa_rope(q, k, v, sink=None, window=128, *, theta=ROPE_THETA_SWA,
                              rope_dim=ROPE_DIM, v_scale=V_SCALE, pos0=0, pos_base=None, o=None,
                              lse=None, scale=None, stream=None, want_lse=True):
    """Sliding-window prefill with the partial RoPE and the value scale applied as Q, K and V
    are loaded: the result of sinkattn_rope_qkv(q, k, v, ...) then sinkattn_prefill_swa, without
    modifying q, k, v. Token l of sequence b sits at position pos0 + pos_base[b] (CUDA int32
    [B] or None) + l. Takes the GQA-packed path (8 query heads per KV head, window <= 128);
    other shapes raise SinkAttnError (UNSUPPORTED)."""
    B, L, Hq, dq = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    if o is None:
        o = torch.empty(B, L, Hq, v.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device)
    a = _prefill_args(q, k, v, sink, o, lse, scale)
    _check_vec("pos_base", pos_base, torch.int32)
    spec = RopeSpec()
    spec.pos_base, spec.pos0, spec.rope_dim = _ptr(pos_base), int(pos0), int(rope_dim)
    spec.theta, spec.v_scale = float(theta), float(v_scale)
    st = lib().sinkattn_prefill_swa_rope(ctypes.byref(a), int(window), ctypes.byref(spec),
                                         _stream(stream))
    _raise(st, "sinkattn_prefill_swa_rope")
    return o, lse


def sinkattn_prefill_ga(q, k, v, sink=None, *, o=None, lse=None, scale=None, stream=None,
                        want_lse=True):
    """Global (full causal) sink attention over whole sequences; arguments as for SWA."""
    return _prefill("ga", q, k, v, sink, 0, o, lse, scale, stream, want_lse)


def sinkattn_prefill_chunk(q, k, v, sink=None, *, prefix, window=0, o=None, lse=None, scale=None,
                           stream=None, want_lse=True):
    """Chunked prefill against cached keys: q [B,L,Hq,192] are the tokens at positions
    prefix .. prefix+L-1; k [B,prefix+L,Hkv,192], v [B,prefix+L,Hkv,128] hold every position
    (the cached prefix, then the chunk). window = 0 full causal, >= 1 sliding window. Returns
    (o [B,L,Hq,128] bf16, lse [B,Hq,L] fp32 or None)."""
    if k.shape[1] != prefix + q.shape[1] or v.shape[1] != prefix + q.shape[1]:
        raise ValueError("k and v must hold prefix + L positions")
    return _prefill("chunk", q, k, v, sink, window, o, lse, scale, stream, want_lse, prefix)


def sinkattn_prefill_chunk_paged(q, k, v, k_pages, v_pages, page_table, sink=None, *, prefix,
                                 window=0, num_pages=None, o=None, lse=None, scale=None,
                                 stream=None, want_lse=True):
    """Chunked prefill against a paged prefix: q, k, v [B, L, ...] are the chunk's own tokens
    (positions prefix .. prefix+L-1); positions 0 .. prefix-1 are row c % page_size of page
    page_table[b, c // page_size] of k_pages [pages, page_size, Hkv, 192] / v_pages [.., 128].
    prefix and page_size must be multiples of 128. Returns (o, lse) as sinkattn_prefill_chunk."""
    _check_bf16("k_pages", k_pages)
    _check_bf16("v_pages", v_pages)
    if page_table.dtype != torch.int32 or not page_table.is_cuda or not page_table.is_contiguous() \
            or page_table.dim() != 2:
        raise ValueError("page_table must be a contiguous 2-D CUDA int32 tensor")
    pk = PagedKV()
    pk.k_pages, pk.v_pages, pk.page_table = _ptr(k_pages), _ptr(v_pages), _ptr(page_table)
    pk.kp_sb, pk.kp_ss, pk.kp_sh = k_pages.stride(0), k_pages.stride(1), k_pages.stride(2)
    pk.vp_sb, pk.vp_ss, pk.vp_sh = v_pages.stride(0), v_pages.stride(1), v_pages.stride(2)
    pk.page_size, pk.max_pages = k_pages.shape[1], page_table.shape[1]
    pk.num_pages = k_pages.shape[0] if num_pages is None else int(num_pages)
    return _prefill("chunk_paged", q, k, v, sink, window, o, lse, scale, stream, want_lse, prefix,
                    pk)


def _host_prefill_args(q, k, v, sink, o, lse, scale):
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda:
            raise ValueError(f"{n} must be a bfloat16 host tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous 4-D tensor")
    if lse is not None and (lse.dtype != torch.float32 or lse.is_cuda or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 host tensor")
    _check_vec("sink", sink, torch.float32)
    B, L, Hq, dq = q.shape
    a = PrefillArgs()
    a.q, a.k, a.v, a.sink, a.o = q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(sink), o.data_ptr()
    a.lse = lse.data_ptr() if lse is not None else None
    a.B, a.L, a.Hq, a.Hkv, a.dq, a.dv = B, L, Hq, k.shape[2], dq, v.shape[3]
    a.scale = scale
    a.q_sb, a.q_sl, a.q_sh = q.stride(0), q.stride(1), q.stride(2)
    a.k_sb, a.k_sl, a.k_sh = k.stride(0), k.stride(1), k.stride(2)
    a.v_sb, a.v_sl, a.v_sh = v.stride(0), v.stride(1), v.stride(2)
    a.o_sb, a.o_sl, a.o_sh = o.stride(0), o.stride(1), o.stride(2)
    return a


def sinkattn_prefill_host_workspace_size(q, k, v, *, chunk=HOST_CHUNK):
    """Device workspace bytes of sinkattn_prefill_host for these (host) tensor shapes."""
    B, L, Hq, dq = q.shape
    a = PrefillArgs()
    a.B, a.L, a.Hq, a.Hkv, a.dq, a.dv = B, L, Hq, k.shape[2], dq, v.shape[3]
    return int(lib().sinkattn_prefill_host_workspace_size(ctypes.byref(a), int(chunk)))


def sinkattn_prefill_host(q, k, v, sink=None, *, window=0, o=None, lse=None, workspace=None,
                          chunk=HOST_CHUNK, scale=None, stream=None, want_lse=True):
    """Prefill with q, k, v and the results in host memory (pinned for the copies to overlap):
    the sequences pass through the device in chunks of `chunk` positions, copies in, kernels and
    copies out overlapping on their own streams. window = 0 full causal (GA), >= 1 sliding
    window (SWA); sink is a CUDA fp32 [Hq] tensor or None; workspace a CUDA uint8 tensor of at
    least sinkattn_prefill_host_workspace_size bytes (allocated if None). Returns (o, lse) host
    tensors, complete once `stream` (default: the current stream) has finished."""
    B, L, Hq, dq = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    if o is None:
        o = torch.empty(B, L, Hq, v.shape[3], dtype=torch.bfloat16, pin_memory=True)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, L, dtype=torch.float32, pin_memory=True)
    a = _host_prefill_args(q, k, v, sink, o, lse, scale)
    need = lib().sinkattn_prefill_host_workspace_size(ctypes.byref(a), int(chunk))
    if workspace is None:
        dev = sink.device if sink is not None else torch.device("cuda", torch.cuda.current_device())
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if workspace.dtype != torch.uint8 or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA uint8 tensor")
    st = lib().sinkattn_prefill_host(ctypes.byref(a), int(window), int(chunk), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    _raise(st, "sinkattn_prefill_host")
    return o, lse


# ----------------------------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------------------------

def _is_fp8_cache(t):
    return isinstance(t, torch.Tensor) and t.dtype in (torch.uint8, torch.float8_e4m3fn)


def _decode_args(kind, q, k_new, v_new, k_cache, v_cache, sink, window, scale, ring_head,
                 ring_len, ctx_len, max_ctx, page_table, page_size, num_pages, o, lse,
                 k_scale=None, v_scale=None):
    for n, t in (("q", q), ("k_new", k_new), ("v_new", v_new)):
        _check_bf16(n, t)
    fp8 = _is_fp8_cache(k_cache)
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if fp8:
            if not _is_fp8_cache(t) or not t.is_cuda or t.dim() != 4 or t.stride(-1) != 1:
                raise ValueError(f"{n}: an FP8 cache is a 4-D CUDA uint8 / float8_e4m3fn tensor "
                                 "with a contiguous last dim (both caches alike)")
        else:
            _check_bf16(n, t)
    if o is not None:
        _check_bf16("o", o)
    _check_vec("sink", sink, torch.float32)
    _check_vec("lse", lse, torch.float32)
    for n, t in (("ring_head", ring_head), ("ring_len", ring_len), ("ctx_len", ctx_len)):
        _check_vec(n, t, torch.int32)
    if page_table is not None and (page_table.dtype != torch.int32 or not page_table.is_cuda
                                   or not page_table.is_contiguous() or page_table.dim() != 2):
        raise ValueError("page_table must be a contiguous 2-D CUDA int32 tensor")
    B, T, Hq, dq = q.shape
    a = DecodeArgs()
    a.kind, a.B, a.T, a.Hq, a.Hkv, a.dq, a.dv = kind, B, T, Hq, k_new.shape[2], dq, v_new.shape[3]
    a.window, a.scale, a.sink = int(window), scale, _ptr(sink)
    a.q, a.q_sb, a.q_st, a.q_sh = _ptr(q), q.stride(0), q.stride(1), q.stride(2)
    a.k_new, a.kn_sb, a.kn_st, a.kn_sh = _ptr(k_new), k_new.stride(0), k_new.stride(1), k_new.stride(2)
    a.v_new, a.vn_sb, a.vn_st, a.vn_sh = _ptr(v_new), v_new.stride(0), v_new.stride(1), v_new.stride(2)
    a.k_cache, a.kc_sb, a.kc_ss, a.kc_sh = (_ptr(k_cache), k_cache.stride(0), k_cache.stride(1),
                                            k_cache.stride(2))
    a.v_cache, a.vc_sb, a.vc_ss, a.vc_sh = (_ptr(v_cache), v_cache.stride(0), v_cache.stride(1),
                                            v_cache.stride(2))
    a.ring_head, a.ring_len = _ptr(ring_head), _ptr(ring_len)
    a.ring_cap = k_cache.shape[1] if kind == KV_RING else 0
    a.ctx_len = _ptr(ctx_len)
    if max_ctx is None:
        if kind == KV_CONTIG:
            max_ctx = k_cache.shape[1]
        elif kind == KV_PAGED:
            max_ctx = page_table.shape[1] * k_cache.shape[1]
        else:
            max_ctx = 0
    a.max_ctx = int(max_ctx)
    a.page_table = _ptr(page_table)
    a.page_size = k_cache.shape[1] if kind == KV_PAGED else int(page_size or 0)
    a.max_pages = page_table.shape[1] if page_table is not None else 0
    a.num_pages = (k_cache.shape[0] if num_pages is None else int(num_pages)) if kind == KV_PAGED else 0
    if o is not None:
        a.o, a.o_sb, a.o_st, a.o_sh = _ptr(o), o.stride(0), o.stride(1), o.stride(2)
    a.lse = _ptr(lse)
    if fp8:
        if k_scale is None or v_scale is None:
            raise ValueError("an FP8 cache needs k_scale and v_scale")
        a.kv_dtype, a.k_scale, a.v_scale = KV_FP8_E4M3, float(k_scale), float(v_scale)
    return a


def sinkattn_decode_workspace_size(kind, q, k_new, v_new, k_cache, v_cache, *, window=0,
                                   ring_head=None, ring_len=None, ctx_len=None, max_ctx=None,
                                   page_table=None, page_size=None, num_pages=None) -> int:
    a = _decode_args(kind, q, k_new, v_new, k_cache, v_cache, None, window, 1.0, ring_head,
                     ring_len, ctx_len, max_ctx, page_table, page_size, num_pages, None, None,
                     1.0, 1.0)
    return int(lib().sinkattn_decode_workspace_size(ctypes.byref(a)))


def sinkattn_decode(kind, q, k_new, v_new, k_cache, v_cache, sink=None, *, window=0,
                    ring_head=None, ring_len=None, ctx_len=None, max_ctx=None, page_table=None,
                    page_size=None, num_pages=None, o=None, lse=None, workspace=None,
                    scale=None, stream=None, want_lse=True, k_scale=None, v_scale=None):
    """Decode / speculative verify of T (1..4) new tokens per sequence against a KV cache.

    kind: KV_RING (k_cache [B,cap,Hkv,192] with ring_head/ring_len int32 [B]), KV_CONTIG
    (k_cache [B,max_ctx,Hkv,192] with ctx_len [B]) or KV_PAGED (k_cache [pages,page,Hkv,192]
    with page_table [B,max_pages] and ctx_len [B]). The new tokens' K/V are not in the cache.
    A uint8 / float8_e4m3fn cache holds E4M3 codes scaled by k_scale / v_scale (FP8 cache).
    Returns (o [B,T,Hq,128] bf16, lse [B,T,Hq] fp32 or None)."""
    B, T, Hq, dq = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    if o is None:
        o = torch.empty(B, T, Hq, v_new.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, T, Hq, dtype=torch.float32, device=q.device)
    a = _decode_args(kind, q, k_new, v_new, k_cache, v_cache, sink, window, scale, ring_head,
                     ring_len, ctx_len, max_ctx, page_table, page_size, num_pages, o, lse,
                     k_scale, v_scale)
    L_ = lib()
    need = int(L_.sinkattn_decode_workspace_size(ctypes.byref(a)))
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if need > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if need > 0 else 0
    st = L_.sinkattn_decode(ctypes.byref(a), ws_ptr, ws_bytes, _stream(stream))
    _raise(st, "sinkattn_decode")
    return o, lse


def sinkattn_decode_noalloc(kind, q, k_new, v_new, k_cache, v_cache, sink=None, *, window=0,
                            ring_head=None, ring_len=None, ctx_len=None, max_ctx=None,
                            page_table=None, page_size=None, num_pages=None, o=None, lse=None,
                            scale=None, stream=None, k_scale=None, v_scale=None):
    """Decode without a workspace, for callers that cannot allocate device memory (a plugin host
    that passes only input/output buffers, a serving loop with all memory reserved up front).
    The library keeps the split-KV partials in its own fixed 16 MiB device array; larger
    problems are rejected (use sinkattn_decode with a workspace). Calls that overlap on the GPU
    race on that array. `o` and `lse` must be given (nothing is allocated here)."""
    B, T, Hq, dq = q.shape
    if o is None or lse is None:
        raise ValueError("sinkattn_decode_noalloc allocates nothing: pass o and lse")
    if scale is None:
        scale = 1.0 / math.sqrt(dq)
    a = _decode_args(kind, q, k_new, v_new, k_cache, v_cache, sink, window, scale, ring_head,
                     ring_len, ctx_len, max_ctx, page_table, page_size, num_pages, o, lse,
                     k_scale, v_scale)
    _raise(lib().sinkattn_decode_noalloc(ctypes.byref(a), _stream(stream)),
           "sinkattn_decode_noalloc")
    return o, lse


def sinkattn_kv_commit(kind, k_new, v_new, n_accept, k_cache, v_cache, *, ring_head=None,
                       ring_len=None, ctx_len=None, max_ctx=None, page_table=None,
                       num_pages=None, stream=None, k_scale=None, v_scale=None,
                       rope_theta=None, rope_dim=ROPE_DIM, commit_v_scale=V_SCALE, pos=None):
    """Append the first n_accept[b] of each sequence's T new tokens to its cache, in place.
    Into an FP8 cache (uint8 / float8_e4m3fn) each element x is stored as the E4M3 code of
    x / scale (k_scale for K, v_scale for V).
    rope_theta given: K is stored with the partial rotary embedding of its first rope_dim dims at
    position pos[b] + u (pos: int32 [B]; None = ctx_len before the commit, not for a ring) and V
    multiplied by commit_v_scale, as sinkattn_rope_qkv would; k_new / v_new are not modified."""
    _check_vec("n_accept", n_accept, torch.int32)
    _check_vec("pos", pos, torch.int32)
    B, T, Hkv, dq = k_new.shape
    q_dummy = k_new  # only the cache-related fields are read
    a = _decode_args(kind, q_dummy, k_new, v_new, k_cache, v_cache, None, 0, 1.0, ring_head,
                     ring_len, ctx_len, max_ctx, page_table, None, num_pages, None, None,
                     k_scale, v_scale)
    if rope_theta is not None:
        a.commit_rope, a.rope_dim, a.rope_theta = 1, int(rope_dim), float(rope_theta)
        a.commit_v_scale, a.commit_pos = float(commit_v_scale), _ptr(pos)
    st = lib().sinkattn_kv_commit(ctypes.byref(a), _ptr(n_accept), _stream(stream))
    _raise(st, "sinkattn_kv_commit")


def sinkattn_rope_qkv(q=None, k=None, v=None, *, theta, rope_dim=ROPE_DIM, v_scale=V_SCALE,
                      pos0=0, pos_base=None, stream=None):
    """Partial RoPE on the first rope_dim dims of q [B,L,Hq,dq] and k [B,L,Hkv,dq], and v
    [B,L,Hkv,dv] times v_scale, all in place (any of the three may be None). Token l of
    sequence b sits at position pos0 + pos_base[b] + l (pos_base: CUDA int32 [B] or None).
    theta: ROPE_THETA_GA or ROPE_THETA_SWA for the pages' model."""
    given = [t for t in (q, k, v) if t is not None]
    for n, t in (("q", q), ("k", k), ("v", v)):
        if t is not None:
            _check_bf16(n, t)
    _check_vec("pos_base", pos_base, torch.int32)
    if not given:
        return
    B, L = given[0].shape[:2]
    if any(tuple(t.shape[:2]) != (B, L) for t in given):
        raise ValueError("q, k and v must share [B, L]")
    if q is not None and k is not None and q.shape[3] != k.shape[3]:
        raise ValueError("q and k must share the head dim")
    if k is not None and v is not None and k.shape[2] != v.shape[2]:
        raise ValueError("k and v must share the KV head count")
    if pos_base is not None and pos_base.numel() != B:
        raise ValueError("pos_base must have B entries")
    a = RopeArgs()
    a.B, a.L = B, L
    a.Hq = q.shape[2] if q is not None else 0
    a.Hkv = k.shape[2] if k is not None else (v.shape[2] if v is not None else 0)
    a.dq = (q if q is not None else k).shape[3] if (q is not None or k is not None) else 0
    a.dv = v.shape[3] if v is not None else 0
    a.rope_dim, a.theta, a.v_scale = int(rope_dim), float(theta), float(v_scale)
    a.pos0, a.pos_base = int(pos0), _ptr(pos_base)
    if q is not None:
        a.q, a.q_sb, a.q_sl, a.q_sh = _ptr(q), q.stride(0), q.stride(1), q.stride(2)
    if k is not None:
        a.k, a.k_sb, a.k_sl, a.k_sh = _ptr(k), k.stride(0), k.stride(1), k.stride(2)
    if v is not None:
        a.v, a.v_sb, a.v_sl, a.v_sh = _ptr(v), v.stride(0), v.stride(1), v.stride(2)
    _raise(lib().sinkattn_rope_qkv(ctypes.byref(a), _stream(stream)), "sinkattn_rope_qkv")


def sinkattn_take_device_error() -> int:
    """Reads and clears the kernels' wait-timeout flag (synchronises the device)."""
    flag = ctypes.c_uint32(0)
    _raise(lib().sinkattn_take_device_error(ctypes.byref(flag)), "sinkattn_take_device_error")
    return int(flag.value)


def sinkattn_prefill_backward(q, k, v, o, lse, dout, sink=None, *, window=0, scale=None,
                              dq=None, dk=None, dv=None, dsink=True, workspace=None, stream=None):
    """Gradients of the whole-sequence prefill (the training variant): given the forward's
    q, k, v, its output o and lse ([B, Hq, L]) and dout = dLoss/dO, returns (dq, dk, dv, dsink)
    as fp32 tensors (dq [B,L,Hq,192], dk [B,L,Hkv,192], dv [B,L,Hkv,128], dsink [Hq] or None
    when dsink=False). window 0: GA, >= 1: SWA."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bf16(n, t)
    _check_vec("sink", sink, torch.float32)
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous CUDA float32 tensor [B, Hq, L]")
    B, L, Hq, dqk = q.shape
    Hkv, dvv = k.shape[2], v.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(B, L, Hq, dqk, **f32) if dq is None else dq
    dk = torch.empty(B, L, Hkv, dqk, **f32) if dk is None else dk
    dv = torch.empty(B, L, Hkv, dvv, **f32) if dv is None else dv
    ds = (torch.empty(Hq, **f32) if dsink is True else dsink) if dsink is not False else None
    a = BackwardArgs()
    a.q, a.k, a.v, a.o, a.dout, a.lse = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse)
    a.sink, a.dq, a.dk, a.dv, a.dsink = _ptr(sink), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds)
    a.B, a.L, a.Hq, a.Hkv, a.d_qk, a.d_v, a.scale = B, L, Hq, Hkv, dqk, dvv, float(scale)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", dout), ("dq", dq), ("dk", dk),
                    ("dv", dv)):
        if t.stride(-1) != 1:
            raise ValueError(f"{name}: the last dim must be contiguous")
        setattr(a, f"{name}_sb", t.stride(0))
        setattr(a, f"{name}_sl", t.stride(1))
        setattr(a, f"{name}_sh", t.stride(2))
    L_ = lib()
    need = int(L_.sinkattn_prefill_backward_workspace_size(ctypes.byref(a)))
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if need > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if need > 0 else 0
    _raise(L_.sinkattn_prefill_backward(ctypes.byref(a), int(window), ws_ptr, ws_bytes,
                                        _stream(stream)), "sinkattn_prefill_backward")
    return dq, dk, dv, ds


def sinkattn_set_wait_limit_ns(ns: int) -> None:
    """How long a kernel on the current device waits on an internal barrier before it gives up
    and records it in the wait-timeout flag (default 10**9 ns; 0 gives up as soon as a wait's
    first, briefly suspending try fails). Process-wide per device; synchronises the device."""
    _raise(lib().sinkattn_set_wait_limit_ns(int(ns)), "sinkattn_set_wait_limit_ns")
