"""The C ABI without a GPU: the library loads, exports every entry point the header declares,
its structs have the layout the Python binding assumes, and invalid arguments are rejected on
the host before any CUDA call."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import build as sa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sinkattn.h")


@pytest.fixture(scope="module")
def L():
    sa_build.build()
    return sa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sinkattn_\w+)\s*\(", text)))


def test_header_and_binding_agree_on_entry_points():
    assert declared_functions() == sorted(sa.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", sa.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sinkattn_\w+)", out))
    missing = set(declared_functions()) - exported
    assert not missing, missing
    for name in declared_functions():
        assert hasattr(L, name)


def test_version_and_status_strings(L):
    assert sa.sinkattn_version() == 1
    assert sa.sinkattn_status_string(0) == "ok"
    for s in range(1, 6):
        assert sa.sinkattn_status_string(s) not in ("ok", "unknown status")
    assert sa.sinkattn_status_string(99) == "unknown status"


C_LAYOUT = r"""
#include <stddef.h>
#include <stdio.h>
#include "sinkattn.h"
#define F(S, f) printf(#S "." #f " %zu\n", offsetof(S, f));
int main(void) {
  printf("sinkattn_prefill_args %zu\n", sizeof(sinkattn_prefill_args));
  printf("sinkattn_decode_args %zu\n", sizeof(sinkattn_decode_args));
  printf("sinkattn_rope_args %zu\n", sizeof(sinkattn_rope_args));
  printf("sinkattn_backward_args %zu\n", sizeof(sinkattn_backward_args));
  printf("sinkattn_paged_kv %zu\n", sizeof(sinkattn_paged_kv));
  printf("sinkattn_rope_spec %zu\n", sizeof(sinkattn_rope_spec));
  %FIELDS%
  return 0;
}
"""


def test_struct_layout_matches_header(tmp_path):
    lines = []
    structs = (("sinkattn_prefill_args", sa.PrefillArgs), ("sinkattn_decode_args", sa.DecodeArgs),
               ("sinkattn_rope_args", sa.RopeArgs), ("sinkattn_backward_args", sa.BackwardArgs),
               ("sinkattn_paged_kv", sa.PagedKV), ("sinkattn_rope_spec", sa.RopeSpec))
    for cname, py in structs:
        for f, _ in py._fields_:
            lines.append(f"F({cname}, {f})")
    src = C_LAYOUT.replace("%FIELDS%", "\n  ".join(lines))
    c = tmp_path / "layout.c"
    exe = tmp_path / "layout"
    c.write_text(src)
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)])
    got = dict(l.rsplit(" ", 1) for l in subprocess.check_output([str(exe)], text=True).splitlines())
    assert int(got["sinkattn_prefill_args"]) == ctypes.sizeof(sa.PrefillArgs)
    assert int(got["sinkattn_decode_args"]) == ctypes.sizeof(sa.DecodeArgs)
    assert int(got["sinkattn_rope_args"]) == ctypes.sizeof(sa.RopeArgs)
    assert int(got["sinkattn_backward_args"]) == ctypes.sizeof(sa.BackwardArgs)
    assert int(got["sinkattn_paged_kv"]) == ctypes.sizeof(sa.PagedKV)
    assert int(got["sinkattn_rope_spec"]) == ctypes.sizeof(sa.RopeSpec)
    for cname, py in structs:
        for f, _ in py._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(py, f).offset, (cname, f)


def _prefill_args(**kw):
    a = sa.PrefillArgs()
    a.q = a.k = a.v = a.o = 0x10000
    a.B, a.L, a.Hq, a.Hkv, a.dq, a.dv = 1, 64, 8, 1, 192, 128
    a.scale = 0.07
    for f in ("q", "k", "v", "o"):
        d = 192 if f in ("q", "k") else 128
        h = 8 if f in ("q", "o") else 1
        setattr(a, f + "_sh", d)
        setattr(a, f + "_sl", d * h)
        setattr(a, f + "_sb", d * h * 64)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(dq=128), 2), (dict(dv=192), 2), (dict(Hkv=3), 2), (dict(B=-1), 1), (dict(Hq=0), 1),
    (dict(q=None), 1), (dict(q=0x10008), 3), (dict(k_sl=100), 3), (dict(o_sh=0), 1),
    (dict(scale=float("inf")), 1), (dict(scale=0.0), 1), (dict(scale=-0.1), 1),
])
def test_prefill_rejects_bad_arguments(L, kw, status):
    a = _prefill_args(**kw)
    assert L.sinkattn_prefill_ga(ctypes.byref(a), None) == status
    assert L.sinkattn_prefill_swa(ctypes.byref(a), 128, None) == status
    assert L.sinkattn_prefill_chunk(ctypes.byref(a), 100, 0, None) == status


def test_chunk_checks_prefix_and_window(L):
    """Rejected before any device work: a negative prefix or window, and a sequence whose
    positions overflow int32; an empty chunk is a no-op."""
    a = _prefill_args()
    assert L.sinkattn_prefill_chunk(ctypes.byref(a), -1, 0, None) == 1
    assert L.sinkattn_prefill_chunk(ctypes.byref(a), 0, -1, None) == 1
    assert L.sinkattn_prefill_chunk(ctypes.byref(a), 0x7fffffff - 10, 0, None) == 1
    assert L.sinkattn_prefill_chunk(ctypes.byref(_prefill_args(L=0)), 5, 0, None) == 0
    assert L.sinkattn_prefill_chunk(None, 0, 0, None) == 1


def test_host_prefill_sizes_and_checks(L):
    """The host-resident prefill: the workspace size follows from the shapes alone (K and V of
    every position, two chunks of Q, O and LSE); arguments are checked before any device work."""
    a = _prefill_args()  # B 1, L 64, 8 / 1 heads, dense strides
    L.sinkattn_prefill_host_workspace_size.restype = ctypes.c_size_t
    size = L.sinkattn_prefill_host_workspace_size(ctypes.byref(a), 128)
    al = lambda x: (x + 255) // 256 * 256
    want = al(64 * 1 * 384) + al(64 * 1 * 256) + 2 * (al(128 * 8 * 384) + al(128 * 8 * 256) + al(8 * 128 * 4))
    assert size == want
    assert L.sinkattn_prefill_host_workspace_size(ctypes.byref(a), 100) == 0
    assert L.sinkattn_prefill_host_workspace_size(ctypes.byref(a), 0) == 0
    assert L.sinkattn_prefill_host_workspace_size(None, 128) == 0
    ws = ctypes.c_void_p(0x20000)
    host = L.sinkattn_prefill_host
    host.argtypes = [ctypes.POINTER(sa.PrefillArgs), ctypes.c_int32, ctypes.c_int32,
                     ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert host(ctypes.byref(a), 128, 100, ws, size, None) == 2          # chunk not 128-aligned
    assert host(ctypes.byref(a), 128, 0, ws, size, None) == 1            # chunk <= 0
    assert host(ctypes.byref(a), -1, 128, ws, size, None) == 1           # negative window
    assert host(ctypes.byref(_prefill_args(k_sl=384)), 128, 128, ws, size, None) == 2  # not dense
    assert host(ctypes.byref(a), 128, 128, None, size, None) == 1        # no workspace
    assert host(ctypes.byref(a), 128, 128, ws, size - 1, None) == 4      # workspace too small
    assert host(ctypes.byref(_prefill_args(L=0)), 128, 128, None, 0, None) == 0


def test_fused_rope_prefill_checks(L):
    """The fused RoPE SWA prefill checks its spec before any device work."""
    f = L.sinkattn_prefill_swa_rope
    f.argtypes = [ctypes.POINTER(sa.PrefillArgs), ctypes.c_int32, ctypes.POINTER(sa.RopeSpec),
                  ctypes.c_void_p]

    def spec(**kw):
        r = sa.RopeSpec()
        r.pos_base, r.pos0, r.rope_dim, r.theta, r.v_scale = None, 0, 64, 1e4, 0.707
        for k, v in kw.items():
            setattr(r, k, v)
        return r
    a = _prefill_args()
    assert f(ctypes.byref(a), 128, None, None) == 1                          # no spec
    assert f(ctypes.byref(a), 0, ctypes.byref(spec()), None) == 1            # window < 1
    assert f(ctypes.byref(a), 128, ctypes.byref(spec(theta=0.0)), None) == 1
    assert f(ctypes.byref(a), 128, ctypes.byref(spec(theta=float("inf"))), None) == 1
    assert f(ctypes.byref(a), 128, ctypes.byref(spec(v_scale=float("nan"))), None) == 1
    for rd in (0, 8, 24, 80, 128):                                           # not 16..64 step 16
        assert f(ctypes.byref(a), 128, ctypes.byref(spec(rope_dim=rd)), None) == 2
    assert f(ctypes.byref(_prefill_args(dq=128)), 128, ctypes.byref(spec()), None) == 2
    assert f(ctypes.byref(_prefill_args(L=0)), 128, ctypes.byref(spec()), None) == 0


def test_prefill_empty_is_ok_and_window_checked(L):
    assert L.sinkattn_prefill_ga(ctypes.byref(_prefill_args(L=0)), None) == 0
    assert L.sinkattn_prefill_ga(ctypes.byref(_prefill_args(B=0, q=None)), None) == 0
    assert L.sinkattn_prefill_swa(ctypes.byref(_prefill_args()), 0, None) == 1
    assert L.sinkattn_prefill_swa(ctypes.byref(_prefill_args()), -5, None) == 1
    assert L.sinkattn_prefill_ga(None, None) == 1


def _decode_args(**kw):
    a = sa.DecodeArgs()
    a.kind, a.B, a.T, a.Hq, a.Hkv, a.dq, a.dv, a.window = 1, 2, 1, 64, 4, 192, 128, 0
    a.scale = 0.07
    a.q = a.k_new = a.v_new = a.k_cache = a.v_cache = a.o = 0x20000
    a.ctx_len = 0x30000
    a.max_ctx = 4096
    for pre, d in (("q", 192), ("kn", 192), ("vn", 128), ("kc", 192), ("vc", 128), ("o", 128)):
        for i, s in enumerate(("sb", "st" if pre in ("q", "kn", "vn", "o") else "ss", "sh")):
            setattr(a, f"{pre}_{s}", d * (4096 if i == 0 else (64 if i == 1 else 1)))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(kind=7), 1), (dict(T=5), 2), (dict(Hkv=2), 2), (dict(Hkv=3), 2), (dict(dq=64), 2),
    (dict(ctx_len=None), 1), (dict(kind=0), 1), (dict(kind=2), 1), (dict(o=None), 1),
    (dict(k_cache=0x20004), 3), (dict(kc_ss=10), 3), (dict(window=-1), 1),
    (dict(kind=2, page_table=0x40000, page_size=128, max_pages=2, num_pages=4), 1),
])
def test_decode_rejects_bad_arguments(L, kw, status):
    a = _decode_args(**kw)
    assert L.sinkattn_decode(ctypes.byref(a), None, 0, None) == status


def test_workspace_size_needs_shapes_only(L):
    a = _decode_args(B=8, max_ctx=262144)
    need = L.sinkattn_decode_workspace_size(ctypes.byref(a))
    for f in ("q", "k_new", "v_new", "k_cache", "v_cache", "o", "ctx_len"):
        b = _decode_args(B=8, max_ctx=262144, **{f: None})
        assert L.sinkattn_decode_workspace_size(ctypes.byref(b)) == need
    for kw in (dict(T=5), dict(Hkv=3), dict(dq=64), dict(kind=7), dict(window=-1)):
        assert L.sinkattn_decode_workspace_size(ctypes.byref(_decode_args(B=8, **kw))) == 0


def test_decode_workspace_sizing(L):
    # GA decode at 262144 tokens of context, 8 x 4 units: split, workspace = partial rows
    a = _decode_args(B=8, max_ctx=262144)
    need = L.sinkattn_decode_workspace_size(ctypes.byref(a))
    assert need > 0 and need % (132 * 4 * 16) == 0
    assert L.sinkattn_decode(ctypes.byref(a), None, 0, None) == 4
    assert L.sinkattn_decode(ctypes.byref(a), ctypes.c_void_p(0x50000), need - 1, None) == 4
    assert L.sinkattn_decode(ctypes.byref(a), ctypes.c_void_p(0x50008), need, None) == 3
    # a 128-slot ring never needs a split
    r = _decode_args(kind=0, ring_head=0x30000, ring_len=0x30100, ring_cap=128, window=128, Hkv=8)
    assert L.sinkattn_decode_workspace_size(ctypes.byref(r)) == 0
    # empty work
    assert L.sinkattn_decode(ctypes.byref(_decode_args(B=0)), None, 0, None) == 0
    assert L.sinkattn_decode(ctypes.byref(_decode_args(T=0)), None, 0, None) == 0


def test_commit_rejects_bad_arguments(L):
    a = _decode_args()
    assert L.sinkattn_kv_commit(ctypes.byref(a), None, None) == 1
    assert L.sinkattn_kv_commit(ctypes.byref(_decode_args(dv=64)), ctypes.c_void_p(0x60000), None) == 2
    assert L.sinkattn_kv_commit(ctypes.byref(_decode_args(kind=0)), ctypes.c_void_p(0x60000), None) == 1
    assert L.sinkattn_kv_commit(ctypes.byref(_decode_args(B=0)), None, None) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(commit_rope=2), 1),                                         # not a flag
    (dict(commit_rope=1, rope_dim=64, rope_theta=0.0), 1),            # theta must be > 0
    (dict(commit_rope=1, rope_dim=64, rope_theta=float("nan")), 1),
    (dict(commit_rope=1, rope_dim=64, rope_theta=1e4, commit_v_scale=float("inf")), 1),
    (dict(commit_rope=1, rope_dim=24, rope_theta=1e4), 2),            # not a multiple of 16
    (dict(commit_rope=1, rope_dim=144, rope_theta=1e4), 2),           # wider than 128
    (dict(commit_rope=1, rope_dim=64, rope_theta=1e4, kind=0, ring_head=0x50000,
          ring_len=0x50100, ring_cap=128), 1),                        # a ring needs commit_pos
])
def test_commit_rope_arguments_are_checked(L, kw, status):
    """Host-side checks of the commit's fused RoPE + value scale: nothing reaches the GPU."""
    a = _decode_args(**kw)
    assert L.sinkattn_kv_commit(ctypes.byref(a), ctypes.c_void_p(0x60000), None) == status


def _paged_kv(**kw):
    pk = sa.PagedKV()
    pk.k_pages, pk.v_pages, pk.page_table = 0x40000, 0x50000, 0x60000
    pk.page_size, pk.max_pages, pk.num_pages = 128, 4, 8
    pk.kp_sh, pk.kp_ss, pk.kp_sb = 192, 192, 192 * 128
    pk.vp_sh, pk.vp_ss, pk.vp_sb = 128, 128, 128 * 128
    for k, v in kw.items():
        setattr(pk, k, v)
    return pk


@pytest.mark.parametrize("prefix,kw,status", [
    (128, dict(page_table=None), 1), (128, dict(page_size=0), 1), (100, {}, 2),
    (128, dict(page_size=64), 2), (640, {}, 1),           # beyond max_pages * page_size
    (128, dict(k_pages=0x40008), 3), (128, dict(vp_ss=12), 3), (128, dict(kp_sb=0), 1),
])
def test_chunk_paged_checks_its_prefix(L, prefix, kw, status):
    """Host-side checks of the paged prefix: nothing reaches the GPU."""
    a = _prefill_args()
    pk = _paged_kv(**kw)
    assert L.sinkattn_prefill_chunk_paged(ctypes.byref(a), ctypes.byref(pk), prefix, 0, None) == status
    assert L.sinkattn_prefill_chunk_paged(ctypes.byref(a), None, 128, 0, None) == 1
    assert L.sinkattn_prefill_chunk_paged(ctypes.byref(a), ctypes.byref(_paged_kv()), 128, -1, None) == 1


def _backward_args(**kw):
    a = sa.BackwardArgs()
    a.q = a.k = a.v = a.o = a.dout = a.lse = a.dq = a.dk = a.dv = 0x10000
    a.B, a.L, a.Hq, a.Hkv, a.d_qk, a.d_v = 1, 64, 8, 1, 192, 128
    a.scale = 0.07
    for t, d, h in (("q", 192, 8), ("k", 192, 1), ("v", 128, 1), ("o", 128, 8), ("do", 128, 8),
                    ("dq", 192, 8), ("dk", 192, 1), ("dv", 128, 1)):
        setattr(a, t + "_sh", d)
        setattr(a, t + "_sl", d * h)
        setattr(a, t + "_sb", d * h * 64)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(d_qk=128), 2), (dict(Hkv=3), 2), (dict(B=-1), 1), (dict(scale=0.0), 1),
    (dict(o=None), 1), (dict(lse=None), 1), (dict(dk=None), 1), (dict(dout=0x10008), 3),
    (dict(q_sl=100), 3), (dict(dq_sl=6), 3), (dict(dv_sh=0), 1),
])
def test_backward_rejects_bad_arguments(L, kw, status):
    """Host-side checks of the prefill backward: nothing reaches the GPU."""
    a = _backward_args(**kw)
    assert L.sinkattn_prefill_backward(ctypes.byref(a), 0, None, 0, None) == status


def test_backward_workspace_and_window(L):
    a = _backward_args()
    need = L.sinkattn_prefill_backward_workspace_size(ctypes.byref(a))
    assert need == 1 * 8 * 64 * 4   # delta: one float per (sequence, head, row)
    assert L.sinkattn_prefill_backward(ctypes.byref(a), 0, None, 0, None) == 4
    assert L.sinkattn_prefill_backward(ctypes.byref(a), -1, None, 0, None) == 1
    assert L.sinkattn_prefill_backward(ctypes.byref(_backward_args(L=0)), 0, None, 0, None) == 0


def _rope_args(**kw):
    a = sa.RopeArgs()
    a.q, a.k, a.v = 0x10000, 0x20000, 0x30000
    a.B, a.L, a.Hq, a.Hkv, a.dq, a.dv, a.rope_dim = 2, 64, 64, 8, 192, 128, 64
    a.theta, a.v_scale = 1e4, 0.707
    for f, d, h in (("q", 192, 64), ("k", 192, 8), ("v", 128, 8)):
        setattr(a, f + "_sh", d)
        setattr(a, f + "_sl", d * h)
        setattr(a, f + "_sb", d * h * 64)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(L=-3), 1), (dict(theta=0.0), 1), (dict(theta=-1e4), 1),
    (dict(theta=float("inf")), 1), (dict(theta=float("nan")), 1), (dict(v_scale=float("nan")), 1),
    (dict(Hq=0), 1), (dict(Hkv=0), 1), (dict(q_sl=0), 1), (dict(v_sh=-128), 1),
    (dict(rope_dim=8), 2), (dict(rope_dim=72), 2), (dict(rope_dim=144), 2), (dict(dq=48), 2),
    (dict(dq=196), 2), (dict(dv=120), 2),
    (dict(q=0x10004), 3), (dict(v=0x30002), 3), (dict(k_sl=100), 3),
])
def test_rope_rejects_bad_arguments(L, kw, status):
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(**kw)), None) == status


def test_rope_empty_and_partial_calls_need_no_device(L):
    """Empty work, or no tensor at all, returns OK before any CUDA call; a tensor that is not
    given is not checked (its head count and strides may be anything)."""
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(B=0)), None) == 0
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(L=0)), None) == 0
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(q=None, k=None, v=None)), None) == 0
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(B=0, q=None, Hq=0, q_sl=0)), None) == 0
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(B=0, v=None, dv=120)), None) == 0
    assert L.sinkattn_rope_qkv(ctypes.byref(_rope_args(B=0, q=None, k=None, rope_dim=0)), None) == 0
    assert L.sinkattn_rope_qkv(None, None) == 1


FP8 = dict(kv_dtype=1, k_scale=0.02, v_scale=0.02)


@pytest.mark.parametrize("kw,status", [
    (dict(kv_dtype=2), 1), (dict(kv_dtype=-1), 1),
    (dict(FP8, k_scale=0.0), 1), (dict(FP8, v_scale=-0.5), 1),
    (dict(FP8, k_scale=float("nan")), 1), (dict(FP8, v_scale=float("inf")), 1),
    # an FP8 cache's strides count bytes: 200 is a whole number of 16-byte bf16 units (8-element
    # multiples) but not of 16 bytes
    (dict(FP8, kc_ss=200), 3), (dict(FP8, vc_sh=136), 3),
])
def test_fp8_cache_arguments_are_checked(L, kw, status):
    a = _decode_args(**kw)
    assert L.sinkattn_decode(ctypes.byref(a), None, 0, None) == status
    assert L.sinkattn_decode_noalloc(ctypes.byref(a), None) == status
    assert L.sinkattn_kv_commit(ctypes.byref(a), ctypes.c_void_p(0x60000), None) == status


def test_fp8_strides_fine_for_bf16_and_workspace_independent_of_dtype(L):
    # the bf16 reading of the same 200-element stride is aligned: that call fails only later,
    # on the missing workspace (a GA context of 4096 tokens needs a split)
    a = _decode_args(kc_ss=200, B=8, max_ctx=262144)
    assert L.sinkattn_decode(ctypes.byref(a), None, 0, None) == 4
    b = _decode_args(B=8, max_ctx=262144, **FP8)
    assert L.sinkattn_decode_workspace_size(ctypes.byref(b)) == \
        L.sinkattn_decode_workspace_size(ctypes.byref(_decode_args(B=8, max_ctx=262144)))


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sa, "library_path", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sa, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        sa.lib()


def test_binding_checks_tensor_types():
    q = torch.zeros(1, 4, 8, 192)
    with pytest.raises(TypeError):
        sa.sinkattn_prefill_ga(q, q, q, o=torch.zeros(1, 4, 8, 128))
