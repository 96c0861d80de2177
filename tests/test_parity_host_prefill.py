"""GPU parity of the host-resident prefill (inputs and outputs in pinned host memory, streamed
through the device chunk by chunk) against the fp64 oracle."""
import math

import pytest
import torch

import oracle
import global_attention_sink_softmax_b200 as sa
from global_attention_sink_softmax_b200 import workloads as W
from parity import assert_close
from test_parity_prefill import rand_inputs, sample_rows

pytestmark = pytest.mark.gpu


def pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("B,L,Hq,Hkv,window,chunk", [
    (1, 1000, 8, 1, 128, 256),   # 4 chunks, ragged last chunk, windows crossing chunk edges
    (2, 640, 16, 2, 0, 128),     # GA, 5 chunks of exactly one tile
    (1, 300, 4, 1, 7, 4096),     # one chunk, shorter than the chunk size
    (2, 513, 8, 8, 200, 256),    # a window longer than a tile
    (1, 129, 64, 4, 0, 128),     # the model's GA heads, a tail of one row
])
def test_host_prefill_matches_oracle(B, L, Hq, Hkv, window, chunk):
    q, k, v, s = rand_inputs(B, L, Hq, Hkv, seed=17 * L + chunk + window)
    sd = s.to("cuda")
    o, lse = sa.sinkattn_prefill_host(pinned(q), pinned(k), pinned(v), sd, window=window,
                                      chunk=chunk)
    torch.cuda.synchronize()
    assert not o.is_cuda and not lse.is_cuda
    ro, rl, _ = oracle.prefill(q, k, v, s, 1 / math.sqrt(192), window)
    assert_close(o, ro, lse.permute(0, 2, 1), rl, f"host B{B} L{L} {Hq}/{Hkv} W{window} c{chunk}")
    assert sa.sinkattn_take_device_error() == 0


def test_host_prefill_equals_device_chunks():
    """Chunk by chunk the host call runs the same kernels as sinkattn_prefill_chunk (the first
    chunk as a whole-sequence prefill), so its result is bit for bit theirs."""
    B, L, Hq, Hkv, window, chunk = 2, 700, 16, 2, 128, 256
    q, k, v, s = rand_inputs(B, L, Hq, Hkv, seed=5)
    dev = "cuda"
    sd = s.to(dev)
    o, lse = sa.sinkattn_prefill_host(pinned(q), pinned(k), pinned(v), sd, window=window,
                                      chunk=chunk)
    torch.cuda.synchronize()
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    for c0 in range(0, L, chunk):
        c1 = min(L, c0 + chunk)
        if c0 == 0:
            oc, lc = sa.sinkattn_prefill_swa(qd[:, :c1].contiguous(), kd[:, :c1].contiguous(),
                                             vd[:, :c1].contiguous(), sd, window)
        else:
            oc, lc = sa.sinkattn_prefill_chunk(qd[:, c0:c1], kd[:, :c1], vd[:, :c1], sd,
                                               prefix=c0, window=window)
        torch.cuda.synchronize()
        assert torch.equal(o[:, c0:c1], oc.cpu()), c0
        assert torch.equal(lse[:, :, c0:c1], lc.cpu()), c0


def test_host_prefill_rejects_device_and_strided_tensors():
    q, k, v, s = rand_inputs(1, 256, 8, 1, seed=1)
    with pytest.raises(ValueError):
        sa.sinkattn_prefill_host(q.cuda(), k, v, s.cuda(), window=128)
    with pytest.raises(ValueError):
        sa.sinkattn_prefill_host(q.transpose(1, 2).contiguous().transpose(1, 2), k, v, s.cuda(),
                                 window=128)
    with pytest.raises(sa.SinkAttnError):  # a chunk that is not a multiple of 128
        sa.sinkattn_prefill_host(pinned(q), pinned(k), pinned(v), s.cuda(), window=128, chunk=100)


def test_host_prefill_full_size_sampled():
    """The headline workload (SWA, B=2, L=32768, 64 Q / 8 KV) through the host call in the
    chunking the benchmark's end-to-end figure uses, on sampled rows."""
    w = W.SWA_PREFILL
    d = W.prefill_inputs(w, device="cuda")
    hq, hk, hv = (pinned(d[x].cpu()) for x in ("q", "k", "v"))
    o, lse = sa.sinkattn_prefill_host(hq, hk, hv, d["sink"], window=w.window)
    torch.cuda.synchronize()
    rows = sample_rows(w.B, w.L, seed=w.seed + 1, extra=12)
    ro, rl, _ = oracle.prefill(hq, hk, hv, d["sink"].cpu(), W.SCALE, w.window, rows=rows)
    idx_b = torch.tensor([r[0] for r in rows])
    idx_i = torch.tensor([r[1] for r in rows])
    assert_close(o[idx_b, idx_i], ro, lse.permute(0, 2, 1)[idx_b, idx_i], rl, w.name + " host")
    assert sa.sinkattn_take_device_error() == 0
