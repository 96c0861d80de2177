// C ABI of the sink-attention library: argument validation, TMA descriptor set-up, split-KV
// sizing and kernel launches. Everything is enqueued on the caller's stream; the library
// allocates no device memory. The kernels live in prefill_kernels.cuh / decode_kernels.cuh;
// the whole library is this one translation unit.
#include <algorithm>
#include <math.h>
#include <mutex>

#include "sinkattn.h"

#include "common.cuh"
#include "decode_kernels.cuh"
#include "decode_fp8_kernels.cuh"
#include "decode_fp8_tma_kernels.cuh"
#include "decode_tma_kernels.cuh"
#include "decode_umma_kernels.cuh"
#include "decode_ring_kernels.cuh"
#include "decode_ring_umma_kernels.cuh"
#include "backward_kernels.cuh"
#include "internal.h"
#include "prefill_kernels.cuh"
#include "prefill_wide_kernels.cuh"
#include "rope_kernels.cuh"
#include "swa_kernels.cuh"

namespace {

using namespace sinkattn;

constexpr int kDQ = 192, kDV = 128;
constexpr int kNumSMs = 148;      // B200; only used to size the split-KV grid
constexpr int kMinSpanKeys = 512; // below this a key span is not split further

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// element strides of bf16 tensors: positive and a whole number of 16-byte units
bool stride_ok(int64_t s) { return s > 0 && (s % 8) == 0; }
// byte strides (one-byte elements): positive multiples of 16
bool stride_ok_bytes(int64_t s) { return s > 0 && (s % 16) == 0; }

// 4-D bf16 map over [B, tokens, heads, d] given as dims {d, heads, tokens, B}; box
// {64, box_heads, box_tokens, 1}, 128-byte swizzle, zero fill outside the tensor.
int make_map(CUtensorMap *map, const void *base, int d, int heads, int tokens, int B,
             int64_t s_head, int64_t s_tok, int64_t s_b, int box_heads, int box_tokens)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return SINKATTN_ERR_CUDA;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)tokens,
                                (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)s_head * 2, (cuuint64_t)s_tok * 2,
                                   (cuuint64_t)s_b * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SINKATTN_OK : SINKATTN_ERR_INVALID_ARG;
}

// 4-D map over one-byte codes [blocks, tokens, heads, d] given as dims {d, heads, tokens,
// blocks}, strides in bytes; box {64, 1, box_tokens, 1} (64-byte rows), 64-byte swizzle, zero
// fill outside the tensor.
int make_map_u8(CUtensorMap *map, const void *base, int d, int heads, int tokens, int blocks,
                int64_t s_head, int64_t s_tok, int64_t s_blk, int box_tokens)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return SINKATTN_ERR_CUDA;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)tokens,
                                (cuuint64_t)blocks};
    const cuuint64_t strides[3] = {(cuuint64_t)s_head, (cuuint64_t)s_tok, (cuuint64_t)s_blk};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_tokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SINKATTN_OK : SINKATTN_ERR_INVALID_ARG;
}

int validate_prefill(const sinkattn_prefill_args *a)
{
    if (!a)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->L < 0 || a->Hq <= 0 || a->Hkv <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->dq != kDQ || a->dv != kDV || a->Hq % a->Hkv != 0)
        return SINKATTN_ERR_UNSUPPORTED;
    if (!isfinite(a->scale) || !(a->scale > 0.f))
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B == 0 || a->L == 0)
        return SINKATTN_OK;
    if (!a->q || !a->k || !a->v || !a->o)
        return SINKATTN_ERR_INVALID_ARG;
    if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->o))
        return SINKATTN_ERR_ALIGNMENT;
    const int64_t s[12] = {a->q_sb, a->q_sl, a->q_sh, a->k_sb, a->k_sl, a->k_sh,
                           a->v_sb, a->v_sl, a->v_sh, a->o_sb, a->o_sl, a->o_sh};
    for (int i = 0; i < 12; ++i) {
        if (s[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if (!stride_ok(s[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    return SINKATTN_OK;
}

// Per-device figures used to shape grids (cached; a device's properties do not change).
struct DeviceInfo {
    int sms = 0, smem_optin = 0;
};

int device_info(DeviceInfo *out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return SINKATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && cache[dev].sms > 0) {
        *out = cache[dev];
        return SINKATTN_OK;
    }
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
        return SINKATTN_ERR_CUDA;
    if (dev >= 0 && dev < 64)
        cache[dev] = d;
    *out = d;
    return SINKATTN_OK;
}

// SWA prefill with the GQA group packed into the MMA rows: possible when G divides 128 and the
// span of P + W - 1 keys (P = 128 / G positions) fits one MMA (<= 256) and shared memory.
int try_prefill_swa_packed(const sinkattn_prefill_args *a, int window, void *stream, bool *done,
                           const sinkattn_rope_spec *rope = nullptr)
{
    *done = false;
    const int G = a->Hq / a->Hkv;
    if (128 % G != 0)
        return SINKATTN_OK;
    const int P = 128 / G;
    if (P % 16 != 0) // the K / V rings advance in 16-key chunks
        return SINKATTN_OK;
    const int64_t span = (int64_t)P + window - 1;
    const int NS = (int)((span + 15) / 16 * 16);
    if (span > 256)
        return SINKATTN_OK;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SINKATTN_OK)
        return st;
    if (swa_packed_smem_bytes(NS, P) > di.smem_optin)
        return SINKATTN_OK;
    CUtensorMap tq, tk, tv, tkc, tvc;
    if ((st = make_map(&tq, a->q, kDQ, a->Hq, a->L, a->B, a->q_sh, a->q_sl, a->q_sb, G, P)))
        return st;
    if ((st = make_map(&tkc, a->k, kDQ, a->Hkv, a->L, a->B, a->k_sh, a->k_sl, a->k_sb, 1, 16)))
        return st;
    if ((st = make_map(&tvc, a->v, kDV, a->Hkv, a->L, a->B, a->v_sh, a->v_sl, a->v_sb, 1, 16)))
        return st;
    if ((st = make_map(&tk, a->k, kDQ, a->Hkv, a->L, a->B, a->k_sh, a->k_sl, a->k_sb, 1, NS)))
        return st;
    if ((st = make_map(&tv, a->v, kDV, a->Hkv, a->L, a->B, a->v_sh, a->v_sl, a->v_sb, 1, NS)))
        return st;
    SwaParams p;
    p.B = a->B;
    p.L = a->L;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.G = G;
    p.P = P;
    p.W = window;
    p.NS = NS;
    p.n_pblk = (a->L + P - 1) / P;
    const int64_t items = (int64_t)a->B * a->Hkv * p.n_pblk;
    if (items > 0x7fffffff)
        return SINKATTN_ERR_UNSUPPORTED;
    p.n_items = (int)items;
    p.scale_log2 = a->scale * kLog2e;
    p.sink = a->sink;
    p.o = a->o;
    p.o_sb = a->o_sb;
    p.o_sl = a->o_sl;
    p.o_sh = a->o_sh;
    p.lse = a->lse;
    p.rope = rope ? 1 : 0;
    p.rope_half = rope ? rope->rope_dim / 2 : 8;
    p.out_mul = rope ? rope->v_scale : 1.f;
    p.pos_base = rope ? rope->pos_base : nullptr;
    p.pos0 = rope ? rope->pos0 : 0;
    for (int i = 0; i < kRopeFusedMaxHalf; ++i)
        p.inv_freq[i] = (rope && i < p.rope_half) ? pow(rope->theta, -2.0 * i / (2.0 * p.rope_half)) : 0.0;
    const int grid = (int)(items < di.sms ? items : di.sms);
    const cudaError_t e =
        launch_prefill_swa_packed(tq, tk, tv, tkc, tvc, p, grid, (cudaStream_t)stream);
    *done = true;
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

// Checks of a paged prefix (sinkattn_prefill_chunk_paged).
int validate_paged_prefix(const sinkattn_paged_kv *kv, int prefix)
{
    if (!kv || !kv->k_pages || !kv->v_pages || !kv->page_table)
        return SINKATTN_ERR_INVALID_ARG;
    if (kv->page_size <= 0 || kv->max_pages <= 0 || kv->num_pages <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (prefix % 128 != 0 || kv->page_size % 128 != 0)
        return SINKATTN_ERR_UNSUPPORTED;
    if ((int64_t)prefix > (int64_t)kv->max_pages * kv->page_size)
        return SINKATTN_ERR_INVALID_ARG;
    if (!aligned16(kv->k_pages) || !aligned16(kv->v_pages))
        return SINKATTN_ERR_ALIGNMENT;
    const int64_t s[6] = {kv->kp_sb, kv->kp_ss, kv->kp_sh, kv->vp_sb, kv->vp_ss, kv->vp_sh};
    for (int i = 0; i < 6; ++i) {
        if (s[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if (!stride_ok(s[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    return SINKATTN_OK;
}

// Prefill of the L query rows at positions prefix .. prefix + L - 1 against keys 0 .. prefix +
// L - 1 (prefix = 0: whole sequences). With `paged`, keys below the prefix come from its pool
// and args->k / v hold the chunk's L positions only.
int run_prefill(const sinkattn_prefill_args *a, int window, int prefix, void *stream,
                const sinkattn_paged_kv *paged = nullptr)
{
    int st = validate_prefill(a);
    if (st != SINKATTN_OK)
        return st;
    if (paged && (st = validate_paged_prefix(paged, prefix)) != SINKATTN_OK)
        return st;
    if (a->B == 0 || a->L == 0)
        return SINKATTN_OK;
    if (prefix < 0 || (int64_t)prefix + a->L > 0x7fffffff)
        return SINKATTN_ERR_INVALID_ARG;
    if (window > 0 && prefix == 0) {
        bool done = false;
        st = try_prefill_swa_packed(a, window, stream, &done);
        if (st != SINKATTN_OK || done)
            return st;
    }
    const int n_kv = paged ? a->L : prefix + a->L;
    CUtensorMap tq, tk, tv, tkp, tvp;
    if ((st = make_map(&tq, a->q, kDQ, a->Hq, a->L, a->B, a->q_sh, a->q_sl, a->q_sb, 1, 128)))
        return st;
    if ((st = make_map(&tk, a->k, kDQ, a->Hkv, n_kv, a->B, a->k_sh, a->k_sl, a->k_sb, 1, 128)))
        return st;
    if ((st = make_map(&tv, a->v, kDV, a->Hkv, n_kv, a->B, a->v_sh, a->v_sl, a->v_sb, 1, 128)))
        return st;
    if (paged) {
        if ((st = make_map(&tkp, paged->k_pages, kDQ, a->Hkv, paged->page_size, paged->num_pages,
                           paged->kp_sh, paged->kp_ss, paged->kp_sb, 1, 128)))
            return st;
        if ((st = make_map(&tvp, paged->v_pages, kDV, a->Hkv, paged->page_size, paged->num_pages,
                           paged->vp_sh, paged->vp_ss, paged->vp_sb, 1, 128)))
            return st;
    } else {
        tkp = tk;
        tvp = tv;
    }
    PrefillParams p;
    p.B = a->B;
    p.L = a->L;
    p.q_off = prefix;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.G = a->Hq / a->Hkv;
    p.window = window;
    p.n_qtiles = (a->L + 127) / 128;
    p.scale_log2 = a->scale * kLog2e;
    p.sink = a->sink;
    p.o = a->o;
    p.o_sb = a->o_sb;
    p.o_sl = a->o_sl;
    p.o_sh = a->o_sh;
    p.lse = a->lse;
    p.paged = paged ? 1 : 0;
    p.page_table = paged ? paged->page_table : nullptr;
    p.page_size = paged ? paged->page_size : 0;
    p.max_pages = paged ? paged->max_pages : 0;
    p.num_pages = paged ? paged->num_pages : 0;
    const cudaError_t e = (window == 0)
                              ? launch_prefill_wide(tq, tk, tv, tkp, tvp, p, (cudaStream_t)stream)
                              : launch_prefill_band(tq, tk, tv, tkp, tvp, p, (cudaStream_t)stream);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

// ---- prefill with host-resident inputs and outputs ---------------------------------------------
// The sequences stream through the device in chunks of `chunk` positions. Copies in (Q, K, V of
// a chunk), the chunk's prefill and copies out (its O and LSE) run on three streams ordered by
// events, with two Q / O / LSE buffers, so while chunk c computes, chunk c + 1 comes in and
// chunk c - 1 goes out: the two PCIe directions run at the same time. K and V stay on the device
// for the whole call (later chunks read earlier keys).
struct HostLayout {
    int64_t chunk, n_chunks;
    int64_t qrow, krow, vrow, orow;       // bytes per position
    size_t off_k, off_v, off_q[2], off_o[2], off_lse[2], total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

HostLayout host_layout(const sinkattn_prefill_args *a, int chunk)
{
    HostLayout h;
    h.chunk = chunk;
    h.n_chunks = (a->L + (int64_t)chunk - 1) / chunk;
    h.qrow = (int64_t)a->Hq * kDQ * 2;
    h.krow = (int64_t)a->Hkv * kDQ * 2;
    h.vrow = (int64_t)a->Hkv * kDV * 2;
    h.orow = (int64_t)a->Hq * kDV * 2;
    size_t off = 0;
    h.off_k = off;
    off += align256((size_t)a->B * a->L * h.krow);
    h.off_v = off;
    off += align256((size_t)a->B * a->L * h.vrow);
    for (int x = 0; x < 2; ++x) {
        h.off_q[x] = off;
        off += align256((size_t)a->B * chunk * h.qrow);
        h.off_o[x] = off;
        off += align256((size_t)a->B * chunk * h.orow);
        h.off_lse[x] = off;
        off += align256((size_t)a->B * a->Hq * chunk * 4);
    }
    h.total = off;
    return h;
}

// Dense [B, L, H, d] layouts only (the host buffers are copied in whole rows).
int validate_host_prefill(const sinkattn_prefill_args *a, int window, int chunk)
{
    int st = validate_prefill(a);
    if (st != SINKATTN_OK)
        return st;
    if (window < 0 || chunk <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (chunk % 128 != 0)
        return SINKATTN_ERR_UNSUPPORTED;
    if (a->B == 0 || a->L == 0)
        return SINKATTN_OK;
    const int64_t qh = kDQ, ql = (int64_t)a->Hq * kDQ, kl = (int64_t)a->Hkv * kDQ;
    const int64_t vl = (int64_t)a->Hkv * kDV, ol = (int64_t)a->Hq * kDV;
    const bool dense = a->q_sh == qh && a->q_sl == ql && a->q_sb == ql * a->L && a->k_sh == kDQ &&
                       a->k_sl == kl && a->k_sb == kl * a->L && a->v_sh == kDV && a->v_sl == vl &&
                       a->v_sb == vl * a->L && a->o_sh == kDV && a->o_sl == ol &&
                       a->o_sb == ol * a->L;
    return dense ? SINKATTN_OK : SINKATTN_ERR_UNSUPPORTED;
}

int run_prefill_host(const sinkattn_prefill_args *a, int window, int chunk, void *ws,
                     size_t ws_bytes, void *stream)
{
    int st = validate_host_prefill(a, window, chunk);
    if (st != SINKATTN_OK)
        return st;
    if (a->B == 0 || a->L == 0)
        return SINKATTN_OK;
    const HostLayout h = host_layout(a, chunk);
    if (!ws || ws_bytes < h.total)
        return !ws ? SINKATTN_ERR_INVALID_ARG : SINKATTN_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws))
        return SINKATTN_ERR_ALIGNMENT;
    uint8_t *w = static_cast<uint8_t *>(ws);
    const cudaStream_t s_comp = (cudaStream_t)stream;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
    cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess)
        e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
    if (e == cudaSuccess)
        e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
    for (int x = 0; x < 2 && e == cudaSuccess; ++x) {
        e = cudaEventCreateWithFlags(&ev_in[x], cudaEventDisableTiming);
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(&ev_comp[x], cudaEventDisableTiming);
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(&ev_out[x], cudaEventDisableTiming);
    }
    // the copies start after the caller's earlier work on `stream`
    if (e == cudaSuccess)
        e = cudaEventRecord(ev_start, s_comp);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(s_in, ev_start, 0);
    if (e == cudaSuccess)
        e = cudaStreamWaitEvent(s_out, ev_start, 0);
    const uint8_t *hq = static_cast<const uint8_t *>(a->q), *hk = static_cast<const uint8_t *>(a->k);
    const uint8_t *hv = static_cast<const uint8_t *>(a->v);
    uint8_t *ho = static_cast<uint8_t *>(a->o);
    uint8_t *hl = reinterpret_cast<uint8_t *>(a->lse);
    for (int64_t c = 0; c < h.n_chunks && e == cudaSuccess && st == SINKATTN_OK; ++c) {
        const int x = (int)(c & 1);
        const int64_t c0 = c * h.chunk, lc = std::min<int64_t>(h.chunk, a->L - c0);
        // in: Q of the chunk into buffer x (free once chunk c - 2 has computed), K and V rows
        if (c >= 2)
            e = cudaStreamWaitEvent(s_in, ev_comp[x], 0);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(w + h.off_q[x], h.chunk * h.qrow, hq + c0 * h.qrow, a->L * h.qrow,
                                  lc * h.qrow, a->B, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(w + h.off_k + c0 * h.krow, a->L * h.krow, hk + c0 * h.krow,
                                  a->L * h.krow, lc * h.krow, a->B, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(w + h.off_v + c0 * h.vrow, a->L * h.vrow, hv + c0 * h.vrow,
                                  a->L * h.vrow, lc * h.vrow, a->B, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess)
            e = cudaEventRecord(ev_in[x], s_in);
        // compute: the chunk's rows against keys 0 .. c0 + lc - 1, into O / LSE buffer x (free
        // once chunk c - 2 has gone out)
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(s_comp, ev_in[x], 0);
        if (e == cudaSuccess && c >= 2)
            e = cudaStreamWaitEvent(s_comp, ev_out[x], 0);
        if (e != cudaSuccess)
            break;
        sinkattn_prefill_args ac = *a;
        ac.q = w + h.off_q[x];
        ac.k = w + h.off_k;
        ac.v = w + h.off_v;
        ac.o = w + h.off_o[x];
        ac.lse = a->lse ? reinterpret_cast<float *>(w + h.off_lse[x]) : nullptr;
        ac.L = (int32_t)lc;
        ac.q_sb = h.chunk * (h.qrow / 2);
        ac.o_sb = h.chunk * (h.orow / 2);
        st = run_prefill(&ac, window, (int)c0, s_comp);
        if (st != SINKATTN_OK)
            break;
        e = cudaEventRecord(ev_comp[x], s_comp);
        // out: O rows and the LSE runs of every (sequence, head)
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(s_out, ev_comp[x], 0);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(ho + c0 * h.orow, a->L * h.orow, w + h.off_o[x], h.chunk * h.orow,
                                  lc * h.orow, a->B, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess && a->lse)
            e = cudaMemcpy2DAsync(hl + c0 * 4, (size_t)a->L * 4, w + h.off_lse[x], (size_t)lc * 4,
                                  lc * 4, (size_t)a->B * a->Hq, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess)
            e = cudaEventRecord(ev_out[x], s_out);
    }
    // the caller's stream completes only after the last copy out
    if (e == cudaSuccess && st == SINKATTN_OK)
        e = cudaStreamWaitEvent(s_comp, ev_out[(h.n_chunks - 1) & 1], 0);
    if (e == cudaSuccess && st == SINKATTN_OK && h.n_chunks >= 2)
        e = cudaStreamWaitEvent(s_comp, ev_out[h.n_chunks & 1], 0);
    // streams and events are released once their pending work is done
    for (int x = 0; x < 2; ++x) {
        if (ev_in[x])
            cudaEventDestroy(ev_in[x]);
        if (ev_comp[x])
            cudaEventDestroy(ev_comp[x]);
        if (ev_out[x])
            cudaEventDestroy(ev_out[x]);
    }
    if (ev_start)
        cudaEventDestroy(ev_start);
    if (s_in)
        cudaStreamDestroy(s_in);
    if (s_out)
        cudaStreamDestroy(s_out);
    if (st != SINKATTN_OK)
        return st;
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

// ---- prefill backward --------------------------------------------------------------------------
int validate_backward(const sinkattn_backward_args *a)
{
    if (!a)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->L < 0 || a->Hq <= 0 || a->Hkv <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->d_qk != kDQ || a->d_v != kDV || a->Hq % a->Hkv != 0)
        return SINKATTN_ERR_UNSUPPORTED;
    if (!isfinite(a->scale) || !(a->scale > 0.f))
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B == 0 || a->L == 0)
        return SINKATTN_OK;
    const void *ptrs[9] = {a->q, a->k, a->v, a->o, a->dout, a->lse, a->dq, a->dk, a->dv};
    for (int i = 0; i < 9; ++i) {
        if (!ptrs[i])
            return SINKATTN_ERR_INVALID_ARG;
        if (!aligned16(ptrs[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    const int64_t sb[15] = {a->q_sb, a->q_sl, a->q_sh, a->k_sb, a->k_sl, a->k_sh, a->v_sb, a->v_sl,
                            a->v_sh, a->o_sb, a->o_sl, a->o_sh, a->do_sb, a->do_sl, a->do_sh};
    for (int i = 0; i < 15; ++i) {
        if (sb[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if (!stride_ok(sb[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    // fp32 gradients: element strides, positive multiples of 4 (16 bytes)
    const int64_t sf[9] = {a->dq_sb, a->dq_sl, a->dq_sh, a->dk_sb, a->dk_sl, a->dk_sh,
                           a->dv_sb, a->dv_sl, a->dv_sh};
    for (int i = 0; i < 9; ++i) {
        if (sf[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if (sf[i] % 4 != 0)
            return SINKATTN_ERR_ALIGNMENT;
    }
    if (a->dsink && !aligned16(a->dsink))
        return SINKATTN_ERR_ALIGNMENT;
    if ((int64_t)a->B * a->Hq * a->L > ((int64_t)1 << 40))
        return SINKATTN_ERR_UNSUPPORTED;
    return SINKATTN_OK;
}

size_t backward_workspace_bytes(const sinkattn_backward_args *a)
{
    return (size_t)a->B * a->Hq * a->L * sizeof(float); // delta
}

// ---- decode sizing ----------------------------------------------------------------------------
struct Split {
    int splits, chunk;
};

// Longest key sequence a (b, kv head) unit can have: used cached tokens + the T new ones.
int64_t max_unit_keys(const sinkattn_decode_args *a)
{
    int64_t cached = (a->kind == SINKATTN_KV_RING) ? a->ring_cap : a->max_ctx;
    if (a->window > 0)
        cached = cached < a->window - 1 ? cached : a->window - 1;
    return cached + a->T;
}

Split plan_split(const sinkattn_decode_args *a)
{
    const int64_t n = max_unit_keys(a);
    const int64_t units = (int64_t)a->B * a->Hkv;
    // about 8 spans per SM (shorter spans even out ragged lengths but each CTA's start and
    // epilogue cost more than that gains)
    int64_t splits = (kNumSMs * 8 + units - 1) / units;
    const int64_t by_len = (n + kMinSpanKeys - 1) / kMinSpanKeys;
    if (splits > by_len)
        splits = by_len;
    if (splits < 1)
        splits = 1;
    int64_t chunk = (n + splits - 1) / splits;
    chunk = (chunk + 127) / 128 * 128; // whole tiles of every decode kernel (64 or 128 keys)
    splits = (n + chunk - 1) / chunk;
    return Split{(int)splits, (int)chunk};
}

size_t workspace_bytes(const sinkattn_decode_args *a, const Split &s)
{
    if (s.splits <= 1)
        return 0;
    const size_t rows = (size_t)a->B * a->Hkv * s.splits * (size_t)(a->T * (a->Hq / a->Hkv));
    return rows * (kDV + 4) * sizeof(float);
}

// The sizes and layout kinds that fix the split plan and hence the workspace size.
int validate_decode_shape(const sinkattn_decode_args *a)
{
    if (!a)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind != SINKATTN_KV_RING && a->kind != SINKATTN_KV_CONTIG && a->kind != SINKATTN_KV_PAGED)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->Hq <= 0 || a->Hkv <= 0 || a->window < 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->dq != kDQ || a->dv != kDV || a->Hq % a->Hkv != 0 || a->T > 4)
        return SINKATTN_ERR_UNSUPPORTED;
    const int G = a->Hq / a->Hkv;
    if (G > 16 || a->T * G > 64)
        return SINKATTN_ERR_UNSUPPORTED;
    if (a->kind == SINKATTN_KV_RING && a->ring_cap <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind != SINKATTN_KV_RING && a->max_ctx < 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind == SINKATTN_KV_PAGED &&
        (a->page_size <= 0 || a->max_pages <= 0 ||
         (int64_t)a->max_ctx > (int64_t)a->max_pages * a->page_size))
        return SINKATTN_ERR_INVALID_ARG;
    return SINKATTN_OK;
}

// The cache element type and, for FP8, its two scales (finite, > 0).
int kv_dtype_check(const sinkattn_decode_args *a)
{
    if (a->kv_dtype == SINKATTN_KV_BF16)
        return SINKATTN_OK;
    if (a->kv_dtype != SINKATTN_KV_FP8_E4M3)
        return SINKATTN_ERR_INVALID_ARG;
    if (!isfinite(a->k_scale) || !(a->k_scale > 0.f) || !isfinite(a->v_scale) ||
        !(a->v_scale > 0.f))
        return SINKATTN_ERR_INVALID_ARG;
    return SINKATTN_OK;
}

int validate_decode(const sinkattn_decode_args *a)
{
    if (!a)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind != SINKATTN_KV_RING && a->kind != SINKATTN_KV_CONTIG && a->kind != SINKATTN_KV_PAGED)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->Hq <= 0 || a->Hkv <= 0 || a->window < 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->dq != kDQ || a->dv != kDV || a->Hq % a->Hkv != 0 || a->T > 4)
        return SINKATTN_ERR_UNSUPPORTED;
    const int G = a->Hq / a->Hkv;
    if (G > 16 || a->T * G > 64)
        return SINKATTN_ERR_UNSUPPORTED;
    if (!isfinite(a->scale) || !(a->scale > 0.f))
        return SINKATTN_ERR_INVALID_ARG;
    if (kv_dtype_check(a) != SINKATTN_OK)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind == SINKATTN_KV_RING) {
        if (a->ring_cap <= 0 || !a->ring_head || !a->ring_len)
            return SINKATTN_ERR_INVALID_ARG;
    } else {
        if (a->max_ctx < 0 || !a->ctx_len)
            return SINKATTN_ERR_INVALID_ARG;
        if (a->kind == SINKATTN_KV_PAGED) {
            if (a->page_size <= 0 || a->max_pages <= 0 || a->num_pages <= 0 || !a->page_table)
                return SINKATTN_ERR_INVALID_ARG;
            if ((int64_t)a->max_ctx > (int64_t)a->max_pages * a->page_size)
                return SINKATTN_ERR_INVALID_ARG;
        }
    }
    if (a->B == 0 || a->T == 0)
        return SINKATTN_OK;
    if (!a->q || !a->k_new || !a->v_new || !a->o || !a->k_cache || !a->v_cache)
        return SINKATTN_ERR_INVALID_ARG;
    const void *ptrs[6] = {a->q, a->k_new, a->v_new, a->k_cache, a->v_cache, a->o};
    for (int i = 0; i < 6; ++i)
        if (!aligned16(ptrs[i]))
            return SINKATTN_ERR_ALIGNMENT;
    const int64_t s[15] = {a->q_sb,  a->q_st,  a->q_sh,  a->kn_sb, a->kn_st,
                           a->kn_sh, a->vn_sb, a->vn_st, a->vn_sh, a->kc_sb,
                           a->kc_ss, a->kc_sh, a->vc_sb, a->vc_ss, a->vc_sh};
    const bool fp8 = a->kv_dtype == SINKATTN_KV_FP8_E4M3;
    for (int i = 0; i < 15; ++i) {
        if (s[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        // cache strides (the last six) of an FP8 cache count bytes
        if ((fp8 && i >= 9) ? !stride_ok_bytes(s[i]) : !stride_ok(s[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    const int64_t so[3] = {a->o_sb, a->o_st, a->o_sh};
    for (int i = 0; i < 3; ++i) {
        if (so[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if (!stride_ok(so[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    return SINKATTN_OK;
}

void fill_decode_params(DecodeParams &p, const sinkattn_decode_args *a, const Split &s, void *ws)
{
    p.kind = a->kind;
    p.B = a->B;
    p.T = a->T;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.G = a->Hq / a->Hkv;
    p.R = a->T * p.G;
    p.MT = (p.R + 15) / 16;
    p.window = a->window;
    p.splits = s.splits;
    p.chunk = s.chunk;
    p.fp8 = a->kv_dtype == SINKATTN_KV_FP8_E4M3;
    p.k_scale = p.fp8 ? a->k_scale : 1.f;
    p.v_scale = p.fp8 ? a->v_scale : 1.f;
    p.k8 = static_cast<const uint8_t *>(a->k_cache);
    p.v8 = static_cast<const uint8_t *>(a->v_cache);
    // an FP8 cache's logits are scale * k_scale * <q, e(c)>
    p.scale_log2 = a->scale * kLog2e * p.k_scale;
    p.sink = a->sink;
    p.q = static_cast<const uint16_t *>(a->q);
    p.k_new = static_cast<const uint16_t *>(a->k_new);
    p.v_new = static_cast<const uint16_t *>(a->v_new);
    p.k_cache = static_cast<const uint16_t *>(a->k_cache);
    p.v_cache = static_cast<const uint16_t *>(a->v_cache);
    p.q_sb = a->q_sb;
    p.q_st = a->q_st;
    p.q_sh = a->q_sh;
    p.kn_sb = a->kn_sb;
    p.kn_st = a->kn_st;
    p.kn_sh = a->kn_sh;
    p.vn_sb = a->vn_sb;
    p.vn_st = a->vn_st;
    p.vn_sh = a->vn_sh;
    p.kc_sb = a->kc_sb;
    p.kc_ss = a->kc_ss;
    p.kc_sh = a->kc_sh;
    p.vc_sb = a->vc_sb;
    p.vc_ss = a->vc_ss;
    p.vc_sh = a->vc_sh;
    p.ring_head = a->ring_head;
    p.ring_len = a->ring_len;
    p.ring_cap = a->ring_cap;
    p.ctx_len = a->ctx_len;
    p.max_ctx = a->max_ctx;
    p.page_table = a->page_table;
    p.page_size = a->page_size;
    p.max_pages = a->max_pages;
    p.num_pages = a->num_pages;
    p.o = static_cast<uint16_t *>(a->o);
    p.o_sb = a->o_sb;
    p.o_st = a->o_st;
    p.o_sh = a->o_sh;
    p.lse = a->lse;
    const size_t rows = (size_t)a->B * a->Hkv * s.splits * (size_t)p.R;
    p.ws_o = static_cast<float *>(ws);
    p.ws_ml = ws ? static_cast<float *>(ws) + rows * kDV : nullptr;
}

// ---- decode without a caller workspace ------------------------------------------------------
// Some callers hand this library only their input and output buffers and have no device
// allocator to lend it: a plugin host whose interface passes fixed buffers, or a serving loop
// whose device memory is all reserved up front, where a cudaMalloc on the decode path would
// block the device or fail under memory pressure. sinkattn_decode_noalloc serves them with a
// split-KV workspace that is a fixed array in the library's own device memory.
constexpr size_t kNoAllocWorkspaceBytes = SINKATTN_NOALLOC_WORKSPACE_BYTES;
static __device__ __align__(256) float g_noalloc_workspace[kNoAllocWorkspaceBytes / sizeof(float)];

std::mutex g_noalloc_mutex;
constexpr int kMaxCachedDevices = 256;
struct NoAllocAddress {
    unsigned long long ctx; // context the address belongs to (0: none cached)
    void *ptr;
};
NoAllocAddress g_noalloc_addr[kMaxCachedDevices] = {};

// Device address of g_noalloc_workspace in the current device's context. Host code cannot use
// the array's name as a device pointer, so the address is looked up with cudaGetSymbolAddress
// the first time a context needs it (with its device current) and kept per device together
// with that context's id: after a device reset the new context's module is loaded afresh, its
// id differs, and the address is looked up again.
cudaError_t noalloc_workspace_ptr(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const bool cached = dev >= 0 && dev < kMaxCachedDevices;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const unsigned long long ctx = current_context_id();
    if (cached && ctx != 0 && g_noalloc_addr[dev].ctx == ctx) {
        *out = g_noalloc_addr[dev].ptr;
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
    if (e != cudaSuccess)
        return e;
    if (cached)
        g_noalloc_addr[dev] = NoAllocAddress{current_context_id(), p};
    *out = p;
    return cudaSuccess;
}

// The split-KV TMA-fed decode kernels take whole 64-key tiles: contiguous caches, and paged
// caches whose pages hold a multiple of 64 tokens (without a window, so tiles stay page-aligned).
// Rings of 128 slots on 8-head groups with up to 4 query tokens (the model's SWA layers, decode
// and verify) go to the tcgen05 ring kernel; other rings of up to 16 rows per item to the
// mma.sync ring kernel; the remaining rings and other page sizes use the cp.async kernel.
bool decode_tma_ok(const sinkattn_decode_args *a, const DecodeParams &)
{
    if (a->kind == SINKATTN_KV_CONTIG)
        return true;
    if (a->kind == SINKATTN_KV_PAGED)
        return a->window == 0 && a->page_size % 64 == 0;
    return false;
}

int run_decode(const sinkattn_decode_args *a, const DecodeParams &p, void *stream)
{
    cudaError_t e;
    if (p.fp8) {
        // whole 64-key tiles of codes by TMA: contiguous caches, pages of a multiple of 64
        // tokens without a window, rings of a multiple of 64 slots in one span; the rest (and a
        // cache the encoder rejects, e.g. an empty one) take the cp.async kernel
        const bool tiles = a->kind == SINKATTN_KV_CONTIG ||
                           (a->kind == SINKATTN_KV_PAGED && a->window == 0 && a->page_size % 64 == 0) ||
                           (a->kind == SINKATTN_KV_RING && a->ring_cap % 64 == 0 && p.splits == 1);
        const int rows = a->kind == SINKATTN_KV_RING ? a->ring_cap
                         : a->kind == SINKATTN_KV_CONTIG ? a->max_ctx
                                                         : a->page_size;
        const int blocks = a->kind == SINKATTN_KV_PAGED ? a->num_pages : a->B;
        CUtensorMap kc, vc;
        if (tiles && rows > 0 &&
            !make_map_u8(&kc, a->k_cache, kDQ, a->Hkv, rows, blocks, a->kc_sh, a->kc_ss, a->kc_sb, 64) &&
            !make_map_u8(&vc, a->v_cache, kDV, a->Hkv, rows, blocks, a->vc_sh, a->vc_ss, a->vc_sb, 64))
            e = launch_decode_fp8_tma(kc, vc, p, (cudaStream_t)stream);
        else
            e = launch_decode_fp8(p, (cudaStream_t)stream);
        return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
    }
    if (a->kind == SINKATTN_KV_RING && a->ring_cap == rv::CAP && p.G == rv::G && a->T <= rv::TMAX &&
        p.splits == 1) {
        // a unit (sequence, KV head) per MMA pass: S = Q K^T over the 128 slots and the new
        // tokens, P V from TMEM
        CUtensorMap q, kc, vc, kn, vn;
        DeviceInfo di;
        int st = device_info(&di);
        if (st != SINKATTN_OK)
            return st;
        if (!make_map(&q, a->q, kDQ, a->Hq, a->T, a->B, a->q_sh, a->q_st, a->q_sb, rv::G, a->T) &&
            !make_map(&kc, a->k_cache, kDQ, a->Hkv, rv::CAP, a->B, a->kc_sh, a->kc_ss, a->kc_sb, 1, rv::CAP) &&
            !make_map(&vc, a->v_cache, kDV, a->Hkv, rv::CAP, a->B, a->vc_sh, a->vc_ss, a->vc_sb, 1, rv::CAP) &&
            !make_map(&kn, a->k_new, kDQ, a->Hkv, a->T, a->B, a->kn_sh, a->kn_st, a->kn_sb, 1, 16) &&
            !make_map(&vn, a->v_new, kDV, a->Hkv, a->T, a->B, a->vn_sh, a->vn_st, a->vn_sb, 1, 16)) {
            e = launch_decode_ring_umma(q, kc, vc, kn, vn, p, di.sms, (cudaStream_t)stream);
            return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
        }
    }
    if (a->kind == SINKATTN_KV_RING && p.R <= 16 && a->ring_cap % 32 == 0 && p.splits == 1) {
        // a ring item per warp, streamed in 32-key chunks
        CUtensorMap kc, vc, kn, vn;
        DeviceInfo di;
        int st = device_info(&di);
        if (st != SINKATTN_OK)
            return st;
        if (!make_map(&kc, a->k_cache, kDQ, a->Hkv, a->ring_cap, a->B, a->kc_sh, a->kc_ss, a->kc_sb, 1, 32) &&
            !make_map(&vc, a->v_cache, kDV, a->Hkv, a->ring_cap, a->B, a->vc_sh, a->vc_ss, a->vc_sb, 1, 32) &&
            !make_map(&kn, a->k_new, kDQ, a->Hkv, a->T, a->B, a->kn_sh, a->kn_st, a->kn_sb, 1, 32) &&
            !make_map(&vn, a->v_new, kDV, a->Hkv, a->T, a->B, a->vn_sh, a->vn_st, a->vn_sb, 1, 32)) {
            e = launch_decode_ring(kc, vc, kn, vn, p, di.sms, (cudaStream_t)stream);
            return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
        }
    }
    if (decode_tma_ok(a, p)) {
        const int rows = a->kind == SINKATTN_KV_CONTIG ? a->max_ctx : a->page_size;
        const int blocks = a->kind == SINKATTN_KV_PAGED ? a->num_pages : a->B;
        // tcgen05 kernel: blocks of more than 16 query rows over 128-key tiles (pages of a
        // multiple of 128 tokens); the mma.sync TMA kernel: the rest, over 64-key tiles
        const bool umma = p.R > 16 && (a->kind != SINKATTN_KV_PAGED || a->page_size % 128 == 0);
        const int new_rows = umma ? 16 : 64;
        const int box = umma ? 128 : 64;
        CUtensorMap kc, vc, kn, vn, q;
        // a cache the tensor-map encoder rejects (e.g. an empty one) takes the cp.async kernel
        if (rows > 0 &&
            !make_map(&kc, a->k_cache, kDQ, a->Hkv, rows, blocks, a->kc_sh, a->kc_ss, a->kc_sb, 1, box) &&
            !make_map(&vc, a->v_cache, kDV, a->Hkv, rows, blocks, a->vc_sh, a->vc_ss, a->vc_sb, 1, box) &&
            !make_map(&kn, a->k_new, kDQ, a->Hkv, a->T, a->B, a->kn_sh, a->kn_st, a->kn_sb, 1, new_rows) &&
            !make_map(&vn, a->v_new, kDV, a->Hkv, a->T, a->B, a->vn_sh, a->vn_st, a->vn_sb, 1, new_rows)) {
            if (!umma) {
                e = launch_decode_tma(kc, vc, kn, vn, p, (cudaStream_t)stream);
                return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
            }
            if (!make_map(&q, a->q, kDQ, a->Hq, a->T, a->B, a->q_sh, a->q_st, a->q_sb, p.G, a->T)) {
                e = launch_decode_umma(q, kc, vc, kn, vn, p, 0, (cudaStream_t)stream);
                return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
            }
        }
    }
    e = launch_decode(p, (cudaStream_t)stream);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

} // namespace

namespace sinkattn {
// Pipeline depth of the split-KV decode kernel: 2 stages let two CTAs share an SM, which
// measured faster than one CTA with 4 stages for every decode workload (GA 262144-token
// context, SWA ring, hybrid verify).
int decode_stages(const DecodeParams &p)
{
    (void)p;
    return 2;
}
} // namespace sinkattn

extern "C" {

const char *sinkattn_status_string(int status)
{
    switch (status) {
    case SINKATTN_OK: return "ok";
    case SINKATTN_ERR_INVALID_ARG: return "invalid argument";
    case SINKATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case SINKATTN_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case SINKATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SINKATTN_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

int sinkattn_version(void) { return SINKATTN_VERSION; }

int sinkattn_prefill_swa(const sinkattn_prefill_args *args, int32_t window, void *stream)
{
    if (window < 1)
        return SINKATTN_ERR_INVALID_ARG;
    return run_prefill(args, window, 0, stream);
}

int sinkattn_prefill_ga(const sinkattn_prefill_args *args, void *stream)
{
    return run_prefill(args, 0, 0, stream);
}

int sinkattn_prefill_chunk(const sinkattn_prefill_args *args, int32_t prefix, int32_t window,
                           void *stream)
{
    if (window < 0)
        return SINKATTN_ERR_INVALID_ARG;
    return run_prefill(args, window, prefix, stream);
}

int sinkattn_prefill_chunk_paged(const sinkattn_prefill_args *args,
                                 const sinkattn_paged_kv *prefix_kv, int32_t prefix,
                                 int32_t window, void *stream)
{
    if (window < 0 || !prefix_kv)
        return SINKATTN_ERR_INVALID_ARG;
    return run_prefill(args, window, prefix, stream, prefix_kv);
}

int sinkattn_prefill_swa_rope(const sinkattn_prefill_args *args, int32_t window,
                              const sinkattn_rope_spec *rope, void *stream)
{
    if (window < 1 || !rope)
        return SINKATTN_ERR_INVALID_ARG;
    if (!(rope->theta > 0.0) || !isfinite(rope->theta) || !isfinite(rope->v_scale))
        return SINKATTN_ERR_INVALID_ARG;
    if (rope->rope_dim < 16 || rope->rope_dim > 2 * kRopeFusedMaxHalf || rope->rope_dim % 16 != 0)
        return SINKATTN_ERR_UNSUPPORTED;
    int st = validate_prefill(args);
    if (st != SINKATTN_OK)
        return st;
    if (args->B == 0 || args->L == 0)
        return SINKATTN_OK;
    bool done = false;
    st = try_prefill_swa_packed(args, window, stream, &done, rope);
    if (st != SINKATTN_OK)
        return st;
    // the fused path is the GQA-packed kernel's: other shapes take the separate pass
    return done ? SINKATTN_OK : SINKATTN_ERR_UNSUPPORTED;
}

size_t sinkattn_prefill_host_workspace_size(const sinkattn_prefill_args *args, int32_t chunk)
{
    if (!args || chunk <= 0 || chunk % 128 != 0 || args->B <= 0 || args->L <= 0 ||
        args->Hq <= 0 || args->Hkv <= 0)
        return 0;
    return host_layout(args, chunk).total;
}

int sinkattn_prefill_host(const sinkattn_prefill_args *args, int32_t window, int32_t chunk,
                          void *workspace, size_t ws_bytes, void *stream)
{
    return run_prefill_host(args, window, chunk, workspace, ws_bytes, stream);
}

size_t sinkattn_decode_workspace_size(const sinkattn_decode_args *args)
{
    if (validate_decode_shape(args) != SINKATTN_OK || args->B == 0 || args->T == 0)
        return 0;
    return workspace_bytes(args, plan_split(args));
}

int sinkattn_decode(const sinkattn_decode_args *args, void *workspace, size_t ws_bytes,
                    void *stream)
{
    int st = validate_decode(args);
    if (st != SINKATTN_OK || args->B == 0 || args->T == 0)
        return st;
    const Split s = plan_split(args);
    const size_t need = workspace_bytes(args, s);
    if (need > 0) {
        if (!workspace || ws_bytes < need)
            return SINKATTN_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(workspace))
            return SINKATTN_ERR_ALIGNMENT;
    }
    DecodeParams p;
    fill_decode_params(p, args, s, need > 0 ? workspace : nullptr);
    return run_decode(args, p, stream);
}

int sinkattn_decode_noalloc(const sinkattn_decode_args *args, void *stream)
{
    int st = validate_decode(args);
    if (st != SINKATTN_OK || args->B == 0 || args->T == 0)
        return st;
    const Split s = plan_split(args);
    const size_t need = workspace_bytes(args, s);
    if (need > kNoAllocWorkspaceBytes)
        return SINKATTN_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    if (need > 0 && noalloc_workspace_ptr(&ws) != cudaSuccess)
        return SINKATTN_ERR_CUDA;
    // Every partial the merge reads is written first by the split kernel of the same call, so
    // whatever an earlier call left in the array needs no clearing.
    DecodeParams p;
    fill_decode_params(p, args, s, need > 0 ? ws : nullptr);
    return run_decode(args, p, stream);
}

int sinkattn_kv_commit(const sinkattn_decode_args *a, const int32_t *n_accept, void *stream)
{
    if (!a || (a->kind != SINKATTN_KV_RING && a->kind != SINKATTN_KV_CONTIG &&
               a->kind != SINKATTN_KV_PAGED))
        return SINKATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->Hkv <= 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->dq != kDQ || a->dv != kDV)
        return SINKATTN_ERR_UNSUPPORTED;
    if (kv_dtype_check(a) != SINKATTN_OK)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->commit_rope != 0 && a->commit_rope != 1)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->commit_rope) {
        if (!(a->rope_theta > 0.0) || !isfinite(a->rope_theta) || !isfinite(a->commit_v_scale))
            return SINKATTN_ERR_INVALID_ARG;
        if (a->kind == SINKATTN_KV_RING && !a->commit_pos)
            return SINKATTN_ERR_INVALID_ARG;
        if (a->rope_dim < 16 || a->rope_dim > 2 * kRopeMaxHalf || a->rope_dim % 16 != 0 ||
            a->rope_dim > kDQ)
            return SINKATTN_ERR_UNSUPPORTED;
    }
    if (a->B == 0 || a->T == 0)
        return SINKATTN_OK;
    if (!n_accept || !a->k_new || !a->v_new || !a->k_cache || !a->v_cache)
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind == SINKATTN_KV_RING && (a->ring_cap <= 0 || !a->ring_head || !a->ring_len))
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind != SINKATTN_KV_RING && (a->max_ctx < 0 || !a->ctx_len))
        return SINKATTN_ERR_INVALID_ARG;
    if (a->kind == SINKATTN_KV_PAGED &&
        (a->page_size <= 0 || a->max_pages <= 0 || a->num_pages <= 0 || !a->page_table))
        return SINKATTN_ERR_INVALID_ARG;
    const void *ptrs[4] = {a->k_new, a->v_new, a->k_cache, a->v_cache};
    for (int i = 0; i < 4; ++i)
        if (!aligned16(ptrs[i]))
            return SINKATTN_ERR_ALIGNMENT;
    const int64_t s[12] = {a->kn_sb, a->kn_st, a->kn_sh, a->vn_sb, a->vn_st, a->vn_sh,
                           a->kc_sb, a->kc_ss, a->kc_sh, a->vc_sb, a->vc_ss, a->vc_sh};
    const bool fp8 = a->kv_dtype == SINKATTN_KV_FP8_E4M3;
    for (int i = 0; i < 12; ++i) {
        if (s[i] <= 0)
            return SINKATTN_ERR_INVALID_ARG;
        if ((fp8 && i >= 6) ? !stride_ok_bytes(s[i]) : !stride_ok(s[i]))
            return SINKATTN_ERR_ALIGNMENT;
    }
    CommitParams p;
    p.fp8 = fp8;
    p.k_scale = fp8 ? a->k_scale : 1.f;
    p.v_scale = fp8 ? a->v_scale : 1.f;
    p.kind = a->kind;
    p.B = a->B;
    p.T = a->T;
    p.Hkv = a->Hkv;
    p.k_new = static_cast<const uint16_t *>(a->k_new);
    p.v_new = static_cast<const uint16_t *>(a->v_new);
    p.kn_sb = a->kn_sb;
    p.kn_st = a->kn_st;
    p.kn_sh = a->kn_sh;
    p.vn_sb = a->vn_sb;
    p.vn_st = a->vn_st;
    p.vn_sh = a->vn_sh;
    p.k_cache = static_cast<uint16_t *>(const_cast<void *>(a->k_cache));
    p.v_cache = static_cast<uint16_t *>(const_cast<void *>(a->v_cache));
    p.kc_sb = a->kc_sb;
    p.kc_ss = a->kc_ss;
    p.kc_sh = a->kc_sh;
    p.vc_sb = a->vc_sb;
    p.vc_ss = a->vc_ss;
    p.vc_sh = a->vc_sh;
    p.ring_head = const_cast<int32_t *>(a->ring_head);
    p.ring_len = const_cast<int32_t *>(a->ring_len);
    p.ring_cap = a->ring_cap;
    p.ctx_len = const_cast<int32_t *>(a->ctx_len);
    p.max_ctx = a->max_ctx;
    p.page_table = a->page_table;
    p.page_size = a->page_size;
    p.max_pages = a->max_pages;
    p.num_pages = a->num_pages;
    p.n_accept = n_accept;
    p.rope_half = a->commit_rope ? a->rope_dim / 2 : 0;
    p.v_mul = a->commit_rope ? a->commit_v_scale : 1.f;
    p.pos = a->commit_rope ? a->commit_pos : nullptr;
    // the same fp64 frequencies as sinkattn_rope_qkv, so both give the same bits
    for (int i = 0; i < kRopeMaxHalf; ++i)
        p.inv_freq[i] = i < p.rope_half ? pow(a->rope_theta, -2.0 * i / (2.0 * p.rope_half)) : 0.0;
    const cudaError_t e = fp8 ? launch_commit_fp8(p, (cudaStream_t)stream)
                              : launch_commit(p, (cudaStream_t)stream);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

int sinkattn_rope_qkv(const sinkattn_rope_args *a, void *stream)
{
    if (!a || a->B < 0 || a->L < 0)
        return SINKATTN_ERR_INVALID_ARG;
    if (!(a->theta > 0.0) || !isfinite(a->theta) || !isfinite(a->v_scale))
        return SINKATTN_ERR_INVALID_ARG;
    if ((a->q && a->Hq <= 0) || ((a->k || a->v) && a->Hkv <= 0))
        return SINKATTN_ERR_INVALID_ARG;
    if ((a->q || a->k) && (a->rope_dim < 16 || a->rope_dim > 2 * kRopeMaxHalf ||
                           a->rope_dim % 16 != 0 || a->dq < a->rope_dim || a->dq % 8 != 0))
        return SINKATTN_ERR_UNSUPPORTED;
    if (a->v && (a->dv <= 0 || a->dv % 16 != 0))
        return SINKATTN_ERR_UNSUPPORTED;
    if (a->B == 0 || a->L == 0 || (!a->q && !a->k && !a->v))
        return SINKATTN_OK;
    const void *ptrs[3] = {a->q, a->k, a->v};
    const int64_t s[9] = {a->q_sb, a->q_sl, a->q_sh, a->k_sb, a->k_sl, a->k_sh,
                          a->v_sb, a->v_sl, a->v_sh};
    for (int i = 0; i < 3; ++i) {
        if (!ptrs[i])
            continue;
        if (!aligned16(ptrs[i]))
            return SINKATTN_ERR_ALIGNMENT;
        for (int j = 0; j < 3; ++j) {
            if (s[3 * i + j] <= 0)
                return SINKATTN_ERR_INVALID_ARG;
            if (!stride_ok(s[3 * i + j]))
                return SINKATTN_ERR_ALIGNMENT;
        }
    }
    {
        // 32-byte units per token; the kernel indexes TOK tokens' worth of them with an int
        const int64_t nc = (a->q || a->k) ? a->rope_dim / 16 : 0;
        const int64_t per_tok = (a->q ? (int64_t)a->Hq * nc : 0) +
                                (a->k ? (int64_t)a->Hkv * nc : 0) +
                                (a->v ? (int64_t)a->Hkv * (a->dv / 16) : 0);
        if (per_tok * 8 > 0x3fffffff)
            return SINKATTN_ERR_UNSUPPORTED;
    }
    RopeParams p;
    p.q = static_cast<uint16_t *>(a->q);
    p.k = static_cast<uint16_t *>(a->k);
    p.v = static_cast<uint16_t *>(a->v);
    p.pos_base = a->pos_base;
    p.pos0 = a->pos0;
    p.B = a->B;
    p.L = a->L;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.half = (a->q || a->k) ? a->rope_dim / 2 : 8;
    p.dv = a->dv;
    p.v_scale = a->v_scale;
    p.q_sb = a->q_sb;
    p.q_sl = a->q_sl;
    p.q_sh = a->q_sh;
    p.k_sb = a->k_sb;
    p.k_sl = a->k_sl;
    p.k_sh = a->k_sh;
    p.v_sb = a->v_sb;
    p.v_sl = a->v_sl;
    p.v_sh = a->v_sh;
    for (int i = 0; i < kRopeMaxHalf; ++i)
        p.inv_freq[i] = i < p.half ? pow(a->theta, -2.0 * i / (2.0 * p.half)) : 0.0;
    const cudaError_t e = launch_rope_qkv(p, (cudaStream_t)stream);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

size_t sinkattn_prefill_backward_workspace_size(const sinkattn_backward_args *args)
{
    if (validate_backward(args) != SINKATTN_OK || args->B == 0 || args->L == 0)
        return 0;
    return backward_workspace_bytes(args);
}

int sinkattn_prefill_backward(const sinkattn_backward_args *a, int32_t window, void *workspace,
                              size_t ws_bytes, void *stream)
{
    if (window < 0)
        return SINKATTN_ERR_INVALID_ARG;
    int st = validate_backward(a);
    if (st != SINKATTN_OK || a->B == 0 || a->L == 0)
        return st;
    const size_t need = backward_workspace_bytes(a);
    if (!workspace || ws_bytes < need)
        return SINKATTN_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace))
        return SINKATTN_ERR_ALIGNMENT;
    CUtensorMap q64, do64, q128, do128, k128, v128;
    if ((st = make_map(&q64, a->q, kDQ, a->Hq, a->L, a->B, a->q_sh, a->q_sl, a->q_sb, 1, 64)) ||
        (st = make_map(&do64, a->dout, kDV, a->Hq, a->L, a->B, a->do_sh, a->do_sl, a->do_sb, 1, 64)) ||
        (st = make_map(&q128, a->q, kDQ, a->Hq, a->L, a->B, a->q_sh, a->q_sl, a->q_sb, 1, 128)) ||
        (st = make_map(&do128, a->dout, kDV, a->Hq, a->L, a->B, a->do_sh, a->do_sl, a->do_sb, 1, 128)) ||
        (st = make_map(&k128, a->k, kDQ, a->Hkv, a->L, a->B, a->k_sh, a->k_sl, a->k_sb, 1, 128)) ||
        (st = make_map(&v128, a->v, kDV, a->Hkv, a->L, a->B, a->v_sh, a->v_sl, a->v_sb, 1, 128)))
        return st;
    BwdParams p;
    p.B = a->B;
    p.L = a->L;
    p.Hq = a->Hq;
    p.Hkv = a->Hkv;
    p.G = a->Hq / a->Hkv;
    p.window = window;
    p.scale = a->scale;
    p.scale_log2 = a->scale * kLog2e;
    p.o = static_cast<const uint16_t *>(a->o);
    p.dout = static_cast<const uint16_t *>(a->dout);
    p.o_sb = a->o_sb;
    p.o_sl = a->o_sl;
    p.o_sh = a->o_sh;
    p.do_sb = a->do_sb;
    p.do_sl = a->do_sl;
    p.do_sh = a->do_sh;
    p.lse = a->lse;
    p.sink = a->sink;
    p.delta = static_cast<float *>(workspace);
    p.dq = a->dq;
    p.dk = a->dk;
    p.dv = a->dv;
    p.dsink = a->dsink;
    p.dq_sb = a->dq_sb;
    p.dq_sl = a->dq_sl;
    p.dq_sh = a->dq_sh;
    p.dk_sb = a->dk_sb;
    p.dk_sl = a->dk_sl;
    p.dk_sh = a->dk_sh;
    p.dv_sb = a->dv_sb;
    p.dv_sl = a->dv_sl;
    p.dv_sh = a->dv_sh;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (a->dsink)
        e = cudaMemsetAsync(a->dsink, 0, sizeof(float) * a->Hq, s);
    if (e == cudaSuccess)
        e = launch_bwd_delta(p, s);
    if (e == cudaSuccess)
        e = launch_bwd_dkdv(q64, k128, v128, do64, p, s);
    if (e == cudaSuccess)
        e = launch_bwd_dq(q128, k128, v128, do128, p, s);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

int sinkattn_set_wait_limit_ns(uint64_t ns)
{
    return set_wait_limit(ns) == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

int sinkattn_take_device_error(uint32_t *flag_out)
{
    if (!flag_out)
        return SINKATTN_ERR_INVALID_ARG;
    const cudaError_t e = read_and_clear_device_error(flag_out);
    return e == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

} // extern "C"
