// Sink-softmax attention decode / speculative verify, split-KV, with TMA tile loads (sm_100a).
//
// Same computation and partial / merge scheme as the cp.async decode kernel (sink-free span
// partials; the sink counted once when spans are merged, "MiMo-V2-Flash 架构 QA" Q3.8). Here a
// producer thread moves each 64-key tile with five bulk tensor copies (3 K boxes, 2 V boxes of
// 64 keys x 64 dims, 128-byte swizzle) into a ring of shared-memory stages, so the consumer
// warps only do math and the load path issues 5 instructions per 40 KB instead of 2560.
//
// Tiles of a (sequence, KV head, span) CTA:
//   contiguous / paged cache: the span's cached keys in position order, 64 per tile (a paged
//     tile never crosses a page: pages hold a multiple of 64 tokens);
//   ring: the ring's slots in physical order (attention does not depend on key order; each slot
//     gets its position from the ring head);
//   then, for the span that holds them, one tile with the T new tokens (rows past T are outside
//     the tensor and arrive as zeros).
// Keys a tile holds but the span must not see are masked; their V rows are zeroed in shared
// memory first, so a zero weight never meets whatever the cache held there.
#pragma once
#include "common.cuh"
#include "decode_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace dt {
constexpr int KT = 64;                       // keys per tile
constexpr int REGION = KT * 128;             // one 64-dim box: 64 rows x 128 B
constexpr int STAGE_K = 3 * REGION;          // 192 dims
constexpr int STAGE_V = 2 * REGION;          // 128 dims
constexpr int STAGE = STAGE_K + STAGE_V;     // 40 KB, 1 KB aligned
constexpr int CONSUMERS = 4;
constexpr int THREADS = 32 * (CONSUMERS + 1);
constexpr int RED_STRIDE = 70;
__host__ __device__ constexpr int smem_bytes(int nstage) { return nstage * STAGE + 256 + 1024; }
} // namespace dt

struct DecodeTiles {
    int n_cache, n_used, first_c, n_total, kb, ke, ring_head;
    int cache_tiles; // tiles of cached keys
    bool has_new;    // plus one tile of new tokens
};

// Tiles of span `split` of sequence b (kt keys each), from its cached length (ring_len or
// ctx_len) and ring head (0 for other caches).
SA_DEV DecodeTiles decode_tiles(const DecodeParams &p, int split, int len, int head, int kt = dt::KT)
{
    DecodeTiles d;
    d.n_cache = max(0, min(len, p.kind == 0 ? p.ring_cap : p.max_ctx));
    d.n_used = (p.window > 0) ? min(d.n_cache, p.window - 1) : d.n_cache;
    d.first_c = d.n_cache - d.n_used;
    d.n_total = d.n_used + p.T;
    d.kb = split * p.chunk;
    d.ke = min(d.kb + p.chunk, d.n_total);
    d.ring_head = (p.kind == 0) ? ((head % p.ring_cap) + p.ring_cap) % p.ring_cap : 0;
    if (p.kind == 0) {
        d.cache_tiles = (d.kb < d.n_used) ? p.ring_cap / kt : 0; // one span holds the ring
    } else {
        const int ce = min(d.ke, d.n_used);
        d.cache_tiles = (ce > d.kb) ? (ce - d.kb + kt - 1) / kt : 0;
    }
    d.has_new = d.ke > d.n_used && d.kb < d.n_total;
    return d;
}

SA_DEV DecodeTiles decode_tiles(const DecodeParams &p, int b, int split)
{
    return p.kind == 0 ? decode_tiles(p, split, p.ring_len[b], p.ring_head[b])
                       : decode_tiles(p, split, p.ctx_len[b], 0);
}

// Whether tile t's keys come from a page that exists (a page id outside the pool hides them).
SA_DEV bool decode_tile_ok(const DecodeParams &p, const DecodeTiles &d, int b, int t)
{
    if (p.kind != 2 || t >= d.cache_tiles)
        return true;
    const int pg = (d.first_c + d.kb + t * dt::KT) / p.page_size;
    if (pg >= p.max_pages)
        return false;
    const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
    return pid >= 0 && pid < p.num_pages;
}

// Validity and position (relative to the first new token) of key i of tile t.
SA_DEV void decode_key(const DecodeParams &p, const DecodeTiles &d, int t, int i, bool tile_ok,
                       bool &valid, int &pos)
{
    if (t < d.cache_tiles) {
        if (p.kind == 0) {
            const int slot = t * dt::KT + i; // slot and head both lie in [0, ring_cap)
            const int c = slot >= d.ring_head ? slot - d.ring_head : slot - d.ring_head + p.ring_cap;
            valid = c >= d.first_c && c < d.n_cache;
            pos = c - d.n_cache;
        } else {
            const int v = d.kb + t * dt::KT + i;
            valid = tile_ok && v < min(d.ke, d.n_used);
            pos = v - d.n_used;
        }
    } else {
        const int v = d.n_used + i;
        valid = i < p.T && v >= d.kb && v < d.ke;
        pos = i;
    }
}

template <int KP, int NSTAGE>
__global__ void __launch_bounds__(dt::THREADS, NSTAGE == 2 ? 2 : 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                      const __grid_constant__ CUtensorMap tmKn, const __grid_constant__ CUtensorMap tmVn,
                      const DecodeParams p)
{
    using namespace dt;
    constexpr int KW = KT / KP; // keys per warp per tile
    constexpr int NT = KW / 8;  // n-tiles of S per warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.MT;
    const int mt = warp % MT, ks = warp / MT;
    const bool active = warp < CONSUMERS && ks < KP;
    const DecodeTiles d = decode_tiles(p, b, split);
    const int ntile = d.cache_tiles + (d.has_new ? 1 : 0);

    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NSTAGE * STAGE);
    uint64_t *empty = full + NSTAGE;
    volatile int *abort = reinterpret_cast<volatile int *>(empty + NSTAGE);
    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], CONSUMERS);
        }
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CONSUMERS) {
        // ---- producer: one thread issues the bulk tensor copies of every tile
        if (lane == 0 && ntile > 0) {
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
            int issued = 0;
            for (int t = 0; t < ntile; ++t) {
                const int st = t % NSTAGE;
                if (t >= NSTAGE && !mbar_wait(&empty[st], ((t / NSTAGE) - 1) & 1, abort, 2u))
                    break;
                uint8_t *sk = smem + st * STAGE, *sv = sk + STAGE_K;
                mbar_arrive_expect_tx(&full[st], STAGE);
                if (t < d.cache_tiles) {
                    int row, blk; // coordinates of the tile's first key: (row, block) = (position, sequence)
                    if (p.kind == 0) {
                        row = t * KT;
                        blk = b;
                    } else if (p.kind == 1) {
                        row = d.first_c + d.kb + t * KT;
                        blk = b;
                    } else {
                        const int c0 = d.first_c + d.kb + t * KT;
                        const int pg = c0 / p.page_size;
                        // a missing page is read at a block outside the pool: zeros, and its keys
                        // are masked by the consumers
                        blk = decode_tile_ok(p, d, b, t) ? p.page_table[(int64_t)b * p.max_pages + pg]
                                                         : p.num_pages;
                        row = c0 - pg * p.page_size;
                    }
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(sk + c * REGION, &tmKc, &full[st], c * 64, g, row, blk);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(sv + c * REGION, &tmVc, &full[st], c * 64, g, row, blk);
                } else {
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(sk + c * REGION, &tmKn, &full[st], c * 64, g, 0, b);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(sv + c * REGION, &tmVn, &full[st], c * 64, g, 0, b);
                }
                issued = t + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int t = max(0, issued - NSTAGE); t < issued; ++t)
                mbar_wait_drain(&full[t % NSTAGE], (t / NSTAGE) & 1);
        }
        __syncwarp();
        return;
    }

    // ---- consumer warps: rows lane/4 and lane/4 + 8 of m-tile mt
    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int ta = min(ra / p.G, p.T - 1), tb = min(rb / p.G, p.T - 1);
    uint32_t qa[12][4];
    {
        const bool va = active && ra < p.R, vb = active && rb < p.R;
        const uint16_t *qra = p.q + (int64_t)b * p.q_sb + (int64_t)ta * p.q_st +
                              (int64_t)(g * p.G + (va ? ra % p.G : 0)) * p.q_sh;
        const uint16_t *qrb = p.q + (int64_t)b * p.q_sb + (int64_t)tb * p.q_st +
                              (int64_t)(g * p.G + (vb ? rb % p.G : 0)) * p.q_sh;
        const int c2 = 2 * (lane & 3);
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
            qa[kk][0] = va ? *reinterpret_cast<const uint32_t *>(qra + kk * 16 + c2) : 0u;
            qa[kk][1] = vb ? *reinterpret_cast<const uint32_t *>(qrb + kk * 16 + c2) : 0u;
            qa[kk][2] = va ? *reinterpret_cast<const uint32_t *>(qra + kk * 16 + 8 + c2) : 0u;
            qa[kk][3] = vb ? *reinterpret_cast<const uint32_t *>(qrb + kk * 16 + 8 + c2) : 0u;
        }
    }
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f, e_a = 0.f, e_b = 0.f;

    for (int t = 0; t < ntile; ++t) {
        const int st = t % NSTAGE;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (t / NSTAGE) & 1, abort, 2u)))
            break;
        if (!active) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
            continue;
        }
        uint8_t *stage = smem + st * STAGE;
        const uint32_t sK = smem_u32(stage), sV = smem_u32(stage + STAGE_K);
        const int key0 = ks * KW; // first key of this warp inside the tile
        const bool tile_ok = decode_tile_ok(p, d, b, t);
        // zero the V rows of this warp's keys that the span must not see, 32 keys at a time
        bool zeroed = false;
#pragma unroll
        for (int k32 = 0; k32 < KW; k32 += 32) {
            bool valid;
            int pos;
            decode_key(p, d, t, key0 + k32 + (lane % KW), tile_ok, valid, pos);
            const unsigned bad = __ballot_sync(0xffffffffu, k32 + lane < KW && !valid);
            if (bad) {
                for (int k = 0; k < 32; ++k) {
                    if (((bad >> k) & 1u) && lane < 16) // 16 lanes x 16 B: both 128-byte halves
                        *reinterpret_cast<uint4 *>(stage + STAGE_K + (lane >> 3) * REGION +
                                                   (key0 + k32 + k) * 128 + (lane & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                zeroed = true;
            }
        }

        // ---- S = Q K^T (K: 3 regions of 64 keys x 128 B, 16-byte chunks XOR-swizzled by key & 7)
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < 6; ++k2) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int key = key0 + nt * 8 + (lane & 7);
                const int ch = 4 * k2 + (lane >> 3); // 16-byte chunk of the 192 dims (0..23)
                const int reg = ch >> 3, cc = (ch & 7) ^ (key & 7);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(sK + reg * REGION + key * 128 + (cc << 4), b0, b1, b2, b3);
                mma_bf16_16816(sacc[nt], qa[2 * k2], b0, b1);
                mma_bf16_16816(sacc[nt], qa[2 * k2 + 1], b2, b3);
            }
        }

        // ---- mask, online softmax (sink-free partial)
        float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kc = nt * 8 + 2 * (lane & 3) + e;
                bool valid;
                int pos;
                decode_key(p, d, t, key0 + kc, tile_ok, valid, pos);
                const bool vis_a = valid && pos <= ta && (p.window <= 0 || pos > ta - p.window);
                const bool vis_b = valid && pos <= tb && (p.window <= 0 || pos > tb - p.window);
                sacc[nt][e] = vis_a ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                sacc[nt][2 + e] = vis_b ? sacc[nt][2 + e] * p.scale_log2 : -INFINITY;
                mxa = fmaxf(mxa, sacc[nt][e]);
                mxb = fmaxf(mxb, sacc[nt][2 + e]);
            }
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        const float mna = fmaxf(m_a, mxa), mnb = fmaxf(m_b, mxb);
        const float alpha_a = (mna == -INFINITY) ? 1.f : fast_exp2(m_a - mna);
        const float alpha_b = (mnb == -INFINITY) ? 1.f : fast_exp2(m_b - mnb);
        const float ua = (mna == -INFINITY) ? 0.f : mna, ub = (mnb == -INFINITY) ? 0.f : mnb;
        m_a = mna;
        m_b = mnb;
        uint32_t pp[NT][2];
        float sa = 0.f, sb = 0.f, xa = 0.f, xb = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float p0 = fast_exp2(sacc[nt][0] - ua), p1 = fast_exp2(sacc[nt][1] - ua);
            const float p2 = fast_exp2(sacc[nt][2] - ub), p3 = fast_exp2(sacc[nt][3] - ub);
            xa += p0 + p1;
            xb += p2 + p3;
            pp[nt][0] = pack_bf16x2(p0, p1);
            pp[nt][1] = pack_bf16x2(p2, p3);
            sa += sum_bf16x2(pp[nt][0]);
            sb += sum_bf16x2(pp[nt][1]);
        }
        l_a = l_a * alpha_a + sa;
        l_b = l_b * alpha_b + sb;
        e_a = e_a * alpha_a + xa;
        e_b = e_b * alpha_b + xb;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            o[i][0] *= alpha_a;
            o[i][1] *= alpha_a;
            o[i][2] *= alpha_b;
            o[i][3] *= alpha_b;
        }

        // ---- O += P V (V: 2 regions of 64 keys x 128 B, swizzled like K)
#pragma unroll
        for (int kq = 0; kq < NT / 2; ++kq) {
            uint32_t a[4];
            a[0] = pp[2 * kq][0];
            a[1] = pp[2 * kq][1];
            a[2] = pp[2 * kq + 1][0];
            a[3] = pp[2 * kq + 1][1];
            const int key = key0 + kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const int ch = 2 * np + (lane >> 4); // 16-byte chunk of the 128 dims (0..15)
                const int reg = ch >> 3, cc = (ch & 7) ^ (key & 7);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(sV + reg * REGION + key * 128 + (cc << 4), b0, b1, b2, b3);
                mma_bf16_16816(o[2 * np], a, b0, b1);
                mma_bf16_16816(o[2 * np + 1], a, b2, b3);
            }
        }
        // generic-proxy writes to the stage must be ordered before the next bulk copy into it
        if (zeroed)
            fence_async_smem();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
    }

    // full row sums across the quad
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    e_a += __shfl_xor_sync(0xffffffffu, e_a, 1);
    e_a += __shfl_xor_sync(0xffffffffu, e_a, 2);
    e_b += __shfl_xor_sync(0xffffffffu, e_b, 1);
    e_b += __shfl_xor_sync(0xffffffffu, e_b, 2);

    // ---- combine the KP key slices of each m-tile (same fragment layout in every warp)
    if (KP > 1) {
        named_bar_sync(1, 32 * CONSUMERS); // every consumer warp is done with the stages
        float *red = reinterpret_cast<float *>(smem);
        if (active && ks > 0) {
            float *dst = red + ((ks * MT + mt) * 32 + lane) * RED_STRIDE;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                dst[4 * i + 0] = o[i][0];
                dst[4 * i + 1] = o[i][1];
                dst[4 * i + 2] = o[i][2];
                dst[4 * i + 3] = o[i][3];
            }
            dst[64] = m_a;
            dst[65] = m_b;
            dst[66] = l_a;
            dst[67] = l_b;
            dst[68] = e_a;
            dst[69] = e_b;
        }
        named_bar_sync(1, 32 * CONSUMERS);
        if (active && ks == 0) {
#pragma unroll
            for (int k2 = 1; k2 < KP; ++k2) {
                const float *src = red + ((k2 * MT + mt) * 32 + lane) * RED_STRIDE;
                const float m2a = src[64], m2b = src[65];
                const float mna = fmaxf(m_a, m2a), mnb = fmaxf(m_b, m2b);
                const float a1 = (mna == -INFINITY) ? 0.f : fast_exp2(m_a - mna);
                const float a2 = (mna == -INFINITY) ? 0.f : fast_exp2(m2a - mna);
                const float b1 = (mnb == -INFINITY) ? 0.f : fast_exp2(m_b - mnb);
                const float b2 = (mnb == -INFINITY) ? 0.f : fast_exp2(m2b - mnb);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    o[i][0] = o[i][0] * a1 + src[4 * i + 0] * a2;
                    o[i][1] = o[i][1] * a1 + src[4 * i + 1] * a2;
                    o[i][2] = o[i][2] * b1 + src[4 * i + 2] * b2;
                    o[i][3] = o[i][3] * b1 + src[4 * i + 3] * b2;
                }
                l_a = l_a * a1 + src[66] * a2;
                l_b = l_b * b1 + src[67] * b2;
                e_a = e_a * a1 + src[68] * a2;
                e_b = e_b * b1 + src[69] * b2;
                m_a = mna;
                m_b = mnb;
            }
        }
    }
    if (!active || ks != 0)
        return;
    decode_write_output(p, b, g, split, ra, rb, lane, o, m_a, m_b, l_a, l_b, e_a, e_b);
}

template <int NSTAGE>
cudaError_t launch_decode_tma_split(const CUtensorMap &kc, const CUtensorMap &vc,
                                    const CUtensorMap &kn, const CUtensorMap &vn,
                                    const DecodeParams &p, cudaStream_t stream)
{
    dim3 grid(p.splits, p.Hkv, p.B);
    const int smem = dt::smem_bytes(NSTAGE);
    if (p.MT == 1)
        decode_tma_kernel<4, NSTAGE><<<grid, dt::THREADS, smem, stream>>>(kc, vc, kn, vn, p);
    else if (p.MT == 2)
        decode_tma_kernel<2, NSTAGE><<<grid, dt::THREADS, smem, stream>>>(kc, vc, kn, vn, p);
    else
        decode_tma_kernel<1, NSTAGE><<<grid, dt::THREADS, smem, stream>>>(kc, vc, kn, vn, p);
    return cudaGetLastError();
}

cudaError_t launch_decode_tma(const CUtensorMap &kc, const CUtensorMap &vc, const CUtensorMap &kn,
                              const CUtensorMap &vn, const DecodeParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        cudaError_t e = cudaSuccess;
        const void *fns[6] = {(const void *)decode_tma_kernel<4, 4>, (const void *)decode_tma_kernel<2, 4>,
                              (const void *)decode_tma_kernel<1, 4>, (const void *)decode_tma_kernel<4, 2>,
                              (const void *)decode_tma_kernel<2, 2>, (const void *)decode_tma_kernel<1, 2>};
        for (int i = 0; i < 6; ++i) {
            e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     dt::smem_bytes(i < 3 ? 4 : 2));
            if (e != cudaSuccess)
                return e;
        }
        return e;
    });
    if (e != cudaSuccess)
        return e;
    e = decode_stages(p) == 2 ? launch_decode_tma_split<2>(kc, vc, kn, vn, p, stream)
                              : launch_decode_tma_split<4>(kc, vc, kn, vn, p, stream);
    if (e != cudaSuccess || p.splits == 1)
        return e;
    return launch_decode_merge(p, stream);
}

} // namespace sinkattn
