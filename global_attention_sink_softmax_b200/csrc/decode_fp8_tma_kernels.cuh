// Decode / speculative verify against an FP8 (E4M3) KV cache, fed by the TMA and widened in
// registers (sm_100a).
//
// Same computation as decode_fp8_kernel (the scales folded in by linearity: logits use
// scale * k_scale on <q, e(c)>, O is v_scale * sum_j w_j e(c'_j); the sink counted once when the
// split-KV partials merge, "MiMo-V2-Flash 架构 QA" Q3.8) and the same work items, (key span, KV
// head, sequence). What changes is how the one-byte codes reach the tensor cores: a producer
// thread moves each 64-key tile of codes with five bulk tensor copies (3 K boxes, 2 V boxes of
// 64 keys x 64 bytes, 64-byte swizzle, 20 KB) into a 4-stage ring, and the consumer warps read
// the codes with ldmatrix and widen them in registers with cvt.rn.f16x2.e4m3x2 (exact), so no
// pass over shared memory and no second barrier per tile is needed.
//
//   S = Q K^T: ldmatrix (8 keys x 16 bytes per matrix) hands thread (g, t) the 4 codes of dims
//     16 s + 4t .. 16 s + 4t + 3 of key g for k-step s; two cvt give the B fragment. The MMA's
//     k order inside a step is therefore (4t, 4t+1 | 4t+2, 4t+3) where mma.sync expects
//     (2t, 2t+1 | 2t+8, 2t+9); Q's A fragment is loaded with the same permutation, and a dot
//     product does not depend on the order of its terms.
//   O += P V: ldmatrix.trans on the code tile hands thread (g, t) the byte pairs (dims 2g, 2g+1)
//     of keys 2t and 2t+1; prmt regroups them into (key 2t, key 2t+1) pairs of dim 2g and of dim
//     2g+1, which are the B fragments of two n-tiles whose column g is dim 2g ("even") and dim
//     2g+1 ("odd"). Thread t then holds the accumulators of dims 16c + 4t .. 16c + 4t + 3 of
//     each 16-dim chunk c, which the epilogue writes in natural order.
//
// New tokens (bf16) are quantised by the producer warp into the last tile's stage exactly as the
// commit stores them (their keys past T are masked and their V rows zeroed, like any key the span
// must not see). Q and P are fp16 (Q rounded once; the row sum that normalises O adds the same
// rounded P values).
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "decode_fp8_kernels.cuh"
#include "decode_kernels.cuh"
#include "decode_tma_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace d8t {
constexpr int KT = 64;                    // keys per tile
constexpr int REGION = KT * 64;           // 4 KB: 64 keys x 64 code bytes, 64-byte swizzle
constexpr int STAGE_K = 3 * REGION;       // 192 dims
constexpr int STAGE = 5 * REGION;         // 20 KB: K then V
constexpr int NSTAGE = 4;
constexpr int CONSUMERS = 4;
constexpr int THREADS = 32 * (CONSUMERS + 1);
constexpr int RED_STRIDE = 70;
constexpr int SMEM_BYTES = NSTAGE * STAGE + 256 + 1024;
constexpr float TAU = 8.0f;               // lazy-rescale threshold (log2 units)
static_assert(CONSUMERS * 32 * RED_STRIDE * 4 <= NSTAGE * STAGE, "combine scratch fits the ring");
} // namespace d8t

// Byte offset of 16-byte chunk ch (0..3) of row r in a 64-byte-swizzled region (64-byte rows:
// the chunk index is XORed with bits 1..2 of the row).
SA_DEV int sw64(int r, int ch) { return r * 64 + ((ch ^ ((r >> 1) & 3)) << 4); }

SA_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// bf16 pair (low element first) -> f16 pair
SA_DEV uint32_t f16x2_of_bf16x2(uint32_t v)
{
    return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// Writes one consumer warp's rows with the P V dims of thread t at 16c + 4t .. 16c + 4t + 3:
// o[2c][.] holds dims 16c + 4t (+0 / +2), o[2c + 1][.] dims 16c + 4t (+1 / +3); elements 0, 1
// row a, 2, 3 row b. O (and the partials) carry v_scale. One span: the final O and LSE with
// the sink; else the span's partial (O, m, l_rounded, l_exact).
SA_DEV void fp8_write_output(const DecodeParams &p, int b, int g, int split, int ra, int rb,
                             int lane, const float (&o)[16][4], float m_a, float m_b, float l_a,
                             float l_b, float e_a, float e_b)
{
    const int t4 = 4 * (lane & 3);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int r = half ? rb : ra;
        if (r >= p.R)
            continue;
        const int e0 = half ? 2 : 0;
        const float m = half ? m_b : m_a, l = half ? l_b : l_a, le = half ? e_b : e_a;
        if (p.splits == 1) {
            const int t = r / p.G, h = g * p.G + r % p.G;
            const float sk = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            const float mf = fmaxf(m, sk);
            const float cm = (m == -INFINITY) ? 0.f : fast_exp2(m - mf);
            const float cs = (sk == -INFINITY) ? 0.f : fast_exp2(sk - mf);
            const float D = le * cm + cs;                      // exact denominator: LSE
            const float scl = p.v_scale * cm / (l * cm + cs);  // rounded-P denominator: O
            uint16_t *orow = p.o + (int64_t)b * p.o_sb + (int64_t)t * p.o_st + (int64_t)h * p.o_sh;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t lo = pack_bf16x2(o[2 * c][e0] * scl, o[2 * c + 1][e0] * scl);
                const uint32_t hi = pack_bf16x2(o[2 * c][e0 + 1] * scl, o[2 * c + 1][e0 + 1] * scl);
                *reinterpret_cast<uint2 *>(orow + 16 * c + t4) = make_uint2(lo, hi);
            }
            if (p.lse && (lane & 3) == 0)
                p.lse[((int64_t)b * p.T + t) * p.Hq + h] = (mf + fast_log2(D)) * kLn2;
        } else {
            const int64_t unit = ((int64_t)b * p.Hkv + g) * p.splits + split;
            float *wo = p.ws_o + (unit * p.R + r) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float4 v4;
                v4.x = o[2 * c][e0] * p.v_scale;
                v4.y = o[2 * c + 1][e0] * p.v_scale;
                v4.z = o[2 * c][e0 + 1] * p.v_scale;
                v4.w = o[2 * c + 1][e0 + 1] * p.v_scale;
                *reinterpret_cast<float4 *>(wo + 16 * c + t4) = v4;
            }
            if ((lane & 3) == 0) {
                float4 ml;
                ml.x = m;
                ml.y = l;
                ml.z = le;
                ml.w = 0.f;
                *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + r) * 4) = ml;
            }
        }
    }
}

template <int KP>
__global__ void __launch_bounds__(d8t::THREADS, 2)
    decode_fp8_tma_kernel(const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                          const DecodeParams p)
{
    using namespace d8t;
    constexpr int KW = KT / KP; // keys per warp per tile
    constexpr int NT = KW / 8;  // n-tiles of S per warp
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // the KV heads of a span are neighbours in the grid: a head's 192-byte K rows share 128-byte
    // lines with the next head's, which then meet in L2 instead of being fetched twice
    const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
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
        // ---- producer warp: lane 0 issues the bulk copies of the cache tiles; the whole warp
        // quantises the new tokens into the last tile's stage
        if (lane == 0) {
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
        }
        int issued = 0;
        for (int t = 0; t < ntile; ++t) {
            const int st = t % NSTAGE;
            bool ok = true;
            if (lane == 0 && t >= NSTAGE)
                ok = mbar_wait(&empty[st], ((t / NSTAGE) - 1) & 1, abort, 2u);
            if (!__shfl_sync(0xffffffffu, ok, 0))
                break;
            uint8_t *sk = smem + st * STAGE, *sv = sk + STAGE_K;
            if (t < d.cache_tiles) {
                if (lane == 0) {
                    int row, blk; // the tile's first key: (row, block) = (position or slot, sequence or page)
                    if (p.kind == 0) {
                        row = t * KT;
                        blk = b;
                    } else if (p.kind == 1) {
                        row = d.first_c + d.kb + t * KT;
                        blk = b;
                    } else {
                        const int c0 = d.first_c + d.kb + t * KT;
                        const int pg = c0 / p.page_size;
                        // a missing page is read at a block outside the pool: zeros, and its
                        // keys are masked by the consumers
                        blk = decode_tile_ok(p, d, b, t) ? p.page_table[(int64_t)b * p.max_pages + pg]
                                                         : p.num_pages;
                        row = c0 - pg * p.page_size;
                    }
                    mbar_arrive_expect_tx(&full[st], STAGE);
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(sk + c * REGION, &tmKc, &full[st], c * 64, g, row, blk);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(sv + c * REGION, &tmVc, &full[st], c * 64, g, row, blk);
                }
            } else {
                // the T new tokens, quantised as the commit stores them: 16 codes per unit,
                // 12 units of K and 8 of V per token
                for (int e = lane; e < p.T * 20; e += 32) {
                    const int u = e / 20, j = e - u * 20;
                    const bool is_k = j < 12;
                    const int unit = is_k ? j : j - 12;
                    const uint16_t *src =
                        is_k ? p.k_new + (int64_t)b * p.kn_sb + (int64_t)u * p.kn_st + (int64_t)g * p.kn_sh
                             : p.v_new + (int64_t)b * p.vn_sb + (int64_t)u * p.vn_st + (int64_t)g * p.vn_sh;
                    const uint4 c = quant16(src + unit * 16, is_k ? p.k_scale : p.v_scale);
                    uint8_t *reg = (is_k ? sk : sv) + (unit >> 2) * REGION;
                    *reinterpret_cast<uint4 *>(reg + sw64(u, unit & 3)) = c;
                }
                fence_async_smem(); // ordered before any later bulk copy into the stage
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&full[st]);
            }
            issued = t + 1;
        }
        // no copy of ours may still be landing when the CTA leaves
        if (lane == 0)
            for (int t = max(0, issued - NSTAGE); t < issued; ++t)
                mbar_wait_drain(&full[t % NSTAGE], (t / NSTAGE) & 1);
        __syncwarp();
        return;
    }

    // ---- consumer warps: rows lane/4 and lane/4 + 8 of m-tile mt
    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int ta = min(ra / p.G, p.T - 1), tb = min(rb / p.G, p.T - 1);
    const int t4 = 4 * (lane & 3);
    // Q as fp16, k index permuted: step s takes dims 16 s + 4t .. +3 (a0 / a2 of row a, a1 / a3
    // of row b)
    uint32_t qa[12][4];
    {
        const bool va = active && ra < p.R, vb = active && rb < p.R;
        const uint16_t *qra = p.q + (int64_t)b * p.q_sb + (int64_t)ta * p.q_st +
                              (int64_t)(g * p.G + (va ? ra % p.G : 0)) * p.q_sh;
        const uint16_t *qrb = p.q + (int64_t)b * p.q_sb + (int64_t)tb * p.q_st +
                              (int64_t)(g * p.G + (vb ? rb % p.G : 0)) * p.q_sh;
#pragma unroll
        for (int s = 0; s < 12; ++s) {
            const uint2 x = va ? *reinterpret_cast<const uint2 *>(qra + 16 * s + t4) : make_uint2(0, 0);
            const uint2 y = vb ? *reinterpret_cast<const uint2 *>(qrb + 16 * s + t4) : make_uint2(0, 0);
            qa[s][0] = f16x2_of_bf16x2(x.x);
            qa[s][2] = f16x2_of_bf16x2(x.y);
            qa[s][1] = f16x2_of_bf16x2(y.x);
            qa[s][3] = f16x2_of_bf16x2(y.y);
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
        // a cached tile whose 64 keys every row sees (no window, a contiguous or paged cache,
        // inside the span's cached keys): no mask and no V rows to zero
        const bool whole = p.kind != 0 && p.window <= 0 && tile_ok && t < d.cache_tiles &&
                           d.kb + (t + 1) * KT <= min(d.ke, d.n_used);
        // zero the V codes of this warp's keys that the span must not see (a NaN code times a
        // zero weight would still be NaN), 32 keys at a time
        bool zeroed = false;
#pragma unroll
        for (int k32 = 0; k32 < KW && !whole; k32 += 32) {
            bool valid;
            int pos;
            decode_key(p, d, t, key0 + k32 + (lane % KW), tile_ok, valid, pos);
            const unsigned bad = __ballot_sync(0xffffffffu, k32 + lane < KW && !valid);
            if (bad) {
                for (int k = 0; k < 32; ++k) {
                    if (((bad >> k) & 1u) && lane < 8) // 8 lanes x 16 B: both 64-byte regions
                        *reinterpret_cast<uint4 *>(stage + STAGE_K + (lane >> 2) * REGION +
                                                   (key0 + k32 + k) * 64 + (lane & 3) * 16) =
                            make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                zeroed = true;
            }
        }

        // ---- S = Q K^T: per n-tile and 64-dim region, one ldmatrix.x4 = 4 k-steps of codes
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int c = 0; c < 3; ++c) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int key = key0 + nt * 8 + (lane & 7);
                uint32_t r[4];
                ldmatrix_x4(sK + c * REGION + sw64(key, lane >> 3), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_f16_16816(sacc[nt], qa[4 * c + j], e4m3x2_to_f16x2(r[j] & 0xffffu),
                                  e4m3x2_to_f16x2(r[j] >> 16));
            }
        }

        // ---- mask, online softmax (sink-free partial) with a lazily raised max
        float mxa = -INFINITY, mxb = -INFINITY;
        if (whole) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    sacc[nt][e] *= p.scale_log2;
                    sacc[nt][2 + e] *= p.scale_log2;
                    mxa = fmaxf(mxa, sacc[nt][e]);
                    mxb = fmaxf(mxb, sacc[nt][2 + e]);
                }
            }
        } else {
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
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        // a row's reference max rises only when the tile's exceeds it by more than TAU (always
        // for the first visible score: m is -inf), so most tiles skip the rescale of O; P stays
        // <= 2^TAU, well inside fp16
        const bool up_a = mxa > m_a + TAU, up_b = mxb > m_b + TAU;
        if (__any_sync(0xffffffffu, up_a || up_b)) {
            const float alpha_a = up_a ? fast_exp2(m_a - mxa) : 1.f; // 0 while m is -inf
            const float alpha_b = up_b ? fast_exp2(m_b - mxb) : 1.f;
            if (up_a)
                m_a = mxa;
            if (up_b)
                m_b = mxb;
            l_a *= alpha_a;
            l_b *= alpha_b;
            e_a *= alpha_a;
            e_b *= alpha_b;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= alpha_a;
                o[i][1] *= alpha_a;
                o[i][2] *= alpha_b;
                o[i][3] *= alpha_b;
            }
        }
        const float ua = (m_a == -INFINITY) ? 0.f : m_a, ub = (m_b == -INFINITY) ? 0.f : m_b;
        uint32_t pp[NT][2];
        float sa = 0.f, sb = 0.f, xa = 0.f, xb = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float p0 = fast_exp2(sacc[nt][0] - ua), p1 = fast_exp2(sacc[nt][1] - ua);
            const float p2 = fast_exp2(sacc[nt][2] - ub), p3 = fast_exp2(sacc[nt][3] - ub);
            xa += p0 + p1;
            xb += p2 + p3;
            pp[nt][0] = pack_f16x2(p0, p1);
            pp[nt][1] = pack_f16x2(p2, p3);
            sa += sum_f16x2(pp[nt][0]);
            sb += sum_f16x2(pp[nt][1]);
        }
        l_a += sa;
        l_b += sb;
        e_a += xa;
        e_b += xb;

        // ---- O += P V: per 16 keys and 32 dims one ldmatrix.x4.trans; prmt splits each
        // register's byte pairs into the "even" (dim 2g) and "odd" (dim 2g + 1) n-tiles
#pragma unroll
        for (int kq = 0; kq < NT / 2; ++kq) {
            uint32_t a[4];
            a[0] = pp[2 * kq][0];
            a[1] = pp[2 * kq][1];
            a[2] = pp[2 * kq + 1][0];
            a[3] = pp[2 * kq + 1][1];
            // lane l addresses row l % 8 of matrix l / 8: keys +0..7 / +8..15, chunks c2, c2 + 1
            const int key = key0 + kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int c2 = 0; c2 < 8; c2 += 2) {
                const int ch = c2 + (lane >> 4); // 16-dim chunk 0..7 (region ch / 4)
                uint32_t r[4];
                ldmatrix_x4_trans(sV + (ch >> 2) * REGION + sw64(key, ch & 3), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t ev = prmt(r[2 * h], r[2 * h + 1], 0x6420u);
                    const uint32_t od = prmt(r[2 * h], r[2 * h + 1], 0x7531u);
                    mma_f16_16816(o[2 * (c2 + h)], a, e4m3x2_to_f16x2(ev & 0xffffu),
                                  e4m3x2_to_f16x2(ev >> 16));
                    mma_f16_16816(o[2 * (c2 + h) + 1], a, e4m3x2_to_f16x2(od & 0xffffu),
                                  e4m3x2_to_f16x2(od >> 16));
                }
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
    fp8_write_output(p, b, g, split, ra, rb, lane, o, m_a, m_b, l_a, l_b, e_a, e_b);
}

cudaError_t launch_decode_fp8_tma(const CUtensorMap &kc, const CUtensorMap &vc,
                                  const DecodeParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        const void *fns[3] = {(const void *)decode_fp8_tma_kernel<4>,
                              (const void *)decode_fp8_tma_kernel<2>,
                              (const void *)decode_fp8_tma_kernel<1>};
        for (int i = 0; i < 3; ++i) {
            const cudaError_t e = cudaFuncSetAttribute(
                fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, d8t::SMEM_BYTES);
            if (e != cudaSuccess)
                return e;
        }
        return cudaSuccess;
    });
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.Hkv, p.splits, p.B);
    if (p.MT == 1)
        decode_fp8_tma_kernel<4><<<grid, d8t::THREADS, d8t::SMEM_BYTES, stream>>>(kc, vc, p);
    else if (p.MT == 2)
        decode_fp8_tma_kernel<2><<<grid, d8t::THREADS, d8t::SMEM_BYTES, stream>>>(kc, vc, p);
    else
        decode_fp8_tma_kernel<1><<<grid, d8t::THREADS, d8t::SMEM_BYTES, stream>>>(kc, vc, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.splits == 1)
        return e;
    return launch_decode_merge(p, stream);
}

} // namespace sinkattn
