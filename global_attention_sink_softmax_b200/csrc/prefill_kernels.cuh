// Sink-softmax attention prefill on tcgen05 tensor cores (sm_100a).
//
// What it computes ("MiMo-V2-Flash 架构 QA" Q3.7/Q3.8; "MiMo-V2-Flash 模型架构深度拆解" CH10.1,
// CH10.3): for each query row i of head h, over the keys j its mask keeps (j <= i, and
// j > i - W for a sliding window W),
//     O_i = sum_j exp(a_ij - m_i) v_j / (exp(sink_h - m_i) + sum_j exp(a_ij - m_i)),
//     a_ij = scale <q_i, k_j>, m_i = max(sink_h, max_j a_ij), LSE_i = m_i + ln(denominator).
//
// Band kernel. One CTA = 128 query rows of one head against the 128-key tiles of its band (row
// i sits at position q_off + i: q_off = 0 for whole sequences, the prefix length for a chunk
// prefilled against cached keys):
// tiles j_lo .. j_hi where the band is [i - W + 1, i] (SWA, at most 2 tiles for W = 128:
// "MiMo-V2-Flash 架构 QA" Q3.6) or [0, i] (GA; tiles above the diagonal are never visited).
//
// Roles (224 threads):
//   warps 0-3  softmax + epilogue: thread t owns query row t (TMEM lane t). It reads its row of
//              S from TMEM, runs the online softmax seeded with the sink (m0 = sink, l0 = 1),
//              writes P (bf16 pairs) back over its S row in TMEM (the A operand of P.V),
//              rescales its O row in TMEM when needed, and at the end normalises O and writes
//              O (bf16) and LSE.
//   warp 4     TMA producer for Q (once) and K tiles (2-stage ring).
//   warp 5     TMA producer for V tiles (2-stage ring).
//   warp 6     TMEM allocator and the single UMMA issuer: S = Q K^T (M128 N128 K16 x 12) into
//              one of three S buffers in TMEM, O += P V (M128 N128 K16 x 8, A = P from TMEM)
//              into O in TMEM (3 x 128 S columns + 128 O columns fill the 512). S_{j+3}
//              reuses the buffer of P_j once P_j V_j is done, long after it was issued.
// The issue order S_0, S_1, {PV_j, S_{j+2}} keeps S two tiles ahead: the tensor cores compute
// S_{j+2} while the softmax warps work on S_j, and S_{j+1} is ready when they finish; the
// softmax waits for PV_{j-1} only when it has to rescale O.
//
// One row sum, of the fp32 P: it normalises O (whose P.V MMA multiplies P rounded to bf16,
// a relative error of at most 2^-9 per weight) and gives LSE. A second sum of the rounded P, for
// O alone, cost three instructions per score pair in the softmax, which sets this kernel's pace
// (5 % of the GA prefill's time).
//
// Lazy rescaling: the running max used for the exponent is only raised when a tile's row max
// exceeds it by more than 8 (log2 units); P values stay <= 2^8 and the final O / l and LSE are
// exact for whatever reference max was used.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace pf {
constexpr int BM = 128;                  // query rows per CTA
constexpr int BN = 128;                  // keys per tile
constexpr int ROW_BYTES = 128;           // one 64-element bf16 chunk row (the swizzle width)
constexpr int Q_REGION = BM * ROW_BYTES; // 16 KB: 128 rows x 64 dims
constexpr int Q_BYTES = 3 * Q_REGION;    // 192 dims
constexpr int K_REGION = BN * ROW_BYTES;
constexpr int K_BYTES = 3 * K_REGION;
constexpr int V_BYTES = 2 * K_REGION;    // 128 dims
constexpr int K_STAGES = 2;
constexpr int V_STAGES = 2;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + K_STAGES * K_BYTES;
constexpr int OFF_BAR = OFF_V + V_STAGES * V_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024; // barriers + 1 KB for aligning the base
constexpr int THREADS = 224;
constexpr int WARP_KLOAD = 4, WARP_VLOAD = 5, WARP_MMA = 6;
constexpr uint32_t TMEM_COLS = 512;
constexpr int S_BUFS = 3;                   // S / P buffers in TMEM, 128 columns each
constexpr uint32_t TMEM_O = S_BUFS * BN;    // O: the last 128 columns
constexpr float TAU = 8.0f;

enum Bar {
    B_Q = 0,
    B_KFULL = 1,   // + K stage
    B_KEMPTY = 3,  // + K stage
    B_VFULL = 5,   // + V stage
    B_VEMPTY = 7,  // + V stage
    B_SFULL = 9,   // + S buffer
    B_PFULL = 12,  // + S buffer
    B_PVDONE = 15, // + S buffer
    B_DRAIN = 18,
    NUM_BARS = 19
};
} // namespace pf

// max(a, b, c) in one instruction (the three-input form of max.f32, sm_100 and later): the row
// maximum over 128 scores takes 64 of them instead of 128.
SA_DEV float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Where key tile j (positions 128 j .. 128 j + 127) of sequence b comes from: the K / V tensors
// at (row, block) = (position, sequence), or, for a paged prefix, a page of the pool below the
// prefix (a page id outside the pool reads zeros) and the chunk's own tensors above it.
struct PrefillTile {
    bool pool;
    int row, blk;
};

SA_DEV PrefillTile prefill_tile(const PrefillParams &p, int b, int j)
{
    const int pos = j * pf::BN;
    if (!p.paged)
        return PrefillTile{false, pos, b};
    if (pos >= p.q_off)
        return PrefillTile{false, pos - p.q_off, b};
    const int pg = pos / p.page_size;
    const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
    return PrefillTile{true, pos - pg * p.page_size, (pid >= 0 && pid < p.num_pages) ? pid : p.num_pages};
}

__global__ void __launch_bounds__(pf::THREADS, 1)
    prefill_band_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKp,
                        const __grid_constant__ CUtensorMap tmVp, const PrefillParams p)
{
    using namespace pf;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- which tile: (query tile, batch, head), head fastest so the CTAs of one KV group run
    // together and share K/V through L2; for GA the longest (last) query tiles go first.
    const int per_tile = p.B * p.Hq;
    const int t_idx = blockIdx.x / per_tile;
    const int qt = (p.window > 0) ? t_idx : (p.n_qtiles - 1 - t_idx);
    const int rem = blockIdx.x - t_idx * per_tile;
    const int b = rem / p.Hq;
    const int h = rem - b * p.Hq;
    const int g = h / p.G;
    const int r0 = qt * BM;                     // first query row of the tile (of the L rows)
    const int r_last = min(r0 + BM, p.L) - 1;
    const int a0 = p.q_off + r0;                // its position in the sequence (keys index it)
    const int k_lo = (p.window > 0) ? max(0, a0 - p.window + 1) : 0;
    const int j_lo = k_lo / BN;
    const int j_hi = (p.q_off + r_last) / BN;
    const int n_tiles = j_hi - j_lo + 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_Q], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], 1);
            mbar_init(&bars[B_VFULL + i], 1);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        for (int i = 0; i < S_BUFS; ++i) {
            mbar_init(&bars[B_SFULL + i], 1);
            mbar_init(&bars[B_PFULL + i], 128);
            mbar_init(&bars[B_PVDONE + i], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == WARP_KLOAD) {
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            mbar_arrive_expect_tx(&bars[B_Q], Q_BYTES);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(smem + OFF_Q + c * Q_REGION, &tmQ, &bars[B_Q], c * 64, h, r0, b);
            int issued = 0;
            for (int idx = 0; idx < n_tiles; ++idx) {
                const int s = idx & 1;
                if (idx >= 2 && !mbar_wait(&bars[B_KEMPTY + s], ((idx >> 1) - 1) & 1, abort, 1u))
                    break;
                const int j = j_lo + idx;
                const PrefillTile tl = prefill_tile(p, b, j);
                mbar_arrive_expect_tx(&bars[B_KFULL + s], K_BYTES);
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + OFF_K + s * K_BYTES + c * K_REGION, tl.pool ? &tmKp : &tmK,
                                &bars[B_KFULL + s], c * 64, g, tl.row, tl.blk);
                issued = idx + 1;
            }
            // make sure no copy of ours is still landing in shared memory when the CTA ends
            for (int idx = max(0, issued - 2); idx < issued; ++idx)
                mbar_wait_drain(&bars[B_KFULL + (idx & 1)], (idx >> 1) & 1);
            mbar_wait_drain(&bars[B_Q], 0);
        }
        __syncwarp();
    } else if (warp == WARP_VLOAD) {
        if (lane == 0) {
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int idx = 0; idx < n_tiles; ++idx) {
                const int vs = idx & 1;
                if (idx >= 2 && !mbar_wait(&bars[B_VEMPTY + vs], ((idx >> 1) - 1) & 1, abort, 1u))
                    break;
                const int j = j_lo + idx;
                const PrefillTile tl = prefill_tile(p, b, j);
                mbar_arrive_expect_tx(&bars[B_VFULL + vs], V_BYTES);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(smem + OFF_V + vs * V_BYTES + c * K_REGION, tl.pool ? &tmVp : &tmV,
                                &bars[B_VFULL + vs], c * 64, g, tl.row, tl.blk);
                issued = idx + 1;
            }
            for (int idx = max(0, issued - 2); idx < issued; ++idx)
                mbar_wait_drain(&bars[B_VFULL + (idx & 1)], (idx >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
            const uint32_t idesc_o = umma_idesc_bf16(BM, 128, 1);
            const uint32_t sQ = smem_u32(smem + OFF_Q);
            const uint32_t sK = smem_u32(smem + OFF_K);
            const uint32_t sV = smem_u32(smem + OFF_V);
            bool ok = mbar_wait(&bars[B_Q], 0, abort, 1u);
            // S_idx = Q K_idx^T into S buffer idx % 3, from K stage idx & 1
            auto issue_s = [&](int idx) -> bool {
                const int ks = idx & 1, sb = idx % S_BUFS;
                if (!mbar_wait(&bars[B_KFULL + ks], (idx >> 1) & 1, abort, 1u))
                    return false;
                // the buffer holds P of tile idx - 3 until its P.V is done
                if (idx >= S_BUFS &&
                    !mbar_wait(&bars[B_PVDONE + sb], (idx / S_BUFS - 1) & 1, abort, 1u))
                    return false;
                tc_fence_after();
                const uint32_t d = tmem + sb * BN;
#pragma unroll
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t off = (kk >> 2) * Q_REGION + (kk & 3) * 32;
                    umma_ss(d, smem_desc_sw128(sQ + off, 16, 1024),
                            smem_desc_sw128(sK + ks * K_BYTES + off, 16, 1024), idesc_s, kk > 0);
                }
                umma_commit(&bars[B_SFULL + sb]);
                umma_commit(&bars[B_KEMPTY + ks]);
                return true;
            };
            // S runs two tiles ahead of P.V: S_0, S_1, then {P.V_idx, S_{idx+2}}. S_{idx+2} goes
            // into the buffer of P_{idx-1}, whose P.V was issued a whole group earlier, so the
            // tensor pipe always has work that does not wait for the softmax, and the softmax
            // warps find S_{idx+1} done when they finish P_idx.
            if (ok)
                ok = issue_s(0);
            if (ok && n_tiles > 1)
                ok = issue_s(1);
            for (int idx = 0; ok && idx < n_tiles; ++idx) {
                const int sb = idx % S_BUFS, vs = idx & 1;
                if (!mbar_wait(&bars[B_PFULL + sb], (idx / S_BUFS) & 1, abort, 1u))
                    break;
                if (!mbar_wait(&bars[B_VFULL + vs], (idx >> 1) & 1, abort, 1u))
                    break;
                tc_fence_after();
                const uint32_t pt = tmem + sb * BN; // P over S
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // A = P (128 rows x 16 keys: 8 TMEM columns of bf16 pairs); B = V (16 keys x
                    // 128 dims, dims contiguous: MN-major, dims 64..127 one 16 KB region further on)
                    umma_ts(tmem + TMEM_O, pt + kk * 8,
                            smem_desc_sw128(sV + vs * V_BYTES + kk * 16 * ROW_BYTES, K_REGION,
                                            1024),
                            idesc_o, (idx > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[B_PVDONE + sb]);
                umma_commit(&bars[B_VEMPTY + vs]);
                if (idx + 2 < n_tiles && !issue_s(idx + 2))
                    break;
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait_drain(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps: thread = query row ----------------
        const int row = threadIdx.x;          // 0..127
        const int rp = r0 + row;              // this query row (of the L rows)
        const int ap = p.q_off + rp;          // its position in the sequence
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
        const float c_l2 = p.scale_log2; // > 0, so max(s) * c = max(s * c)
        // m_run: reference max (log2 units); l_exact: sum of fp32 P (normalises O, gives LSE),
        // seeded with the sink: m_0 = sink, l_0 = exp(sink - m_0) = 1.
        float m_run = sink_l2;
        float l_exact = (sink_l2 > -INFINITY) ? 1.f : 0.f;
        bool ok = true;
        for (int idx = 0; idx < n_tiles; ++idx) {
            const int sb = idx % S_BUFS;
            const int kbase = (j_lo + idx) * BN;
            ok = warp_wait(&bars[B_SFULL + sb], (idx / S_BUFS) & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            // The row's 128 scores in one TMEM round trip, kept in registers: the row maximum,
            // then P from the same registers (1.5 % faster on GA prefill than two rolled passes
            // of four 32-column loads each).
            const uint32_t saddr = tmem + lane_addr + sb * BN;
            // mask only on tiles that cross the diagonal or the window's lower edge
            const bool need_mask = (kbase + BN - 1 > a0) ||
                                   (p.window > 0 && kbase < a0 + BM - p.window);
            const int hi = ap - kbase;                                       // keep c <= hi
            const int lo = (p.window > 0) ? ap - p.window + 1 - kbase : -BN; // keep c >= lo
            // eight independent running maxima: short dependency chains
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx8[i] = -INFINITY;
            uint32_t sr[128];
            tmem_ld128(saddr, sr);
            if (need_mask) {
#pragma unroll
                for (int e = 0; e < 128; ++e)
                    if (e > hi || e < lo)
                        sr[e] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int e = 0; e < 128; e += 2)
                mx8[(e >> 1) & 7] =
                    fmax3(mx8[(e >> 1) & 7], __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            mx *= c_l2;
            // The first tile sets the exact max (m = max(sink, row max)), so rows that see few
            // keys get their dominant term exactly 1; later tiles raise it lazily.
            const bool rescale = (idx == 0) ? (mx > m_run) : (mx > m_run + TAU);
            float alpha = 1.f;
            if (rescale) {
                alpha = fast_exp2(m_run - mx); // 0 when m_run is -inf
                l_exact *= alpha;
                m_run = mx;
            }
            // O is only touched when one of this warp's rows raises its max: then wait for the
            // P.V of the previous tile (O up to date) and rescale. Otherwise P of this tile goes
            // into its own S buffer while that P.V may still run.
            if (idx > 0 && __any_sync(0xffffffffu, rescale)) {
                const int pb = (idx - 1) % S_BUFS;
                ok = warp_wait(&bars[B_PVDONE + pb], ((idx - 1) / S_BUFS) & 1, abort);
                if (!ok)
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32_sync(tmem + lane_addr + TMEM_O + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem + lane_addr + TMEM_O + c * 32, o);
                }
                tmem_st_wait();
            }
            const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
            float pe[4] = {0.f, 0.f, 0.f, 0.f};
            // P (bf16 pairs: keys 2c, 2c + 1 in column c) over this row's S in TMEM: chunk c0's
            // 16 columns of P land on scores already read (columns < c0 + 32)
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const float e0 = fast_exp2(fmaf(__uint_as_float(sr[c0 + 2 * u]), c_l2, neg_m));
                    const float e1 = fast_exp2(fmaf(__uint_as_float(sr[c0 + 2 * u + 1]), c_l2, neg_m));
                    pk[u] = pack_bf16x2(e0, e1);
                    pe[u & 3] += e0 + e1;
                }
                tmem_st8(saddr + c0 / 2, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
                tmem_st8(saddr + c0 / 2 + 8, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14],
                         pk[15]);
            }
            l_exact += (pe[0] + pe[1]) + (pe[2] + pe[3]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + sb]);
        }
        if (ok && n_tiles > 0)
            ok = warp_wait(&bars[B_PVDONE + (n_tiles - 1) % S_BUFS],
                           ((n_tiles - 1) / S_BUFS) & 1, abort);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l_exact;
            const bool valid = rp < p.L;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.o_sb +
                                  (int64_t)rp * p.o_sl + (int64_t)h * p.o_sh;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32_sync(tmem + lane_addr + TMEM_O + c * 32, o);
                if (valid) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(o[v4 * 8 + 0]) * inv_l,
                                           __uint_as_float(o[v4 * 8 + 1]) * inv_l);
                        pk.y = pack_bf16x2(__uint_as_float(o[v4 * 8 + 2]) * inv_l,
                                           __uint_as_float(o[v4 * 8 + 3]) * inv_l);
                        pk.z = pack_bf16x2(__uint_as_float(o[v4 * 8 + 4]) * inv_l,
                                           __uint_as_float(o[v4 * 8 + 5]) * inv_l);
                        pk.w = pack_bf16x2(__uint_as_float(o[v4 * 8 + 6]) * inv_l,
                                           __uint_as_float(o[v4 * 8 + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + v4 * 8) = pk;
                    }
                }
            }
            if (valid && p.lse)
                p.lse[((int64_t)b * p.Hq + h) * p.L + rp] = (m_run + fast_log2(l_exact)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_prefill_band(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                const CUtensorMap &tmV, const CUtensorMap &tmKp,
                                const CUtensorMap &tmVp, const PrefillParams &p,
                                cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(prefill_band_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    pf::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = (int64_t)p.n_qtiles * p.B * p.Hq;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    prefill_band_kernel<<<(unsigned)blocks, pf::THREADS, pf::SMEM_BYTES, stream>>>(tmQ, tmK, tmV,
                                                                                    tmKp, tmVp, p);
    return cudaGetLastError();
}

} // namespace sinkattn
