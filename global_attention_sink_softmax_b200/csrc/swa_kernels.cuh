// Sliding-window sink attention prefill, GQA-packed and persistent (sm_100a, tcgen05).
//
// Same result as the band kernel ("MiMo-V2-Flash 架构 QA" Q3.7/Q3.8 with the window of
// "MiMo-V2-Flash 模型架构深度拆解" CH10.3), arranged for the HBM-bound SWA case.
//
// Work item = (sequence b, KV head g, block of P = 128 / G consecutive positions). Its 128 MMA
// rows are the P positions x the G query heads of the group (row = position * G + head), so
// one K/V span feeds the whole GQA group inside the CTA. The span is the NS = roundup16(P + W - 1)
// keys ending at the block's last position: every row's W-key window lies inside it, and only
// the first / last few columns of each row are masked. One MMA pass per item: S = Q K^T
// (M128 x NS x 192) and O = P V (M128 x 128 x NS); no online rescaling is needed.
//
// The grid is one persistent CTA per SM walking a contiguous run of items (positions fastest,
// so consecutive items share most of their span in L2). Q is double-buffered in shared memory
// and streams one item ahead; K of item n+1 loads once S of item n is computed, V of item n+1
// once P.V of item n is done. S is double-buffered in tensor memory (2 x NS columns), and the
// softmax writes P (bf16) over the scores it has consumed, so P.V takes its A operand straight
// from tensor memory; O (128 columns) is read out by a separate epilogue warpgroup.
//
// Roles (352 threads): warps 0-3 softmax (thread = row = TMEM lane): a max pass and an exp pass
// over the row's scores, P back into TMEM, row statistics to shared memory; warps 4-7
// epilogue: O / l and LSE to global memory; warp 8 TMA producer for Q and K, warp 10 for V;
// warp 9 TMEM allocator + single-thread UMMA issuer, issuing S_0, {S_{n+1}, PV_n}. Waits are
// bounded as in the band kernel.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace sw {
constexpr int THREADS = 352;
constexpr int WARP_LOAD = 8, WARP_MMA = 9, WARP_VLOAD = 10;
constexpr int ROW = 128;          // bytes per swizzled row (64 bf16)
constexpr int Q_REGION = 128 * ROW;
constexpr int Q_BYTES = 3 * Q_REGION;
constexpr int MAX_NS = 192;       // S double buffer (2 x 192) + O (128) = 512 TMEM columns
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 384;  // S buffer i at i * NS; P of that item overwrites its first NS/2
constexpr int GROUP = 3;          // 16-column TMEM loads per round trip

enum Bar {
    Q_FULL = 0,      // + Q buffer
    Q_EMPTY = 2,     // + Q buffer
    K_FULL = 4, K_EMPTY, V_FULL, V_EMPTY,
    S_FULL = 8,      // + S buffer
    S_FREE = 10,     // + S buffer (S and the P that overwrote it are consumed)
    P_FULL = 12, PV_DONE, O_FREE,
    STATS_FULL = 15, // + stats buffer
    STATS_FREE = 17, // + stats buffer
    DRAIN = 19, NUM_BARS
};

__host__ __device__ constexpr bool counted_by_rows(int i)
{
    return i == P_FULL || i == O_FREE || (i >= STATS_FULL && i < STATS_FREE + 2);
}

// shared-memory plan for a key span of ns keys (ns a multiple of 16)
__host__ __device__ constexpr int k_bytes(int ns) { return 3 * ns * ROW; }
__host__ __device__ constexpr int v_bytes(int ns) { return 2 * ns * ROW; }
__host__ __device__ constexpr int off_k() { return 2 * Q_BYTES; }
__host__ __device__ constexpr int off_v(int ns) { return off_k() + k_bytes(ns); }
__host__ __device__ constexpr int off_stats(int ns) { return off_v(ns) + v_bytes(ns); }
__host__ __device__ constexpr int off_bar(int ns) { return off_stats(ns) + 2 * 128 * 16; }
__host__ __device__ constexpr int smem_bytes(int ns) { return off_bar(ns) + 256 + 1024; }
} // namespace sw

// Loads GROUP 16-column chunks of a row's scores (one TMEM round trip).
SA_DEV void swa_load_group(uint32_t taddr, int g0, int nch, uint32_t (&r)[sw::GROUP][16])
{
    using namespace sw;
#pragma unroll
    for (int k = 0; k < GROUP; ++k)
        if (g0 + k < nch)
            tmem_ld16(taddr + (g0 + k) * 16, r[k]);
    tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < GROUP; ++k)
#pragma unroll
        for (int i = 0; i < 16; i += 8)
            asm volatile("" : "+r"(r[k][i]), "+r"(r[k][i + 1]), "+r"(r[k][i + 2]), "+r"(r[k][i + 3]),
                         "+r"(r[k][i + 4]), "+r"(r[k][i + 5]), "+r"(r[k][i + 6]),
                         "+r"(r[k][i + 7])::"memory");
}

// Row max of the raw visible scores of one row.
SA_DEV float swa_row_max(uint32_t taddr, int NS, int lo, int hi)
{
    using namespace sw;
    float mx = -INFINITY;
    for (int g0 = 0; g0 < NS / 16; g0 += GROUP) {
        uint32_t r[GROUP][16];
        swa_load_group(taddr, g0, NS / 16, r);
#pragma unroll
        for (int k = 0; k < GROUP; ++k) {
            if (g0 + k >= NS / 16)
                break;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c = (g0 + k) * 16 + u;
                if (c >= lo && c <= hi)
                    mx = fmaxf(mx, __uint_as_float(r[k][u]));
            }
        }
    }
    return mx;
}

// P = 2^(s c - m) for the visible columns of one row, as bf16 pairs written back into the
// same TMEM row (key 2j, 2j+1 -> column j, over scores already read); returns the sums of
// fp32 P (se) and of bf16-rounded P (sr). With m the true max (the sink or the largest score)
// the dominant term is exactly 1.
SA_DEV void swa_softmax_exp(uint32_t taddr, int NS, int lo, int hi, float c_l2, float m,
                            float &se, float &sr)
{
    using namespace sw;
    const float neg_m = (m == -INFINITY) ? 0.f : -m;
    se = 0.f;
    sr = 0.f;
    for (int g0 = 0; g0 < NS / 16; g0 += GROUP) {
        uint32_t r[GROUP][16];
        swa_load_group(taddr, g0, NS / 16, r);
#pragma unroll
        for (int k = 0; k < GROUP; ++k) {
            const int ch = g0 + k;
            if (ch >= NS / 16)
                break;
            uint32_t pk[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
                const int c = ch * 16 + u;
                const float x0 = (c >= lo && c <= hi) ? __uint_as_float(r[k][u]) : -INFINITY;
                const float x1 = (c + 1 >= lo && c + 1 <= hi) ? __uint_as_float(r[k][u + 1]) : -INFINITY;
                const float e0 = fast_exp2(fmaf(x0, c_l2, neg_m));
                const float e1 = fast_exp2(fmaf(x1, c_l2, neg_m));
                se += e0 + e1;
                pk[u / 2] = pack_bf16x2(e0, e1);
                sr += sum_bf16x2(pk[u / 2]);
            }
            tmem_st8(taddr + ch * 8, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
        }
    }
    tmem_st_wait();
}

__global__ void __launch_bounds__(sw::THREADS, 1)
    prefill_swa_packed_kernel(const __grid_constant__ CUtensorMap tmQ,
                              const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const SwaParams p)
{
    using namespace sw;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = p.NS;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + off_bar(NS));
    float4 *stats = reinterpret_cast<float4 *>(smem + off_stats(NS)); // [2][128]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // contiguous run of items for this CTA
    const int it0 = (int)(((int64_t)blockIdx.x * p.n_items) / gridDim.x);
    const int it1 = (int)(((int64_t)(blockIdx.x + 1) * p.n_items) / gridDim.x);
    const int cnt = it1 - it0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i)
            mbar_init(&bars[i], counted_by_rows(i) ? 128 : 1);
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

    if (warp == WARP_LOAD) {
        if (lane == 0 && cnt > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            int issued = 0;
            for (int n = 0; n < cnt; ++n) {
                const int item = it0 + n;
                const int pblk = item % p.n_pblk;
                const int bg = item / p.n_pblk;
                const int g = bg % p.Hkv, b = bg / p.Hkv;
                const int p0 = pblk * p.P;
                const int ks = p0 + p.P - NS;
                const int qb = n & 1;
                // Q buffer qb was read by S of item n - 2; K by S of item n - 1
                if (n >= 2 && !mbar_wait(&bars[Q_EMPTY + qb], ((n >> 1) - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[Q_FULL + qb], Q_BYTES);
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + qb * Q_BYTES + c * Q_REGION, &tmQ, &bars[Q_FULL + qb],
                                c * 64, g * p.G, p0, b);
                if (n > 0 && !mbar_wait(&bars[K_EMPTY], (n - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[K_FULL], k_bytes(NS));
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + off_k() + c * NS * ROW, &tmK, &bars[K_FULL], c * 64, g, ks, b);
                issued = n + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int n = max(0, issued - 2); n < issued; ++n)
                mbar_wait_drain(&bars[Q_FULL + (n & 1)], (n >> 1) & 1);
            if (issued > 0)
                mbar_wait_drain(&bars[K_FULL], (issued - 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_VLOAD) {
        if (lane == 0 && cnt > 0) {
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int n = 0; n < cnt; ++n) {
                const int item = it0 + n;
                const int pblk = item % p.n_pblk;
                const int bg = item / p.n_pblk;
                const int g = bg % p.Hkv, b = bg / p.Hkv;
                const int ks = pblk * p.P + p.P - NS;
                // V of item n is free once P.V of item n - 1 is done
                if (n > 0 && !mbar_wait(&bars[V_EMPTY], (n - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[V_FULL], v_bytes(NS));
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(smem + off_v(NS) + c * NS * ROW, &tmV, &bars[V_FULL], c * 64, g, ks, b);
                issued = n + 1;
            }
            if (issued > 0)
                mbar_wait_drain(&bars[V_FULL], (issued - 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0 && cnt > 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, NS, 0);
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            const uint32_t sK = smem_u32(smem + off_k());
            const uint32_t sV = smem_u32(smem + off_v(NS));
            const int ksteps_pv = NS / 16;
            // S of item n into S buffer n & 1
            auto issue_s = [&](int n) -> bool {
                const int sb = n & 1;
                if (!mbar_wait(&bars[Q_FULL + sb], (n >> 1) & 1, abort, 1u) ||
                    !mbar_wait(&bars[K_FULL], n & 1, abort, 1u))
                    return false;
                // S buffer sb held S and P of item n - 2: free once that P.V is done
                if (n >= 2 && !mbar_wait(&bars[S_FREE + sb], ((n >> 1) - 1) & 1, abort, 1u))
                    return false;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + sb * Q_BYTES);
#pragma unroll
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    umma_ss(tmem + sb * NS, smem_desc_sw128(sQ + (kk >> 2) * Q_REGION + koff, 16, 1024),
                            smem_desc_sw128(sK + (kk >> 2) * NS * ROW + koff, 16, 1024), idesc_s,
                            kk > 0);
                }
                umma_commit(&bars[S_FULL + sb]);
                umma_commit(&bars[Q_EMPTY + sb]);
                umma_commit(&bars[K_EMPTY]);
                return true;
            };
            // issue order S_0, {S_{n+1}, PV_n}: the next item's S is computed while this item's
            // softmax runs
            bool ok = issue_s(0);
            for (int n = 0; ok && n < cnt; ++n) {
                if (n + 1 < cnt && !issue_s(n + 1))
                    break;
                if (!mbar_wait(&bars[P_FULL], n & 1, abort, 1u) ||
                    !mbar_wait(&bars[V_FULL], n & 1, abort, 1u))
                    break;
                // O was read out by the epilogue of item n - 1
                if (n >= 1 && !mbar_wait(&bars[O_FREE], (n - 1) & 1, abort, 1u))
                    break;
                tc_fence_after();
                const uint32_t pt = tmem + (n & 1) * NS; // P: 16 keys per 8 columns
                for (int kk = 0; kk < ksteps_pv; ++kk)
                    umma_ts(tmem + TMEM_O, pt + kk * 8,
                            smem_desc_sw128(sV + kk * 16 * ROW, NS * ROW, 1024), idesc_o, kk > 0);
                umma_commit(&bars[PV_DONE]);
                umma_commit(&bars[V_EMPTY]);
                umma_commit(&bars[S_FREE + (n & 1)]);
            }
            umma_commit(&bars[DRAIN]);
            mbar_wait_drain(&bars[DRAIN], 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- softmax warps: thread = MMA row ----------------
        const int row = threadIdx.x;
        const int l_local = row / p.G, h_local = row - l_local * p.G;
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        for (int n = 0; n < cnt; ++n) {
            const int item = it0 + n;
            const int pblk = item % p.n_pblk;
            const int g = (item / p.n_pblk) % p.Hkv;
            const int p0 = pblk * p.P;
            const int ks = p0 + p.P - NS;
            const int l = p0 + l_local;
            const int h = g * p.G + h_local;
            // visible columns: ks + c in [max(l - W + 1, 0), l]
            const int hi = l - ks;
            const int lo = max(l - p.W + 1, 0) - ks;
            const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            const int sb = n & 1;
            if (!warp_wait(&bars[S_FULL + sb], (n >> 1) & 1, abort))
                break;
            tc_fence_after();
            // m = max(sink, max_j a_j) in log2 units (the max includes the sink)
            const uint32_t saddr = tmem + lane_addr + sb * NS;
            const float mx = swa_row_max(saddr, NS, lo, hi);
            const float m = fmaxf(sink_l2, mx * p.scale_log2);
            float se, sr;
            swa_softmax_exp(saddr, NS, lo, hi, p.scale_log2, m, se, sr);
            tc_fence_before();
            mbar_arrive(&bars[P_FULL]);
            // the sink seeds both sums: exp(sink - m)
            const float s0 = (sink_l2 == -INFINITY) ? 0.f : fast_exp2(sink_l2 - m);
            // statistics for the epilogue; buffer sb was last read by the epilogue of n - 2
            if (n >= 2 && !warp_wait(&bars[STATS_FREE + sb], ((n >> 1) - 1) & 1, abort))
                break;
            stats[sb * 128 + row] = make_float4(m, s0 + se, s0 + sr, 0.f);
            mbar_arrive(&bars[STATS_FULL + sb]);
        }
    } else {
        // ---------------- epilogue warps: O = (P V) / l_round, LSE = m + log2(l_exact) ----
        const int row = threadIdx.x - 128;
        const int l_local = row / p.G, h_local = row - l_local * p.G;
        const uint32_t lane_addr = (uint32_t)((warp - 4) * 32) << 16;
        for (int n = 0; n < cnt; ++n) {
            const int item = it0 + n;
            const int pblk = item % p.n_pblk;
            const int bg = item / p.n_pblk;
            const int g = bg % p.Hkv, b = bg / p.Hkv;
            const int l = pblk * p.P + l_local;
            const int h = g * p.G + h_local;
            const int sb = n & 1;
            if (!warp_wait(&bars[STATS_FULL + sb], (n >> 1) & 1, abort) ||
                !warp_wait(&bars[PV_DONE], n & 1, abort))
                break;
            tc_fence_after();
            const float4 st = stats[sb * 128 + row];
            mbar_arrive(&bars[STATS_FREE + sb]);
            const float inv_l = 1.f / st.z;
            const bool valid = l < p.L;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.o_sb +
                                  (int64_t)l * p.o_sl + (int64_t)h * p.o_sh;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32_sync(tmem + lane_addr + TMEM_O + c * 32, o);
                if (c == 3) {
                    // O is read: the next P.V may overwrite it
                    tc_fence_before();
                    mbar_arrive(&bars[O_FREE]);
                }
                if (valid) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * inv_l,
                                           __uint_as_float(o[v * 8 + 1]) * inv_l);
                        pk.y = pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * inv_l,
                                           __uint_as_float(o[v * 8 + 3]) * inv_l);
                        pk.z = pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * inv_l,
                                           __uint_as_float(o[v * 8 + 5]) * inv_l);
                        pk.w = pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * inv_l,
                                           __uint_as_float(o[v * 8 + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + v * 8) = pk;
                    }
                }
            }
            if (valid && p.lse)
                p.lse[((int64_t)b * p.Hq + h) * p.L + l] = (st.x + fast_log2(st.y)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

int swa_packed_smem_bytes(int ns) { return ns <= sw::MAX_NS ? sw::smem_bytes(ns) : 1 << 30; }

cudaError_t launch_prefill_swa_packed(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                      const CUtensorMap &tmV, const SwaParams &p, int grid,
                                      cudaStream_t stream)
{
    static int configured_devices = 0; // bit per device: shared-memory opt-in done
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 32 && !(configured_devices & (1 << dev))) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess)
            return e;
        e = cudaFuncSetAttribute(prefill_swa_packed_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (e != cudaSuccess)
            return e;
        configured_devices |= (1 << dev);
    }
    if (grid <= 0)
        return cudaSuccess;
    prefill_swa_packed_kernel<<<grid, sw::THREADS, sw::smem_bytes(p.NS), stream>>>(tmQ, tmK, tmV, p);
    return cudaGetLastError();
}

} // namespace sinkattn
