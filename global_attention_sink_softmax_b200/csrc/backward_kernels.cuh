// Backward of the sink-softmax attention prefill on tcgen05 tensor cores (sm_100a): the training
// variant.
//
// The sink is a per-head logit appended after the scaled, masked scores, softmaxed with them and
// dropped ("MiMo-V2-Flash 模型架构深度拆解" CH10.1), so its gradient is that column's softmax
// gradient with a zero value. With P_ij = exp(a_ij - LSE_i), LSE the forward's (sink included),
//     delta_i = <dO_i, O_i>,   dS_ij = P_ij (<dO_i, v_j> - delta_i),
//     dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,   dv_j = sum_i P_ij dO_i,
//     dsink_h = -sum_i exp(sink_h - LSE_i) delta_i,
// the sums over i running over every query row of the KV head's GQA group. P is recomputed from
// the saved LSE, so no row maximum is needed and a tile's columns can be handled in any order.
//
// Three launches:
//   bwd_delta_kernel  one warp per 32 rows of one (sequence, head): delta, and dsink by one atomic
//                     per warp;
//   bwd_dkdv_kernel   one CTA per (128-key tile, sequence, KV head), looping over the group's
//                     heads and 64-row query blocks; dK and dV accumulate in tensor memory;
//   bwd_dq_kernel     one CTA per (128-row query tile, sequence, head), looping over the key
//                     tiles its rows see; dQ accumulates in tensor memory.
// All contractions are tcgen05 MMAs (kind::f16, bf16 in, fp32 accumulate): S and dP with both
// operands K-major in shared memory, dV / dK / dQ with P or dS from tensor memory (bf16 pairs)
// and Q, dO or K as an MN-major B operand. Waits are bounded as in the forward kernels.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

// ---------------------------------------------------------------------------------------------
// delta and dsink
// ---------------------------------------------------------------------------------------------
namespace bd {
constexpr int ROWS = 32; // rows per warp
constexpr int WARPS = 8;
} // namespace bd

__global__ void __launch_bounds__(bd::WARPS * 32) bwd_delta_kernel(const BwdParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = (int64_t)blockIdx.x * bd::WARPS + (threadIdx.x >> 5);
    const int nblk = (p.L + bd::ROWS - 1) / bd::ROWS;
    if (w >= (int64_t)p.B * p.Hq * nblk)
        return;
    const int blk = (int)(w % nblk);
    const int bh = (int)(w / nblk);
    const int h = bh % p.Hq, b = bh / p.Hq;
    const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
    float acc = 0.f;
    for (int r = 0; r < bd::ROWS; ++r) {
        const int i = blk * bd::ROWS + r;
        if (i >= p.L)
            break;
        // lane covers dims 4 lane .. 4 lane + 3 of the 128
        const uint2 x = *reinterpret_cast<const uint2 *>(
            p.dout + (int64_t)b * p.do_sb + (int64_t)i * p.do_sl + (int64_t)h * p.do_sh + 4 * lane);
        const uint2 y = *reinterpret_cast<const uint2 *>(
            p.o + (int64_t)b * p.o_sb + (int64_t)i * p.o_sl + (int64_t)h * p.o_sh + 4 * lane);
        float d = __uint_as_float(x.x << 16) * __uint_as_float(y.x << 16);
        d = fmaf(__uint_as_float(x.x & 0xffff0000u), __uint_as_float(y.x & 0xffff0000u), d);
        d = fmaf(__uint_as_float(x.y << 16), __uint_as_float(y.y << 16), d);
        d = fmaf(__uint_as_float(x.y & 0xffff0000u), __uint_as_float(y.y & 0xffff0000u), d);
#pragma unroll
        for (int s = 16; s > 0; s >>= 1)
            d += __shfl_xor_sync(0xffffffffu, d, s);
        const int64_t row = ((int64_t)b * p.Hq + h) * p.L + i;
        if (lane == 0) {
            p.delta[row] = d;
            if (sink_l2 > -INFINITY)
                acc += fast_exp2(sink_l2 - p.lse[row] * kLog2e) * d;
        }
    }
    if (lane == 0 && p.dsink && acc != 0.f)
        atomicAdd(&p.dsink[h], -acc);
}

// ---------------------------------------------------------------------------------------------
// shared by the two MMA kernels
// ---------------------------------------------------------------------------------------------
namespace bw {
constexpr int ROW = 128;                 // bytes per swizzled row (64 bf16)
constexpr int R128 = 128 * ROW;          // 16 KB: 128 rows x 64 dims
constexpr int R64 = 64 * ROW;            // 8 KB: 64 rows x 64 dims
constexpr int THREADS = 192;             // warps 0-3 rows, warp 4 TMA producer, warp 5 MMA
constexpr int WARP_LOAD = 4, WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 512;
} // namespace bw

// Two 32-column loads, then one wait; the wait names the registers so no use of them can be
// scheduled before it.
SA_DEV void tmem_ld32x2_sync(uint32_t ta, uint32_t (&a)[32], uint32_t tb, uint32_t (&b)[32])
{
    tmem_ld32(ta, a);
    tmem_ld32(tb, b);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        asm volatile("" : "+r"(a[i]), "+r"(a[i + 1]), "+r"(a[i + 2]), "+r"(a[i + 3]),
                     "+r"(a[i + 4]), "+r"(a[i + 5]), "+r"(a[i + 6]), "+r"(a[i + 7])::"memory");
        asm volatile("" : "+r"(b[i]), "+r"(b[i + 1]), "+r"(b[i + 2]), "+r"(b[i + 3]),
                     "+r"(b[i + 4]), "+r"(b[i + 5]), "+r"(b[i + 6]), "+r"(b[i + 7])::"memory");
    }
}

// 32 rows x 16 columns of packed bf16 pairs into tensor memory (two 8-column stores)
SA_DEV void tmem_st16(uint32_t taddr, const uint32_t (&w)[16])
{
    tmem_st8(taddr, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    tmem_st8(taddr + 8, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
}

// ---------------------------------------------------------------------------------------------
// dQ: one CTA per (128-row query tile, sequence, head)
// ---------------------------------------------------------------------------------------------
// Per key tile j of the band: S = Q K_j^T and dP = dO V_j^T into tensor memory; the row warps
// (thread = query row) turn them into dS = P (dP - delta) as bf16 pairs in 64 columns of their
// own; dQ += dS K_j with K_j as the MN-major B operand. K is double-buffered (it serves S and
// dQ), V single-buffered (it serves dP only). S_{j+1} is issued as soon as the row warps have
// read S_j and dP_j (SDP_FREE), so it runs while they compute dS_j; dP_{j+1} follows dQ_j
// (V_{j+1} lands after dP_j has read V_j); the row warps store dS_{j+1} once dQ_j has read dS_j.
namespace bq {
using namespace bw;
constexpr int OFF_Q = 0;                  // 3 x 16 KB
constexpr int OFF_DO = OFF_Q + 3 * R128;  // 2 x 16 KB
constexpr int OFF_K = OFF_DO + 2 * R128;  // 2 stages x 48 KB
constexpr int OFF_V = OFF_K + 6 * R128;   // 32 KB
constexpr int OFF_BAR = OFF_V + 2 * R128;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DS = 448; // tensor-memory columns
enum Bar { QD_FULL = 0, K_FULL = 1, K_EMPTY = 3, V_FULL = 5, V_EMPTY = 6, S_FULL = 7, DS_FULL = 8,
           DQ_DONE = 9, DRAIN = 10, SDP_FREE = 11, NUM_BARS = 12 };
} // namespace bq

__global__ void __launch_bounds__(bw::THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p)
{
    using namespace bq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // (query tile, sequence, head), head fastest; for GA the longest (last) query tiles first
    const int per_tile = p.B * p.Hq;
    const int t_idx = blockIdx.x / per_tile;
    const int n_qt = (p.L + 127) / 128;
    const int qt = (p.window > 0) ? t_idx : (n_qt - 1 - t_idx);
    const int rem = blockIdx.x - t_idx * per_tile;
    const int b = rem / p.Hq, h = rem - b * p.Hq, g = h / p.G;
    const int q0 = qt * 128;
    const int q_last = min(q0 + 128, p.L) - 1;
    const int j_lo = (p.window > 0) ? max(0, q0 - p.window + 1) / 128 : 0;
    const int j_hi = q_last / 128;
    const int n_tiles = j_hi - j_lo + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i)
            mbar_init(&bars[i], (i == DS_FULL || i == SDP_FREE) ? 128 : 1);
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
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(&bars[QD_FULL], 5 * R128);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(smem + OFF_Q + c * R128, &tmQ, &bars[QD_FULL], c * 64, h, q0, b);
            for (int c = 0; c < 2; ++c)
                tma_load_4d(smem + OFF_DO + c * R128, &tmDO, &bars[QD_FULL], c * 64, h, q0, b);
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int ks = j & 1, kt = j_lo + j;
                if (j >= 2 && !mbar_wait(&bars[K_EMPTY + ks], ((j >> 1) - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[K_FULL + ks], 3 * R128);
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + OFF_K + ks * 3 * R128 + c * R128, &tmK, &bars[K_FULL + ks],
                                c * 64, g, kt * 128, b);
                k_issued = j + 1;
                if (j >= 1 && !mbar_wait(&bars[V_EMPTY], (j - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[V_FULL], 2 * R128);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(smem + OFF_V + c * R128, &tmV, &bars[V_FULL], c * 64, g, kt * 128, b);
                v_issued = j + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int j = max(0, k_issued - 2); j < k_issued; ++j)
                mbar_wait_drain(&bars[K_FULL + (j & 1)], (j >> 1) & 1);
            if (v_issued > 0)
                mbar_wait_drain(&bars[V_FULL], (v_issued - 1) & 1);
            mbar_wait_drain(&bars[QD_FULL], 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, 128, 0);
            const uint32_t idesc_q = umma_idesc_bf16(128, 192, 1);
            const uint32_t sQ = smem_u32(smem + OFF_Q), sDO = smem_u32(smem + OFF_DO);
            const uint32_t sK = smem_u32(smem + OFF_K), sV = smem_u32(smem + OFF_V);
            bool ok = mbar_wait(&bars[QD_FULL], 0, abort, 1u);
            // S_j = Q K_j^T (its K stage landed) and dP_j = dO V_j^T (V landed); both into
            // columns the row warps have finished reading for tile j - 1
            auto issue_s = [&](int j) -> bool {
                const uint32_t kb = sK + (j & 1) * 3 * R128;
                if (!mbar_wait(&bars[K_FULL + (j & 1)], (j >> 1) & 1, abort, 1u))
                    return false;
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t off = (kk >> 2) * R128 + (kk & 3) * 32;
                    umma_ss(tmem + T_S, smem_desc_sw128(sQ + off, 16, 1024),
                            smem_desc_sw128(kb + off, 16, 1024), idesc_s, kk > 0);
                }
                return true;
            };
            auto issue_dp = [&](int j) -> bool {
                if (!mbar_wait(&bars[V_FULL], j & 1, abort, 1u))
                    return false;
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * R128 + (kk & 3) * 32;
                    umma_ss(tmem + T_DP, smem_desc_sw128(sDO + off, 16, 1024),
                            smem_desc_sw128(sV + off, 16, 1024), idesc_s, kk > 0);
                }
                umma_commit(&bars[S_FULL]);
                umma_commit(&bars[V_EMPTY]);
                return true;
            };
            if (ok && n_tiles > 0)
                ok = issue_s(0) && issue_dp(0);
            // tile j + 1's S runs while the row warps turn tile j into dS, and its dP after
            // dQ_j (V_{j+1} is loaded only once dP_j has read V_j)
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int ks = j & 1;
                const uint32_t kb = sK + ks * 3 * R128;
                const bool more = j + 1 < n_tiles;
                if (more && (!mbar_wait(&bars[SDP_FREE], j & 1, abort, 1u) || !issue_s(j + 1)))
                    break;
                if (!mbar_wait(&bars[DS_FULL], j & 1, abort, 1u))
                    break;
                tc_fence_after();
                // dQ += dS K_j: A = dS (128 rows x 16 keys per step, 8 columns of bf16 pairs),
                // B = K_j (16 keys x 192 dims, dims contiguous: MN-major, 64-dim regions 16 KB apart)
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + T_DQ, tmem + T_DS + kk * 8,
                            smem_desc_sw128(kb + kk * 16 * ROW, R128, 1024), idesc_q,
                            (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&bars[DQ_DONE]);
                umma_commit(&bars[K_EMPTY + ks]);
                if (more && !issue_dp(j + 1))
                    break;
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[DRAIN]);
            mbar_wait_drain(&bars[DRAIN], 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- row warps: thread = query row = TMEM lane ----------------
        const int row = threadIdx.x;
        const int i = q0 + row;
        const bool valid = i < p.L;
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const int64_t lrow = ((int64_t)b * p.Hq + h) * p.L + i;
        // P = 2^(s c - LSE log2 e): rows past L get +inf (P = 0)
        const float lse2 = valid ? p.lse[lrow] * kLog2e : INFINITY;
        const float delta = valid ? p.delta[lrow] : 0.f;
        const float c_l2 = p.scale_log2;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int kbase = (j_lo + j) * 128;
            ok = warp_wait(&bars[S_FULL], j & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            const int hi = min(i, p.L - 1) - kbase;                             // keep c <= hi
            const int lo = (p.window > 0) ? i - p.window + 1 - kbase : -128;   // keep c >= lo
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t s[32], dp[32];
                tmem_ld32x2_sync(tmem + lane_addr + T_S + c * 32, s, tmem + lane_addr + T_DP + c * 32, dp);
                if (c == 3) {
                    // tile j's S and dP are all read: the issuer may compute tile j + 1's
                    tc_fence_before();
                    mbar_arrive(&bars[SDP_FREE]);
                }
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float d2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = c * 32 + 2 * e + u;
                        const bool vis = col <= hi && col >= lo;
                        const float pr = vis ? fast_exp2(fmaf(__uint_as_float(s[2 * e + u]), c_l2, -lse2)) : 0.f;
                        d2[u] = pr * (__uint_as_float(dp[2 * e + u]) - delta);
                    }
                    w[e] = pack_bf16x2(d2[0], d2[1]);
                }
                // dS (bf16 pairs) into its own 64 columns, once dQ_{j-1} has read tile j - 1's
                if (c == 0 && j > 0) {
                    ok = warp_wait(&bars[DQ_DONE], (j - 1) & 1, abort);
                    if (!ok)
                        break;
                    tc_fence_after();
                }
                tmem_st16(tmem + lane_addr + T_DS + c * 16, w);
            }
            if (!ok)
                break;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[DS_FULL]);
        }
        if (ok)
            ok = warp_wait(&bars[DQ_DONE], (n_tiles - 1) & 1, abort);
        if (ok) {
            tc_fence_after();
            float *drow = p.dq + (int64_t)b * p.dq_sb + (int64_t)i * p.dq_sl + (int64_t)h * p.dq_sh;
#pragma unroll 1
            for (int c = 0; c < 6; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem + lane_addr + T_DQ + c * 32, r);
                if (valid) {
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4) {
                        float4 f;
                        f.x = __uint_as_float(r[4 * v4 + 0]) * p.scale;
                        f.y = __uint_as_float(r[4 * v4 + 1]) * p.scale;
                        f.z = __uint_as_float(r[4 * v4 + 2]) * p.scale;
                        f.w = __uint_as_float(r[4 * v4 + 3]) * p.scale;
                        *reinterpret_cast<float4 *>(drow + c * 32 + 4 * v4) = f;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------------------------
// dK, dV: one CTA per (128-key tile, sequence, KV head)
// ---------------------------------------------------------------------------------------------
// The CTA holds its K and V tiles and walks the steps (head hh of the group, 64-row query block
// qb) whose rows see its keys. Per step: S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 64
// rows) into tensor memory; the row warps (thread = key row) form P^T = exp(S^T c - LSE) and
// dS^T = P^T (dP^T - delta) for the 64 rows, as bf16 pairs in their own columns; then
// dV += P^T dO and dK += dS^T Q, with dO and Q as MN-major B operands. A step's Q, dO, LSE and
// delta come in a 3-stage ring. The two halves of a step overlap with the neighbouring steps:
// S^T and dP^T of step s + 1 are computed as soon as the row warps have read those of step s
// (SDP_FREE), while the row warps work, and the row warps store P^T / dS^T of step s + 1 once the
// dV / dK MMAs of step s have read theirs (DKV_DONE).
namespace bk {
using namespace bw;
constexpr int QB = 64;                         // query rows per step
constexpr int ST_Q = 0;                        // 3 x 8 KB
constexpr int ST_DO = 3 * R64;                 // 2 x 8 KB
constexpr int ST_LSE = 5 * R64;                // 64 floats of LSE log2 e, then 64 of delta
constexpr int STAGE = 5 * R64 + 1024;          // 41 KB, 1 KB aligned
constexpr int NST = 3;
constexpr int OFF_K = 0;                       // 3 x 16 KB
constexpr int OFF_V = 3 * R128;                // 2 x 16 KB
constexpr int OFF_ST = 5 * R128;               // stages
constexpr int OFF_BAR = OFF_ST + NST * STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t T_S = 0, T_DP = 64, T_P = 128, T_DS = 160, T_DV = 192, T_DK = 320;
enum Bar { KV_FULL = 0, ST_FULL = 1, ST_EMPTY = 4, S_FULL = 7, P_FULL = 8, DONE = 9,
           SDP_FREE = 10, DKV_DONE = 11, NUM_BARS = 12 };
} // namespace bk

__global__ void __launch_bounds__(bw::THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p)
{
    using namespace bk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // (key tile, sequence, KV head), KV head fastest; the first key tiles (most rows) first
    const int per_tile = p.B * p.Hkv;
    const int kt = blockIdx.x / per_tile;
    const int rem = blockIdx.x - kt * per_tile;
    const int b = rem / p.Hkv, g = rem - b * p.Hkv;
    const int k0 = kt * 128;
    const int k_last = min(k0 + 128, p.L) - 1;
    // rows that see a key of the tile: from k0 (causal) to k_last + W - 1 (window) or L - 1
    const int qb_lo = k0 / QB;
    const int q_hi = (p.window > 0) ? min(p.L - 1, k_last + p.window - 1) : p.L - 1;
    const int qb_hi = q_hi / QB;
    const int nqb = qb_hi - qb_lo + 1;
    const int n_steps = p.G * nqb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i)
            mbar_init(&bars[i], (i == P_FULL || i == SDP_FREE) ? 128 : 1);
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
        // ---- producer: the K / V tiles once; per step Q, dO by TMA and 64 LSE / delta values
        // by the warp's lanes
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(&bars[KV_FULL], 5 * R128);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(smem + OFF_K + c * R128, &tmK, &bars[KV_FULL], c * 64, g, k0, b);
            for (int c = 0; c < 2; ++c)
                tma_load_4d(smem + OFF_V + c * R128, &tmV, &bars[KV_FULL], c * 64, g, k0, b);
        }
        int issued = 0;
        for (int s = 0; s < n_steps; ++s) {
            const int st = s % NST;
            bool ok = true;
            if (lane == 0 && s >= NST)
                ok = mbar_wait(&bars[ST_EMPTY + st], ((s / NST) - 1) & 1, abort, 1u);
            if (!__shfl_sync(0xffffffffu, ok, 0))
                break;
            const int h = g * p.G + s / nqb;
            const int q0 = (qb_lo + s % nqb) * QB;
            uint8_t *stage = smem + OFF_ST + st * STAGE;
            float *lse2 = reinterpret_cast<float *>(stage + ST_LSE);
            const int64_t lrow = ((int64_t)b * p.Hq + h) * p.L;
            for (int e = lane; e < QB; e += 32) {
                const int i = q0 + e;
                lse2[e] = i < p.L ? p.lse[lrow + i] * kLog2e : INFINITY; // rows past L: P = 0
                lse2[QB + e] = i < p.L ? p.delta[lrow + i] : 0.f;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars[ST_FULL + st], 5 * R64);
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(stage + ST_Q + c * R64, &tmQ, &bars[ST_FULL + st], c * 64, h, q0, b);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(stage + ST_DO + c * R64, &tmDO, &bars[ST_FULL + st], c * 64, h, q0, b);
            }
            issued = s + 1;
        }
        // no copy of ours may still be landing when the CTA leaves
        if (lane == 0) {
            for (int s = max(0, issued - NST); s < issued; ++s)
                mbar_wait_drain(&bars[ST_FULL + s % NST], (s / NST) & 1);
            mbar_wait_drain(&bars[KV_FULL], 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, QB, 0);
            const uint32_t idesc_v = umma_idesc_bf16(128, 128, 1);
            const uint32_t idesc_k = umma_idesc_bf16(128, 192, 1);
            const uint32_t sK = smem_u32(smem + OFF_K), sV = smem_u32(smem + OFF_V);
            bool ok = mbar_wait(&bars[KV_FULL], 0, abort, 1u);
            // S^T = K Q^T and dP^T = V dO^T of step s into their columns (the row warps have read
            // those of step s - 1)
            auto issue_sdp = [&](int s) -> bool {
                const int st = s % NST;
                const uint32_t sQ = smem_u32(smem + OFF_ST + st * STAGE + ST_Q);
                const uint32_t sDO = smem_u32(smem + OFF_ST + st * STAGE + ST_DO);
                if (!mbar_wait(&bars[ST_FULL + st], (s / NST) & 1, abort, 1u))
                    return false;
                tc_fence_after();
                // S^T: A = 128 keys (K-major), B = 64 rows (K-major), 12 k-steps of 16 dims
#pragma unroll 1
                for (int kk = 0; kk < 12; ++kk)
                    umma_ss(tmem + T_S,
                            smem_desc_sw128(sK + (kk >> 2) * R128 + (kk & 3) * 32, 16, 1024),
                            smem_desc_sw128(sQ + (kk >> 2) * R64 + (kk & 3) * 32, 16, 1024),
                            idesc_s, kk > 0);
                // dP^T, 8 k-steps of 16 dims
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    umma_ss(tmem + T_DP,
                            smem_desc_sw128(sV + (kk >> 2) * R128 + (kk & 3) * 32, 16, 1024),
                            smem_desc_sw128(sDO + (kk >> 2) * R64 + (kk & 3) * 32, 16, 1024),
                            idesc_s, kk > 0);
                umma_commit(&bars[S_FULL]);
                return true;
            };
            if (ok && n_steps > 0)
                ok = issue_sdp(0);
            for (int s = 0; ok && s < n_steps; ++s) {
                const int st = s % NST;
                const uint32_t sQ = smem_u32(smem + OFF_ST + st * STAGE + ST_Q);
                const uint32_t sDO = smem_u32(smem + OFF_ST + st * STAGE + ST_DO);
                // step s + 1's S^T / dP^T, once the row warps hold step s's
                if (s + 1 < n_steps) {
                    if (!mbar_wait(&bars[SDP_FREE], s & 1, abort, 1u) || !issue_sdp(s + 1))
                        break;
                }
                if (!mbar_wait(&bars[P_FULL], s & 1, abort, 1u))
                    break;
                tc_fence_after();
                // dV += P^T dO and dK += dS^T Q: A from tensor memory (128 keys x 16 rows per step,
                // 8 columns of bf16 pairs); B = dO / Q (16 rows x 128 / 192 dims, dims contiguous:
                // MN-major, 64-dim regions 8 KB apart)
#pragma unroll 1
                for (int kk = 0; kk < QB / 16; ++kk) {
                    umma_ts(tmem + T_DV, tmem + T_P + kk * 8,
                            smem_desc_sw128(sDO + kk * 16 * ROW, R64, 1024), idesc_v,
                            (s > 0 || kk > 0) ? 1u : 0u);
                    umma_ts(tmem + T_DK, tmem + T_DS + kk * 8,
                            smem_desc_sw128(sQ + kk * 16 * ROW, R64, 1024), idesc_k,
                            (s > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[ST_EMPTY + st]);
                umma_commit(&bars[DKV_DONE]);
            }
            // every MMA of ours has finished before the row warps read dK / dV and TMEM is freed
            umma_commit(&bars[DONE]);
            mbar_wait_drain(&bars[DONE], 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- row warps: thread = key row = TMEM lane ----------------
        const int key = k0 + threadIdx.x;
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const float c_l2 = p.scale_log2;
        bool ok = true;
        for (int s = 0; s < n_steps; ++s) {
            const int st = s % NST;
            const int q0 = (qb_lo + s % nqb) * QB;
            const float *lse2 = reinterpret_cast<const float *>(smem + OFF_ST + st * STAGE + ST_LSE);
            // the stage's LSE / delta (written by the producer's lanes before its barrier
            // completed), then this step's S^T and dP^T
            ok = warp_wait(&bars[ST_FULL + st], (s / NST) & 1, abort) &&
                 warp_wait(&bars[S_FULL], s & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            // row i sees this key when key <= i and (no window or key > i - W)
            const int lo = key - q0;                                               // keep c >= lo
            const int hi = (p.window > 0) ? key + p.window - 1 - q0 : (1 << 30);   // keep c <= hi
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                uint32_t sv[32], dp[32];
                tmem_ld32x2_sync(tmem + lane_addr + T_S + c * 32, sv, tmem + lane_addr + T_DP + c * 32, dp);
                if (c == 1) {
                    // step s's S^T / dP^T are all read: the issuer may compute step s + 1's
                    tc_fence_before();
                    mbar_arrive(&bars[SDP_FREE]);
                }
                uint32_t wp[16], wd[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float pr[2], ds[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = c * 32 + 2 * e + u;
                        const bool vis = col >= lo && col <= hi;
                        pr[u] = vis ? fast_exp2(fmaf(__uint_as_float(sv[2 * e + u]), c_l2, -lse2[col])) : 0.f;
                        ds[u] = pr[u] * (__uint_as_float(dp[2 * e + u]) - lse2[QB + col]);
                    }
                    wp[e] = pack_bf16x2(pr[0], pr[1]);
                    wd[e] = pack_bf16x2(ds[0], ds[1]);
                }
                // P^T / dS^T of step s - 1 must have been read by its dV / dK MMAs
                if (c == 0 && s > 0) {
                    ok = warp_wait(&bars[DKV_DONE], (s - 1) & 1, abort);
                    if (!ok)
                        break;
                    tc_fence_after();
                }
                tmem_st16(tmem + lane_addr + T_P + c * 16, wp);
                tmem_st16(tmem + lane_addr + T_DS + c * 16, wd);
            }
            if (!ok)
                break;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[P_FULL]);
        }
        if (ok)
            ok = warp_wait(&bars[DONE], 0, abort);
        if (ok) {
            tc_fence_after();
            const bool valid = key < p.L;
            float *vrow = p.dv + (int64_t)b * p.dv_sb + (int64_t)key * p.dv_sl + (int64_t)g * p.dv_sh;
            float *krow = p.dk + (int64_t)b * p.dk_sb + (int64_t)key * p.dk_sl + (int64_t)g * p.dk_sh;
#pragma unroll 1
            for (int c = 0; c < 10; ++c) {
                uint32_t r[32];
                tmem_ld32_sync(tmem + lane_addr + T_DV + c * 32, r); // dV (4 chunks), then dK (6)
                if (valid) {
                    float *dst = c < 4 ? vrow + c * 32 : krow + (c - 4) * 32;
                    const float f = c < 4 ? 1.f : p.scale;
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        *reinterpret_cast<float4 *>(dst + 4 * v4) =
                            make_float4(__uint_as_float(r[4 * v4]) * f, __uint_as_float(r[4 * v4 + 1]) * f,
                                        __uint_as_float(r[4 * v4 + 2]) * f, __uint_as_float(r[4 * v4 + 3]) * f);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_bwd_delta(const BwdParams &p, cudaStream_t stream)
{
    const int64_t warps = (int64_t)p.B * p.Hq * ((p.L + bd::ROWS - 1) / bd::ROWS);
    const int64_t blocks = (warps + bd::WARPS - 1) / bd::WARPS;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    bwd_delta_kernel<<<(unsigned)blocks, bd::WARPS * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                            const CUtensorMap &dout, const BwdParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    bk::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = (int64_t)((p.L + 127) / 128) * p.B * p.Hkv;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    bwd_dkdv_kernel<<<(unsigned)blocks, bw::THREADS, bk::SMEM_BYTES, stream>>>(q, k, v, dout, p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                          const CUtensorMap &dout, const BwdParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    bq::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    const int64_t blocks = (int64_t)((p.L + 127) / 128) * p.B * p.Hq;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    bwd_dq_kernel<<<(unsigned)blocks, bw::THREADS, bq::SMEM_BYTES, stream>>>(q, k, v, dout, p);
    return cudaGetLastError();
}

} // namespace sinkattn
