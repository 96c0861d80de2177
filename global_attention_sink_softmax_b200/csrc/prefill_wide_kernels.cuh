// Full-causal (GA) sink-softmax prefill with two softmax warpgroups per CTA (sm_100a, tcgen05).
//
// Same result as the band kernel ("MiMo-V2-Flash 架构 QA" Q3.7/Q3.8; the GA layers' causal mask
// of "MiMo-V2-Flash 模型架构深度拆解" CH10.3): for each query row i of head h,
//     O_i = sum_{j <= i} exp(a_ij - m_i) v_j / (exp(sink_h - m_i) + sum_{j <= i} exp(a_ij - m_i)).
// What changes is how a CTA walks its keys. One CTA still owns 128 query rows of one head, but it
// takes the keys 256 at a time: the two 128-key halves of a pair go to two softmax warpgroups that
// run at the same time, so each SMSP holds two softmax warps (the band kernel has one), and S
// takes half as many UMMA instructions per key.
//
// Per pair t (keys 256 t .. 256 t + 255; the last pair may have its upper half past the diagonal,
// in which case that half is neither loaded nor multiplied):
//   S = Q [K_0 K_1]^T   one M128 N256 K16 x 12 chain, half x into TMEM columns 128 x (the two K
//                       halves interleave by 64-dim region in shared memory, so the 256 keys of
//                       a region form one K-major operand)
//   row max             each warpgroup over its half, then swapped through shared memory so both
//                       use the same running max m (and rescale O by the same factor)
//   P_x = 2^(S_x c - m) bf16 pairs into TMEM columns 256 + 64 x (P has its own columns: S's can
//                       take S_{t+1} as soon as the scores sit in registers)
//   O += [P_0 P_1] V    M128 N128 K16 x 16 from TMEM P and the two V halves in shared memory
// Issue order S_0, then {S_{t+1}, P V_t}: the tensor cores compute the next pair's scores while
// the softmax warps work on this pair's, and P V_t follows as soon as P_t is written.
//
// Each warpgroup keeps its own row sum of the fp32 P (the sink's 1 in warpgroup 0); the two are
// added in the epilogue, which normalises O (warpgroup x writes dims 64 x .. 64 x + 63) and gives
// LSE. The running max is raised lazily (only when a pair's max exceeds it by more than 8 in log2
// units, the first pair setting it exactly), so P <= 2^8.
//
// Roles (384 threads): warps 0-3 softmax of half 0, warps 4-7 of half 1 (thread = query row =
// TMEM lane, warp w reading lanes 32 (w mod 4) ..); warp 8 the TMA producer for Q, K and V; warp 9
// allocates TMEM (all 512 columns: S 256, P 128, O 128) and is the single-thread UMMA issuer;
// warps 10-11 only complete the third warpgroup, whose registers go to the softmax warpgroups.
// Shared memory: Q 48 KB, K 2 x 48 KB, V 2 x 32 KB (one pair), the max exchange 2 KB. Every wait
// is bounded as in the band kernel.
#pragma once
#include "common.cuh"
#include "internal.h"
#include "prefill_kernels.cuh"

namespace sinkattn {

namespace pw {
constexpr int BM = 128;                  // query rows per CTA
constexpr int BN = 128;                  // keys per half
constexpr int ROW_BYTES = 128;           // one 64-element bf16 chunk row (the swizzle width)
constexpr int Q_REGION = BM * ROW_BYTES; // 16 KB: 128 rows x 64 dims
constexpr int Q_BYTES = 3 * Q_REGION;    // 192 dims
constexpr int K_REGION = BN * ROW_BYTES;
constexpr int K_BYTES = 3 * K_REGION;    // one half: 128 keys x 192 dims
constexpr int V_BYTES = 2 * K_REGION;    // one half: 128 keys x 128 dims
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;   // region c (dims 64 c ..) at + 2 c K_REGION, half x at + x K_REGION
constexpr int OFF_V = OFF_K + 2 * K_BYTES;
constexpr int OFF_X = OFF_V + 2 * V_BYTES; // float [2 parity][2 half][128 rows]
constexpr int OFF_BAR = OFF_X + 2 * 2 * BM * 4;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024; // barriers + 1 KB for aligning the base
constexpr int THREADS = 384;
constexpr int WARP_LOAD = 8, WARP_MMA = 9;
// launched at 168 registers a thread (384 x 168 = 64512); the third warpgroup gives up 112 of
// them, the two softmax warpgroups take 56 more: 2 x 128 x 224 + 128 x 56 = 64512
constexpr int REGS_LAUNCH = 168, REGS_SOFTMAX = 224, REGS_ROLES = 56;
static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_ROLES <= THREADS * REGS_LAUNCH, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_P = 256; // P_x at + 64 x
constexpr uint32_t TMEM_O = 384;
constexpr float TAU = 8.0f;

enum Bar {
    QFULL = 0,
    KFULL = 1,   // + half
    KEMPTY = 3,  // + half
    VFULL = 5,
    VEMPTY = 6,
    SFULL = 7,   // + half
    SFREE = 9,   // + half (128 arrivals: the half's warpgroup has its scores in registers)
    PFULL = 11,  // 256 arrivals
    PVDONE = 12,
    XCH = 13,    // + parity * 4 + lane quarter (64 arrivals: warps q and q + 4)
    DRAIN = 21,
    NUM = 22
};
// per-warpgroup register budget (every warp of the warpgroup executes it)
template <int N> SA_DEV void regs_raise() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> SA_DEV void regs_lower() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
} // namespace pw

__global__ void __launch_bounds__(pw::THREADS, 1)
    prefill_wide_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKp,
                        const __grid_constant__ CUtensorMap tmVp, const PrefillParams p)
{
    using namespace pw;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *xchg = reinterpret_cast<float *>(smem + OFF_X);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // (query tile, sequence, head), head fastest so the CTAs of one KV group run together and
    // share K / V through L2; the longest (last) query tiles first
    const int per_tile = p.B * p.Hq;
    const int t_idx = blockIdx.x / per_tile;
    const int qt = p.n_qtiles - 1 - t_idx;
    const int rem = blockIdx.x - t_idx * per_tile;
    const int b = rem / p.Hq;
    const int h = rem - b * p.Hq;
    const int g = h / p.G;
    const int r0 = qt * BM;
    const int r_last = min(r0 + BM, p.L) - 1;
    const int a0 = p.q_off + r0;
    const int n_tiles = (p.q_off + r_last) / BN + 1; // 128-key tiles 0 .. n_tiles - 1
    const int n_pairs = (n_tiles + 1) >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM; ++i) {
            uint32_t cnt = 1;
            if (i == SFREE || i == SFREE + 1)
                cnt = 128;
            else if (i == PFULL)
                cnt = 256;
            else if (i >= XCH && i < XCH + 8)
                cnt = 64;
            mbar_init(&bars[i], cnt);
        }
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
        regs_lower<REGS_ROLES>();
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(&bars[QFULL], Q_BYTES);
            for (int c = 0; c < 3; ++c)
                tma_load_4d(smem + OFF_Q + c * Q_REGION, &tmQ, &bars[QFULL], c * 64, h, r0, b);
            int k_issued[2] = {0, 0}, v_issued = 0; // phases started, per K half and for V
            // K half x of pair t, once S of pair t - 1 has read that half; a half past the
            // diagonal is not loaded (its barrier phase completes with no bytes)
            auto load_k = [&](int t) -> bool {
                for (int x = 0; x < 2; ++x) {
                    if (t >= 1 && !mbar_wait(&bars[KEMPTY + x], (t - 1) & 1, abort, 1u))
                        return false;
                    const int j = 2 * t + x;
                    k_issued[x] = t + 1;
                    if (j >= n_tiles) {
                        mbar_arrive(&bars[KFULL + x]);
                        continue;
                    }
                    const PrefillTile tl = prefill_tile(p, b, j);
                    mbar_arrive_expect_tx(&bars[KFULL + x], K_BYTES);
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + OFF_K + (2 * c + x) * K_REGION,
                                    tl.pool ? &tmKp : &tmK, &bars[KFULL + x], c * 64, g, tl.row,
                                    tl.blk);
                }
                return true;
            };
            // both V halves of pair t, once P V of pair t - 1 is done
            auto load_v = [&](int t) -> bool {
                if (t >= 1 && !mbar_wait(&bars[VEMPTY], (t - 1) & 1, abort, 1u))
                    return false;
                v_issued = t + 1;
                const int halves = (2 * t + 1 < n_tiles) ? 2 : 1;
                mbar_arrive_expect_tx(&bars[VFULL], halves * V_BYTES);
                for (int x = 0; x < halves; ++x) {
                    const PrefillTile tl = prefill_tile(p, b, 2 * t + x);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem + OFF_V + x * V_BYTES + c * K_REGION,
                                    tl.pool ? &tmVp : &tmV, &bars[VFULL], c * 64, g, tl.row, tl.blk);
                }
                return true;
            };
            // The stages free up in the order S_0, S_1, P V_0, S_2, P V_1, ...: K of pair t + 1
            // (read by S_t) before V of pair t (read by P V_{t-1}).
            bool ok = load_k(0) && load_v(0);
            if (ok && n_pairs > 1)
                ok = load_k(1);
            for (int t = 1; ok && t < n_pairs; ++t) {
                if (t + 1 < n_pairs && !(ok = load_k(t + 1)))
                    break;
                ok = load_v(t);
            }
            // make sure no copy of ours is still landing in shared memory when the CTA ends
            for (int x = 0; x < 2; ++x)
                if (k_issued[x] > 0)
                    mbar_wait_drain(&bars[KFULL + x], (k_issued[x] - 1) & 1);
            if (v_issued > 0)
                mbar_wait_drain(&bars[VFULL], (v_issued - 1) & 1);
            mbar_wait_drain(&bars[QFULL], 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        regs_lower<REGS_ROLES>();
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
            const uint32_t idesc_o = umma_idesc_bf16(BM, 128, 1);
            const uint32_t sQ = smem_u32(smem + OFF_Q);
            const uint32_t sK = smem_u32(smem + OFF_K);
            const uint32_t sV = smem_u32(smem + OFF_V);
            bool ok = mbar_wait(&bars[QFULL], 0, abort, 1u);
            // S of pair t into TMEM columns 0..255 (half x at 128 x) in one M128 N256 chain (the
            // two K halves interleave by 64-dim region, so keys 0..255 of a region are one
            // K-major operand), N128 when the upper half lies past the diagonal; issued once both
            // halves' softmax warps have read pair t - 1's scores
            const uint32_t idesc_s2 = umma_idesc_bf16(BM, 2 * BN, 0);
            auto issue_s = [&](int t) -> bool {
                for (int x = 0; x < 2; ++x)
                    if (!mbar_wait(&bars[KFULL + x], t & 1, abort, 1u))
                        return false;
                for (int x = 0; t >= 1 && x < 2; ++x)
                    if (!mbar_wait(&bars[SFREE + x], (t - 1) & 1, abort, 1u))
                        return false;
                tc_fence_after();
                const uint32_t idesc = (2 * t + 1 < n_tiles) ? idesc_s2 : idesc_s;
#pragma unroll
                for (int kk = 0; kk < 12; ++kk)
                    umma_ss(tmem, smem_desc_sw128(sQ + (kk >> 2) * Q_REGION + (kk & 3) * 32, 16, 1024),
                            smem_desc_sw128(sK + (kk >> 2) * 2 * K_REGION + (kk & 3) * 32, 16, 1024),
                            idesc, kk > 0);
                for (int x = 0; x < 2; ++x) {
                    umma_commit(&bars[SFULL + x]);
                    umma_commit(&bars[KEMPTY + x]);
                }
                return true;
            };
            // O += P_t V_t: A = P (128 rows x 16 keys per step, 8 TMEM columns of bf16 pairs),
            // B = V (16 keys x 128 dims, MN-major, dims 64..127 one 16 KB region further on)
            auto issue_pv = [&](int t) -> bool {
                if (!mbar_wait(&bars[PFULL], t & 1, abort, 1u))
                    return false;
                if (!mbar_wait(&bars[VFULL], t & 1, abort, 1u))
                    return false;
                tc_fence_after();
                const int nk = (2 * t + 1 < n_tiles) ? 16 : 8;
#pragma unroll 1
                for (int kk = 0; kk < nk; ++kk)
                    umma_ts(tmem + TMEM_O, tmem + TMEM_P + kk * 8,
                            smem_desc_sw128(sV + (kk >> 3) * V_BYTES + (kk & 7) * 16 * ROW_BYTES,
                                            K_REGION, 1024),
                            idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&bars[PVDONE]);
                umma_commit(&bars[VEMPTY]);
                return true;
            };
            if (ok)
                ok = issue_s(0);
            for (int t = 0; ok && t < n_pairs; ++t) {
                if (t + 1 < n_pairs)
                    ok = issue_s(t + 1);
                ok = ok && issue_pv(t);
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[DRAIN]);
            mbar_wait_drain(&bars[DRAIN], 0);
        }
        __syncwarp();
    } else if (warp < 8) {
        regs_raise<REGS_SOFTMAX>();
        // ---------------- softmax warps: half x, thread = query row ----------------
        const int x = warp >> 2;
        const int q = warp & 3;
        const int row = q * 32 + lane;        // 0..127
        const int rp = r0 + row;              // this query row (of the L rows)
        const int ap = p.q_off + rp;          // its position in the sequence
        const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
        const uint32_t saddr = tmem + lane_addr + x * BN;
        const uint32_t paddr = tmem + lane_addr + TMEM_P + x * 64;
        const uint32_t oaddr = tmem + lane_addr + TMEM_O + x * 64;
        const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
        const float c_l2 = p.scale_log2; // > 0, so max(s) * c = max(s * c)
        // m_run: reference max (log2 units), the same in both halves; l_part: this half's sum
        // of fp32 P, the sink's exp(sink - m_0) = 1 counted in half 0.
        float m_run = sink_l2;
        float l_part = (x == 0 && sink_l2 > -INFINITY) ? 1.f : 0.f;
        bool ok = true;
        // swap a per-row value with the other half's warp over the same rows (slot s parity)
        auto swap_rows = [&](int s, float v, float &other) -> bool {
            xchg[((s & 1) * 2 + x) * BM + row] = v;
            mbar_arrive(&bars[XCH + (s & 1) * 4 + q]);
            if (!warp_wait(&bars[XCH + (s & 1) * 4 + q], (s >> 1) & 1, abort))
                return false;
            other = xchg[((s & 1) * 2 + (x ^ 1)) * BM + row];
            return true;
        };
        for (int t = 0; t < n_pairs; ++t) {
            const int j = 2 * t + x;
            const bool present = j < n_tiles;
            const int kbase = j * BN;
            ok = warp_wait(&bars[SFULL + x], t & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            uint32_t sr[128];
            float mx = -INFINITY;
            if (present) {
                tmem_ld128(saddr, sr);
                // the scores sit in registers: S_{t+1} may overwrite this half's columns
                tc_fence_before();
                mbar_arrive(&bars[SFREE + x]);
                if (kbase + BN - 1 > a0) { // the half crosses the diagonal
                    const int hi = ap - kbase;
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (e > hi)
                            sr[e] = __float_as_uint(-INFINITY);
                }
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx8[i] = -INFINITY;
#pragma unroll
                for (int e = 0; e < 128; e += 2)
                    mx8[(e >> 1) & 7] =
                        fmax3(mx8[(e >> 1) & 7], __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
                mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                           fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                mx *= c_l2;
            } else {
                mbar_arrive(&bars[SFREE + x]);
            }
            float mo;
            if (!(ok = swap_rows(t, mx, mo)))
                break;
            mx = fmaxf(mx, mo);
            // the first pair sets the exact max (m = max(sink, row max)); later pairs raise it
            // lazily. Both halves see the same values, so they take the same decisions.
            const bool rescale = (t == 0) ? (mx > m_run) : (mx > m_run + TAU);
            float alpha = 1.f;
            if (rescale) {
                alpha = fast_exp2(m_run - mx); // 0 when m_run is -inf
                l_part *= alpha;
                m_run = mx;
            }
            const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
            uint32_t pk[64];
            if (present) {
                float pe[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int u = 0; u < 64; ++u) {
                    const float e0 = fast_exp2(fmaf(__uint_as_float(sr[2 * u]), c_l2, neg_m));
                    const float e1 = fast_exp2(fmaf(__uint_as_float(sr[2 * u + 1]), c_l2, neg_m));
                    pk[u] = pack_bf16x2(e0, e1);
                    pe[u & 3] += e0 + e1;
                }
                l_part += (pe[0] + pe[1]) + (pe[2] + pe[3]);
            }
            // P's columns and O are free once P V of the previous pair is done
            if (t > 0) {
                ok = warp_wait(&bars[PVDONE], (t - 1) & 1, abort);
                if (!ok)
                    break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < 2; ++c) {
                        uint32_t o[32];
                        tmem_ld32_sync(oaddr + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(oaddr + c * 32, o);
                    }
                }
            }
            if (present) {
                // P (bf16 pairs: keys 2c, 2c + 1 of this half in column c)
#pragma unroll
                for (int c = 0; c < 64; c += 8)
                    tmem_st8(paddr + c, pk[c], pk[c + 1], pk[c + 2], pk[c + 3], pk[c + 4],
                             pk[c + 5], pk[c + 6], pk[c + 7]);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[PFULL]);
        }
        if (ok && n_pairs > 0)
            ok = warp_wait(&bars[PVDONE], (n_pairs - 1) & 1, abort);
        float l_other = 0.f;
        if (ok)
            ok = swap_rows(n_pairs, l_part, l_other);
        if (ok) {
            tc_fence_after();
            const float l_exact = l_part + l_other;
            const float inv_l = 1.f / l_exact;
            const bool valid = rp < p.L;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.o_sb +
                                  (int64_t)rp * p.o_sl + (int64_t)h * p.o_sh + x * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                tmem_ld32_sync(oaddr + c * 32, o);
                if (valid) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 pkv;
                        pkv.x = pack_bf16x2(__uint_as_float(o[v4 * 8 + 0]) * inv_l,
                                            __uint_as_float(o[v4 * 8 + 1]) * inv_l);
                        pkv.y = pack_bf16x2(__uint_as_float(o[v4 * 8 + 2]) * inv_l,
                                            __uint_as_float(o[v4 * 8 + 3]) * inv_l);
                        pkv.z = pack_bf16x2(__uint_as_float(o[v4 * 8 + 4]) * inv_l,
                                            __uint_as_float(o[v4 * 8 + 5]) * inv_l);
                        pkv.w = pack_bf16x2(__uint_as_float(o[v4 * 8 + 6]) * inv_l,
                                            __uint_as_float(o[v4 * 8 + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + v4 * 8) = pkv;
                    }
                }
            }
            if (valid && x == 0 && p.lse)
                p.lse[((int64_t)b * p.Hq + h) * p.L + rp] = (m_run + fast_log2(l_exact)) * kLn2;
        }
    } else {
        regs_lower<REGS_ROLES>(); // warps 10-11: nothing to do but give up registers
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_prefill_wide(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                const CUtensorMap &tmV, const CUtensorMap &tmKp,
                                const CUtensorMap &tmVp, const PrefillParams &p,
                                cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(prefill_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    pw::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    if (p.window != 0)
        return cudaErrorInvalidValue;
    const int64_t blocks = (int64_t)p.n_qtiles * p.B * p.Hq;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    prefill_wide_kernel<<<(unsigned)blocks, pw::THREADS, pw::SMEM_BYTES, stream>>>(tmQ, tmK, tmV,
                                                                                    tmKp, tmVp, p);
    return cudaGetLastError();
}

} // namespace sinkattn
