// Full-causal (GA) sink-attention prefill, two query heads per CTA (sm_100a, tcgen05).
//
// Same result as the band kernel ("MiMo-V2-Flash 架构 QA" Q3.7/Q3.8; the GA layers' causal mask
// of "MiMo-V2-Flash 模型架构深度拆解" CH10.3). What changes is the work of a CTA: the 128 query rows
// of one query tile for two heads of the same GQA group, A and B. Each K / V tile is loaded once
// and feeds both heads, and the heads' softmax warpgroups take turns with the tensor cores: while
// warpgroup A turns S_A into P_A, the MMA issuer runs S_B, and so on. An M128 N128 K16 UMMA costs
// about the same issue time whatever its operands, so the tensor pipe is kept busy by giving it a
// second head's work to do while the first head's softmax runs, instead of by deeper buffering.
//
// Tensor memory: S_A / P_A (128 columns), O_A (128), S_B / P_B (128), O_B (128). Issue order per
// key tile j: S_A(0), S_B(0), then {PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)}; S_x(j+1) is issued once
// PV_x(j) has read P_x(j), which lies over S_x.
//
// Roles (384 threads): warps 0-3 softmax + epilogue of head A, warps 4-7 of head B (thread = row
// = TMEM lane); warp 8 TMA producer for both Q tiles and the K tiles (2 stages); warp 9 for the V
// tiles (1 stage); warp 10 TMEM allocator and the single-thread UMMA issuer; warp 11 idle. The
// softmax warpgroups take registers from the fourth. Shared memory: two Q
// tiles (96 KB), two K stages (96 KB), one V stage (32 KB). Waits are bounded as in the band
// kernel. Used for full-causal prefill (whole sequences, or a chunk after a prefix, contiguous or
// paged) when the group has an even number of heads.
#pragma once
#include "common.cuh"
#include "internal.h"
#include "prefill_kernels.cuh"

namespace sinkattn {

namespace pq {
using namespace pf;
constexpr int Q_OFF = 0;                          // head x's Q tile at x * Q_BYTES
constexpr int K_OFF = 2 * Q_BYTES;                // 2 stages
constexpr int V_OFF = K_OFF + 2 * K_BYTES;        // 1 stage
constexpr int BAR_OFF = V_OFF + V_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
constexpr int THREADS = 384;
constexpr int WARP_K = 8, WARP_V = 9, WARP_M = 10; // warp 11 only completes warpgroup 2
// launched at 168 registers a thread (384 x 168 = 64512); warpgroup 2 gives up 96 of them, the
// two softmax warpgroups take 48 more: 2 x 128 x 216 + 128 x 72 = 64512
constexpr int REGS_LAUNCH = 168, REGS_SOFTMAX = 216, REGS_ROLES = 72;
static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_ROLES <= THREADS * REGS_LAUNCH, "register split");
enum Bar {
    QFULL = 0,
    KFULL = 1,   // + K stage
    KEMPTY = 3,  // + K stage
    VFULL = 5,
    VEMPTY = 6,
    SFULL = 7,   // + head
    PFULL = 9,   // + head
    PVDONE = 11, // + head
    DRAIN = 13,
    NUM = 14
};
// Per-warpgroup register budget (all four warps of the warpgroup execute it). The budgets of
// all warpgroups must add up to at most the registers the block was launched with.
template <int N> SA_DEV void regs_raise() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> SA_DEV void regs_lower() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
SA_DEV uint32_t t_s(int x) { return (uint32_t)x * 256; }       // S_x / P_x
SA_DEV uint32_t t_o(int x) { return (uint32_t)x * 256 + 128; } // O_x
} // namespace pq

__global__ void __launch_bounds__(pq::THREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKp,
                        const __grid_constant__ CUtensorMap tmVp, const PrefillParams p)
{
    using namespace pq;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // (query tile, sequence, head pair), pair fastest so a group's CTAs read the same K / V
    // tiles at about the same time; the longest (last) query tiles first
    const int npair = p.Hq / 2;
    const int per_tile = p.B * npair;
    const int t_idx = blockIdx.x / per_tile;
    const int qt = p.n_qtiles - 1 - t_idx;
    const int rem = blockIdx.x - t_idx * per_tile;
    const int b = rem / npair;
    const int h0 = 2 * (rem - b * npair);
    const int g = h0 / p.G; // h0 and h0 + 1 share KV head g (G is even)
    const int r0 = qt * BM;
    const int r_last = min(r0 + BM, p.L) - 1;
    const int a0 = p.q_off + r0;
    const int n_tiles = (p.q_off + r_last) / BN + 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM; ++i)
            mbar_init(&bars[i], (i == PFULL || i == PFULL + 1) ? 128 : 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == WARP_M) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp >= 8) {
        regs_lower<REGS_ROLES>();
        if (warp == WARP_K) {
            if (lane == 0) {
                tma_prefetch_desc(&tmQ);
                tma_prefetch_desc(&tmK);
                mbar_arrive_expect_tx(&bars[QFULL], 2 * Q_BYTES);
                for (int x = 0; x < 2; ++x)
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + Q_OFF + x * Q_BYTES + c * Q_REGION, &tmQ, &bars[QFULL],
                                    c * 64, h0 + x, r0, b);
                int issued = 0;
                for (int j = 0; j < n_tiles; ++j) {
                    const int s = j & 1;
                    // stage s was read by S_A and S_B of tile j - 2
                    if (j >= 2 && !mbar_wait(&bars[KEMPTY + s], ((j >> 1) - 1) & 1, abort, 1u))
                        break;
                    const PrefillTile tl = prefill_tile(p, b, j);
                    mbar_arrive_expect_tx(&bars[KFULL + s], K_BYTES);
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + K_OFF + s * K_BYTES + c * K_REGION, tl.pool ? &tmKp : &tmK,
                                    &bars[KFULL + s], c * 64, g, tl.row, tl.blk);
                    issued = j + 1;
                }
                // no copy of ours may still be landing when the CTA ends
                for (int j = max(0, issued - 2); j < issued; ++j)
                    mbar_wait_drain(&bars[KFULL + (j & 1)], (j >> 1) & 1);
                mbar_wait_drain(&bars[QFULL], 0);
            }
            __syncwarp();
        } else if (warp == WARP_V) {
            if (lane == 0) {
                tma_prefetch_desc(&tmV);
                int issued = 0;
                for (int j = 0; j < n_tiles; ++j) {
                    // the stage was read by PV_A and PV_B of tile j - 1
                    if (j >= 1 && !mbar_wait(&bars[VEMPTY], (j - 1) & 1, abort, 1u))
                        break;
                    const PrefillTile tl = prefill_tile(p, b, j);
                    mbar_arrive_expect_tx(&bars[VFULL], V_BYTES);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem + V_OFF + c * K_REGION, tl.pool ? &tmVp : &tmV, &bars[VFULL],
                                    c * 64, g, tl.row, tl.blk);
                    issued = j + 1;
                }
                if (issued > 0)
                    mbar_wait_drain(&bars[VFULL], (issued - 1) & 1);
            }
            __syncwarp();
        } else if (warp == WARP_M) {
            if (lane == 0) {
                const uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
                const uint32_t idesc_o = umma_idesc_bf16(BM, 128, 1);
                const uint32_t sK = smem_u32(smem + K_OFF), sV = smem_u32(smem + V_OFF);
                bool ok = mbar_wait(&bars[QFULL], 0, abort, 1u);
                // S_x(j) = Q_x K_j^T into S_x, once P_x(j - 1) (over S_x) has been read by PV_x(j - 1)
                auto issue_s = [&](int x, int j) -> bool {
                    const int ks = j & 1;
                    if (x == 0 && !mbar_wait(&bars[KFULL + ks], (j >> 1) & 1, abort, 1u))
                        return false;
                    if (j >= 1 && !mbar_wait(&bars[PVDONE + x], (j - 1) & 1, abort, 1u))
                        return false;
                    tc_fence_after();
                    const uint32_t sQ = smem_u32(smem + Q_OFF + x * Q_BYTES);
    #pragma unroll 1
                    for (int kk = 0; kk < 12; ++kk) {
                        const uint32_t off = (kk >> 2) * Q_REGION + (kk & 3) * 32;
                        umma_ss(tmem + t_s(x), smem_desc_sw128(sQ + off, 16, 1024),
                                smem_desc_sw128(sK + ks * K_BYTES + off, 16, 1024), idesc_s, kk > 0);
                    }
                    umma_commit(&bars[SFULL + x]);
                    if (x == 1)
                        umma_commit(&bars[KEMPTY + ks]); // both heads' S have read K stage ks
                    return true;
                };
                // O_x += P_x(j) V_j, A = P_x from TMEM
                auto issue_pv = [&](int x, int j) -> bool {
                    if (x == 0 && !mbar_wait(&bars[VFULL], j & 1, abort, 1u))
                        return false;
                    if (!mbar_wait(&bars[PFULL + x], j & 1, abort, 1u))
                        return false;
                    tc_fence_after();
    #pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(tmem + t_o(x), tmem + t_s(x) + kk * 8,
                                smem_desc_sw128(sV + kk * 16 * ROW_BYTES, K_REGION, 1024), idesc_o,
                                (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bars[PVDONE + x]);
                    if (x == 1)
                        umma_commit(&bars[VEMPTY]); // both heads' PV have read the V stage
                    return true;
                };
                if (ok)
                    ok = issue_s(0, 0) && issue_s(1, 0);
                for (int j = 0; ok && j < n_tiles; ++j) {
                    const bool more = j + 1 < n_tiles;
                    ok = issue_pv(0, j) && (!more || issue_s(0, j + 1)) && issue_pv(1, j) &&
                         (!more || issue_s(1, j + 1));
                }
                // every MMA of ours has finished before TMEM is released
                umma_commit(&bars[DRAIN]);
                mbar_wait_drain(&bars[DRAIN], 0);
            }
            __syncwarp();
        }
    } else {
        regs_raise<REGS_SOFTMAX>();
        // ---------------- softmax warps of head x: thread = query row = TMEM lane ----------------
        const int x = warp >> 2;
        const int h = h0 + x;
        const int row = threadIdx.x & 127;
        const int rp = r0 + row;     // this query row (of the L rows)
        const int ap = p.q_off + rp; // its position in the sequence
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t sbase = tmem + lane_addr + t_s(x), obase = tmem + lane_addr + t_o(x);
        const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
        const float c_l2 = p.scale_log2; // > 0, so max(s) * c = max(s * c)
        // m_run: reference max (log2 units); l_exact: sum of fp32 P (gives LSE); l_round: sum
        // of the bf16-rounded P that P V multiplies (normalises O). Both start with the sink:
        // m_0 = sink, l_0 = exp(sink - m_0) = 1.
        float m_run = sink_l2;
        float l_exact = (sink_l2 > -INFINITY) ? 1.f : 0.f;
        float l_round = l_exact;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int kbase = j * BN;
            ok = warp_wait(&bars[SFULL + x], j & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            uint32_t raw[128];
            tmem_ld128(sbase, raw);
            float xs[128]; // raw scores q.k; masked keys -inf
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx8[i] = -INFINITY;
            if (kbase + BN - 1 > a0) { // the tile crosses the diagonal
                const int hi = ap - kbase;
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    xs[c] = (c <= hi) ? __uint_as_float(raw[c]) : -INFINITY;
                    mx8[c & 7] = fmaxf(mx8[c & 7], xs[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    xs[c] = __uint_as_float(raw[c]);
                    mx8[c & 7] = fmaxf(mx8[c & 7], xs[c]);
                }
            }
            float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            mx *= c_l2;
            // the first tile sets the exact max; later tiles raise it lazily
            const bool rescale = (j == 0) ? (mx > m_run) : (mx > m_run + TAU);
            float alpha = 1.f;
            if (rescale) {
                alpha = fast_exp2(m_run - mx); // 0 when m_run is -inf
                l_exact *= alpha;
                l_round *= alpha;
                m_run = mx;
            }
            // O is touched only when one of this warp's rows raises its max: then wait for the
            // previous tile's P V (O up to date) and rescale
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                ok = warp_wait(&bars[PVDONE + x], (j - 1) & 1, abort);
                if (!ok)
                    break;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32_sync(obase + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(obase + c * 32, o);
                }
                tmem_st_wait();
            }
            const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
            float pe[4] = {0.f, 0.f, 0.f, 0.f}, pr[4] = {0.f, 0.f, 0.f, 0.f};
            // P (bf16 pairs: keys 2c, 2c + 1 in column c) over this row's S
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
                uint32_t pk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float e0 = fast_exp2(fmaf(xs[c16 * 16 + 2 * u], c_l2, neg_m));
                    const float e1 = fast_exp2(fmaf(xs[c16 * 16 + 2 * u + 1], c_l2, neg_m));
                    pk[u] = pack_bf16x2(e0, e1);
                    pe[u & 3] += e0 + e1;
                    pr[u & 3] += sum_bf16x2(pk[u]);
                }
                tmem_st8(sbase + c16 * 8, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            }
            l_exact += (pe[0] + pe[1]) + (pe[2] + pe[3]);
            l_round += (pr[0] + pr[1]) + (pr[2] + pr[3]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[PFULL + x]);
        }
        if (ok)
            ok = warp_wait(&bars[PVDONE + x], (n_tiles - 1) & 1, abort);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l_round;
            const bool valid = rp < p.L;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (int64_t)b * p.o_sb +
                                  (int64_t)rp * p.o_sl + (int64_t)h * p.o_sh;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32_sync(obase + c * 32, o);
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
    if (warp == WARP_M) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_prefill_pair(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                const CUtensorMap &tmV, const CUtensorMap &tmKp,
                                const CUtensorMap &tmVp, const PrefillParams &p,
                                cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    pq::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    if (p.window != 0 || p.G % 2 != 0)
        return cudaErrorInvalidValue;
    const int64_t blocks = (int64_t)p.n_qtiles * p.B * (p.Hq / 2);
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    prefill_pair_kernel<<<(unsigned)blocks, pq::THREADS, pq::SMEM_BYTES, stream>>>(tmQ, tmK, tmV,
                                                                                    tmKp, tmVp, p);
    return cudaGetLastError();
}

} // namespace sinkattn
