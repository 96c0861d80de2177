// Sink-softmax attention decode and speculative verify on a 128-slot sliding-window ring, on
// the tensor cores (tcgen05, sm_100a).
//
// Same computation as the other decode kernels: each query row attends to the keys of its
// window (the ring's cached tokens, then the step's new tokens up to its own), with the sink
// counted once in the softmax denominator ("MiMo-V2-Flash 架构 QA" Q3.8; the window of
// "MiMo-V2-Flash 模型架构深度拆解" CH10.3). The model's SWA layers keep a ring of 128 slots per
// sequence and KV head, and a verify step brings T <= 4 tokens for the G = 8 query heads of a
// group: 32 rows against 132 keys. Such a unit (80 KB of K / V) is too small for a CTA to spend
// its latency on alone, and its 32 x 128 fp32 output does not fit one warp's registers, so:
//
// - a persistent CTA walks a contiguous run of units with two shared-memory stages for Q and K
//   (released once S is computed) and two for V (released after P V), each filled by its own
//   loader warp: the next units' tiles land by TMA while this one is computed;
// - one MMA pass per unit: S = Q K^T (M128 N144 K192: the 128 ring slots in physical order,
//   then a 16-row box of new tokens whose rows past T arrive as zeros), P written over S in
//   TMEM as bf16 pairs, O = P V (M128 N128 K144, P from TMEM);
// - the 32 query rows of a unit fill one TMEM lane quarter, so one warp holds them all and the
//   softmax's exponentials run on 32 useful lanes: Q's region holds one 8-row swizzle atom per
//   token (row 8 t + h = token t, head h), and the A descriptor of an odd unit starts 4 KB
//   before its Q, so its rows land in lanes 32 .. 63 (the MMA's other rows read neighbouring
//   bytes and are never used);
// - warp 0 takes the even units (lanes 0 .. 31) and warp 1 the odd ones (lanes 32 .. 63), on
//   two SMSPs, so the two units in flight do not share an exponential unit (S double-buffered
//   in TMEM, O handed over); warp 2 loads Q and K, warp 4 V, one thread of warp 3 issues the
//   MMAs: S of the next unit goes in before P V of this one;
// - launched as a programmatic dependent: the next launch's CTAs are set up while this one
//   drains, and none reads global memory before the kernels ahead of it have completed.
//
// Masks: slot s holds the token of age index cl = (s - head) mod 128 (0 the oldest); it is a
// key iff first_c <= cl < n_cache, and row t sees it iff also cl >= n_cache + t - W + 1: the
// slots a row does not see form one circular run, kept as a bit mask per 48-column group. New
// token i is seen by row t iff i < T, i <= t and i > t - W. V rows of slots that hold no key
// are zeroed before P V reads them (their P is 0, but the slot may hold anything).
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace rv {
constexpr int G = 8;                       // query heads per KV head
constexpr int TMAX = 4;                    // new tokens per step
constexpr int CAP = 128;                   // ring slots
constexpr int NK = CAP + 16;               // keys per unit: ring slots + a 16-row new-token box
constexpr int ROW = 128;                   // bytes per swizzled row (64 bf16)
constexpr int Q_REGION = TMAX * 1024;      // one 8-row atom per token
constexpr int Q_BYTES = 3 * Q_REGION;
constexpr int KV_REGION = NK * ROW;        // 18 KB
constexpr int K_BYTES = 3 * KV_REGION;
constexpr int V_BYTES = 2 * KV_REGION;
constexpr int QK_STAGE = Q_BYTES + K_BYTES; // Q and K of a unit, released after S
constexpr int OFF_V = 2 * QK_STAGE;          // V of a unit, released after P V
constexpr int OFF_BAR = OFF_V + 2 * V_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int WARP_LOAD = 2, WARP_MMA = 3, WARP_VLOAD = 4; // warps 0 / 1: softmax of even / odd units
constexpr int THREADS = 160;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 384;           // S buffer i at i * NK

enum Bar {
    QK_FULL = 0,  // + stage: Q and K landed
    QK_EMPTY = 2, // + stage: S of the stage's unit done
    V_FULL = 4,   // + stage: V landed
    V_EMPTY = 6,  // + stage: P V of the stage's unit done
    S_FULL = 8,   // + S buffer (= warpgroup = stage)
    S_FREE = 10,  // + S buffer: the P written over it is consumed
    P_FULL = 12,  // + warpgroup: P in TMEM, the stage's stray V rows zeroed
    PV_DONE = 14, // + warpgroup
    O_FREE = 16,
    DRAIN = 17,
    NUM_BARS = 18
};
__host__ __device__ constexpr bool counted_by_rows(int i)
{
    return i == P_FULL || i == P_FULL + 1 || i == O_FREE;
}
constexpr int ROW_THREADS = 32; // one softmax warp per unit
static_assert(NUM_BARS * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
static_assert(SMEM_BYTES <= 232448, "two stages fit the opt-in shared memory");
} // namespace rv

// A unit's ring occupancy: keys are the slots of age index in [first_c, n_cache).
struct RvUnit {
    int b, g, n_cache, first_c, head;
};

SA_DEV RvUnit rv_unit(const DecodeParams &p, int u)
{
    RvUnit x;
    x.g = u % p.Hkv;
    x.b = u / p.Hkv;
    x.n_cache = max(0, min(p.ring_len[x.b], rv::CAP));
    const int n_used = (p.window > 0) ? min(x.n_cache, p.window - 1) : x.n_cache;
    x.first_c = x.n_cache - n_used;
    x.head = p.ring_head[x.b] & (rv::CAP - 1);
    return x;
}

// Bits of the columns [x, y) that fall in the 48-column group starting at c0, relative to c0.
SA_DEV uint64_t rv_bits(int x, int y, int c0)
{
    const int a = max(x, c0) - c0, b = min(y, c0 + 48) - c0;
    return a < b ? (((1ull << (b - a)) - 1ull) << a) : 0ull;
}

// The hidden columns of a row among c0 .. c0 + 47: ring slots outside the row's keys, which form
// one circular run of k slots from slot e (e = the slot after the newest key, k = 128 - the
// keys the row sees), and new tokens outside i_lo .. i_hi (columns 128 + i).
SA_DEV uint64_t rv_hidden48(int c0, int e, int k, int i_lo, int i_hi)
{
    uint64_t m = rv_bits(e, min(e + k, rv::CAP), c0) | rv_bits(0, e + k - rv::CAP, c0);
    return m | rv_bits(rv::CAP, rv::CAP + i_lo, c0) | rv_bits(rv::CAP + i_hi + 1, rv::NK, c0);
}

// -inf in the hidden columns (bit u of `hidden` = column c0 + u); most groups have none.
SA_DEV void rv_mask48(uint32_t (&r)[48], uint64_t hidden)
{
    if (hidden == 0ull)
        return;
#pragma unroll
    for (int u = 0; u < 48; ++u)
        if ((hidden >> u) & 1ull)
            r[u] = __float_as_uint(-INFINITY);
}

__global__ void __launch_bounds__(rv::THREADS, 1)
    decode_ring_umma_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmKc,
                            const __grid_constant__ CUtensorMap tmVc,
                            const __grid_constant__ CUtensorMap tmKn,
                            const __grid_constant__ CUtensorMap tmVn, const DecodeParams p)
{
    using namespace rv;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // contiguous run of units (sequence, KV head) for this CTA
    const int n_units = p.B * p.Hkv;
    const int u0 = (int)(((int64_t)blockIdx.x * n_units) / gridDim.x);
    const int u1 = (int)(((int64_t)(blockIdx.x + 1) * n_units) / gridDim.x);
    const int cnt = u1 - u0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i)
            mbar_init(&bars[i], counted_by_rows(i) ? ROW_THREADS : 1);
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
    // Programmatic dependent launch: the next kernel in the stream may start its own set-up now;
    // this one reads no global memory before the kernels ahead of it have completed and their
    // writes are visible (without a programmatic launch both are no-ops).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == WARP_LOAD || warp == WARP_VLOAD) {
        // Q and K (warp 8) or V (warp 10) of unit n into stage n & 1, once the unit n - 2 that
        // held it is done with it
        const bool is_v = warp == WARP_VLOAD;
        if (lane == 0 && cnt > 0) {
            const CUtensorMap *m0 = is_v ? &tmVc : &tmKc, *m1 = is_v ? &tmVn : &tmKn;
            tma_prefetch_desc(m0);
            tma_prefetch_desc(m1);
            if (!is_v)
                tma_prefetch_desc(&tmQ);
            const int full0 = is_v ? V_FULL : QK_FULL, empty0 = is_v ? V_EMPTY : QK_EMPTY;
            const uint32_t bytes = is_v ? (uint32_t)V_BYTES : (uint32_t)(3 * p.T * 1024 + K_BYTES);
            const int nreg = is_v ? 2 : 3;
            int issued = 0;
            for (int n = 0; n < cnt; ++n) {
                const int s = n & 1;
                if (n >= 2 && !mbar_wait(&bars[empty0 + s], ((n >> 1) - 1) & 1, abort, 2u))
                    break;
                const int u = u0 + n, g = u % p.Hkv, b = u / p.Hkv;
                uint8_t *kv = is_v ? smem + OFF_V + s * V_BYTES : smem + s * QK_STAGE + Q_BYTES;
                uint64_t *full = &bars[full0 + s];
                mbar_arrive_expect_tx(full, bytes);
                for (int c = 0; c < nreg; ++c) {
                    if (!is_v) // the T tokens' G heads: token t's 8-row atom at t KB
                        tma_load_4d(smem + s * QK_STAGE + c * Q_REGION, &tmQ, full, c * 64, g * G, 0, b);
                    tma_load_4d(kv + c * KV_REGION, m0, full, c * 64, g, 0, b);
                    tma_load_4d(kv + c * KV_REGION + CAP * ROW, m1, full, c * 64, g, 0, b);
                }
                issued = n + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int n = max(0, issued - 2); n < issued; ++n)
                mbar_wait_drain(&bars[full0 + (n & 1)], (n >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0 && cnt > 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, NK, 0);
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            // A: Q in 8-row groups 1 KB apart (token t's atom is group t of an even unit, group
            // 4 + t of an odd one); B: the unit's 144 keys, 8-row groups 1 KB apart; V: N = 128
            // dims in two 64-dim regions (leading offset), K = keys in 8-row groups (stride
            // offset)
            // (stage 1: the start address advanced by the stage size >> 4; shared memory < 256 KB,
            // so the field never carries)
            const uint64_t qd0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
            const uint64_t kd0 = smem_desc_sw128(smem_u32(smem + Q_BYTES), 16, 1024);
            const uint64_t vd0 = smem_desc_sw128(smem_u32(smem + OFF_V), KV_REGION, 1024);
            constexpr uint32_t kQK16 = QK_STAGE >> 4, kV16 = V_BYTES >> 4;
            auto issue_s = [&](int n) -> bool {
                const int s = n & 1;
                if (!mbar_wait(&bars[QK_FULL + s], (n >> 1) & 1, abort, 2u))
                    return false;
                // S buffer s held S and P of unit n - 2: free once that P V is done
                if (n >= 2 && !mbar_wait(&bars[S_FREE + s], ((n >> 1) - 1) & 1, abort, 2u))
                    return false;
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t qo = (uint32_t)((kk >> 2) * Q_REGION + (kk & 3) * 32) >> 4;
                    const uint32_t ko = (uint32_t)((kk >> 2) * KV_REGION + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + s * NK, qd0 + s * (kQK16 - (4096 >> 4)) + qo, kd0 + s * kQK16 + ko,
                            idesc_s, kk > 0);
                }
                umma_commit(&bars[S_FULL + s]);
                umma_commit(&bars[QK_EMPTY + s]);
                return true;
            };
            // issue order S_0, {S_{n+1}, PV_n}
            bool ok = issue_s(0);
            for (int n = 0; ok && n < cnt; ++n) {
                const int s = n & 1;
                if (n + 1 < cnt && !issue_s(n + 1))
                    break;
                if (!mbar_wait(&bars[P_FULL + s], (n >> 1) & 1, abort, 2u) ||
                    !mbar_wait(&bars[V_FULL + s], (n >> 1) & 1, abort, 2u))
                    break;
                // O was read out by the warpgroup of unit n - 1
                if (n >= 1 && !mbar_wait(&bars[O_FREE], (n - 1) & 1, abort, 2u))
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < NK / 16; ++kk)
                    umma_ts(tmem + TMEM_O, tmem + s * NK + kk * 8,
                            vd0 + s * kV16 + (uint32_t)((kk * 16 * ROW) >> 4), idesc_o, kk > 0);
                umma_commit(&bars[PV_DONE + s]);
                umma_commit(&bars[V_EMPTY + s]);
                umma_commit(&bars[S_FREE + s]);
            }
            umma_commit(&bars[DRAIN]);
            mbar_wait_drain(&bars[DRAIN], 0);
        }
        __syncwarp();
    } else if (warp < 2) {
        // ------- softmax + epilogue: warp wg takes units n = wg, wg + 2, ... in TMEM lanes
        // 32 wg .. 32 wg + 31; lane 8 t + h is query row (token t, head g G + h)
        const int wg = warp;
        const int t = lane >> 3, hl = lane & 7;
        const bool row_ok = t < p.T;
        const uint32_t lane_addr = (uint32_t)(wg * 32) << 16;
        const float c_l2 = p.scale_log2;
        for (int n = wg; n < cnt; n += 2) {
            const RvUnit x = rv_unit(p, u0 + n);
            const int h = x.g * G + hl;
            // visible: ring slots of age index in [lo, n_cache), i.e. the circular run of
            // slots from head + lo; hidden: the other 128 - (n_cache - lo) slots from
            // head + n_cache; new tokens i_lo .. t
            const int lo = p.window > 0 ? max(x.first_c, x.n_cache + t - p.window + 1) : x.first_c;
            const int hid_e = (x.head + x.n_cache) & (CAP - 1);
            const int hid_k = CAP - max(0, x.n_cache - lo);
            const int i_lo = p.window > 0 ? max(0, t - p.window + 1) : 0;
            const int i_hi = min(t, p.T - 1);
            const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            if (!warp_wait(&bars[S_FULL + wg], (n >> 1) & 1, abort))
                break;
            tc_fence_after();
            // the row's 144 scores in one TMEM round trip (a CTA of five warps leaves each
            // thread room for them in registers), masked; the row max; then P
            const uint32_t saddr = tmem + lane_addr + wg * NK;
            uint32_t sv[NK];
            tmem_ld32(saddr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(saddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_ld32(saddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
            tmem_ld32(saddr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
            tmem_ld16(saddr + 128, *reinterpret_cast<uint32_t(*)[16]>(&sv[128]));
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < NK; i += 8)
                asm volatile("" : "+r"(sv[i]), "+r"(sv[i + 1]), "+r"(sv[i + 2]), "+r"(sv[i + 3]),
                             "+r"(sv[i + 4]), "+r"(sv[i + 5]), "+r"(sv[i + 6]), "+r"(sv[i + 7])::"memory");
#pragma unroll
            for (int c0 = 0; c0 < NK; c0 += 48)
                rv_mask48(*reinterpret_cast<uint32_t(*)[48]>(&sv[c0]),
                          rv_hidden48(c0, hid_e, hid_k, i_lo, i_hi));
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int u = 0; u < NK; ++u)
                mx4[u & 3] = fmaxf(mx4[u & 3], __uint_as_float(sv[u]));
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            // m = max(sink, max_j a_j) in log2 units (the max includes the sink)
            const float m = fmaxf(sink_l2, mx * c_l2);
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            // P = 2^(s c - m) as bf16 pairs over S's first 72 columns; the row sum of the fp32 P
            // normalises O (the P V MMA multiplies P rounded to bf16) and gives LSE
            float pe[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < NK / 16; ++k) {
                uint32_t pk[8];
#pragma unroll
                for (int u = 0; u < 16; u += 2) {
                    const float e0 = fast_exp2(fmaf(__uint_as_float(sv[k * 16 + u]), c_l2, neg_m));
                    const float e1 = fast_exp2(fmaf(__uint_as_float(sv[k * 16 + u + 1]), c_l2, neg_m));
                    pe[(u >> 1) & 3] += e0 + e1;
                    pk[u >> 1] = pack_bf16x2(e0, e1);
                }
                tmem_st8(saddr + k * 8, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            }
            // V rows of slots that hold no key: zeros (lane = slot mod 32), once V has landed,
            // seen by P V through the async proxy
            {
                bool any = false;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int cl = (lane + 32 * i - x.head) & (CAP - 1);
                    any |= cl < x.first_c || cl >= x.n_cache;
                }
                if (__any_sync(0xffffffffu, any)) {
                    if (!warp_wait(&bars[V_FULL + wg], (n >> 1) & 1, abort))
                        break;
#pragma unroll 1
                    for (int i = 0; i < 4; ++i) {
                        const int slot = lane + 32 * i, cl = (slot - x.head) & (CAP - 1);
                        if (cl >= x.first_c && cl < x.n_cache)
                            continue;
                        uint8_t *vrow = smem + OFF_V + wg * V_BYTES + slot * ROW;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            *reinterpret_cast<uint4 *>(vrow + j * 16) = make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(vrow + KV_REGION + j * 16) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[P_FULL + wg]);
            // the sink seeds both sums: exp(sink - m)
            const float s0 = (sink_l2 == -INFINITY) ? 0.f : fast_exp2(sink_l2 - m);
            const float l_exact = s0 + ((pe[0] + pe[1]) + (pe[2] + pe[3]));

            // epilogue: O = (P V) / l_exact, LSE = m + log2(l_exact)
            if (!warp_wait(&bars[PV_DONE + wg], (n >> 1) & 1, abort))
                break;
            tc_fence_after();
            const float inv_l = 1.f / l_exact;
            uint16_t *orow = p.o + (int64_t)x.b * p.o_sb + (int64_t)(row_ok ? t : 0) * p.o_st + (int64_t)h * p.o_sh;
            {
                uint32_t o[128];
                tmem_ld128(tmem + lane_addr + TMEM_O, o);
                // O is read: the next P V may overwrite it
                tc_fence_before();
                mbar_arrive(&bars[O_FREE]);
                if (row_ok) {
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        uint4 pk;
                        pk.x = pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * inv_l,
                                           __uint_as_float(o[v * 8 + 1]) * inv_l);
                        pk.y = pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * inv_l,
                                           __uint_as_float(o[v * 8 + 3]) * inv_l);
                        pk.z = pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * inv_l,
                                           __uint_as_float(o[v * 8 + 5]) * inv_l);
                        pk.w = pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * inv_l,
                                           __uint_as_float(o[v * 8 + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + v * 8) = pk;
                    }
                }
            }
            if (row_ok && p.lse)
                p.lse[((int64_t)x.b * p.T + t) * p.Hq + h] = (m + fast_log2(l_exact)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_decode_ring_umma(const CUtensorMap &q, const CUtensorMap &kc, const CUtensorMap &vc,
                                    const CUtensorMap &kn, const CUtensorMap &vn, const DecodeParams &p,
                                    int sms, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(decode_ring_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    rv::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    const int units = p.B * p.Hkv;
    // launched as a programmatic dependent: its CTAs are placed and set up (barriers, TMEM)
    // while the kernel before it finishes, and wait for it before reading memory
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units < sms ? units : sms);
    cfg.blockDim = dim3(rv::THREADS);
    cfg.dynamicSmemBytes = rv::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_ring_umma_kernel, q, kc, vc, kn, vn, p);
}

} // namespace sinkattn
