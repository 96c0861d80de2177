// Sink-softmax attention decode / speculative verify on tcgen05 tensor cores (sm_100a).
//
// Same computation and split-KV partial / merge scheme as the mma.sync decode kernels (sink-free
// span partials, the sink counted once when spans are merged: "MiMo-V2-Flash 架构 QA" Q3.8). It
// serves query blocks of more than 16 rows: T new tokens x G heads of one KV group, up to 64
// rows, as in a 4-token draft verify on a 16-head group. There every KV byte feeds 64 FLOP,
// which the warp-level mma.sync path cannot sustain at HBM speed; here both contractions are
// 128-row UMMAs with TMEM accumulators:
//   S = Q K^T   M 128, N 64 keys, K 16 x 12          (A = Q from shared memory)
//   O += P V    M 128, N 128 dims, K 16 keys x 4     (A = P from TMEM, written over S)
//
// Row layout. The R query rows are loaded F = 128 / RP times (RP = 32 or 64 >= R): TMEM lane L
// holds query row r = L % RP and owns key part jp = L / RP of every 64-key tile (64 / F keys).
// Each lane runs its own online softmax over its part (its P is zero on the other parts), so
// the F lanes of a row are F partial softmaxes over disjoint keys, merged once at the end the
// way split-KV partials are. All 128 lanes do softmax work and no lane waits for another.
//
// Roles (192 threads): warps 0-3 softmax + epilogue (thread = TMEM lane); warp 4 TMA producer
// (Q and the new tokens once, then the 64-key cache tiles through a 4-stage ring); warp 5 TMEM
// allocator and the single UMMA issuer, in the order S_0, {S_j+1, PV_j}.
//
// Cache tiles are those of the TMA decode kernel (contiguous, or pages of a multiple of 64
// tokens); the T new tokens follow as one 16-row box (rows past T arrive as zeros) through an
// N = 16 step. V rows of keys a tile holds but the span must not see are zeroed in shared
// memory before P V reads them, so a zero weight never meets whatever the cache held there.
#pragma once
#include "common.cuh"
#include "decode_kernels.cuh"
#include "decode_tma_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace du {
constexpr int KT = 64;                             // keys per cache tile
constexpr int REGION = KT * 128;                   // 8 KB: 64 keys x 64 dims, 128B swizzle
constexpr int STAGE = 5 * REGION;                  // K (3 regions) + V (2 regions): 40 KB
constexpr int NSTAGE = 4;
constexpr int Q_REGION = 128 * 128;                // 16 KB: 128 MMA rows x 64 dims
constexpr int NEW_ROWS = 16;                       // new-token box (T <= 4 rows + zero fill)
constexpr int NEW_REGION = NEW_ROWS * 128;         // 2 KB
constexpr int OFF_Q = 0;
constexpr int OFF_NEWK = 3 * Q_REGION;             // 48 KB
constexpr int OFF_NEWV = OFF_NEWK + 3 * NEW_REGION;
constexpr int OFF_STAGE = OFF_NEWV + 2 * NEW_REGION; // 58 KB, 1 KB aligned
constexpr int OFF_BAR = OFF_STAGE + NSTAGE * STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;   // barriers + 1 KB to align the base
constexpr int THREADS = 192;
constexpr int WARP_LOAD = 4, WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TMEM_S = 0;                     // S buffer i at column 64 i; P over it
constexpr uint32_t TMEM_O = 128;
constexpr float TAU = 8.0f;                        // lazy-rescale threshold (log2 units)
constexpr int MERGE_STRIDE = 36;                   // floats per row of the merge buffer

enum Bar {
    B_QN = 0,                 // Q and the new tokens
    B_FULL = 1,               // + stage
    B_EMPTY = B_FULL + NSTAGE,
    B_SFULL = B_EMPTY + NSTAGE, // + S buffer
    B_PFULL = B_SFULL + 2,
    B_PVDONE = B_PFULL + 2,
    B_DRAIN = B_PVDONE + 2,
    NUM_BARS = B_DRAIN + 1
};
} // namespace du

// Online-softmax step over NC scores of one lane (raw q.k, masked ones -inf): raises the
// reference max when a score exceeds it by more than TAU (or on the first visible score),
// returns P = 2^(s c - m) as bf16 pairs and adds the fp32 and the rounded sums.
template <int NC>
SA_DEV bool du_softmax(const float (&x)[NC], float c_l2, float &m, float &l_round, float &l_exact,
                       float &alpha, uint32_t (&pk)[NC / 2])
{
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < NC; ++c)
        mx4[c & 3] = fmaxf(mx4[c & 3], x[c]);
    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c_l2;
    const bool rescale = mx > m + du::TAU; // always true for the first finite max (m = -inf)
    alpha = 1.f;
    if (rescale) {
        alpha = fast_exp2(m - mx); // 0 while m is -inf
        l_round *= alpha;
        l_exact *= alpha;
        m = mx;
    }
    const float neg_m = (m == -INFINITY) ? 0.f : -m;
    float pe[2] = {0.f, 0.f}, pr[2] = {0.f, 0.f};
#pragma unroll
    for (int u = 0; u < NC / 2; ++u) {
        const float e0 = fast_exp2(fmaf(x[2 * u], c_l2, neg_m));
        const float e1 = fast_exp2(fmaf(x[2 * u + 1], c_l2, neg_m));
        pk[u] = pack_bf16x2(e0, e1);
        pe[u & 1] += e0 + e1;
        pr[u & 1] += sum_bf16x2(pk[u]);
    }
    l_exact += pe[0] + pe[1];
    l_round += pr[0] + pr[1];
    return rescale;
}

template <int F>
__global__ void __launch_bounds__(du::THREADS, 1)
    decode_umma_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmKc,
                       const __grid_constant__ CUtensorMap tmVc,
                       const __grid_constant__ CUtensorMap tmKn,
                       const __grid_constant__ CUtensorMap tmVn, const DecodeParams p)
{
    using namespace du;
    constexpr int RP = 128 / F;  // MMA rows per key part
    constexpr int KPT = KT / F;  // keys of a cache tile per part
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const DecodeTiles d = decode_tiles(p, b, split);
    const int ct = d.cache_tiles;
    const int nsteps = ct + (d.has_new ? 1 : 0);

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QN], 1);
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&bars[B_FULL + i], 1);
            mbar_init(&bars[B_EMPTY + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
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

    if (warp == WARP_LOAD) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && nsteps > 0) {
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
            const uint32_t qbytes = (uint32_t)(F * 3 * p.R * 128);
            mbar_arrive_expect_tx(&bars[B_QN], qbytes + (d.has_new ? 5u * NEW_REGION : 0u));
            // Q rows (t, h) of this group: box {64 dims, G heads, T tokens}, row r = t G + h,
            // once per key part at MMA row jp * RP
            for (int jp = 0; jp < F; ++jp)
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + OFF_Q + c * Q_REGION + jp * RP * 128, &tmQ, &bars[B_QN],
                                c * 64, g * p.G, 0, b);
            if (d.has_new) {
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + OFF_NEWK + c * NEW_REGION, &tmKn, &bars[B_QN], c * 64, g, 0, b);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(smem + OFF_NEWV + c * NEW_REGION, &tmVn, &bars[B_QN], c * 64, g, 0, b);
            }
            int issued = 0;
            for (int t = 0; t < ct; ++t) {
                const int st = t % NSTAGE;
                if (t >= NSTAGE && !mbar_wait(&bars[B_EMPTY + st], ((t / NSTAGE) - 1) & 1, abort, 2u))
                    break;
                uint8_t *sk = smem + OFF_STAGE + st * STAGE;
                mbar_arrive_expect_tx(&bars[B_FULL + st], STAGE);
                const int c0 = d.first_c + d.kb + t * KT; // first cached token of the tile
                int row = c0, blk = b;
                if (p.kind == 2) {
                    const int pg = c0 / p.page_size;
                    // a missing page is read at a block outside the pool (zeros); the softmax
                    // warps mask its keys
                    blk = decode_tile_ok(p, d, b, t) ? p.page_table[(int64_t)b * p.max_pages + pg]
                                                     : p.num_pages;
                    row = c0 - pg * p.page_size;
                }
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(sk + c * REGION, &tmKc, &bars[B_FULL + st], c * 64, g, row, blk);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d(sk + (3 + c) * REGION, &tmVc, &bars[B_FULL + st], c * 64, g, row, blk);
                issued = t + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int t = max(0, issued - NSTAGE); t < issued; ++t)
                mbar_wait_drain(&bars[B_FULL + t % NSTAGE], (t / NSTAGE) & 1);
            mbar_wait_drain(&bars[B_QN], 0);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ---------------- UMMA issuer ----------------
        if (lane == 0 && nsteps > 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, KT, 0);
            const uint32_t idesc_n = umma_idesc_bf16(128, NEW_ROWS, 0);
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            const uint32_t sQ = smem_u32(smem + OFF_Q);
            const uint32_t sKn = smem_u32(smem + OFF_NEWK), sVn = smem_u32(smem + OFF_NEWV);
            bool ok = mbar_wait(&bars[B_QN], 0, abort, 2u);
            // S_j = Q K_j^T into S buffer j & 1, once P V of step j - 2 has read that buffer
            auto issue_s = [&](int j) -> bool {
                const int sb = j & 1;
                if (j >= 2 && !mbar_wait(&bars[B_PVDONE + sb], ((j - 2) >> 1) & 1, abort, 2u))
                    return false;
                uint32_t kb_addr = sKn, kreg = NEW_REGION, idesc = idesc_n;
                if (j < ct) {
                    const int st = j % NSTAGE;
                    if (!mbar_wait(&bars[B_FULL + st], (j / NSTAGE) & 1, abort, 2u))
                        return false;
                    kb_addr = smem_u32(smem + OFF_STAGE + st * STAGE);
                    kreg = REGION;
                    idesc = idesc_s;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    umma_ss(tmem + TMEM_S + sb * 64,
                            smem_desc_sw128(sQ + (kk >> 2) * Q_REGION + koff, 16, 1024),
                            smem_desc_sw128(kb_addr + (kk >> 2) * kreg + koff, 16, 1024), idesc,
                            kk > 0);
                }
                umma_commit(&bars[B_SFULL + sb]);
                return true;
            };
            if (ok)
                ok = issue_s(0);
            for (int j = 0; ok && j < nsteps; ++j) {
                if (j + 1 < nsteps && !issue_s(j + 1))
                    break;
                if (!mbar_wait(&bars[B_PFULL + (j & 1)], (j >> 1) & 1, abort, 2u))
                    break;
                tc_fence_after();
                const uint32_t pt = tmem + TMEM_S + (j & 1) * 64; // P: 16 keys per 8 columns
                if (j < ct) {
                    // B = V (16 keys x 128 dims, dims contiguous: MN-major; dims 64..127 one
                    // region further on)
                    const uint32_t sV = smem_u32(smem + OFF_STAGE + (j % NSTAGE) * STAGE + 3 * REGION);
#pragma unroll
                    for (int kk = 0; kk < KT / 16; ++kk)
                        umma_ts(tmem + TMEM_O, pt + kk * 8,
                                smem_desc_sw128(sV + kk * 16 * 128, REGION, 1024), idesc_o,
                                (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bars[B_PVDONE + (j & 1)]);
                    umma_commit(&bars[B_EMPTY + j % NSTAGE]);
                } else {
                    umma_ts(tmem + TMEM_O, pt, smem_desc_sw128(sVn, NEW_REGION, 1024), idesc_o,
                            j > 0 ? 1u : 0u);
                    umma_commit(&bars[B_PVDONE + (j & 1)]);
                }
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait_drain(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else if (nsteps > 0) {
        // ---------------- softmax warps: thread = TMEM lane = (key part, query row) ----------
        const int L = threadIdx.x;
        const int jp = L / RP, r = L % RP; // jp is warp-uniform (RP >= 32)
        const bool row_ok = r < p.R;
        const int t = row_ok ? r / p.G : 0;
        const int h = g * p.G + (row_ok ? r % p.G : 0);
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const float c_l2 = p.scale_log2;
        float m = -INFINITY, l_round = 0.f, l_exact = 0.f;
        bool ok = true;
        for (int j = 0; j < nsteps; ++j) {
            const int sb = j & 1;
            ok = warp_wait(&bars[B_SFULL + sb], (j >> 1) & 1, abort);
            if (!ok)
                break;
            tc_fence_after();
            const uint32_t saddr = tmem + lane_addr + TMEM_S + sb * 64;
            float alpha;
            bool rescale;
            if (j < ct) {
                const bool tile_ok = decode_tile_ok(p, d, b, j);
                const int v0 = d.kb + j * KT; // span index of the tile's first key
                const bool all_valid = tile_ok && v0 + KT <= min(d.ke, d.n_used);
                // cached keys sit before every new token; the window may cut the oldest
                const bool all_vis = all_valid && (p.window <= 0 || v0 - d.n_used > p.T - 1 - p.window);
                if (!all_valid) {
                    // zero the V rows of keys outside the span: lane L takes key L % 64, half L / 64
                    bool valid;
                    int pos;
                    decode_key(p, d, j, L & 63, tile_ok, valid, pos);
                    if (!valid) {
                        uint4 *row = reinterpret_cast<uint4 *>(smem + OFF_STAGE + (j % NSTAGE) * STAGE +
                                                               (3 + (L >> 6)) * REGION + (L & 63) * 128);
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            row[u] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_async_smem();
                }
                uint32_t raw[KPT];
                if constexpr (KPT == 32) {
                    tmem_ld32_sync(saddr + jp * KPT, raw);
                } else {
                    tmem_ld16_sync(saddr + jp * KPT, raw);
                }
                float x[KPT];
                if (all_vis && row_ok) {
#pragma unroll
                    for (int c = 0; c < KPT; ++c)
                        x[c] = __uint_as_float(raw[c]);
                } else {
#pragma unroll
                    for (int c = 0; c < KPT; ++c) {
                        bool valid;
                        int pos;
                        decode_key(p, d, j, jp * KPT + c, tile_ok, valid, pos);
                        const bool vis = row_ok && valid && pos <= t &&
                                         (p.window <= 0 || pos > t - p.window);
                        x[c] = vis ? __uint_as_float(raw[c]) : -INFINITY;
                    }
                }
                uint32_t pk[KPT / 2];
                rescale = du_softmax<KPT>(x, c_l2, m, l_round, l_exact, alpha, pk);
                // P of this lane's part; zeros on the other parts (columns = key pairs)
#pragma unroll
                for (int jj = 0; jj < F; ++jj) {
                    if (jj != jp)
                        continue;
#pragma unroll
                    for (int q8 = 0; q8 < KT / 16; ++q8) {
                        const int rel = q8 * 8 - jj * (KPT / 2); // first column relative to the part
                        if (rel >= 0 && rel < KPT / 2)
                            tmem_st8(saddr + q8 * 8, pk[rel + 0], pk[rel + 1], pk[rel + 2],
                                     pk[rel + 3], pk[rel + 4], pk[rel + 5], pk[rel + 6], pk[rel + 7]);
                        else
                            tmem_st8(saddr + q8 * 8, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u);
                    }
                }
            } else {
                // the new tokens: 16 columns, keys 16 / F * jp .. of this lane's part
                uint32_t raw[16];
                tmem_ld16_sync(saddr, raw);
                float x[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    bool valid;
                    int pos;
                    decode_key(p, d, j, c, true, valid, pos);
                    const bool vis = row_ok && valid && c / (16 / F) == jp && pos <= t &&
                                     (p.window <= 0 || pos > t - p.window);
                    x[c] = vis ? __uint_as_float(raw[c]) : -INFINITY;
                }
                uint32_t pk[8];
                rescale = du_softmax<16>(x, c_l2, m, l_round, l_exact, alpha, pk);
                tmem_st8(saddr, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
            }
            // O holds P V up to step j - 1: rescale it to the new reference max
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                ok = warp_wait(&bars[B_PVDONE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort);
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
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + sb]);
        }
        if (ok)
            ok = warp_wait(&bars[B_PVDONE + ((nsteps - 1) & 1)], ((nsteps - 1) >> 1) & 1, abort);
        tc_fence_after();

        // ---- merge the F key parts of each row (every softmax thread takes every barrier) ----
        float4 *mlbuf = reinterpret_cast<float4 *>(smem + OFF_Q);         // Q is no longer read
        float *obuf = reinterpret_cast<float *>(smem + OFF_Q + 128 * 16); // [F-1][RP][STRIDE]
        mlbuf[L] = make_float4(m, l_round, l_exact, 0.f);
        named_bar_sync(1, 128);
        float mf = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < F; ++jj)
            mf = fmaxf(mf, mlbuf[jj * RP + r].x);
        float lr = 0.f, le = 0.f;
#pragma unroll
        for (int jj = 0; jj < F; ++jj) {
            const float4 ml = mlbuf[jj * RP + r];
            const float c = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - mf);
            lr += ml.y * c;
            le += ml.z * c;
        }
        const float a_self = (m == -INFINITY) ? 0.f : fast_exp2(m - mf);
        const bool writer = jp == 0 && row_ok;
        // final scaling (single span: the sink applied once) or the span's partial
        float scl = 1.f, lse = 0.f;
        if (writer && p.splits == 1) {
            const float sk = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            const float mf2 = fmaxf(mf, sk);
            const float cm = (mf == -INFINITY) ? 0.f : fast_exp2(mf - mf2);
            const float cs = (sk == -INFINITY) ? 0.f : fast_exp2(sk - mf2);
            scl = cm / (lr * cm + cs);
            lse = (mf2 + fast_log2(le * cm + cs)) * kLn2;
        }
        const int64_t unit = ((int64_t)b * p.Hkv + g) * p.splits + split;
        uint16_t *orow = p.o + (int64_t)b * p.o_sb + (int64_t)t * p.o_st + (int64_t)h * p.o_sh;
        float *wrow = p.ws_o ? p.ws_o + (unit * p.R + r) * 128 : nullptr;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32_sync(tmem + lane_addr + TMEM_O + c * 32, o);
            if (jp > 0) {
                float4 *dst = reinterpret_cast<float4 *>(obuf + ((jp - 1) * RP + r) * MERGE_STRIDE);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    dst[k] = make_float4(__uint_as_float(o[4 * k]) * a_self,
                                         __uint_as_float(o[4 * k + 1]) * a_self,
                                         __uint_as_float(o[4 * k + 2]) * a_self,
                                         __uint_as_float(o[4 * k + 3]) * a_self);
            }
            named_bar_sync(1, 128);
            if (writer && ok && !*abort) {
                float acc[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    acc[e] = __uint_as_float(o[e]) * a_self;
#pragma unroll
                for (int jj = 1; jj < F; ++jj) {
                    const float4 *src = reinterpret_cast<const float4 *>(obuf + ((jj - 1) * RP + r) * MERGE_STRIDE);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float4 v = src[k];
                        acc[4 * k] += v.x;
                        acc[4 * k + 1] += v.y;
                        acc[4 * k + 2] += v.z;
                        acc[4 * k + 3] += v.w;
                    }
                }
                if (p.splits == 1) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint4 pk;
                        pk.x = pack_bf16x2(acc[8 * k + 0] * scl, acc[8 * k + 1] * scl);
                        pk.y = pack_bf16x2(acc[8 * k + 2] * scl, acc[8 * k + 3] * scl);
                        pk.z = pack_bf16x2(acc[8 * k + 4] * scl, acc[8 * k + 5] * scl);
                        pk.w = pack_bf16x2(acc[8 * k + 6] * scl, acc[8 * k + 7] * scl);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + 8 * k) = pk;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        *reinterpret_cast<float4 *>(wrow + c * 32 + 4 * k) =
                            make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
                }
            }
            named_bar_sync(1, 128);
        }
        if (writer && ok && !*abort) {
            if (p.splits == 1) {
                if (p.lse)
                    p.lse[((int64_t)b * p.T + t) * p.Hq + h] = lse;
            } else {
                *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + r) * 4) =
                    make_float4(mf, lr, le, 0.f);
            }
        }
    } else {
        // an empty span: its partial has no keys (the merge skips l = 0)
        const int L = threadIdx.x;
        if (L < p.R && p.splits > 1) {
            const int64_t unit = ((int64_t)b * p.Hkv + g) * p.splits + split;
            *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + L) * 4) =
                make_float4(-INFINITY, 0.f, 0.f, 0.f);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

cudaError_t launch_decode_umma(const CUtensorMap &q, const CUtensorMap &kc, const CUtensorMap &vc,
                               const CUtensorMap &kn, const CUtensorMap &vn, const DecodeParams &p,
                               cudaStream_t stream)
{
    static int configured_devices = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 32 && !(configured_devices & (1 << dev))) {
        e = cudaFuncSetAttribute(decode_umma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 du::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_umma_kernel<4>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, du::SMEM_BYTES);
        if (e != cudaSuccess)
            return e;
        configured_devices |= (1 << dev);
    }
    dim3 grid(p.splits, p.Hkv, p.B);
    if (p.R > 32)
        decode_umma_kernel<2><<<grid, du::THREADS, du::SMEM_BYTES, stream>>>(q, kc, vc, kn, vn, p);
    else
        decode_umma_kernel<4><<<grid, du::THREADS, du::SMEM_BYTES, stream>>>(q, kc, vc, kn, vn, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.splits == 1)
        return e;
    return launch_decode_merge(p, stream);
}

} // namespace sinkattn
