// Sink-softmax attention decode / speculative verify on tcgen05 tensor cores (sm_100a).
//
// Same computation and split-KV partial / merge scheme as the mma.sync decode kernels (sink-free
// span partials, the sink counted once when spans are merged: "MiMo-V2-Flash 架构 QA" Q3.8).
// It serves query blocks of 17..64 rows (T new tokens x G heads of one KV group, as in a
// 4-token draft verify on a 16-head group), where every KV byte feeds 64 FLOP: more than the
// warp-level mma.sync path sustains at HBM speed. Both contractions are 128-row UMMAs with TMEM
// accumulators, over 128-key steps so each instruction carries as much work as it can:
//   S = Q K^T   M 128, N 128 keys (16 for the new tokens), K 16 x 12   (A = Q in shared memory)
//   O += P V    M 128, N 128 dims, K 16 keys x 8                       (A = P in TMEM, over S)
//
// Row layout. The R query rows are loaded F = 128 / RP times (RP = 32 or 64 >= R): TMEM lane L
// holds query row r = L % RP and owns key part jp = L / RP of every 128-key step (128 / F keys).
// Each lane runs its own online softmax over its part (its P is zero on the other parts), so
// the F lanes of a row are F partial softmaxes over disjoint keys, merged once at the end the
// way split-KV partials are. All 128 lanes do softmax work and no lane waits for another.
//
// Pipelines. K and V stream through separate 2-stage rings: a K stage is free as soon as its S
// MMA has read it, a V stage once P V has. S is double-buffered in TMEM, so S of the next step
// runs on the tensor cores while the softmax warps work on this one. One thread issues the
// MMAs from two queues (S and P V) and never lets a ready P V wait behind an S whose keys are
// still loading.
//
// Work items are (span, KV head, sequence), span-major so the longest spans start first; a CTA
// takes items blockIdx.x, + gridDim.x, ... (one CTA per item, unless the host caps the grid).
//
// Roles (224 threads):
//   warps 0-3  softmax + epilogue, thread = TMEM lane;
//   warp 4     TMA producer of the cache tiles (K and V rings, run ahead across items);
//   warp 5     TMEM allocator and the UMMA issuer;
//   warp 6     TMA producer of each item's Q (once per key part) and new tokens (one 16-row box,
//              rows past T arrive as zeros).
//
// Cache tiles: contiguous caches and pages of a multiple of 128 tokens in position order; a
// ring's slots in physical order (each slot gets its position from the ring head). V rows of
// keys a tile holds but the span must not see are zeroed in shared memory before P V reads
// them, so a zero weight never meets whatever the cache held there.
#pragma once
#include "common.cuh"
#include "decode_kernels.cuh"
#include "decode_tma_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace du {
constexpr int KT = 128;                            // keys per cache step
constexpr int REGION = KT * 128;                   // 16 KB: 128 rows x 64 dims, 128B swizzle
constexpr int K_STAGE = 3 * REGION;                // 48 KB
constexpr int V_STAGE = 2 * REGION;                // 32 KB
constexpr int NK = 2, NV = 2;                      // ring depths
constexpr int NEW_ROWS = 16;                       // new-token box (T <= 4 rows + zero fill)
constexpr int NEW_REGION = NEW_ROWS * 128;         // 2 KB
constexpr int MERGE_COLS = 32;                     // O columns merged per round
constexpr int MERGE_STRIDE = MERGE_COLS + 4;       // floats per row of the merge buffer
constexpr int OFF_Q = 0;                           // 3 regions of 128 MMA rows
// Once every MMA of an item is done the Q region holds the epilogue's merge data (row
// statistics [128] float4, then the key parts' O rows [F - 1][RP][MERGE_STRIDE] floats); the
// next item's Q waits for the merge.
constexpr int OFF_ML = OFF_Q;
constexpr int OFF_OBUF = OFF_Q + 128 * 16;
constexpr int OFF_NEWK = 3 * REGION;               // 48 KB
constexpr int OFF_NEWV = OFF_NEWK + 3 * NEW_REGION;
constexpr int OFF_K = OFF_NEWV + 2 * NEW_REGION;   // 58 KB, 1 KB aligned
constexpr int OFF_V = OFF_K + NK * K_STAGE;
constexpr int OFF_BAR = OFF_V + NV * V_STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;   // barriers + 1 KB to align the base
constexpr int THREADS = 224;
constexpr int WARP_TILES = 4, WARP_MMA = 5, WARP_ITEM = 6;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 256;                   // S buffer b at column 128 b (P over it)
constexpr float TAU = 8.0f;                        // lazy-rescale threshold (log2 units)

enum Bar {
    B_QFULL = 0,              // an item's Q and new tokens have landed
    B_MERGED = 1,             // the item is merged: Q region (scratch) and new tokens free
    B_KFULL = 2,              // + K stage
    B_KEMPTY = B_KFULL + NK,
    B_VFULL = B_KEMPTY + NK,  // + V stage
    B_VEMPTY = B_VFULL + NV,
    B_SFULL = B_VEMPTY + NV,  // + S buffer
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

// The keys of step j (index 0..127 in a cache tile, 0..15 among the new tokens) as at most two
// intervals [a0, a1) u [b0, b1): those present in the span or, with `row`, those query row t may
// see (cached keys precede every new token; the window may cut the oldest). A ring tile can
// hold the span's keys in two pieces, where the ring wraps.
struct KeySpan {
    int a0, a1, b0, b1;
    SA_DEV bool has(int i) const { return (i >= a0 && i < a1) || (i >= b0 && i < b1); }
    SA_DEV bool covers(int n) const
    {
        return (a0 <= 0 && a1 >= n) || (b0 <= 0 && b1 >= n) || (b0 <= 0 && b1 >= a0 && a1 >= n) ||
               (a0 <= 0 && a1 >= b0 && b1 >= n);
    }
};

SA_DEV KeySpan du_span(const DecodeParams &p, const DecodeTiles &d, int j, bool tile_ok, bool row,
                       int t)
{
    KeySpan s{0, 0, 0, 0};
    const bool win = row && p.window > 0;
    if (j < d.cache_tiles) {
        if (p.kind == 0) {
            // logical index c = slot - head (mod ring_cap) in [clo, n_cache): unwrapped slots
            // head + clo .. head + n_cache, once as they are and once less a ring's length
            const int clo = win ? max(d.first_c, d.n_cache + t - p.window + 1) : d.first_c;
            s.a0 = d.ring_head + clo - j * du::KT;
            s.a1 = d.ring_head + d.n_cache - j * du::KT;
            s.b0 = s.a0 - p.ring_cap;
            s.b1 = s.a1 - p.ring_cap;
        } else if (tile_ok) {
            // span index v = kb + KT j + i in [vlo, min(ke, n_used))
            const int base = d.kb + j * du::KT;
            const int vlo = win ? max(d.kb, d.n_used + t - p.window + 1) : d.kb;
            s.a0 = vlo - base;
            s.a1 = min(d.ke, d.n_used) - base;
        }
    } else {
        // new token i: span index n_used + i in [kb, ke), i < T; the row sees i <= t
        s.a0 = max(0, d.kb - d.n_used);
        s.a1 = min(p.T, d.ke - d.n_used);
        if (row) {
            s.a1 = min(s.a1, t + 1);
            if (p.window > 0)
                s.a0 = max(s.a0, t - p.window + 1);
        }
    }
    return s;
}

// One work item: (span, KV head, sequence) and its steps (cache tiles, then the new tokens).
struct DuItem {
    int split, g, b, ct, nsteps;
    DecodeTiles d;
};

// The per-sequence scalars an item needs (cached length, ring head), loaded one item ahead so
// the load latency overlaps the current item.
struct DuRaw {
    int len, head;
};

SA_DEV DuRaw du_raw(const DecodeParams &p, int it, int n_items)
{
    DuRaw r{0, 0};
    if (it < n_items) {
        const int b = (it % (p.Hkv * p.B)) / p.Hkv;
        r.len = p.kind == 0 ? p.ring_len[b] : p.ctx_len[b];
        r.head = p.kind == 0 ? p.ring_head[b] : 0;
    }
    return r;
}

SA_DEV DuItem du_item(const DecodeParams &p, int it, const DuRaw &raw)
{
    DuItem x;
    // span-major: the first spans of all (sequence, head) units come first, so the CTAs with
    // the most keys start first and the short last spans fill the tail
    const int units = p.Hkv * p.B;
    x.split = it / units;
    x.b = (it % units) / p.Hkv;
    x.g = it % p.Hkv;
    x.d = decode_tiles(p, x.split, raw.len, raw.head, du::KT);
    x.ct = x.d.cache_tiles;
    x.nsteps = x.ct + (x.d.has_new ? 1 : 0);
    return x;
}

// Page of the cache tile t of item (b, span d): the page id, or -1 for a page outside the pool
// (its keys are hidden); contiguous caches and rings have no pages (0).
SA_DEV int du_page(const DecodeParams &p, const DecodeTiles &d, int b, int t)
{
    if (p.kind != 2)
        return 0;
    const int pg = (d.first_c + d.kb + t * du::KT) / p.page_size;
    if (pg >= p.max_pages)
        return -1;
    const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
    return (pid >= 0 && pid < p.num_pages) ? pid : -1;
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
    constexpr int KPT = KT / F;  // keys of a cache step per part
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *go_on = reinterpret_cast<volatile int *>(tmem_slot + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = p.splits * p.Hkv * p.B;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QFULL], 1);
        mbar_init(&bars[B_MERGED], 128);
        for (int i = 0; i < NK; ++i) {
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&bars[B_VFULL + i], 1);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[B_SFULL + i], 1);
            mbar_init(&bars[B_PFULL + i], 128);
            mbar_init(&bars[B_PVDONE + i], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort = 0;
        *go_on = 1;
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

    if (warp == WARP_TILES) {
        // ---------------- cache tiles: K and V rings across all items ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
            int tt = 0;       // tiles issued
            int k_issued = 0; // tiles whose K copy was issued (one more than tt if a V wait failed)
            bool ok = true;
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                for (int t = 0; t < x.ct; ++t, ++tt) {
                    int row, blk = x.b;
                    if (p.kind == 0) { // ring: slots in physical order
                        row = t * KT;
                    } else {
                        row = x.d.first_c + x.d.kb + t * KT; // first cached token of the tile
                        if (p.kind == 2) {
                            // a missing page is read at a block outside the pool (zeros); the
                            // softmax warps mask its keys
                            const int pid = du_page(p, x.d, x.b, t);
                            blk = pid >= 0 ? pid : p.num_pages;
                            row -= (row / p.page_size) * p.page_size;
                        }
                    }
                    const int ks = tt % NK, vs = tt % NV;
                    if (tt >= NK && !mbar_wait(&bars[B_KEMPTY + ks], ((tt / NK) - 1) & 1, abort, 2u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sk = smem + OFF_K + ks * K_STAGE;
                    mbar_arrive_expect_tx(&bars[B_KFULL + ks], K_STAGE);
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(sk + c * REGION, &tmKc, &bars[B_KFULL + ks], c * 64, x.g, row, blk);
                    k_issued = tt + 1;
                    if (tt >= NV && !mbar_wait(&bars[B_VEMPTY + vs], ((tt / NV) - 1) & 1, abort, 2u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sv = smem + OFF_V + vs * V_STAGE;
                    mbar_arrive_expect_tx(&bars[B_VFULL + vs], V_STAGE);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(sv + c * REGION, &tmVc, &bars[B_VFULL + vs], c * 64, x.g, row, blk);
                }
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int t = max(0, k_issued - NK); t < k_issued; ++t)
                mbar_wait_drain(&bars[B_KFULL + t % NK], (t / NK) & 1);
            for (int t = max(0, tt - NV); t < tt; ++t)
                mbar_wait_drain(&bars[B_VFULL + t % NV], (t / NV) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_ITEM) {
        // ---------------- Q and the new tokens of each item ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            const uint32_t qbytes = (uint32_t)(F * 3 * p.R * 128);
            int n = 0; // non-empty items loaded
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                if (x.nsteps == 0)
                    continue;
                // the Q region doubles as the previous item's merge scratch
                if (n >= 1 && !mbar_wait(&bars[B_MERGED], (n - 1) & 1, abort, 2u))
                    break;
                mbar_arrive_expect_tx(&bars[B_QFULL], qbytes + (x.d.has_new ? 5u * NEW_REGION : 0u));
                // rows (t, h) of the group: box {64 dims, G heads, T tokens}, row r = t G + h,
                // once per key part at MMA row jp * RP
                for (int jp = 0; jp < F; ++jp)
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + OFF_Q + c * REGION + jp * RP * 128, &tmQ, &bars[B_QFULL],
                                    c * 64, x.g * p.G, 0, x.b);
                if (x.d.has_new) {
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + OFF_NEWK + c * NEW_REGION, &tmKn, &bars[B_QFULL], c * 64,
                                    x.g, 0, x.b);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem + OFF_NEWV + c * NEW_REGION, &tmVn, &bars[B_QFULL], c * 64,
                                    x.g, 0, x.b);
                }
                ++n;
            }
            if (n > 0)
                mbar_wait_drain(&bars[B_QFULL], (n - 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ---------------- UMMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, KT, 0);
            const uint32_t idesc_n = umma_idesc_bf16(128, NEW_ROWS, 0);
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            const uint64_t qd = smem_desc_sw128(smem_u32(smem + OFF_Q), 16, 1024);
            const uint32_t sKn = smem_u32(smem + OFF_NEWK);
            int n = 0, tt = 0, J = 0; // items, cache tiles and steps before this item
            bool ok = true;
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                if (x.nsteps == 0)
                    continue;
                if (!mbar_wait(&bars[B_QFULL], n & 1, abort, 2u))
                    break;
                // Step j (global jg = J + j) uses S buffer jg & 1. S needs its keys landed and
                // the buffer read by the P V two steps back; P V needs P and its V landed.
                auto s_ready = [&](int j) -> bool {
                    const int jg = J + j;
                    if (jg >= 2 && !mbar_test(&bars[B_PVDONE + (jg & 1)], ((jg - 2) >> 1) & 1))
                        return false;
                    const int tg = tt + j;
                    return j >= x.ct || mbar_test(&bars[B_KFULL + tg % NK], (tg / NK) & 1);
                };
                auto issue_s = [&](int j) {
                    const int jg = J + j;
                    uint32_t kb_addr = sKn, kreg = NEW_REGION, idesc = idesc_n;
                    if (j < x.ct) {
                        kb_addr = smem_u32(smem + OFF_K + ((tt + j) % NK) * K_STAGE);
                        kreg = REGION;
                        idesc = idesc_s;
                    }
                    // descriptors advanced by the k-step's byte offset (the start-address field
                    // counts 16-byte units; shared memory < 256 KB)
                    const uint64_t kd = smem_desc_sw128(kb_addr, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 12; ++kk) {
                        const uint32_t koff = (kk & 3) * 32;
                        umma_ss(tmem + (jg & 1) * 128, qd + (((kk >> 2) * REGION + koff) >> 4),
                                kd + (((kk >> 2) * kreg + koff) >> 4), idesc, kk > 0);
                    }
                    umma_commit(&bars[B_SFULL + (jg & 1)]);
                    if (j < x.ct)
                        umma_commit(&bars[B_KEMPTY + (tt + j) % NK]); // K stage read
                };
                auto pv_ready = [&](int j) -> bool {
                    const int jg = J + j;
                    if (!mbar_test(&bars[B_PFULL + (jg & 1)], (jg >> 1) & 1))
                        return false;
                    const int tg = tt + j;
                    return j >= x.ct || mbar_test(&bars[B_VFULL + tg % NV], (tg / NV) & 1);
                };
                auto issue_pv = [&](int j) {
                    const int jg = J + j;
                    const uint32_t pt = tmem + (jg & 1) * 128; // P: 16 keys per 8 columns
                    if (j < x.ct) {
                        // B = V (16 keys x 128 dims, dims contiguous: MN-major; dims 64..127 one
                        // region further on)
                        const int vs = (tt + j) % NV;
                        const uint64_t vd = smem_desc_sw128(smem_u32(smem + OFF_V + vs * V_STAGE), REGION, 1024);
#pragma unroll
                        for (int kk = 0; kk < KT / 16; ++kk)
                            umma_ts(tmem + TMEM_O, pt + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_o,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&bars[B_PVDONE + (jg & 1)]);
                        umma_commit(&bars[B_VEMPTY + vs]);
                    } else {
                        umma_ts(tmem + TMEM_O, pt, smem_desc_sw128(smem_u32(smem + OFF_NEWV), NEW_REGION, 1024),
                                idesc_o, j > 0 ? 1u : 0u);
                        umma_commit(&bars[B_PVDONE + (jg & 1)]);
                    }
                };
                int ns = 0, np = 0; // S and P V issued
                uint64_t idle_since = 0;
                while (np < x.nsteps) {
                    if (np < ns && pv_ready(np)) {
                        tc_fence_after();
                        issue_pv(np++);
                        idle_since = 0;
                    } else if (ns < x.nsteps && ns < np + 2 && s_ready(ns)) {
                        tc_fence_after();
                        issue_s(ns++);
                        idle_since = 0;
                    } else {
                        if (*abort) {
                            ok = false;
                            break;
                        }
                        const uint64_t now = globaltimer_ns();
                        if (idle_since == 0) {
                            idle_since = now;
                        } else if (now - idle_since > kWaitLimitNs) {
                            *abort = 1;
                            atomicOr(&g_device_error, 2u);
                            ok = false;
                            break;
                        }
                    }
                }
                J += x.nsteps;
                tt += x.ct;
                ++n;
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait_drain(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else {
        // ---------- softmax warps: thread = TMEM lane = (key part, query row) ----------
        const int L = threadIdx.x;
        const int jp = L / RP, r = L % RP; // jp is warp-uniform (RP >= 32)
        const bool row_ok = r < p.R;
        const int t = row_ok ? r / p.G : 0;
        const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
        const float c_l2 = p.scale_log2;
        float4 *ml = reinterpret_cast<float4 *>(smem + OFF_ML);     // [128], after the MMAs
        float *obuf = reinterpret_cast<float *>(smem + OFF_OBUF);   // [F-1][RP][..], after the MMAs
        int n = 0, tt = 0, J = 0;
        DuRaw raw = du_raw(p, blockIdx.x, n_items);
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const DuItem x = du_item(p, it, raw);
            raw = du_raw(p, it + gridDim.x, n_items);
            const int64_t unit = ((int64_t)x.b * p.Hkv + x.g) * p.splits + x.split;
            if (x.nsteps == 0) {
                // an empty span: its partial has no keys (the merge skips l = 0)
                if (L < p.R && p.splits > 1)
                    *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + L) * 4) =
                        make_float4(-INFINITY, 0.f, 0.f, 0.f);
                continue;
            }
            const DecodeTiles &d = x.d;
            const int h = x.g * p.G + (row_ok ? r % p.G : 0);
            const float sink_h = p.sink ? p.sink[h] : -INFINITY; // used at the end of the item
            float m = -INFINITY, l_round = 0.f, l_exact = 0.f;
            bool ok = true;
            for (int j = 0; j < x.nsteps; ++j) {
                const int jg = J + j, sb = jg & 1;
                // Cache tiles and the new tokens take the same path: the new tokens are keys
                // 0..T-1 of an N = 16 step, which all fall in key part 0 (the other parts'
                // columns hold stale values and are masked).
                const bool cache = j < x.ct;
                // a paged tile's page, looked up before the wait so the load's latency hides
                const int pid = cache ? du_page(p, d, x.b, j) : 0;
                ok = warp_wait(&bars[B_SFULL + sb], (jg >> 1) & 1, abort);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t saddr = tmem + lane_addr + sb * 128;
                const bool tile_ok = pid >= 0;
                if (cache) {
                    const KeySpan present = du_span(p, d, j, tile_ok, false, 0);
                    if (!present.covers(KT)) {
                        // zero the V rows of keys outside the span: lane L takes key L, both
                        // halves, once the tile's V has landed
                        const int tg = tt + j;
                        ok = warp_wait(&bars[B_VFULL + tg % NV], (tg / NV) & 1, abort);
                        if (!ok)
                            break;
                        if (!present.has(L)) {
                            uint8_t *vrow = smem + OFF_V + (tg % NV) * V_STAGE + L * 128;
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                *reinterpret_cast<uint4 *>(vrow + u * 16) = make_uint4(0u, 0u, 0u, 0u);
                                *reinterpret_cast<uint4 *>(vrow + REGION + u * 16) = make_uint4(0u, 0u, 0u, 0u);
                            }
                        }
                        fence_async_smem();
                    }
                }
                uint32_t raw_s[KPT];
                if constexpr (KPT == 64) {
                    tmem_ld32(saddr + jp * KPT, *reinterpret_cast<uint32_t(*)[32]>(&raw_s[0]));
                    tmem_ld32(saddr + jp * KPT + 32, *reinterpret_cast<uint32_t(*)[32]>(&raw_s[32]));
                    tmem_ld_wait();
                } else {
                    tmem_ld32_sync(saddr + jp * KPT, *reinterpret_cast<uint32_t(*)[32]>(&raw_s[0]));
                }
                const KeySpan vis = row_ok ? du_span(p, d, j, tile_ok, true, t) : KeySpan{0, 0, 0, 0};
                float xs[KPT];
                if (vis.a0 <= jp * KPT && vis.a1 >= (jp + 1) * KPT) { // every key of the part
#pragma unroll
                    for (int c = 0; c < KPT; ++c)
                        xs[c] = __uint_as_float(raw_s[c]);
                } else {
#pragma unroll
                    for (int c = 0; c < KPT; ++c)
                        xs[c] = vis.has(jp * KPT + c) ? __uint_as_float(raw_s[c]) : -INFINITY;
                }
                uint32_t pk[KPT / 2];
                float alpha;
                const bool rescale = du_softmax<KPT>(xs, c_l2, m, l_round, l_exact, alpha, pk);
                // P over S: this lane's part at columns jp KPT / 2 .., zeros on the other parts
#pragma unroll
                for (int q = 0; q < KPT / 16; ++q)
                    tmem_st8(saddr + jp * (KPT / 2) + q * 8, pk[8 * q], pk[8 * q + 1], pk[8 * q + 2],
                             pk[8 * q + 3], pk[8 * q + 4], pk[8 * q + 5], pk[8 * q + 6], pk[8 * q + 7]);
#pragma unroll
                for (int q8 = 0; q8 < KT / 16; ++q8)
                    if (q8 / (KPT / 16) != jp)
                        tmem_st8(saddr + q8 * 8, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u);
                // O holds P V up to step j - 1: rescale it to the new reference max (the first
                // step's P V overwrites O)
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                    ok = warp_wait(&bars[B_PVDONE + ((jg - 1) & 1)], ((jg - 1) >> 1) & 1, abort);
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
            const int jl = J + x.nsteps - 1;
            if (ok)
                ok = warp_wait(&bars[B_PVDONE + (jl & 1)], (jl >> 1) & 1, abort);
            tc_fence_after();
            J += x.nsteps;
            tt += x.ct;

            // ---- merge the F key parts of each row (all MMAs of the item are done: the Q
            // region is scratch); every softmax thread takes every barrier
            ml[L] = make_float4(m, l_round, l_exact, 0.f);
            if (L == 0)
                *go_on = !*abort; // one decision for the four warps, read after the barriers
            named_bar_sync(1, 128);
            float mf = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < F; ++jj)
                mf = fmaxf(mf, ml[jj * RP + r].x);
            float lr = 0.f, le = 0.f;
#pragma unroll
            for (int jj = 0; jj < F; ++jj) {
                const float4 v4 = ml[jj * RP + r];
                const float c = (v4.x == -INFINITY) ? 0.f : fast_exp2(v4.x - mf);
                lr += v4.y * c;
                le += v4.z * c;
            }
            const float a_self = (m == -INFINITY) ? 0.f : fast_exp2(m - mf);
            const bool writer = jp == 0 && row_ok;
            // final scaling (single span: the sink applied once) or the span's partial
            float scl = 1.f, lse = 0.f;
            if (writer && p.splits == 1) {
                const float sk = sink_h * kLog2e;
                const float mf2 = fmaxf(mf, sk);
                const float cm = (mf == -INFINITY) ? 0.f : fast_exp2(mf - mf2);
                const float cs = (sk == -INFINITY) ? 0.f : fast_exp2(sk - mf2);
                scl = cm / (lr * cm + cs);
                lse = (mf2 + fast_log2(le * cm + cs)) * kLn2;
            }
            uint16_t *orow = p.o + (int64_t)x.b * p.o_sb + (int64_t)t * p.o_st + (int64_t)h * p.o_sh;
            float *wrow = p.ws_o ? p.ws_o + (unit * p.R + r) * 128 : nullptr;
            const bool cont = *go_on != 0;
            const bool write = writer && ok && cont;
#pragma unroll 1
            for (int c = 0; c < 128 / MERGE_COLS; ++c) {
                uint32_t o[MERGE_COLS];
                tmem_ld32_sync(tmem + lane_addr + TMEM_O + c * MERGE_COLS, o);
                if (jp > 0) {
                    float4 *dst = reinterpret_cast<float4 *>(obuf + ((jp - 1) * RP + r) * MERGE_STRIDE);
#pragma unroll
                    for (int q = 0; q < MERGE_COLS / 4; ++q)
                        dst[q] = make_float4(__uint_as_float(o[4 * q]) * a_self,
                                             __uint_as_float(o[4 * q + 1]) * a_self,
                                             __uint_as_float(o[4 * q + 2]) * a_self,
                                             __uint_as_float(o[4 * q + 3]) * a_self);
                }
                named_bar_sync(1, 128);
                if (write) {
                    float v[MERGE_COLS];
#pragma unroll
                    for (int e = 0; e < MERGE_COLS; ++e)
                        v[e] = __uint_as_float(o[e]) * a_self;
#pragma unroll
                    for (int jj = 1; jj < F; ++jj) {
                        const float4 *src = reinterpret_cast<const float4 *>(
                            obuf + ((jj - 1) * RP + r) * MERGE_STRIDE);
#pragma unroll
                        for (int q = 0; q < MERGE_COLS / 4; ++q) {
                            const float4 w4 = src[q];
                            v[4 * q] += w4.x;
                            v[4 * q + 1] += w4.y;
                            v[4 * q + 2] += w4.z;
                            v[4 * q + 3] += w4.w;
                        }
                    }
                    const int col = c * MERGE_COLS;
                    if (p.splits == 1) {
#pragma unroll
                        for (int q = 0; q < MERGE_COLS / 8; ++q) {
                            uint4 pk;
                            pk.x = pack_bf16x2(v[8 * q + 0] * scl, v[8 * q + 1] * scl);
                            pk.y = pack_bf16x2(v[8 * q + 2] * scl, v[8 * q + 3] * scl);
                            pk.z = pack_bf16x2(v[8 * q + 4] * scl, v[8 * q + 5] * scl);
                            pk.w = pack_bf16x2(v[8 * q + 6] * scl, v[8 * q + 7] * scl);
                            *reinterpret_cast<uint4 *>(orow + col + 8 * q) = pk;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < MERGE_COLS / 4; ++q)
                            *reinterpret_cast<float4 *>(wrow + col + 4 * q) =
                                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
                named_bar_sync(1, 128);
            }
            // O and the merge scratch are free: the next item may load its Q and new tokens
            tc_fence_before();
            mbar_arrive(&bars[B_MERGED]);
            if (write) {
                if (p.splits == 1) {
                    if (p.lse)
                        p.lse[((int64_t)x.b * p.T + t) * p.Hq + h] = lse;
                } else {
                    *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + r) * 4) =
                        make_float4(mf, lr, le, 0.f);
                }
            }
            ++n;
            if (!cont)
                break;
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
                               int max_ctas, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        cudaError_t e = cudaFuncSetAttribute(
            decode_umma_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, du::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(decode_umma_kernel<4>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, du::SMEM_BYTES);
        return e;
    });
    if (e != cudaSuccess)
        return e;
    const int n_items = p.splits * p.Hkv * p.B;
    const int grid = (max_ctas > 0 && max_ctas < n_items) ? max_ctas : n_items;
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
