// Sink-softmax attention decode / speculative verify on tcgen05 tensor cores (sm_100a).
//
// Same computation and split-KV partial / merge scheme as the mma.sync decode kernels (sink-free
// span partials, the sink counted once when spans are merged: "MiMo-V2-Flash 架构 QA" Q3.8).
// Both contractions are 128-row UMMAs with TMEM accumulators and A operands in TMEM:
//   S = Q K^T   M 128, N 64 keys (16 for the new tokens), K 16 x 12  (A = Q in TMEM)
//   O += P V    M 128, N 128 dims, K 16 keys per instruction        (A = P in TMEM, over S)
// It serves query blocks of 17..64 rows (T new tokens x G heads of one KV group, as in a
// 4-token draft verify on a 16-head group), where every KV byte feeds 64 FLOP: more than the
// warp-level mma.sync path sustains at HBM speed.
//
// Row layout. The R query rows are loaded F = 128 / RP times (RP = 32 or 64 >= R): TMEM lane L
// holds query row r = L % RP and owns key part jp = L / RP of every 64-key tile (64 / F keys).
// Each lane runs its own online softmax over its part (its P is zero on the other parts), so
// the F lanes of a row are F partial softmaxes over disjoint keys, merged once at the end the
// way split-KV partials are. All 128 lanes do softmax work and no lane waits for another.
//
// Two softmax warpgroups take alternate tiles (warpgroup g the steps j = g, g + 2, ...), each
// with its own S buffer and O accumulator in TMEM; at the end of an item warpgroup 0 folds
// warpgroup 1's O into its own (same lanes) and then merges the key parts in shared memory.
//
// Work items are (span, KV head, sequence), span-major so the longest spans start first; a CTA
// takes items blockIdx.x, + gridDim.x, ... (one CTA per item, unless the host caps the grid).
//
// Roles (352 threads):
//   warps 0-7  softmax + epilogue (two warpgroups), thread = TMEM lane; warpgroup 0 also writes
//              each item's Q rows into TMEM;
//   warp 8     TMA producer of the 64-key cache tiles (5-stage ring, runs ahead across items);
//   warp 9     TMEM allocator and the single UMMA issuer, which keeps an S queue and a P V
//              queue and never lets a ready P V wait behind an S whose tile is still loading;
//   warp 10    TMA producer of each item's new tokens (one 16-row box, rows past T arrive as
//              zeros).
//
// Cache tiles: contiguous caches and pages of a multiple of 64 tokens in position order; a
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
constexpr int KT = 64;                             // keys per cache tile
constexpr int REGION = KT * 128;                   // 8 KB: 64 keys x 64 dims, 128B swizzle
constexpr int STAGE = 5 * REGION;                  // K (3 regions) + V (2 regions): 40 KB
constexpr int NSTAGE = 5;
constexpr int NEW_ROWS = 16;                       // new-token box (T <= 4 rows + zero fill)
constexpr int NEW_REGION = NEW_ROWS * 128;         // 2 KB
constexpr int MERGE_COLS = 32;                     // O columns merged per round
constexpr int MERGE_STRIDE = MERGE_COLS + 4;       // floats per row of the merge buffer
constexpr int OFF_NEWK = 0;                        // new K: 3 regions
constexpr int OFF_NEWV = OFF_NEWK + 3 * NEW_REGION; // new V: 2 regions
// Once every MMA of an item is done (and until the next item's new tokens load) the start of
// shared memory holds the epilogue's merge data: row statistics [128] (float4), then the key
// parts' O rows [F - 1][RP][MERGE_STRIDE] floats.
constexpr int OFF_ML0 = 0;
constexpr int OFF_OBUF = OFF_ML0 + 128 * 16;
constexpr int OFF_ML1 = 16 * 1024;                 // warpgroup 1's row statistics [128]
constexpr int OFF_STAGE = OFF_ML1 + 2 * 1024;      // 18 KB, 1 KB aligned
constexpr int OFF_BAR = OFF_STAGE + NSTAGE * STAGE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;   // barriers + 1 KB to align the base
constexpr int THREADS = 352;
constexpr int WARP_TILES = 8, WARP_MMA = 9, WARP_ITEM = 10;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: S of warpgroup g at 64 g (P over it); O of warpgroup g at 128 + 128 g; Q (the
// A operand of S = Q K^T, dims 2c and 2c + 1 in column c) at 384
constexpr uint32_t TMEM_O = 128;
constexpr uint32_t TMEM_Q = 384;
constexpr float TAU = 8.0f;                        // lazy-rescale threshold (log2 units)

enum Bar {
    B_NEWFULL = 0,            // an item's new tokens have landed
    B_QT = 1,                 // an item's Q is in TMEM (warpgroup 0)
    B_MERGED = 2,             // warpgroup 0 has merged an item: new-token buffers and O_1 free
    B_FULL = 3,               // + stage
    B_EMPTY = B_FULL + NSTAGE,
    B_SFULL = B_EMPTY + NSTAGE, // + warpgroup
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

// The keys of step j (index 0..63 in a cache tile, 0..15 among the new tokens) as at most two
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
            // span index v = kb + 64 j + i in [vlo, min(ke, n_used))
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
    x.d = decode_tiles(p, x.split, raw.len, raw.head);
    x.ct = x.d.cache_tiles;
    x.nsteps = x.ct + (x.d.has_new ? 1 : 0);
    return x;
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
    volatile int *go_on = reinterpret_cast<volatile int *>(tmem_slot + 2); // [2], per item parity
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = p.splits * p.Hkv * p.B;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_NEWFULL], 1);
        mbar_init(&bars[B_QT], 128);
        mbar_init(&bars[B_MERGED], 128);
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
        go_on[0] = go_on[1] = 1;
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
        // ---------------- cache tiles: one 3-stage ring across all items ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tmKc);
            tma_prefetch_desc(&tmVc);
            int tt = 0; // tiles issued
            bool ok = true;
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                for (int t = 0; t < x.ct; ++t, ++tt) {
                    const int st = tt % NSTAGE;
                    if (tt >= NSTAGE && !mbar_wait(&bars[B_EMPTY + st], ((tt / NSTAGE) - 1) & 1, abort, 2u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sk = smem + OFF_STAGE + st * STAGE;
                    mbar_arrive_expect_tx(&bars[B_FULL + st], STAGE);
                    int row, blk = x.b;
                    if (p.kind == 0) { // ring: slots in physical order
                        row = t * KT;
                    } else {
                        row = x.d.first_c + x.d.kb + t * KT; // first cached token of the tile
                        if (p.kind == 2) {
                            const int pg = row / p.page_size;
                            // a missing page is read at a block outside the pool (zeros); the
                            // softmax warps mask its keys
                            blk = decode_tile_ok(p, x.d, x.b, t)
                                      ? p.page_table[(int64_t)x.b * p.max_pages + pg]
                                      : p.num_pages;
                            row -= pg * p.page_size;
                        }
                    }
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(sk + c * REGION, &tmKc, &bars[B_FULL + st], c * 64, x.g, row, blk);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(sk + (3 + c) * REGION, &tmVc, &bars[B_FULL + st], c * 64, x.g, row, blk);
                }
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int t = max(0, tt - NSTAGE); t < tt; ++t)
                mbar_wait_drain(&bars[B_FULL + t % NSTAGE], (t / NSTAGE) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_ITEM) {
        // ---------------- the new tokens of each item ----------------
        if (lane == 0) {
            int n = 0; // non-empty items
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                if (x.nsteps == 0)
                    continue;
                // the new-token buffers double as the previous item's merge scratch
                if (n >= 1 && !mbar_wait(&bars[B_MERGED], (n - 1) & 1, abort, 2u))
                    break;
                mbar_arrive_expect_tx(&bars[B_NEWFULL], x.d.has_new ? 5u * NEW_REGION : 0u);
                if (x.d.has_new) {
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + OFF_NEWK + c * NEW_REGION, &tmKn, &bars[B_NEWFULL], c * 64,
                                    x.g, 0, x.b);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem + OFF_NEWV + c * NEW_REGION, &tmVn, &bars[B_NEWFULL], c * 64,
                                    x.g, 0, x.b);
                }
                ++n;
            }
            if (n > 0)
                mbar_wait_drain(&bars[B_NEWFULL], (n - 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ---------------- UMMA issuer ----------------
        // Step j of an item belongs to warpgroup g = j & 1 and is its k-th step overall.
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(128, KT, 0);
            const uint32_t idesc_n = umma_idesc_bf16(128, NEW_ROWS, 0);
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            const uint32_t sKn = smem_u32(smem + OFF_NEWK);
            int n = 0, tt = 0;     // items and cache tiles before this item
            int cg0 = 0, cg1 = 0;  // steps of each warpgroup before this item
            bool ok = true;
            DuRaw raw = du_raw(p, blockIdx.x, n_items);
            for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
                const DuItem x = du_item(p, it, raw);
                raw = du_raw(p, it + gridDim.x, n_items);
                if (x.nsteps == 0)
                    continue;
                if (!mbar_wait(&bars[B_QT], n & 1, abort, 2u) ||
                    !mbar_wait(&bars[B_NEWFULL], n & 1, abort, 2u))
                    break;
                // One thread issues both queues in order (S_0, S_1, ...; PV_0, PV_1, ...) and
                // never blocks one behind the other: a P V whose P is ready goes first (it frees
                // a stage), an S goes as soon as its tile has landed and its warpgroup's S
                // buffer has been read by the previous P V.
                auto s_ready = [&](int j) -> bool {
                    const int g = j & 1, k = (g ? cg1 : cg0) + (j >> 1);
                    if (k >= 1 && !mbar_test(&bars[B_PVDONE + g], (k - 1) & 1))
                        return false;
                    const int tg = tt + j;
                    return j >= x.ct || mbar_test(&bars[B_FULL + tg % NSTAGE], (tg / NSTAGE) & 1);
                };
                auto issue_s = [&](int j) {
                    const int g = j & 1;
                    uint32_t kb_addr = sKn, kreg = NEW_REGION, idesc = idesc_n;
                    if (j < x.ct) {
                        kb_addr = smem_u32(smem + OFF_STAGE + ((tt + j) % NSTAGE) * STAGE);
                        kreg = REGION;
                        idesc = idesc_s;
                    }
                    // B descriptors of the later k-steps: the start-address field (16-byte
                    // units, shared memory < 256 KB) advanced by the step's byte offset
                    const uint64_t kd = smem_desc_sw128(kb_addr, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 12; ++kk)
                        umma_ts(tmem + g * 64, tmem + TMEM_Q + kk * 8,
                                kd + (((kk >> 2) * kreg + (kk & 3) * 32) >> 4), idesc, kk > 0 ? 1u : 0u);
                    umma_commit(&bars[B_SFULL + g]);
                };
                auto pv_ready = [&](int j) -> bool {
                    const int g = j & 1, k = (g ? cg1 : cg0) + (j >> 1);
                    return mbar_test(&bars[B_PFULL + g], k & 1);
                };
                auto issue_pv = [&](int j) {
                    const int g = j & 1;
                    const uint32_t pt = tmem + g * 64;            // P: 16 keys per 8 columns
                    const uint32_t od = tmem + TMEM_O + g * 128;  // this warpgroup's O
                    if (j < x.ct) {
                        // B = V (16 keys x 128 dims, dims contiguous: MN-major; dims 64..127 one
                        // region further on)
                        const int st = (tt + j) % NSTAGE;
                        const uint64_t vd = smem_desc_sw128(
                            smem_u32(smem + OFF_STAGE + st * STAGE + 3 * REGION), REGION, 1024);
#pragma unroll
                        for (int kk = 0; kk < KT / 16; ++kk)
                            umma_ts(od, pt + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_o,
                                    (j >= 2 || kk > 0) ? 1u : 0u);
                        umma_commit(&bars[B_PVDONE + g]);
                        umma_commit(&bars[B_EMPTY + st]);
                    } else {
                        umma_ts(od, pt, smem_desc_sw128(smem_u32(smem + OFF_NEWV), NEW_REGION, 1024),
                                idesc_o, j >= 2 ? 1u : 0u);
                        umma_commit(&bars[B_PVDONE + g]);
                    }
                };
                int ns = 0, np = 0; // S and P V issued
                uint64_t idle_since = 0;
                while (np < x.nsteps) {
                    if (np < ns && pv_ready(np)) {
                        tc_fence_after();
                        issue_pv(np++);
                        idle_since = 0;
                    } else if (ns < x.nsteps && s_ready(ns)) {
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
                cg0 += (x.nsteps + 1) >> 1;
                cg1 += x.nsteps >> 1;
                tt += x.ct;
                ++n;
            }
            // every MMA of ours has finished before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait_drain(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else {
        // ---------- softmax warpgroups: thread = TMEM lane = (key part, query row) ----------
        // Warpgroup grp takes the steps j = grp, grp + 2, ... of every item into its own O.
        const int grp = warp >> 2;
        const int L = (warp & 3) * 32 + lane;
        const int jp = L / RP, r = L % RP; // jp is warp-uniform (RP >= 32)
        const bool row_ok = r < p.R;
        const int t = row_ok ? r / p.G : 0;
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t o_addr = tmem + lane_addr + TMEM_O + grp * 128;
        const float c_l2 = p.scale_log2;
        float4 *ml0 = reinterpret_cast<float4 *>(smem + OFF_ML0);  // [128], after the MMAs
        float4 *ml1 = reinterpret_cast<float4 *>(smem + OFF_ML1);  // [128]
        float *obuf = reinterpret_cast<float *>(smem + OFF_OBUF);  // [F-1][RP][..], after the MMAs
        int n = 0, tt = 0, cg = 0;
        DuRaw raw = du_raw(p, blockIdx.x, n_items);
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const DuItem x = du_item(p, it, raw);
            raw = du_raw(p, it + gridDim.x, n_items);
            const int64_t unit = ((int64_t)x.b * p.Hkv + x.g) * p.splits + x.split;
            if (x.nsteps == 0) {
                // an empty span: its partial has no keys (the merge skips l = 0)
                if (grp == 0 && L < p.R && p.splits > 1)
                    *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + L) * 4) =
                        make_float4(-INFINITY, 0.f, 0.f, 0.f);
                continue;
            }
            const DecodeTiles &d = x.d;
            const int h = x.g * p.G + (row_ok ? r % p.G : 0);
            if (grp == 0) {
                // this lane's query row into TMEM (the A operand of S; rows past R are zero).
                // The previous item's MMAs are all done: its merge came after them.
                const uint4 *qrow = reinterpret_cast<const uint4 *>(
                    p.q + (int64_t)x.b * p.q_sb + (int64_t)t * p.q_st + (int64_t)h * p.q_sh);
#pragma unroll 1
                for (int c = 0; c < 3; ++c) {
                    uint32_t v[32];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint4 w = row_ok ? __ldg(qrow + c * 8 + u) : make_uint4(0u, 0u, 0u, 0u);
                        v[4 * u] = w.x;
                        v[4 * u + 1] = w.y;
                        v[4 * u + 2] = w.z;
                        v[4 * u + 3] = w.w;
                    }
                    tmem_st32(tmem + lane_addr + TMEM_Q + c * 32, v);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars[B_QT]);
            }
            const float sink_h = (grp == 0 && p.sink) ? p.sink[h] : -INFINITY; // used at the end
            float m = -INFINITY, l_round = 0.f, l_exact = 0.f;
            bool ok = true;
            int k = cg;
            for (int j = grp; j < x.nsteps; j += 2, ++k) {
                // Cache tiles and the new tokens take the same path: the new tokens are keys
                // 0..T-1 of an N = 16 step, which all fall in key part 0 (the other parts'
                // columns hold stale values and are masked).
                const bool cache = j < x.ct;
                // a paged tile's page id, loaded before the wait so its latency hides there
                const int pg = cache && p.kind == 2 ? (d.first_c + d.kb + j * KT) / p.page_size : 0;
                const int pid = cache && p.kind == 2 && pg < p.max_pages
                                    ? __ldg(p.page_table + (int64_t)x.b * p.max_pages + pg)
                                    : -1;
                ok = warp_wait(&bars[B_SFULL + grp], k & 1, abort);
                if (!ok)
                    break;
                tc_fence_after();
                const uint32_t saddr = tmem + lane_addr + grp * 64;
                const bool tile_ok = !cache || p.kind != 2 || (pid >= 0 && pid < p.num_pages);
                if (cache) {
                    const KeySpan present = du_span(p, d, j, tile_ok, false, 0);
                    if (!present.covers(KT)) {
                        // zero the V rows of keys outside the span: lane L takes key L % 64,
                        // half L / 64
                        if (!present.has(L & 63)) {
                            uint4 *row = reinterpret_cast<uint4 *>(
                                smem + OFF_STAGE + ((tt + j) % NSTAGE) * STAGE +
                                (3 + (L >> 6)) * REGION + (L & 63) * 128);
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                row[u] = make_uint4(0u, 0u, 0u, 0u);
                        }
                        fence_async_smem();
                    }
                }
                uint32_t raw_s[KPT];
                if constexpr (KPT == 32) {
                    tmem_ld32_sync(saddr + jp * KPT, raw_s);
                } else {
                    tmem_ld16_sync(saddr + jp * KPT, raw_s);
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
                // O holds this warpgroup's P V of the item up to its previous step: rescale it
                // to the new reference max (its first step's P V overwrites O)
                if (j >= 2 && __any_sync(0xffffffffu, rescale)) {
                    ok = warp_wait(&bars[B_PVDONE + grp], (k - 1) & 1, abort);
                    if (!ok)
                        break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32_sync(o_addr + c * 32, o);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(o_addr + c * 32, o);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars[B_PFULL + grp]);
            }
            if (ok && k > cg) {
                const int kl = k - 1;
                ok = warp_wait(&bars[B_PVDONE + grp], kl & 1, abort);
            }
            tc_fence_after();
            cg = k;
            tt += x.ct;

            // ---- warpgroup 1 hands its row statistics to warpgroup 0; one decision to go on
            if (grp == 1) {
                ml1[L] = make_float4(m, l_round, l_exact, ok ? 1.f : 0.f);
                if (L == 0)
                    go_on[n & 1] = !*abort;
            }
            named_bar_sync(2, 256);
            const bool cont = go_on[n & 1] != 0;
            if (grp == 1) {
                ++n;
                if (!cont)
                    break;
                continue;
            }

            // ---- warpgroup 0: combine the two warpgroups (same lanes), then the F key parts
            const float4 s1 = ml1[L];
            const bool has1 = x.nsteps >= 2;
            ok = ok && s1.w != 0.f;
            const float m01 = fmaxf(m, has1 ? s1.x : -INFINITY);
            const float a0 = (m == -INFINITY) ? 0.f : fast_exp2(m - m01);
            const float a1 = (!has1 || s1.x == -INFINITY) ? 0.f : fast_exp2(s1.x - m01);
            const float lr01 = l_round * a0 + (has1 ? s1.y * a1 : 0.f);
            const float le01 = l_exact * a0 + (has1 ? s1.z * a1 : 0.f);
            ml0[L] = make_float4(m01, lr01, le01, 0.f);
            named_bar_sync(1, 128);
            float mf = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < F; ++jj)
                mf = fmaxf(mf, ml0[jj * RP + r].x);
            float lr = 0.f, le = 0.f;
#pragma unroll
            for (int jj = 0; jj < F; ++jj) {
                const float4 ml = ml0[jj * RP + r];
                const float c = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - mf);
                lr += ml.y * c;
                le += ml.z * c;
            }
            // this lane's O = a0 O_0 + a1 O_1, brought to the row's reference max mf
            const float sc = (m01 == -INFINITY) ? 0.f : fast_exp2(m01 - mf);
            const float b0 = a0 * sc, b1 = a1 * sc;
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
            const bool write = writer && ok && cont;
#pragma unroll 1
            for (int c = 0; c < 128 / MERGE_COLS; ++c) {
                uint32_t o[MERGE_COLS], o1[MERGE_COLS];
                tmem_ld32(tmem + lane_addr + TMEM_O + c * MERGE_COLS, o);
                if (has1)
                    tmem_ld32(tmem + lane_addr + TMEM_O + 128 + c * MERGE_COLS, o1);
                tmem_ld_wait();
                float v[MERGE_COLS];
#pragma unroll
                for (int e = 0; e < MERGE_COLS; ++e)
                    v[e] = __uint_as_float(o[e]) * b0 + (has1 ? __uint_as_float(o1[e]) * b1 : 0.f);
                if (jp > 0) {
                    float4 *dst = reinterpret_cast<float4 *>(obuf + ((jp - 1) * RP + r) * MERGE_STRIDE);
#pragma unroll
                    for (int q = 0; q < MERGE_COLS / 4; ++q)
                        dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
                named_bar_sync(1, 128);
                if (write) {
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
            // warpgroup 1's O is read and the merge scratch is dead: the next item may load
            // its new tokens and overwrite O_1
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
