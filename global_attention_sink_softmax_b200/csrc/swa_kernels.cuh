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
// The grid is one persistent CTA per SM walking a contiguous run of items (positions fastest).
// Consecutive items of one (sequence, KV head) share all but P of their span's keys, so K and V
// sit in shared-memory rings of 16-key chunks and each item loads only its new chunk, one item
// ahead (the first item of a run loads the whole span). S is computed over the whole ring in
// slot order, one M128 N160 chain (10 slots of 16 keys; the slot outside the span is masked), so
// a span that wraps around the ring costs no extra MMAs. Q is double-buffered and streams one
// item ahead. S is double-buffered in tensor memory; two warpgroups own one S buffer each and
// work on consecutive items at the same time. Each reads its row of S (three 16-column chunks per
// TMEM round trip, the span's chunks in slot order), writes P (bf16) back over it (slot s's P in
// the 8 columns at 8 s, over scores already read), so P.V takes its A operand straight from tensor
// memory, then reads O (128 columns), frees it for the other warpgroup's P.V and writes O / l and
// LSE. Loops are kept rolled so the code of the four warp roles fits the SM's instruction caches.
//
// Specialised for the 144-key span of G = 8 query heads per KV head (P = 16) and W <= 128.
//
// Roles (480 threads): warps 0-3 and 4-7 softmax + epilogue (even / odd items; thread = row =
// TMEM lane); warp 8 TMA producer for Q and K, warp 10 for V; warp 9 TMEM allocator +
// single-thread UMMA issuer, issuing S_0, {S_{n+1}, PV_n}; warps 11-14 apply the partial RoPE to
// each Q tile and each new K chunk as they land, when asked to (the rotary dims lie in the first
// 64-dim region of a tile; the issuer then waits for the rotated tiles instead of the copies),
// and the value scale multiplies O. Waits are bounded as in the band kernel.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace sw {
constexpr int THREADS = 480;
constexpr int WARP_LOAD = 8, WARP_MMA = 9, WARP_VLOAD = 10;
constexpr int WARP_ROPE = 11, ROPE_WARPS = 4; // warps 11-14 rotate (fused RoPE)
constexpr int ROW = 128;          // bytes per swizzled row (64 bf16)
constexpr int Q_REGION = 128 * ROW;
constexpr int Q_BYTES = 3 * Q_REGION;
constexpr int CHUNK = 16 * ROW;   // one 16-key chunk of one 64-dim region
constexpr int NSC = 144;          // key span: P + W - 1 rounded up to 16 (G = 8, W <= 128)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 384;  // S buffer i at i * 16 R (R ring slots); P of that item over it

enum Bar {
    Q_FULL = 0,   // + Q buffer
    Q_EMPTY = 2,  // + Q buffer
    K_FULL = 4,   // + item parity
    K_EMPTY = 6,  // + item parity
    V_FULL = 8,   // + item parity
    V_EMPTY = 10, // + item parity
    S_FULL = 12,  // + S buffer (= warpgroup)
    S_FREE = 14,  // + S buffer (S and the P that overwrote it are consumed)
    P_FULL = 16,  // + warpgroup
    PV_DONE = 18, // + warpgroup
    O_FREE = 20,
    DRAIN = 21,
    Q_ROT = 22,   // + Q buffer: Q rotated (fused RoPE)
    K_ROT = 24,   // + item parity: the item's new K chunks rotated
    NUM_BARS = 26
};

__host__ __device__ constexpr bool counted_by_rows(int i)
{
    return i == P_FULL || i == P_FULL + 1 || i == O_FREE;
}
__host__ __device__ constexpr bool counted_by_rope_warps(int i)
{
    return i == Q_ROT || i == Q_ROT + 1 || i == K_ROT || i == K_ROT + 1;
}

// K and V rings: R = NSC / 16 + P / 16 chunks of 16 keys per 64-dim region (the span plus the
// chunks the next item adds, so those load while the current span is still in use).
__host__ __device__ constexpr int ring_chunks(int p) { return NSC / 16 + p / 16; }
// two S buffers of 16 R columns (S over the whole ring) below O
static_assert(2 * 16 * ring_chunks(16) <= (int)TMEM_O, "S buffers fit below O in tensor memory");
__host__ __device__ constexpr int k_bytes(int p) { return 3 * ring_chunks(p) * CHUNK; }
__host__ __device__ constexpr int v_bytes(int p) { return 2 * ring_chunks(p) * CHUNK; }
__host__ __device__ constexpr int off_k() { return 2 * Q_BYTES; }
__host__ __device__ constexpr int off_v(int p) { return off_k() + k_bytes(p); }
__host__ __device__ constexpr int off_bar(int p) { return off_v(p) + v_bytes(p); }
// Fused RoPE tables: the pair frequencies, then (cos, sin) of the item's P query positions and
// of its A * 16 new keys, per rotary pair
__host__ __device__ constexpr int off_rope(int p) { return off_bar(p) + 256; }
__host__ __device__ constexpr int rope_bytes(int p)
{
    return ROPE_WARPS * kRopeFusedMaxHalf * 8 + p * kRopeFusedMaxHalf * 8; // frequencies, table
}
__host__ __device__ constexpr int smem_bytes(int p) { return off_rope(p) + rope_bytes(p) + 1024; }
static_assert(NUM_BARS * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit their 256 bytes");
} // namespace sw

struct SwaItem {
    int b, g, p0, ks;
    bool fresh; // first item of a (sequence, KV head) run: the whole span is loaded
};

SA_DEV SwaItem swa_item(const SwaParams &p, int item, bool first_of_cta)
{
    SwaItem it;
    const int pblk = item % p.n_pblk;
    const int bg = item / p.n_pblk;
    it.g = bg % p.Hkv;
    it.b = bg / p.Hkv;
    it.p0 = pblk * p.P;
    it.ks = it.p0 + p.P - sw::NSC;
    it.fresh = first_of_cta || pblk == 0;
    return it;
}

// Ring bookkeeping. Consecutive items of one run move the span by A = P / 16 chunks; `base` is
// the ring slot of the span's first chunk, span chunk i sits in slot (base + i) mod R.
SA_DEV int swa_next_base(const SwaParams &p, const SwaItem &it, int base)
{
    const int R = sw::ring_chunks(p.P), A = p.P / 16;
    return it.fresh ? 0 : (base + A) % R;
}

// Rotates the 8 pairs of 16-byte chunk c (dims 8c .. 8c + 7) of a 128-byte swizzled row with
// their partners nch chunks further on (dims half + 8c ..), in shared memory; cs: the 8 pairs'
// (cos, sin). Row `row` of a tile (1 KB-aligned atoms of 8 rows) sits at `rowp`.
SA_DEV void swa_rotate_chunk(uint8_t *rowp, int row, int c, int nch, const float2 *cs)
{
    uint4 *a = reinterpret_cast<uint4 *>(rowp + ((c ^ (row & 7)) << 4));
    uint4 *b = reinterpret_cast<uint4 *>(rowp + (((c + nch) ^ (row & 7)) << 4));
    uint4 x = *a, y = *b;
    rope_rotate8(x, y, cs);
    *a = x;
    *b = y;
}

// Fused RoPE of a whole key span (the first item of a run loads all NSC keys into ring slots
// 0 .. SC - 1): region 0 of key r sits in slot r / 16, row r % 16. Rotator warp rw takes keys
// r = rw, rw + 4, ...; lane = (key, chunk c). Angles computed here, key by key. Out of line: it
// runs once per run of items, and its code stays out of the rotators' loop.
__device__ __noinline__ void swa_rope_span(uint8_t *kring, int ks, int L, int64_t mb, const double *wf,
                                           int nch, int rw, int lane)
{
    const int c = lane & 3;
    for (int rr = lane >> 2; rr < sw::NSC / sw::ROPE_WARPS; rr += 8) {
        const int r = rr * sw::ROPE_WARPS + rw;
        const int key = ks + r;
        if (c >= nch || key < 0 || key >= L)
            continue; // a row outside the sequence: zeros from the copy, masked
        float2 csk[8];
#pragma unroll 1
        for (int j = 0; j < 8; ++j)
            csk[j] = rope_cos_sin(mb + key, wf[c * 8 + j]);
        swa_rotate_chunk(kring + (r >> 4) * sw::CHUNK + (r & 15) * sw::ROW, r & 15, c, nch, csk);
    }
}

// Loads the 16-column chunks of ring slots s0, s1, s2 of a row of S (one TMEM round trip).
SA_DEV void swa_ld48(uint32_t taddr, int s0, int s1, int s2, uint32_t (&r)[48])
{
    tmem_ld16(taddr + s0 * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
    tmem_ld16(taddr + s1 * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
    tmem_ld16(taddr + s2 * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[32]));
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 48; i += 8)
        asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]),
                     "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])::"memory");
}

// -inf outside span offsets [lo, hi] for three chunks whose first keys sit at span offsets k0, k1,
// k2 (skipped when all are inside)
SA_DEV void swa_mask48(uint32_t (&r)[48], int k0, int k1, int k2, int lo, int hi)
{
    if (min(k0, min(k1, k2)) >= lo && max(k0, max(k1, k2)) + 15 <= hi)
        return;
#pragma unroll
    for (int u = 0; u < 48; ++u) {
        const int k = (u < 16 ? k0 : u < 32 ? k1 : k2) + (u & 15);
        if (k < lo || k > hi)
            r[u] = __float_as_uint(-INFINITY);
    }
}

// The i-th chunk of the span in ring-slot order (i = 0 .. SC - 1): every slot but `out`, the one
// the span leaves out; its offset in the span is 16 ((slot - base) mod R).
SA_DEV int swa_span_slot(int i, int out) { return i + (i >= out ? 1 : 0); }
SA_DEV int swa_span_off(int slot, int base, int R) { return 16 * (slot >= base ? slot - base : slot + R - base); }

__global__ void __launch_bounds__(sw::THREADS, 1)
    prefill_swa_packed_kernel(const __grid_constant__ CUtensorMap tmQ,
                              const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV,
                              const __grid_constant__ CUtensorMap tmKc,
                              const __grid_constant__ CUtensorMap tmVc, const SwaParams p)
{
    using namespace sw;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int SC = NSC / 16;
    const int R = ring_chunks(p.P), A = p.P / 16;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + off_bar(p.P));
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // contiguous run of items for this CTA
    const int it0 = (int)(((int64_t)blockIdx.x * p.n_items) / gridDim.x);
    const int it1 = (int)(((int64_t)(blockIdx.x + 1) * p.n_items) / gridDim.x);
    const int cnt = it1 - it0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i)
            mbar_init(&bars[i], counted_by_rows(i) ? 128 : counted_by_rope_warps(i) ? ROPE_WARPS : 1);
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
            int issued = 0, base = 0;
            for (int n = 0; n < cnt; ++n) {
                const SwaItem it = swa_item(p, it0 + n, n == 0);
                base = swa_next_base(p, it, base);
                const int qb = n & 1;
                // Q buffer qb was read by S of item n - 2
                if (n >= 2 && !mbar_wait(&bars[Q_EMPTY + qb], ((n >> 1) - 1) & 1, abort, 1u))
                    break;
                mbar_arrive_expect_tx(&bars[Q_FULL + qb], Q_BYTES);
                for (int c = 0; c < 3; ++c)
                    tma_load_4d(smem + qb * Q_BYTES + c * Q_REGION, &tmQ, &bars[Q_FULL + qb],
                                c * 64, it.g * p.G, it.p0, it.b);
                uint64_t *kf = &bars[K_FULL + (n & 1)];
                if (it.fresh) {
                    // the whole span, slots 0 .. SC-1: wait for S of the previous item
                    if (n >= 1 && !mbar_wait(&bars[K_EMPTY + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort, 1u))
                        break;
                    mbar_arrive_expect_tx(kf, 3 * NSC * ROW);
                    for (int c = 0; c < 3; ++c)
                        tma_load_4d(smem + off_k() + c * R * CHUNK, &tmK, kf, c * 64, it.g, it.ks, it.b);
                } else {
                    // A new chunks over the slots of item n - 2's first chunks
                    if (n >= 2 && !mbar_wait(&bars[K_EMPTY + (n & 1)], ((n - 2) >> 1) & 1, abort, 1u))
                        break;
                    mbar_arrive_expect_tx(kf, 3 * A * CHUNK);
                    for (int a = 0; a < A; ++a) {
                        const int slot = (base + SC - A + a) % R;
                        const int key0 = it.ks + NSC - (A - a) * 16;
                        for (int c = 0; c < 3; ++c)
                            tma_load_4d(smem + off_k() + c * R * CHUNK + slot * CHUNK, &tmKc, kf,
                                        c * 64, it.g, key0, it.b);
                    }
                }
                issued = n + 1;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int n = max(0, issued - 2); n < issued; ++n) {
                mbar_wait_drain(&bars[Q_FULL + (n & 1)], (n >> 1) & 1);
                mbar_wait_drain(&bars[K_FULL + (n & 1)], (n >> 1) & 1);
            }
        }
        __syncwarp();
    } else if (warp == WARP_VLOAD) {
        if (lane == 0 && cnt > 0) {
            tma_prefetch_desc(&tmV);
            int issued = 0, base = 0;
            for (int n = 0; n < cnt; ++n) {
                const SwaItem it = swa_item(p, it0 + n, n == 0);
                base = swa_next_base(p, it, base);
                uint64_t *vf = &bars[V_FULL + (n & 1)];
                if (it.fresh) {
                    if (n >= 1 && !mbar_wait(&bars[V_EMPTY + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort, 1u))
                        break;
                    mbar_arrive_expect_tx(vf, 2 * NSC * ROW);
                    for (int c = 0; c < 2; ++c)
                        tma_load_4d(smem + off_v(p.P) + c * R * CHUNK, &tmV, vf, c * 64, it.g,
                                    it.ks, it.b);
                } else {
                    if (n >= 2 && !mbar_wait(&bars[V_EMPTY + (n & 1)], ((n - 2) >> 1) & 1, abort, 1u))
                        break;
                    mbar_arrive_expect_tx(vf, 2 * A * CHUNK);
                    for (int a = 0; a < A; ++a) {
                        const int slot = (base + SC - A + a) % R;
                        const int key0 = it.ks + NSC - (A - a) * 16;
                        for (int c = 0; c < 2; ++c)
                            tma_load_4d(smem + off_v(p.P) + c * R * CHUNK + slot * CHUNK, &tmVc,
                                        vf, c * 64, it.g, key0, it.b);
                    }
                }
                issued = n + 1;
            }
            for (int n = max(0, issued - 2); n < issued; ++n)
                mbar_wait_drain(&bars[V_FULL + (n & 1)], (n >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        if (lane == 0 && cnt > 0) {
            const uint32_t idesc_o = umma_idesc_bf16(128, 128, 1);
            // Operand descriptors are built once; a k-step or a ring slot only advances the
            // start-address field (16-byte units; shared memory < 256 KB, so it never carries).
            // This thread shares its SMSP with two softmax warps, so it issues few instructions;
            // its loops stay rolled (the kernel's code must fit the instruction caches).
            const uint64_t kd0 = smem_desc_sw128(smem_u32(smem + off_k()), 16, 1024);
            const uint64_t vd0 = smem_desc_sw128(smem_u32(smem + off_v(p.P)), R * CHUNK, 1024);
            const uint64_t qd0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
            const uint64_t qd1 = smem_desc_sw128(smem_u32(smem + Q_BYTES), 16, 1024);
            const uint32_t region16 = (uint32_t)(R * CHUNK) >> 4; // one 64-dim region of a ring
            int base_s = 0;
            int base_even = 0, base_odd = 0; // ring slot of the span's first key, per item parity
            int pblk = (it0 % p.n_pblk) - 1; // position block of the last item issued
            // S of item n into S buffer n & 1 (warpgroup n & 1), over all R ring slots in slot
            // order (one N = 16 R MMA per k-step, whether or not the span wraps; the slot outside
            // the span is masked by the softmax). A CTA's items are consecutive, so the position
            // block and the ring base advance without division.
            const uint32_t idesc_s = umma_idesc_bf16(128, 16 * R, 0);
            auto issue_s = [&](int n) -> bool {
                pblk = (pblk + 1 == p.n_pblk) ? 0 : pblk + 1;
                const int nb_ = base_s + p.P / 16;
                base_s = (n == 0 || pblk == 0) ? 0 : (nb_ >= R ? nb_ - R : nb_);
                if (n & 1)
                    base_odd = base_s;
                else
                    base_even = base_s;
                const int sb = n & 1;
                // the tiles as loaded, or once rotated (fused RoPE)
                if (!mbar_wait(&bars[(p.rope ? Q_ROT : Q_FULL) + sb], (n >> 1) & 1, abort, 1u) ||
                    !mbar_wait(&bars[(p.rope ? K_ROT : K_FULL) + (n & 1)], (n >> 1) & 1, abort, 1u))
                    return false;
                // S buffer sb held S and P of item n - 2: free once that P.V is done
                if (n >= 2 && !mbar_wait(&bars[S_FREE + sb], ((n >> 1) - 1) & 1, abort, 1u))
                    return false;
                tc_fence_after();
                const uint64_t qd = sb ? qd1 : qd0;
                const uint32_t d = tmem + sb * 16 * R;
#pragma unroll 1
                for (int kk = 0; kk < 12; ++kk) {
                    const uint32_t qo = (uint32_t)((kk >> 2) * Q_REGION + (kk & 3) * 32) >> 4;
                    const uint32_t ko = (kk >> 2) * region16 + (((kk & 3) * 32) >> 4);
                    umma_ss(d, qd + qo, kd0 + ko, idesc_s, kk > 0);
                }
                umma_commit(&bars[S_FULL + sb]);
                umma_commit(&bars[Q_EMPTY + sb]);
                umma_commit(&bars[K_EMPTY + (n & 1)]);
                return true;
            };
            // issue order S_0, {S_{n+1}, PV_n}
            bool ok = issue_s(0);
            for (int n = 0; ok && n < cnt; ++n) {
                const int base_pv = (n & 1) ? base_odd : base_even; // set by issue_s(n)
                if (n + 1 < cnt && !issue_s(n + 1))
                    break;
                if (!mbar_wait(&bars[P_FULL + (n & 1)], (n >> 1) & 1, abort, 1u) ||
                    !mbar_wait(&bars[V_FULL + (n & 1)], (n >> 1) & 1, abort, 1u))
                    break;
                // O was read out by the warpgroup of item n - 1
                if (n >= 1 && !mbar_wait(&bars[O_FREE], (n - 1) & 1, abort, 1u))
                    break;
                tc_fence_after();
                const uint32_t pt = tmem + (n & 1) * 16 * R; // P of slot s: 8 columns at 8 s
#pragma unroll 1
                for (int kk = 0; kk < SC; ++kk) {
                    int slot = base_pv + kk;
                    slot = slot >= R ? slot - R : slot;
                    umma_ts(tmem + TMEM_O, pt + slot * 8, vd0 + (uint32_t)((slot * CHUNK) >> 4),
                            idesc_o, kk > 0);
                }
                umma_commit(&bars[PV_DONE + (n & 1)]);
                umma_commit(&bars[V_EMPTY + (n & 1)]);
                umma_commit(&bars[S_FREE + (n & 1)]);
            }
            umma_commit(&bars[DRAIN]);
            mbar_wait_drain(&bars[DRAIN], 0);
        }
        __syncwarp();
    } else if (warp >= WARP_ROPE && warp < WARP_ROPE + ROPE_WARPS) {
        // ------- fused partial RoPE: Q tiles and the new K chunks, rotated in shared memory by
        // four warps. Warp rw owns query positions rw * 4 .. rw * 4 + 3 of each item (P = 16:
        // their 32 Q rows, and the new keys at those positions, since the span ends at the item's
        // last position) and its own rows of the (cos, sin) table, so the warps never wait for
        // one another; each releases its share of an item with one arrival on each of Q_ROT and
        // K_ROT. Lane = (position, chunk c of 8 rotary pairs, half of the heads): it holds its 8
        // pairs' (cos, sin) in registers and applies them to 4 Q rows (heads hb * 4 .. + 3) and,
        // in head half 0, to the new key at its position; the 8 lanes of a quarter warp touch 8
        // distinct bank groups. The loop is kept small and rolled: its code shares the SM's
        // instruction caches with the softmax warps' loops, and more code here slows those.
        if (p.rope && cnt > 0) {
            const int rw = warp - WARP_ROPE;
            const int half = p.rope_half, nch = half / 8;
            const int c = lane & 3, hb = (lane >> 2) & 1, pos = lane >> 3;
            // the frequencies in shared memory (a per-lane index into the kernel's parameters
            // serialises the warp; done once), this lane's own in a register
            double *wf = reinterpret_cast<double *>(smem + off_rope(p.P)) + rw * kRopeFusedMaxHalf;
            float2 *cs = reinterpret_cast<float2 *>(smem + off_rope(p.P) + ROPE_WARPS * kRopeFusedMaxHalf * 8) +
                         rw * 4 * kRopeFusedMaxHalf; // [4][half], this warp's positions
            wf[lane] = p.inv_freq[lane];
            const double w_lane = wf[lane];
            __syncwarp();
            // consecutive items: the position block and the sequence advance without division
            int pblk = it0 % p.n_pblk, bg = it0 / p.n_pblk, base = 0;
            int64_t mb = p.pos0 + (p.pos_base ? p.pos_base[bg / p.Hkv] : 0);
            for (int n = 0; n < cnt; ++n) {
                const bool fresh = n == 0 || pblk == 0;
                base = fresh ? 0 : (base + 1 == R ? 0 : base + 1);
                const int p0 = pblk * 16;
                // (cos, sin) of the warp's 4 positions: lane = rotary pair
                if (lane < half) {
#pragma unroll 1
                    for (int l = 0; l < 4; ++l)
                        cs[l * half + lane] = rope_cos_sin(mb + p0 + rw * 4 + l, w_lane);
                }
                __syncwarp();
                // the item's Q tile and K chunks (one lane polls)
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&bars[Q_FULL + (n & 1)], (n >> 1) & 1, abort, 1u) &&
                         mbar_wait(&bars[K_FULL + (n & 1)], (n >> 1) & 1, abort, 1u);
                if (!__shfl_sync(0xffffffffu, (int)ok, 0))
                    break;
                // the first item of a run loaded its whole span: rotate it here (rare)
                if (fresh)
                    swa_rope_span(smem + off_k(), p0 + 16 - NSC, p.L, mb, wf, nch, rw, lane);
                if (c < nch) {
                    float2 csl[8];
                    const float4 *src = reinterpret_cast<const float4 *>(cs + pos * half + c * 8);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 v = src[j];
                        csl[2 * j] = make_float2(v.x, v.y);
                        csl[2 * j + 1] = make_float2(v.z, v.w);
                    }
                    // tasks 0-3: the Q rows; task 4: the new key (slot base + SC - 1 of the
                    // ring, row = its position in the chunk), unless the span was just rotated
                    const int key = p0 + rw * 4 + pos;
                    const int ntask = (!fresh && hb == 0 && key < p.L) ? 5 : 4;
                    uint8_t *q0 = smem + (n & 1) * Q_BYTES;
#pragma unroll 1
                    for (int t = 0; t < ntask; ++t) {
                        int row = rw * 32 + pos * 8 + hb * 4 + t;
                        uint8_t *rowp = q0 + row * ROW;
                        if (t == 4) {
                            const int slot = base + SC - 1 >= R ? base + SC - 1 - R : base + SC - 1;
                            row = rw * 4 + pos;
                            rowp = smem + off_k() + slot * CHUNK + row * ROW;
                        }
                        swa_rotate_chunk(rowp, row, c, nch, csl);
                    }
                }
                // generic stores before the tensor cores' reads; then release this warp's share
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars[Q_ROT + (n & 1)]);
                    mbar_arrive(&bars[K_ROT + (n & 1)]);
                }
                if (++pblk == p.n_pblk) {
                    pblk = 0;
                    ++bg;
                    if (n + 1 < cnt) // the next item's sequence (none past the CTA's last item)
                        mb = p.pos0 + (p.pos_base ? p.pos_base[bg / p.Hkv] : 0);
                }
            }
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------- softmax + epilogue warpgroups: wg handles items n = wg, wg + 2, ...; thread = row
        const int wg = warp >> 2;
        const int row = threadIdx.x & 127;
        const int l_local = row / p.G, h_local = row - l_local * p.G;
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        const float c_l2 = p.scale_log2;
        for (int n = wg; n < cnt; n += 2) {
            const SwaItem it = swa_item(p, it0 + n, n == 0);
            const int l = it.p0 + l_local;
            const int h = it.g * p.G + h_local;
            // visible span offsets: ks + c in [max(l - W + 1, 0), l]
            const int hi = l - it.ks;
            const int lo = max(l - p.W + 1, 0) - it.ks;
            // ring slot of the span's first chunk (the issuer's base for this item) and the slot
            // the span leaves out
            const int base = (min(n, it.p0 / p.P) * A) % R;
            const int out = (base + SC) % R;
            const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            if (!warp_wait(&bars[S_FULL + wg], (n >> 1) & 1, abort))
                break;
            tc_fence_after();
            // Row max, then P, three of the span's chunks (in slot order) per TMEM round trip.
            // The loops stay rolled: the kernel's code must fit the instruction caches of an SM
            // that runs four different warp roles.
            const uint32_t saddr = tmem + lane_addr + wg * 16 * R;
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
            for (int i0 = 0; i0 < SC; i0 += 3) {
                const int s0 = swa_span_slot(i0, out), s1 = swa_span_slot(i0 + 1, out),
                          s2 = swa_span_slot(i0 + 2, out);
                uint32_t r[48];
                swa_ld48(saddr, s0, s1, s2, r);
                swa_mask48(r, swa_span_off(s0, base, R), swa_span_off(s1, base, R),
                           swa_span_off(s2, base, R), lo, hi);
#pragma unroll
                for (int u = 0; u < 48; ++u)
                    mx4[u & 3] = fmaxf(mx4[u & 3], __uint_as_float(r[u]));
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            // m = max(sink, max_j a_j) in log2 units (the max includes the sink)
            const float m = fmaxf(sink_l2, mx * c_l2);
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            // P = 2^(s c - m) as bf16 pairs over the consumed scores; the row sum of the fp32 P
            // normalises O and gives LSE
            float pe[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int i0 = 0; i0 < SC; i0 += 3) {
                const int s0 = swa_span_slot(i0, out), s1 = swa_span_slot(i0 + 1, out),
                          s2 = swa_span_slot(i0 + 2, out);
                uint32_t r[48];
                swa_ld48(saddr, s0, s1, s2, r);
                swa_mask48(r, swa_span_off(s0, base, R), swa_span_off(s1, base, R),
                           swa_span_off(s2, base, R), lo, hi);
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    uint32_t pk[8];
#pragma unroll
                    for (int u = 0; u < 16; u += 2) {
                        const float e0 = fast_exp2(fmaf(__uint_as_float(r[k * 16 + u]), c_l2, neg_m));
                        const float e1 = fast_exp2(fmaf(__uint_as_float(r[k * 16 + u + 1]), c_l2, neg_m));
                        pe[(u >> 1) & 3] += e0 + e1;
                        pk[u >> 1] = pack_bf16x2(e0, e1);
                    }
                    // P of slot s over S columns 8 s .. 8 s + 7, scores of slot s / 2 <= s,
                    // already read (slots go in increasing order)
                    tmem_st8(saddr + (k == 0 ? s0 : k == 1 ? s1 : s2) * 8, pk[0], pk[1], pk[2],
                             pk[3], pk[4], pk[5], pk[6], pk[7]);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[P_FULL + wg]);
            // the sink seeds both sums: exp(sink - m)
            const float s0 = (sink_l2 == -INFINITY) ? 0.f : fast_exp2(sink_l2 - m);
            const float l_exact = s0 + ((pe[0] + pe[1]) + (pe[2] + pe[3]));

            // epilogue: O = (P V) / l_exact, LSE = m + log2(l_exact)
            if (!warp_wait(&bars[PV_DONE + wg], (n >> 1) & 1, abort))
                break;
            tc_fence_after();
            const bool valid = l < p.L;
            const float inv_l = p.out_mul / l_exact; // the value scale (fused RoPE) rides on 1 / l
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.o) + (int64_t)it.b * p.o_sb +
                                  (int64_t)l * p.o_sl + (int64_t)h * p.o_sh;
#pragma unroll 1
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
                p.lse[((int64_t)it.b * p.Hq + h) * p.L + l] = (m + fast_log2(l_exact)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

int swa_packed_smem_bytes(int ns, int P)
{
    // this kernel is specialised for a 144-key span (G = 8 query heads per KV head, W <= 128)
    return (ns == sw::NSC && P == 16) ? sw::smem_bytes(P) : 1 << 30;
}

cudaError_t launch_prefill_swa_packed(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                      const CUtensorMap &tmV, const CUtensorMap &tmKc,
                                      const CUtensorMap &tmVc, const SwaParams &p, int grid,
                                      cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int dev) {
        int optin = 0;
        cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess)
            return e;
        return cudaFuncSetAttribute(prefill_swa_packed_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    });
    if (e != cudaSuccess)
        return e;
    if (grid <= 0)
        return cudaSuccess;
    prefill_swa_packed_kernel<<<grid, sw::THREADS, sw::smem_bytes(p.P), stream>>>(
        tmQ, tmK, tmV, tmKc, tmVc, p);
    return cudaGetLastError();
}

} // namespace sinkattn
