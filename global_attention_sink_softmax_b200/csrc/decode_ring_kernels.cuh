// Sink-softmax attention decode on a sliding-window ring cache, one warp per (sequence, KV head)
// item (sm_100a).
//
// Same computation as the other decode kernels (the sink counted once per row: "MiMo-V2-Flash
// 架构 QA" Q3.8; the window of "MiMo-V2-Flash 模型架构深度拆解" CH10.3). A ring item is small:
// ring_cap slots of 640 bytes (80 KB for the 128-slot ring) plus T new tokens, read once. What
// costs time is not arithmetic but the latency of bringing each item in, so here every warp
// owns whole items and works alone: it streams its item in 32-key chunks through a private
// double buffer filled by the TMA (3 K boxes + 2 V boxes of 32 keys x 64 dims, 128-byte
// swizzle), runs S = Q K^T and O += P V on mma.sync with Q in registers, and writes O and LSE.
// No warp waits for another, and the CTAs are persistent (warp w of CTA c takes items
// c * WARPS + w, + WARPS * gridDim.x, ...): each warp's chunks form one stream across its items,
// kept two chunks ahead, so the next item's first chunks are in flight while this one finishes.
//
// Rows: an item is one m16 tile of the R = T G query rows of a (sequence, KV head) unit; a
// unit with more than 16 rows is MT items, taken by neighbouring warps, whose chunk reads of
// the same K/V meet in L2.
// Chunks: the ring's slots in physical order (each slot gets its position from the ring head;
// attention does not depend on key order), then the new tokens as one box whose rows past T
// arrive as zeros. V rows of slots outside the span (an unfilled ring, or the oldest slot that
// the window drops) are zeroed in shared memory before P V reads them.
#pragma once
#include "common.cuh"
#include "decode_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace dr {
constexpr int KC = 32;                     // keys per chunk
constexpr int REGION = KC * 128;           // 4 KB: 32 keys x 64 dims
constexpr int CHUNK = 5 * REGION;          // K (3 regions) + V (2 regions): 20 KB
constexpr int WARPS = 5;
constexpr int THREADS = 32 * WARPS;
constexpr int OFF_BAR = WARPS * 2 * CHUNK; // 200 KB of chunk buffers
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
} // namespace dr

__global__ void __launch_bounds__(dr::THREADS, 1)
    decode_ring_kernel(const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                       const __grid_constant__ CUtensorMap tmKn, const __grid_constant__ CUtensorMap tmVn,
                       const DecodeParams p)
{
    using namespace dr;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 2 * WARPS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * WARPS; ++i)
            mbar_init(&bars[i], 1);
        *abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    uint64_t *full = bars + 2 * warp;
    uint8_t *bufs = smem + warp * 2 * CHUNK;
    const int items = p.B * p.Hkv * p.MT;
    const int stride = gridDim.x * WARPS;
    const int c2 = 2 * (lane & 3);

    // An item: sequence b, KV head g, its ring's occupancy, and its chunks (cache chunks while
    // the span holds cached keys, then one chunk of new tokens).
    struct Item {
        int b, g, mt, n_cache, first_c, head, ncc, nch;
    };
    auto plan = [&](int u) {
        Item x;
        x.mt = u % p.MT;
        x.g = (u / p.MT) % p.Hkv;
        x.b = u / (p.MT * p.Hkv);
        x.n_cache = max(0, min(p.ring_len[x.b], p.ring_cap));
        const int n_used = (p.window > 0) ? min(x.n_cache, p.window - 1) : x.n_cache;
        x.first_c = x.n_cache - n_used;
        x.head = ((p.ring_head[x.b] % p.ring_cap) + p.ring_cap) % p.ring_cap;
        x.ncc = n_used > 0 ? p.ring_cap / KC : 0;
        x.nch = x.ncc + 1;
        return x;
    };

    // Issue cursor (lane 0): the next (item, chunk) of this warp's stream; chunk n of the stream
    // goes to buffer n & 1.
    int iu = blockIdx.x * WARPS + warp, ic = 0, issued = 0, used = 0;
    Item ii;
    if (lane == 0 && iu < items)
        ii = plan(iu);
    auto issue_next = [&]() {
        while (iu < items && ic >= ii.nch) {
            iu += stride;
            ic = 0;
            if (iu < items)
                ii = plan(iu);
        }
        if (iu >= items)
            return;
        const int bi = issued & 1;
        uint8_t *dst = bufs + bi * CHUNK;
        mbar_arrive_expect_tx(&full[bi], CHUNK);
        if (ic < ii.ncc) {
            for (int x = 0; x < 3; ++x)
                tma_load_4d(dst + x * REGION, &tmKc, &full[bi], x * 64, ii.g, ic * KC, ii.b);
            for (int x = 0; x < 2; ++x)
                tma_load_4d(dst + (3 + x) * REGION, &tmVc, &full[bi], x * 64, ii.g, ic * KC, ii.b);
        } else {
            for (int x = 0; x < 3; ++x)
                tma_load_4d(dst + x * REGION, &tmKn, &full[bi], x * 64, ii.g, 0, ii.b);
            for (int x = 0; x < 2; ++x)
                tma_load_4d(dst + (3 + x) * REGION, &tmVn, &full[bi], x * 64, ii.g, 0, ii.b);
        }
        ++ic;
        ++issued;
    };
    if (lane == 0) {
        issue_next();
        issue_next();
    }

    bool ok = true;
    for (int u = blockIdx.x * WARPS + warp; ok && u < items; u += stride) {
        const Item it = plan(u);
        const int b = it.b, g = it.g, n_cache = it.n_cache, first_c = it.first_c, head = it.head;
        const int ncc = it.ncc, nch = it.nch;
        const int ra = it.mt * 16 + (lane >> 2), rb = ra + 8; // this lane's two query rows
        const int ta = min(ra / p.G, p.T - 1), tb = min(rb / p.G, p.T - 1);
        // key i of chunk c: present in the span, and its position (relative to the first new
        // token)
        auto key = [&](int c, int i, bool &valid, int &pos) {
            if (c < ncc) {
                const int s = c * KC + i; // slot and head both lie in [0, ring_cap)
                const int cl = s >= head ? s - head : s - head + p.ring_cap;
                valid = cl >= first_c && cl < n_cache;
                pos = cl - n_cache;
            } else {
                valid = i < p.T;
                pos = i;
            }
        };

        // Q fragments: rows ra and rb (query token t, head g G + r % G), zero past R
        uint32_t qa[12][4];
        {
            const bool va = ra < p.R, vb = rb < p.R;
            const uint16_t *qra = p.q + (int64_t)b * p.q_sb + (int64_t)ta * p.q_st +
                                  (int64_t)(g * p.G + (va ? ra % p.G : 0)) * p.q_sh;
            const uint16_t *qrb = p.q + (int64_t)b * p.q_sb + (int64_t)tb * p.q_st +
                                  (int64_t)(g * p.G + (vb ? rb % p.G : 0)) * p.q_sh;
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
                qa[kk][0] = va ? *reinterpret_cast<const uint32_t *>(qra + kk * 16 + c2) : 0u;
                qa[kk][1] = vb ? *reinterpret_cast<const uint32_t *>(qrb + kk * 16 + c2) : 0u;
                qa[kk][2] = va ? *reinterpret_cast<const uint32_t *>(qra + kk * 16 + 8 + c2) : 0u;
                qa[kk][3] = vb ? *reinterpret_cast<const uint32_t *>(qrb + kk * 16 + 8 + c2) : 0u;
            }
        }
        float o[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f, e_a = 0.f, e_b = 0.f;

        for (int c = 0; c < nch; ++c, ++used) {
            const int bi = used & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&full[bi], (used >> 1) & 1, abort, 2u));
            if (!ok)
                break;
            uint8_t *buf = bufs + bi * CHUNK;
            const uint32_t sK = smem_u32(buf), sV = smem_u32(buf + 3 * REGION);
            // zero the V rows of keys outside the span (the new tokens' rows past T are zeros)
            bool zeroed = false;
            if (c < ncc) {
                bool valid;
                int pos;
                key(c, lane, valid, pos);
                const unsigned bad = __ballot_sync(0xffffffffu, !valid);
                if (bad) {
                    for (int k = 0; k < KC; ++k)
                        if (((bad >> k) & 1u) && lane < 16) // 16 lanes x 16 B: both 128-byte halves
                            *reinterpret_cast<uint4 *>(buf + (3 + (lane >> 3)) * REGION + k * 128 +
                                                       (lane & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
                    __syncwarp();
                    zeroed = true;
                }
            }

            // ---- S = Q K^T (K: 3 regions of 32 keys x 128 B, 16-byte chunks XOR-swizzled)
            float sacc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
                sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < 6; ++k2) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int kr = nt * 8 + (lane & 7);
                    const int ch = 4 * k2 + (lane >> 3); // 16-byte chunk of the 192 dims
                    const int cc = (ch & 7) ^ (kr & 7);
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(sK + (ch >> 3) * REGION + kr * 128 + (cc << 4), b0, b1, b2, b3);
                    mma_bf16_16816(sacc[nt], qa[2 * k2], b0, b1);
                    mma_bf16_16816(sacc[nt], qa[2 * k2 + 1], b2, b3);
                }
            }

            // ---- mask, online softmax (single span: the sink joins at the end)
            float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    bool valid;
                    int pos;
                    key(c, nt * 8 + c2 + e, valid, pos);
                    const bool vis_a = valid && pos <= ta && (p.window <= 0 || pos > ta - p.window);
                    const bool vis_b = valid && pos <= tb && (p.window <= 0 || pos > tb - p.window);
                    sacc[nt][e] = vis_a ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                    sacc[nt][2 + e] = vis_b ? sacc[nt][2 + e] * p.scale_log2 : -INFINITY;
                    mxa = fmaxf(mxa, sacc[nt][e]);
                    mxb = fmaxf(mxb, sacc[nt][2 + e]);
                }
            }
            mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
            mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
            mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
            mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
            const float mna = fmaxf(m_a, mxa), mnb = fmaxf(m_b, mxb);
            const float alpha_a = (mna == -INFINITY) ? 1.f : fast_exp2(m_a - mna);
            const float alpha_b = (mnb == -INFINITY) ? 1.f : fast_exp2(m_b - mnb);
            const float ua = (mna == -INFINITY) ? 0.f : mna, ub = (mnb == -INFINITY) ? 0.f : mnb;
            m_a = mna;
            m_b = mnb;
            uint32_t pp[4][2];
            float sa = 0.f, sb = 0.f, xa = 0.f, xb = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const float p0 = fast_exp2(sacc[nt][0] - ua), p1 = fast_exp2(sacc[nt][1] - ua);
                const float p2 = fast_exp2(sacc[nt][2] - ub), p3 = fast_exp2(sacc[nt][3] - ub);
                xa += p0 + p1;
                xb += p2 + p3;
                pp[nt][0] = pack_bf16x2(p0, p1);
                pp[nt][1] = pack_bf16x2(p2, p3);
                sa += sum_bf16x2(pp[nt][0]);
                sb += sum_bf16x2(pp[nt][1]);
            }
            l_a = l_a * alpha_a + sa;
            l_b = l_b * alpha_b + sb;
            e_a = e_a * alpha_a + xa;
            e_b = e_b * alpha_b + xb;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                o[i][0] *= alpha_a;
                o[i][1] *= alpha_a;
                o[i][2] *= alpha_b;
                o[i][3] *= alpha_b;
            }

            // ---- O += P V (V: 2 regions of 32 keys x 128 B, swizzled like K)
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) {
                uint32_t a[4];
                a[0] = pp[2 * kq][0];
                a[1] = pp[2 * kq][1];
                a[2] = pp[2 * kq + 1][0];
                a[3] = pp[2 * kq + 1][1];
                const int kr = kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    const int ch = 2 * np + (lane >> 4); // 16-byte chunk of the 128 dims
                    const int cc = (ch & 7) ^ (kr & 7);
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(sV + (ch >> 3) * REGION + kr * 128 + (cc << 4), b0, b1, b2, b3);
                    mma_bf16_16816(o[2 * np], a, b0, b1);
                    mma_bf16_16816(o[2 * np + 1], a, b2, b3);
                }
            }
            // the buffer is read (and our zeros are ordered before the next bulk copy into it)
            if (zeroed)
                fence_async_smem();
            __syncwarp();
            if (lane == 0)
                issue_next(); // into the buffer just read: two chunks stay in flight
        }
        if (!ok)
            break;
        // full row sums across the quad, then O and LSE with the sink
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        e_a += __shfl_xor_sync(0xffffffffu, e_a, 1);
        e_a += __shfl_xor_sync(0xffffffffu, e_a, 2);
        e_b += __shfl_xor_sync(0xffffffffu, e_b, 1);
        e_b += __shfl_xor_sync(0xffffffffu, e_b, 2);
        decode_write_output(p, b, g, 0, ra, rb, lane, o, m_a, m_b, l_a, l_b, e_a, e_b);
    }
    // no copy of ours may still be landing when the CTA leaves: chunks used .. issued - 1 (lane 0
    // issued them; `used` is the same in every lane)
    if (lane == 0)
        for (int n = used; n < issued; ++n)
            mbar_wait_drain(&full[n & 1], (n >> 1) & 1);
    __syncwarp();
}

cudaError_t launch_decode_ring(const CUtensorMap &kc, const CUtensorMap &vc, const CUtensorMap &kn,
                               const CUtensorMap &vn, const DecodeParams &p, int sms,
                               cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        return cudaFuncSetAttribute(decode_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    dr::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    const int items = p.B * p.Hkv * p.MT;
    const int ctas = (items + dr::WARPS - 1) / dr::WARPS;
    decode_ring_kernel<<<ctas < sms ? ctas : sms, dr::THREADS, dr::SMEM_BYTES, stream>>>(kc, vc, kn, vn, p);
    return cudaGetLastError();
}

} // namespace sinkattn
