// Sink-softmax attention decode / speculative verify (sm_100a), split-KV.
//
// One CTA = (sequence b, KV head g, key span). Its rows are the T x G query rows that read KV
// head g (T new tokens x the G query heads of the GQA group), so every K/V row fetched from HBM
// serves the whole group. The span's keys stream through a 4-stage cp.async ring in shared
// memory (16-byte vector loads, XOR-swizzled rows for conflict-free ldmatrix). The two
// contractions S = Q K^T and O += P V run on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate); row max / row sum use quad warp shuffles. Partials are sink-free:
//     m_p = max_j a_j, l_p = sum_j exp(a_j - m_p), O_p = sum_j exp(a_j - m_p) v_j
// and the sink is counted exactly once when the spans are merged ("MiMo-V2-Flash 架构 QA" Q3.8):
//     m = max(sink, max_p m_p), D = exp(sink - m) + sum_p l_p exp(m_p - m),
//     O = sum_p O_p exp(m_p - m) / D, LSE = m + ln D.
// With a single span the same kernel applies the sink and writes O / LSE itself.
//
// Key order inside a (b, g) unit: the used cached tokens oldest first, then the T new tokens.
// A cached token c (0 = oldest of n) sits at position c - n, new token u at u; new query t sees
// positions p <= t and, with a window W, p > t - W (so only the newest W - 1 cached tokens can
// ever be visible and older ones are not read).
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace dec {
constexpr int KT = 64;                 // keys per shared-memory tile
constexpr int KROW = 384, VROW = 256;  // bytes per K row (192 dims) / V row (128 dims)
constexpr int STAGE_K = KT * KROW;
constexpr int STAGE_V = KT * VROW;
constexpr int STAGE = STAGE_K + STAGE_V + KT; // + one validity byte per key
constexpr int THREADS = 128;
// cp.async ring depth and CTAs per SM: 4 stages (160 KB, 1 CTA / SM) or 2 stages (80 KB,
// 2 CTAs / SM)
__host__ __device__ constexpr int smem_bytes(int nstage) { return nstage * STAGE; }
constexpr int RED_STRIDE = 70;         // floats per lane in the cross-warp combine
} // namespace dec

struct KeyRows {
    const uint16_t *k, *v;
    bool valid;
};

// Global rows of virtual key v of unit (b, g).
SA_DEV KeyRows key_rows(const DecodeParams &p, int b, int g, int v, int n_used, int first_c,
                        int ring_head)
{
    KeyRows r{p.k_new, p.v_new, false};
    if (v < n_used) {
        const int c = first_c + v;
        int64_t ko, vo;
        if (p.kind == 0) { // ring
            const int slot = (ring_head + c) % p.ring_cap;
            ko = (int64_t)b * p.kc_sb + (int64_t)slot * p.kc_ss + (int64_t)g * p.kc_sh;
            vo = (int64_t)b * p.vc_sb + (int64_t)slot * p.vc_ss + (int64_t)g * p.vc_sh;
        } else if (p.kind == 1) { // contiguous
            ko = (int64_t)b * p.kc_sb + (int64_t)c * p.kc_ss + (int64_t)g * p.kc_sh;
            vo = (int64_t)b * p.vc_sb + (int64_t)c * p.vc_ss + (int64_t)g * p.vc_sh;
        } else { // paged
            const int pg = c / p.page_size;
            if (pg >= p.max_pages)
                return r;
            const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
            if (pid < 0 || pid >= p.num_pages)
                return r;
            const int rr = c - pg * p.page_size;
            ko = (int64_t)pid * p.kc_sb + (int64_t)rr * p.kc_ss + (int64_t)g * p.kc_sh;
            vo = (int64_t)pid * p.vc_sb + (int64_t)rr * p.vc_ss + (int64_t)g * p.vc_sh;
        }
        r.k = p.k_cache + ko;
        r.v = p.v_cache + vo;
        r.valid = true;
    } else {
        const int u = v - n_used;
        r.k = p.k_new + (int64_t)b * p.kn_sb + (int64_t)u * p.kn_st + (int64_t)g * p.kn_sh;
        r.v = p.v_new + (int64_t)b * p.vn_sb + (int64_t)u * p.vn_st + (int64_t)g * p.vn_sh;
        r.valid = true;
    }
    return r;
}

// Issue the cp.async copies of one tile: thread pairs share a key, each copies half its K row
// (12 x 16 B) and half its V row (8 x 16 B). Invalid keys are zero-filled and flagged.
SA_DEV void load_tile(const DecodeParams &p, uint8_t *stage, int vt, int ke, int b, int g,
                      int n_used, int first_c, int ring_head)
{
    using namespace dec;
    const int key = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int v = vt + key;
    KeyRows r{p.k_new, p.v_new, false};
    if (v < ke)
        r = key_rows(p, b, g, v, n_used, first_c, ring_head);
    uint8_t *sk = stage + key * KROW;
    uint8_t *sv = stage + STAGE_K + key * VROW;
#pragma unroll
    for (int i = 0; i < 12; ++i) {
        const int ch = half * 12 + i;
        cp_async16(sk + ((ch ^ (key & 7)) << 4), r.k + ch * 8, r.valid);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int ch = half * 8 + i;
        cp_async16(sv + ((ch ^ (key & 7)) << 4), r.v + ch * 8, r.valid);
    }
    if (half == 0)
        stage[STAGE_K + STAGE_V + key] = r.valid ? 1 : 0;
}

// Writes the result of one consumer warp's rows (lane/4 and lane/4 + 8 of its m-tile): with a
// single span, the final O and LSE (the sink applied once: m_f = max(m, sink),
// D = l e^(m - m_f) + e^(sink - m_f)); otherwise the span's partial (O, m, l_rounded, l_exact).
SA_DEV void decode_write_output(const DecodeParams &p, int b, int g, int split, int ra, int rb,
                                int lane, const float (&o)[16][4], float m_a, float m_b,
                                float l_a, float l_b, float e_a, float e_b)
{
    const int c2 = 2 * (lane & 3);
    if (p.splits == 1) {
        // apply the sink once and finish: m_f = max(m, sink), D = l e^(m - m_f) + e^(sink - m_f)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int r = half ? rb : ra;
            if (r >= p.R)
                continue;
            const int t = r / p.G, h = g * p.G + r % p.G;
            const float m = half ? m_b : m_a, l = half ? l_b : l_a, le = half ? e_b : e_a;
            const float sk = p.sink ? p.sink[h] * kLog2e : -INFINITY;
            const float mf = fmaxf(m, sk);
            const float cm = (m == -INFINITY) ? 0.f : fast_exp2(m - mf);
            const float cs = (sk == -INFINITY) ? 0.f : fast_exp2(sk - mf);
            const float D = le * cm + cs;         // exact denominator: LSE
            const float scl = cm / (l * cm + cs); // rounded-P denominator: O
            uint16_t *orow = p.o + (int64_t)b * p.o_sb + (int64_t)t * p.o_st + (int64_t)h * p.o_sh;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float x0 = (half ? o[i][2] : o[i][0]) * scl;
                const float x1 = (half ? o[i][3] : o[i][1]) * scl;
                *reinterpret_cast<uint32_t *>(orow + i * 8 + c2) = pack_bf16x2(x0, x1);
            }
            if (p.lse && (lane & 3) == 0)
                p.lse[((int64_t)b * p.T + t) * p.Hq + h] = (mf + fast_log2(D)) * kLn2;
        }
    } else {
        const int64_t unit = ((int64_t)b * p.Hkv + g) * p.splits + split;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int r = half ? rb : ra;
            if (r >= p.R)
                continue;
            float *wo = p.ws_o + (unit * p.R + r) * 128;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float2 v2;
                v2.x = half ? o[i][2] : o[i][0];
                v2.y = half ? o[i][3] : o[i][1];
                *reinterpret_cast<float2 *>(wo + i * 8 + c2) = v2;
            }
            if ((lane & 3) == 0) {
                float4 ml;
                ml.x = half ? m_b : m_a;
                ml.y = half ? l_b : l_a;
                ml.z = half ? e_b : e_a;
                ml.w = 0.f;
                *reinterpret_cast<float4 *>(p.ws_ml + (unit * p.R + r) * 4) = ml;
            }
        }
    }
}

template <int KP, int NSTAGE>
SA_DEV void decode_body(const DecodeParams &p, uint8_t *smem)
{
    using namespace dec;
    constexpr int KW = KT / KP; // keys per warp per tile
    constexpr int NT = KW / 8;  // n-tiles of S per warp
    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = p.MT;
    const int mt = warp % MT, ks = warp / MT;
    const bool active = ks < KP;

    int n_cache = (p.kind == 0) ? p.ring_len[b] : p.ctx_len[b];
    n_cache = max(0, min(n_cache, p.kind == 0 ? p.ring_cap : p.max_ctx));
    const int n_used = (p.window > 0) ? min(n_cache, p.window - 1) : n_cache;
    const int first_c = n_cache - n_used;
    const int n_total = n_used + p.T;
    const int kb = split * p.chunk;
    const int ke = min(kb + p.chunk, n_total);
    const int ntile = (ke > kb) ? (ke - kb + KT - 1) / KT : 0;
    const int ring_head = (p.kind == 0) ? ((p.ring_head[b] % p.ring_cap) + p.ring_cap) % p.ring_cap : 0;

    // rows of this warp: lane/4 and lane/4 + 8 of m-tile mt
    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int ta = min(ra / p.G, p.T - 1), tb = min(rb / p.G, p.T - 1);

    // Q fragments (A operand, 12 k-steps of 16 dims), zero for padding rows
    uint32_t qa[12][4];
    {
        const bool va = active && ra < p.R, vb = active && rb < p.R;
        const uint16_t *qra = p.q + (int64_t)b * p.q_sb + (int64_t)ta * p.q_st +
                              (int64_t)(g * p.G + (va ? ra % p.G : 0)) * p.q_sh;
        const uint16_t *qrb = p.q + (int64_t)b * p.q_sb + (int64_t)tb * p.q_st +
                              (int64_t)(g * p.G + (vb ? rb % p.G : 0)) * p.q_sh;
        const int c2 = 2 * (lane & 3);
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
    // per row: running max m, sum of bf16-rounded P (l*, normalises O) and of fp32 P (e*, LSE)
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f, e_a = 0.f, e_b = 0.f;

    // prologue: NSTAGE - 1 tiles in flight
#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
        if (s < ntile)
            load_tile(p, smem + s * STAGE, kb + s * KT, ke, b, g, n_used, first_c, ring_head);
        cp_async_commit();
    }

    for (int it = 0; it < ntile; ++it) {
        cp_async_wait<NSTAGE - 2>();
        __syncthreads();
        {
            const int nx = it + NSTAGE - 1;
            if (nx < ntile)
                load_tile(p, smem + (nx % NSTAGE) * STAGE, kb + nx * KT, ke, b, g, n_used,
                          first_c, ring_head);
            cp_async_commit();
        }
        if (!active)
            continue;
        const uint8_t *stage = smem + (it % NSTAGE) * STAGE;
        const uint32_t sK = smem_u32(stage), sV = smem_u32(stage + STAGE_K);
        const uint8_t *vflag = stage + STAGE_K + STAGE_V;
        const int key0 = ks * KW; // first key of this warp inside the tile

        // ---- S = Q K^T
        float sacc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < 6; ++k2) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int key = key0 + nt * 8 + (lane & 7);
                const int ch = 4 * k2 + (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(sK + key * KROW + ((ch ^ (key & 7)) << 4), b0, b1, b2, b3);
                mma_bf16_16816(sacc[nt], qa[2 * k2], b0, b1);
                mma_bf16_16816(sacc[nt], qa[2 * k2 + 1], b2, b3);
            }
        }

        // ---- mask, online softmax (sink-free partial)
        const int vbase = kb + it * KT + key0;
        float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kc = nt * 8 + 2 * (lane & 3) + e;
                const int v = vbase + kc;
                const int pos = v - n_used;
                const bool ok = vflag[key0 + kc] != 0;
                const bool vis_a = ok && pos <= ta && (p.window <= 0 || pos > ta - p.window);
                const bool vis_b = ok && pos <= tb && (p.window <= 0 || pos > tb - p.window);
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
        // P in bf16 pairs: [nt][0] row a, [nt][1] row b; the row sums add these same rounded
        // values so the weights of numerator and denominator agree
        uint32_t pp[NT][2];
        float sa = 0.f, sb = 0.f, xa = 0.f, xb = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
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

        // ---- O += P V
#pragma unroll
        for (int kq = 0; kq < NT / 2; ++kq) {
            uint32_t a[4];
            a[0] = pp[2 * kq][0];
            a[1] = pp[2 * kq][1];
            a[2] = pp[2 * kq + 1][0];
            a[3] = pp[2 * kq + 1][1];
            const int key = key0 + kq * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const int ch = 2 * np + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(sV + key * VROW + ((ch ^ (key & 7)) << 4), b0, b1, b2, b3);
                mma_bf16_16816(o[2 * np], a, b0, b1);
                mma_bf16_16816(o[2 * np + 1], a, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

    // full row sums across the quad
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    e_a += __shfl_xor_sync(0xffffffffu, e_a, 1);
    e_a += __shfl_xor_sync(0xffffffffu, e_a, 2);
    e_b += __shfl_xor_sync(0xffffffffu, e_b, 1);
    e_b += __shfl_xor_sync(0xffffffffu, e_b, 2);

    // ---- combine the KP key slices of each m-tile (same fragment layout in every warp)
    if (KP > 1) {
        __syncthreads(); // all warps are done with the stages
        float *red = reinterpret_cast<float *>(smem);
        if (active && ks > 0) {
            float *dst = red + ((ks * MT + mt) * 32 + lane) * RED_STRIDE;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                dst[4 * i + 0] = o[i][0];
                dst[4 * i + 1] = o[i][1];
                dst[4 * i + 2] = o[i][2];
                dst[4 * i + 3] = o[i][3];
            }
            dst[64] = m_a;
            dst[65] = m_b;
            dst[66] = l_a;
            dst[67] = l_b;
            dst[68] = e_a;
            dst[69] = e_b;
        }
        __syncthreads();
        if (active && ks == 0) {
#pragma unroll
            for (int k2 = 1; k2 < KP; ++k2) {
                const float *src = red + ((k2 * MT + mt) * 32 + lane) * RED_STRIDE;
                const float m2a = src[64], m2b = src[65];
                const float mna = fmaxf(m_a, m2a), mnb = fmaxf(m_b, m2b);
                const float a1 = (mna == -INFINITY) ? 0.f : fast_exp2(m_a - mna);
                const float a2 = (mna == -INFINITY) ? 0.f : fast_exp2(m2a - mna);
                const float b1 = (mnb == -INFINITY) ? 0.f : fast_exp2(m_b - mnb);
                const float b2 = (mnb == -INFINITY) ? 0.f : fast_exp2(m2b - mnb);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    o[i][0] = o[i][0] * a1 + src[4 * i + 0] * a2;
                    o[i][1] = o[i][1] * a1 + src[4 * i + 1] * a2;
                    o[i][2] = o[i][2] * b1 + src[4 * i + 2] * b2;
                    o[i][3] = o[i][3] * b1 + src[4 * i + 3] * b2;
                }
                l_a = l_a * a1 + src[66] * a2;
                l_b = l_b * b1 + src[67] * b2;
                e_a = e_a * a1 + src[68] * a2;
                e_b = e_b * b1 + src[69] * b2;
                m_a = mna;
                m_b = mnb;
            }
        }
    }
    if (!active || ks != 0)
        return;

    decode_write_output(p, b, g, split, ra, rb, lane, o, m_a, m_b, l_a, l_b, e_a, e_b);
}

// KP = warps that split each tile's keys: 4 when the unit has one 16-row m-tile (T x G <= 16),
// 2 for two m-tiles, 1 for three or four.
template <int KP, int NSTAGE>
__global__ void __launch_bounds__(dec::THREADS, NSTAGE == 2 ? 2 : 1)
    decode_split_kernel(const DecodeParams p)
{
    extern __shared__ __align__(128) uint8_t dsmem[];
    decode_body<KP, NSTAGE>(p, dsmem);
}

// Merge the spans of each query row, counting the sink once. One warp per (b, t, h) row; each
// lane owns 4 of the 128 output dims.
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + warp;
    if (row >= (int64_t)p.B * p.T * p.Hq)
        return;
    const int h = (int)(row % p.Hq);
    const int t = (int)((row / p.Hq) % p.T);
    const int b = (int)(row / ((int64_t)p.Hq * p.T));
    const int g = h / p.G;
    const int r = t * p.G + (h - g * p.G);
    const float sk = p.sink ? p.sink[h] * kLog2e : -INFINITY;
    float m = sk, l = (sk == -INFINITY) ? 0.f : 1.f, le = l;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t unit0 = ((int64_t)b * p.Hkv + g) * p.splits;
    for (int s = 0; s < p.splits; ++s) {
        const int64_t idx = (unit0 + s) * p.R + r;
        const float4 ml = *reinterpret_cast<const float4 *>(p.ws_ml + idx * 4);
        if (!(ml.y > 0.f))
            continue;
        const float mn = fmaxf(m, ml.x);
        const float a = (m == -INFINITY) ? 0.f : fast_exp2(m - mn);
        const float c = fast_exp2(ml.x - mn);
        const float4 v = *reinterpret_cast<const float4 *>(p.ws_o + idx * 128 + lane * 4);
        acc.x = acc.x * a + v.x * c;
        acc.y = acc.y * a + v.y * c;
        acc.z = acc.z * a + v.z * c;
        acc.w = acc.w * a + v.w * c;
        l = l * a + ml.y * c;
        le = le * a + ml.z * c;
        m = mn;
    }
    const float inv = 1.f / l;
    uint16_t *orow = p.o + (int64_t)b * p.o_sb + (int64_t)t * p.o_st + (int64_t)h * p.o_sh;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(orow + lane * 4) = pk;
    if (p.lse && lane == 0)
        p.lse[((int64_t)b * p.T + t) * p.Hq + h] = (m + fast_log2(le)) * kLn2;
}

cudaError_t launch_decode_merge(const DecodeParams &p, cudaStream_t stream)
{
    const int64_t rows = (int64_t)p.B * p.T * p.Hq;
    decode_merge_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int NSTAGE>
cudaError_t launch_decode_split(const DecodeParams &p, cudaStream_t stream)
{
    dim3 grid(p.splits, p.Hkv, p.B);
    const int smem = dec::smem_bytes(NSTAGE);
    if (p.MT == 1)
        decode_split_kernel<4, NSTAGE><<<grid, dec::THREADS, smem, stream>>>(p);
    else if (p.MT == 2)
        decode_split_kernel<2, NSTAGE><<<grid, dec::THREADS, smem, stream>>>(p);
    else
        decode_split_kernel<1, NSTAGE><<<grid, dec::THREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

int decode_stages(const DecodeParams &p);

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        cudaError_t e = cudaSuccess;
        const void *fns[6] = {(const void *)decode_split_kernel<4, 4>,
                              (const void *)decode_split_kernel<2, 4>,
                              (const void *)decode_split_kernel<1, 4>,
                              (const void *)decode_split_kernel<4, 2>,
                              (const void *)decode_split_kernel<2, 2>,
                              (const void *)decode_split_kernel<1, 2>};
        for (int i = 0; i < 6; ++i) {
            e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     dec::smem_bytes(i < 3 ? 4 : 2));
            if (e != cudaSuccess)
                return e;
        }
        return e;
    });
    if (e != cudaSuccess)
        return e;
    e = decode_stages(p) == 2 ? launch_decode_split<2>(p, stream) : launch_decode_split<4>(p, stream);
    if (e != cudaSuccess || p.splits == 1)
        return e;
    return launch_decode_merge(p, stream);
}

// ---------------------------------------------------------------------------------------------
// Cache commit: one CTA per sequence copies its accepted tokens, then thread 0 advances that
// sequence's ring head / length or context length (only this CTA reads them).
// ---------------------------------------------------------------------------------------------
// The work of one thread: one 16-byte piece (8 values) of a new token's K or V head row, or,
// when the commit rotates K, the two K pieces c and c + rope_half / 8 whose dims are the rotation
// pairs (i, i + rope_dim / 2).
struct CommitPiece {
    int is_k, c0, c1; // c1 < 0: one piece
};

SA_DEV int commit_pieces_per_head(const CommitParams &p) { return 24 - p.rope_half / 8 + 16; }

SA_DEV CommitPiece commit_piece(const CommitParams &p, int idx)
{
    const int nrp = p.rope_half / 8; // rotated piece pairs
    const int nk = 24 - nrp;         // K work items: the pairs, then the unrotated pieces
    if (idx < nrp)
        return CommitPiece{1, idx, idx + nrp};
    if (idx < nk)
        return CommitPiece{1, idx + nrp, -1};
    return CommitPiece{0, idx - nk, -1};
}

// The piece(s) of new token u, KV head gh, of sequence b as the cache stores them: rotated at
// position `pos` (a K pair) or multiplied by v_mul (V, when the commit transforms), else as
// given. The arithmetic is the RoPE pass's, so both give the same bits.
SA_DEV void commit_load(const CommitParams &p, const CommitPiece &pc, int b, int u, int gh,
                        int64_t pos, uint4 &x0, uint4 &x1)
{
    const uint16_t *row =
        pc.is_k ? p.k_new + (int64_t)b * p.kn_sb + (int64_t)u * p.kn_st + (int64_t)gh * p.kn_sh
                : p.v_new + (int64_t)b * p.vn_sb + (int64_t)u * p.vn_st + (int64_t)gh * p.vn_sh;
    x0 = *reinterpret_cast<const uint4 *>(row + pc.c0 * 8);
    if (pc.c1 >= 0) {
        x1 = *reinterpret_cast<const uint4 *>(row + pc.c1 * 8);
        float2 cs[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            cs[j] = rope_cos_sin(pos, p.inv_freq[pc.c0 * 8 + j]);
        rope_rotate8(x0, x1, cs);
    } else if (!pc.is_k && p.rope_half > 0) {
        scale8(x0, p.v_mul);
    }
}

// Where token u of sequence b goes: its K and V row offsets (elements for a bf16 cache, bytes
// for an FP8 one); false if it falls outside the cache (dropped).
SA_DEV bool commit_dst(const CommitParams &p, int b, int u, int head, int len, int ctx,
                       int64_t &kdst, int64_t &vdst)
{
    if (p.kind == 0) {
        const int slot = (head + len + u) % p.ring_cap;
        kdst = (int64_t)b * p.kc_sb + (int64_t)slot * p.kc_ss;
        vdst = (int64_t)b * p.vc_sb + (int64_t)slot * p.vc_ss;
        return true;
    }
    const int pos = ctx + u;
    if (pos >= p.max_ctx)
        return false;
    if (p.kind == 1) {
        kdst = (int64_t)b * p.kc_sb + (int64_t)pos * p.kc_ss;
        vdst = (int64_t)b * p.vc_sb + (int64_t)pos * p.vc_ss;
        return true;
    }
    const int pg = pos / p.page_size;
    if (pg >= p.max_pages)
        return false;
    const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
    if (pid < 0 || pid >= p.num_pages)
        return false;
    const int rr = pos - pg * p.page_size;
    kdst = (int64_t)pid * p.kc_sb + (int64_t)rr * p.kc_ss;
    vdst = (int64_t)pid * p.vc_sb + (int64_t)rr * p.vc_ss;
    return true;
}

// The sequence's cache state before the commit, and the advance after it (thread 0, once every
// thread of the CTA is done).
struct CommitState {
    int head, len, ctx, n;
};

SA_DEV CommitState commit_state(const CommitParams &p, int b)
{
    CommitState c{0, 0, 0, max(0, min(p.n_accept[b], p.T))};
    if (p.kind == 0) {
        c.head = ((p.ring_head[b] % p.ring_cap) + p.ring_cap) % p.ring_cap;
        c.len = max(0, min(p.ring_len[b], p.ring_cap));
    } else {
        c.ctx = max(0, min(p.ctx_len[b], p.max_ctx));
    }
    return c;
}

SA_DEV void commit_advance(const CommitParams &p, int b, const CommitState &c)
{
    if (p.kind == 0) {
        const int over = max(0, c.len + c.n - p.ring_cap);
        p.ring_len[b] = min(p.ring_cap, c.len + c.n);
        p.ring_head[b] = (c.head + over) % p.ring_cap;
    } else {
        p.ctx_len[b] = min(c.ctx + c.n, p.max_ctx);
    }
}

__global__ void __launch_bounds__(128) kv_commit_kernel(const __grid_constant__ CommitParams p)
{
    const int b = blockIdx.x;
    const CommitState cs = commit_state(p, b);
    const int pph = commit_pieces_per_head(p);
    const int per_tok = p.Hkv * pph;
    const int64_t pos0 = p.pos ? (int64_t)p.pos[b] : (int64_t)cs.ctx;
    for (int i = threadIdx.x; i < cs.n * per_tok; i += blockDim.x) {
        const int u = i / per_tok;
        const int rem = i - u * per_tok;
        const int gh = rem / pph;
        const CommitPiece pc = commit_piece(p, rem - gh * pph);
        int64_t kdst, vdst;
        if (!commit_dst(p, b, u, cs.head, cs.len, cs.ctx, kdst, vdst))
            continue;
        uint4 x0, x1;
        commit_load(p, pc, b, u, gh, pos0 + u, x0, x1);
        uint16_t *row = pc.is_k ? p.k_cache + kdst + (int64_t)gh * p.kc_sh
                                : p.v_cache + vdst + (int64_t)gh * p.vc_sh;
        *reinterpret_cast<uint4 *>(row + pc.c0 * 8) = x0;
        if (pc.c1 >= 0)
            *reinterpret_cast<uint4 *>(row + pc.c1 * 8) = x1;
    }
    __syncthreads();
    if (threadIdx.x == 0)
        commit_advance(p, b, cs);
}

cudaError_t launch_commit(const CommitParams &p, cudaStream_t stream)
{
    kv_commit_kernel<<<p.B, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t set_wait_limit(uint64_t ns)
{
    cudaError_t e = cudaDeviceSynchronize(); // no kernel of ours runs while the limit changes
    if (e != cudaSuccess)
        return e;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}

cudaError_t read_and_clear_device_error(uint32_t *flag)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(flag, g_device_error, sizeof(uint32_t));
    if (e != cudaSuccess)
        return e;
    const uint32_t zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
}

} // namespace sinkattn
