// Decode / speculative verify against an FP8 (E4M3) KV cache, and the commit into one.
//
// The cache holds one-byte E4M3 codes, one fp32 scale per tensor: a K code c stands for
// e4m3(c) * k_scale, a V code for e4m3(c) * v_scale (the pages size a KV slot at one byte and
// speak of FP8 inference, "MiMo-V2-Flash Technical Report" paper notes; the format and the
// scaling are this library's reading). Attention is linear in both scales:
//     a_j = scale * <q, k_scale e(c_j)> = (scale * k_scale) * <q, e(c_j)>,
//     O   = sum_j w_j v_scale e(c'_j)   = v_scale * sum_j w_j e(c'_j),
// so the tensor cores multiply the E4M3 values themselves, which fp16 holds exactly (4
// significant bits, exponents -9..8), scale * k_scale goes into the logit scale and v_scale
// into O. The T new tokens (bf16) are quantised on load exactly as the commit stores them, so
// every key and value of the attention is a cache value.
//
// Structure: the split-KV decode of the bf16 cp.async kernel (one CTA = (key span, KV head,
// sequence), its T x G query rows on mma.sync m16n8k16, sink-free partials merged with the sink
// counted once). The codes stream through a 3-stage cp.async ring of 20 KB stages; each tile is
// then widened in shared memory into the f16 layout of the bf16 kernel (rows of 384 / 256
// bytes, 16-byte chunks XOR-swizzled by key), with cvt.rn.f16x2.e4m3x2 (exact), and read with
// ldmatrix as there. Q is rounded once to fp16 (exact inside fp16's normal range, so |q| must
// stay below 65504); P is rounded to fp16 for the P.V product and the row sum that normalises
// O adds the same rounded values.
#pragma once
#include <cuda_fp16.h>

#include "common.cuh"
#include "decode_kernels.cuh"
#include "internal.h"

namespace sinkattn {

namespace d8 {
constexpr int KT = dec::KT;                   // 64 keys per tile
constexpr int KROW8 = 192, VROW8 = 128;       // code bytes per K / V row
constexpr int STAGE_K8 = KT * KROW8;          // 12 KB
constexpr int STAGE_V8 = KT * VROW8;          // 8 KB
constexpr int FLAG8 = STAGE_K8 + STAGE_V8;    // one validity byte per key
constexpr int STAGE8 = (FLAG8 + KT + 127) / 128 * 128; // 20608 bytes, 128-byte aligned slots
constexpr int NSTAGE = 3;
constexpr int OFF_TILE = NSTAGE * STAGE8;     // the widened f16 tile (dec::STAGE bytes)
constexpr int SMEM = OFF_TILE + dec::STAGE;   // 102848 bytes: two CTAs per SM
constexpr int THREADS = dec::THREADS;
static_assert(STAGE8 % 16 == 0 && OFF_TILE % 128 == 0, "16-byte chunks, aligned tile");
} // namespace d8

// D (16x8 fp32) += A (16x16 fp16, row) * B (16x8 fp16, col)
SA_DEV void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

SA_DEV uint32_t pack_f16x2(float lo, float hi)
{
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

SA_DEV float sum_f16x2(uint32_t v)
{
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&v));
    return f.x + f.y;
}

// bf16 pair -> fp16 pair (round to nearest even; exact inside fp16's normal range)
SA_DEV uint32_t bf16x2_to_f16x2(uint32_t v)
{
    return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// Two E4M3 codes (low byte first) -> their fp16 values (exact)
SA_DEV uint32_t e4m3x2_to_f16x2(uint32_t codes16)
{
    uint32_t r;
    const uint16_t c = (uint16_t)codes16;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c));
    return r;
}

// The E4M3 codes of x0 / scale (low byte) and x1 / scale: fp32 division (correctly rounded),
// then the nearest E4M3 value, ties to even, saturating to +-448
SA_DEV uint32_t quant_e4m3x2(float x0, float x1, float scale)
{
    const float y0 = __fdiv_rn(x0, scale), y1 = __fdiv_rn(x1, scale);
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(y1), "f"(y0));
    return r;
}

// 16 bf16 values (two 16-byte loads) -> 16 codes (one 16-byte value)
SA_DEV uint4 quant16(const uint16_t *src, float scale)
{
    const uint4 a = reinterpret_cast<const uint4 *>(src)[0];
    const uint4 b = reinterpret_cast<const uint4 *>(src)[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        c[i] = quant_e4m3x2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u), scale);
    return make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16),
                      c[6] | (c[7] << 16));
}

// Byte offsets of cached token c of unit (b, g) in the K / V code caches; false for a page the
// table does not map.
SA_DEV bool fp8_cache_offsets(const DecodeParams &p, int b, int g, int c, int ring_head,
                              int64_t &ko, int64_t &vo)
{
    if (p.kind == 0) { // ring
        const int slot = (ring_head + c) % p.ring_cap;
        ko = (int64_t)b * p.kc_sb + (int64_t)slot * p.kc_ss;
        vo = (int64_t)b * p.vc_sb + (int64_t)slot * p.vc_ss;
    } else if (p.kind == 1) { // contiguous
        ko = (int64_t)b * p.kc_sb + (int64_t)c * p.kc_ss;
        vo = (int64_t)b * p.vc_sb + (int64_t)c * p.vc_ss;
    } else { // paged
        const int pg = c / p.page_size;
        if (pg >= p.max_pages)
            return false;
        const int pid = p.page_table[(int64_t)b * p.max_pages + pg];
        if (pid < 0 || pid >= p.num_pages)
            return false;
        const int rr = c - pg * p.page_size;
        ko = (int64_t)pid * p.kc_sb + (int64_t)rr * p.kc_ss;
        vo = (int64_t)pid * p.vc_sb + (int64_t)rr * p.vc_ss;
    }
    ko += (int64_t)g * p.kc_sh;
    vo += (int64_t)g * p.vc_sh;
    return true;
}

// One tile of codes into a staging slot: thread pairs share a key, each moving half its K row
// (6 x 16 B) and half its V row (4 x 16 B). Cached keys come by cp.async; a new token's bf16
// row is quantised here and stored; keys past the span and unmapped pages are zero-filled and
// flagged invalid.
SA_DEV void load_tile_fp8(const DecodeParams &p, uint8_t *stage, int vt, int ke, int b, int g,
                          int n_used, int first_c, int ring_head)
{
    using namespace d8;
    const int key = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int v = vt + key;
    uint8_t *sk = stage + key * KROW8 + half * 96;
    uint8_t *sv = stage + STAGE_K8 + key * VROW8 + half * 64;
    bool valid = false;
    if (v < ke && v >= n_used) {
        const int u = v - n_used;
        const uint16_t *kr = p.k_new + (int64_t)b * p.kn_sb + (int64_t)u * p.kn_st +
                             (int64_t)g * p.kn_sh + half * 96;
        const uint16_t *vr = p.v_new + (int64_t)b * p.vn_sb + (int64_t)u * p.vn_st +
                             (int64_t)g * p.vn_sh + half * 64;
#pragma unroll
        for (int i = 0; i < 6; ++i)
            *reinterpret_cast<uint4 *>(sk + i * 16) = quant16(kr + i * 16, p.k_scale);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4 *>(sv + i * 16) = quant16(vr + i * 16, p.v_scale);
        valid = true;
    } else {
        const uint8_t *kr = p.k8, *vr = p.v8; // not read when zero-filling
        if (v < ke) {
            int64_t ko = 0, vo = 0;
            valid = fp8_cache_offsets(p, b, g, first_c + v, ring_head, ko, vo);
            if (valid) {
                kr = p.k8 + ko + half * 96;
                vr = p.v8 + vo + half * 64;
            }
        }
#pragma unroll
        for (int i = 0; i < 6; ++i)
            cp_async16(sk + i * 16, kr + i * 16, valid);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            cp_async16(sv + i * 16, vr + i * 16, valid);
    }
    if (half == 0)
        stage[FLAG8 + key] = valid ? 1 : 0;
}

// Widen a staged tile of codes into the f16 tile the consumers read (the bf16 kernel's layout:
// K rows of 24 and V rows of 16 sixteen-byte chunks, chunk ch of key at (ch ^ (key & 7))).
SA_DEV void widen_tile_fp8(const uint8_t *st, uint8_t *tile)
{
    using namespace d8;
    for (int i = threadIdx.x; i < KT * 20; i += THREADS) {
        const int key = i / 20, j = i - key * 20;
        const bool is_k = j < 12;
        const uint4 c = is_k ? *reinterpret_cast<const uint4 *>(st + key * KROW8 + j * 16)
                             : *reinterpret_cast<const uint4 *>(st + STAGE_K8 + key * VROW8 +
                                                                 (j - 12) * 16);
        uint8_t *row = is_k ? tile + key * dec::KROW : tile + dec::STAGE_K + key * dec::VROW;
        const int ch = 2 * (is_k ? j : j - 12);
        uint4 h0, h1;
        h0.x = e4m3x2_to_f16x2(c.x & 0xffffu);
        h0.y = e4m3x2_to_f16x2(c.x >> 16);
        h0.z = e4m3x2_to_f16x2(c.y & 0xffffu);
        h0.w = e4m3x2_to_f16x2(c.y >> 16);
        h1.x = e4m3x2_to_f16x2(c.z & 0xffffu);
        h1.y = e4m3x2_to_f16x2(c.z >> 16);
        h1.z = e4m3x2_to_f16x2(c.w & 0xffffu);
        h1.w = e4m3x2_to_f16x2(c.w >> 16);
        *reinterpret_cast<uint4 *>(row + ((ch ^ (key & 7)) << 4)) = h0;
        *reinterpret_cast<uint4 *>(row + (((ch + 1) ^ (key & 7)) << 4)) = h1;
    }
    if (threadIdx.x < KT)
        tile[dec::STAGE_K + dec::STAGE_V + threadIdx.x] = st[FLAG8 + threadIdx.x];
}

template <int KP>
__global__ void __launch_bounds__(d8::THREADS, 2) decode_fp8_kernel(const DecodeParams p)
{
    using namespace dec;
    constexpr int NSTAGE = d8::NSTAGE;
    constexpr int KW = KT / KP; // keys per warp per tile
    constexpr int NT = KW / 8;  // n-tiles of S per warp
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *tile = smem + d8::OFF_TILE;
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

    const int ra = mt * 16 + (lane >> 2), rb = ra + 8;
    const int ta = min(ra / p.G, p.T - 1), tb = min(rb / p.G, p.T - 1);

    // Q fragments in fp16 (A operand, 12 k-steps of 16 dims), zero for padding rows
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
            qa[kk][0] = va ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qra + kk * 16 + c2)) : 0u;
            qa[kk][1] = vb ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrb + kk * 16 + c2)) : 0u;
            qa[kk][2] = va ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qra + kk * 16 + 8 + c2)) : 0u;
            qa[kk][3] = vb ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrb + kk * 16 + 8 + c2)) : 0u;
        }
    }

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f, e_a = 0.f, e_b = 0.f;

#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
        if (s < ntile)
            load_tile_fp8(p, smem + s * d8::STAGE8, kb + s * KT, ke, b, g, n_used, first_c,
                          ring_head);
        cp_async_commit();
    }

    for (int it = 0; it < ntile; ++it) {
        cp_async_wait<NSTAGE - 2>();
        __syncthreads(); // tile `it` staged; every warp is done with the f16 tile of it - 1
        {
            const int nx = it + NSTAGE - 1;
            if (nx < ntile)
                load_tile_fp8(p, smem + (nx % NSTAGE) * d8::STAGE8, kb + nx * KT, ke, b, g,
                              n_used, first_c, ring_head);
            cp_async_commit();
        }
        widen_tile_fp8(smem + (it % NSTAGE) * d8::STAGE8, tile);
        __syncthreads();
        if (!active)
            continue;
        const uint32_t sK = smem_u32(tile), sV = smem_u32(tile + STAGE_K);
        const uint8_t *vflag = tile + STAGE_K + STAGE_V;
        const int key0 = ks * KW;

        // ---- S = Q e(K)^T
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
                mma_f16_16816(sacc[nt], qa[2 * k2], b0, b1);
                mma_f16_16816(sacc[nt], qa[2 * k2 + 1], b2, b3);
            }
        }

        // ---- mask, online softmax (sink-free partial); scale_log2 includes k_scale
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
        uint32_t pp[NT][2];
        float sa = 0.f, sb = 0.f, xa = 0.f, xb = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float p0 = fast_exp2(sacc[nt][0] - ua), p1 = fast_exp2(sacc[nt][1] - ua);
            const float p2 = fast_exp2(sacc[nt][2] - ub), p3 = fast_exp2(sacc[nt][3] - ub);
            xa += p0 + p1;
            xb += p2 + p3;
            pp[nt][0] = pack_f16x2(p0, p1);
            pp[nt][1] = pack_f16x2(p2, p3);
            sa += sum_f16x2(pp[nt][0]);
            sb += sum_f16x2(pp[nt][1]);
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

        // ---- O += P e(V)
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
                mma_f16_16816(o[2 * np], a, b0, b1);
                mma_f16_16816(o[2 * np + 1], a, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

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
        __syncthreads(); // every warp is done with the staging ring and the tile
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
    // the values were e(c): O of the cache's values is v_scale times this (partials merge
    // linearly, so the partials carry it too)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        o[i][0] *= p.v_scale;
        o[i][1] *= p.v_scale;
        o[i][2] *= p.v_scale;
        o[i][3] *= p.v_scale;
    }
    decode_write_output(p, b, g, split, ra, rb, lane, o, m_a, m_b, l_a, l_b, e_a, e_b);
}

cudaError_t launch_decode_fp8(const DecodeParams &p, cudaStream_t stream)
{
    static PerContextOnce configured; // shared-memory opt-in, once per context
    cudaError_t e = configured.run([](int) {
        cudaError_t e = cudaSuccess;
        const void *fns[3] = {(const void *)decode_fp8_kernel<4>, (const void *)decode_fp8_kernel<2>,
                              (const void *)decode_fp8_kernel<1>};
        for (int i = 0; i < 3; ++i) {
            e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, d8::SMEM);
            if (e != cudaSuccess)
                return e;
        }
        return e;
    });
    if (e != cudaSuccess)
        return e;
    dim3 grid(p.splits, p.Hkv, p.B);
    if (p.MT == 1)
        decode_fp8_kernel<4><<<grid, d8::THREADS, d8::SMEM, stream>>>(p);
    else if (p.MT == 2)
        decode_fp8_kernel<2><<<grid, d8::THREADS, d8::SMEM, stream>>>(p);
    else
        decode_fp8_kernel<1><<<grid, d8::THREADS, d8::SMEM, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.splits == 1)
        return e;
    return launch_decode_merge(p, stream);
}

// Commit into an FP8 cache: as kv_commit_kernel (the same pieces, rotated / scaled first when
// the commit transforms), each 8-value bf16 piece quantised to 8 codes by the decode's rule for
// new tokens.
SA_DEV uint2 quant_piece(const uint4 &x, float scale)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        c[j] = quant_e4m3x2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u), scale);
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__global__ void __launch_bounds__(128) kv_commit_fp8_kernel(const __grid_constant__ CommitParams p)
{
    const int b = blockIdx.x;
    const CommitState cs = commit_state(p, b);
    uint8_t *k8 = reinterpret_cast<uint8_t *>(p.k_cache);
    uint8_t *v8 = reinterpret_cast<uint8_t *>(p.v_cache);
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
        uint8_t *row = pc.is_k ? k8 + kdst + (int64_t)gh * p.kc_sh : v8 + vdst + (int64_t)gh * p.vc_sh;
        const float scale = pc.is_k ? p.k_scale : p.v_scale;
        *reinterpret_cast<uint2 *>(row + pc.c0 * 8) = quant_piece(x0, scale);
        if (pc.c1 >= 0)
            *reinterpret_cast<uint2 *>(row + pc.c1 * 8) = quant_piece(x1, scale);
    }
    __syncthreads();
    if (threadIdx.x == 0)
        commit_advance(p, b, cs);
}

cudaError_t launch_commit_fp8(const CommitParams &p, cudaStream_t stream)
{
    kv_commit_fp8_kernel<<<p.B, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

} // namespace sinkattn
