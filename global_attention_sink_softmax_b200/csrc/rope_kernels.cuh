// Partial rotary position embedding and the value scale, fused into one in-place pass over
// Q, K and V: the steps the attention module runs between the Q/K/V projection and the
// attention core ("MiMo-V2-Flash 模型架构深度拆解" CH10.3: value_states * v_scale (0.707), split
// Q/K into 64 rotary | 128 no-pe dims, rotate the first 64, concatenate).
//
// Rotation ("MiMo-V2-Flash 模型架构深度拆解" CH3.5, CH8.1, CH10.5; "MiMo-V2-Flash 架构 QA" Q2.7): at
// position m, dimension pair i (0 <= i < rope_dim/2) turns by m * w_i with
// w_i = theta^(-2i/rope_dim) (theta 5e6 on GA layers, 1e4 on SWA layers); the pair is dims
// (i, i + rope_dim/2):
//     y_i              = x_i cos - x_{i+rope_dim/2} sin
//     y_{i+rope_dim/2} = x_{i+rope_dim/2} cos + x_i sin
// Dims rope_dim .. d-1 are not touched (not even read). V is multiplied by v_scale.
//
// Precision (rope_cos_sin, rope_rotate8 in common.cuh): the angle m * w_i is formed in fp64 (w_i
// from the host in fp64) and range-reduced in fp64 before sincosf; the rotation runs in fp32 and
// each result is rounded once to bf16 (nearest even).
//
// Work split: a CTA takes TOK tokens. Its threads first compute (cos, sin) for every
// (token, pair) into shared memory (the angle depends on the token only, so one value serves
// all Hq + Hkv heads), then stream 32-byte units: for a Q or K head, 8 pairs (16 bytes from
// each half of its rotary part); for a V head, 16 consecutive values. The pass is HBM-bound:
// it reads and writes exactly the rotary part of every Q/K head and all of V.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace sinkattn {

namespace rp {
constexpr int THREADS = 256;
constexpr int TOK = 8; // tokens per CTA
} // namespace rp

// One unit of work: where its two 16-byte pieces live and what to do with them.
struct RopeUnit {
    uint4 *p0, *p1;
    int pair0;  // first pair index (rotation), or -1 for a value unit, -2 for none
};

__device__ __forceinline__ RopeUnit rope_unit(const RopeParams &p, int64_t t0, int ntk,
                                              int per_tok, int q_units, int k_units, int e)
{
    RopeUnit r;
    r.pair0 = -2;
    r.p0 = r.p1 = nullptr;
    if (e >= ntk * per_tok)
        return r;
    const int tt = e / per_tok;
    int u = e - tt * per_tok;
    const int64_t t = t0 + tt;
    const int b = (int)(t / p.L);
    const int l = (int)(t - (int64_t)b * p.L);
    const int nc = p.half >> 3; // 16-byte chunks per half of the rotary part
    if (u < q_units + k_units) {
        uint16_t *row;
        int c;
        if (u < q_units) {
            const int h = u / nc;
            c = u - h * nc;
            row = p.q + (int64_t)b * p.q_sb + (int64_t)l * p.q_sl + (int64_t)h * p.q_sh;
        } else {
            u -= q_units;
            const int g = u / nc;
            c = u - g * nc;
            row = p.k + (int64_t)b * p.k_sb + (int64_t)l * p.k_sl + (int64_t)g * p.k_sh;
        }
        r.p0 = reinterpret_cast<uint4 *>(row + c * 8);
        r.p1 = reinterpret_cast<uint4 *>(row + p.half + c * 8);
        r.pair0 = tt * p.half + c * 8; // index into the (cos, sin) table
    } else {
        u -= q_units + k_units;
        const int nv = p.dv >> 4; // 16-value units per V head
        const int g = u / nv;
        const int c = u - g * nv;
        uint16_t *row = p.v + (int64_t)b * p.v_sb + (int64_t)l * p.v_sl + (int64_t)g * p.v_sh;
        r.p0 = reinterpret_cast<uint4 *>(row + c * 16);
        r.p1 = r.p0 + 1;
        r.pair0 = -1;
    }
    return r;
}

__device__ __forceinline__ void rope_apply(const RopeUnit &r, uint4 a, uint4 b,
                                           const float2 *cs, float v_scale)
{
    if (r.pair0 == -2)
        return;
    if (r.pair0 >= 0) {
        rope_rotate8(a, b, cs + r.pair0); // pairs pair0 .. pair0 + 7: first half in a
    } else {
        scale8(a, v_scale);
        scale8(b, v_scale);
    }
    *r.p0 = a;
    *r.p1 = b;
}

__global__ void __launch_bounds__(rp::THREADS) rope_qkv_kernel(const __grid_constant__ RopeParams p)
{
    using namespace rp;
    __shared__ float2 cs[TOK * kRopeMaxHalf]; // (cos, sin) of token tt, pair i at tt * half + i
    const int nc = p.half >> 3;
    const int q_units = p.q ? p.Hq * nc : 0;
    const int k_units = p.k ? p.Hkv * nc : 0;
    const int v_units = p.v ? p.Hkv * (p.dv >> 4) : 0;
    const int per_tok = q_units + k_units + v_units;
    const int64_t ntok = (int64_t)p.B * p.L;
    const int64_t t0 = (int64_t)blockIdx.x * TOK;
    const int ntk = (int)min((int64_t)TOK, ntok - t0);

    if (q_units + k_units > 0) {
        for (int e = threadIdx.x; e < ntk * p.half; e += THREADS) {
            const int tt = e / p.half, i = e - tt * p.half;
            const int64_t t = t0 + tt;
            const int b = (int)(t / p.L);
            const int l = (int)(t - (int64_t)b * p.L);
            const int64_t m = p.pos0 + (p.pos_base ? (int64_t)p.pos_base[b] : 0) + l;
            cs[e] = rope_cos_sin(m, p.inv_freq[i]);
        }
        __syncthreads();
    }
    // two units per thread per round, both loads in flight before either is used
    for (int e = threadIdx.x; e < ntk * per_tok; e += 2 * THREADS) {
        const RopeUnit u0 = rope_unit(p, t0, ntk, per_tok, q_units, k_units, e);
        const RopeUnit u1 = rope_unit(p, t0, ntk, per_tok, q_units, k_units, e + THREADS);
        const uint4 a0 = *u0.p0, b0 = *u0.p1;
        uint4 a1 = make_uint4(0, 0, 0, 0), b1 = a1;
        if (u1.pair0 != -2) {
            a1 = *u1.p0;
            b1 = *u1.p1;
        }
        rope_apply(u0, a0, b0, cs, p.v_scale);
        rope_apply(u1, a1, b1, cs, p.v_scale);
    }
}

cudaError_t launch_rope_qkv(const RopeParams &p, cudaStream_t stream)
{
    const int64_t ntok = (int64_t)p.B * p.L;
    const int64_t blocks = (ntok + rp::TOK - 1) / rp::TOK;
    if (blocks <= 0)
        return cudaSuccess;
    if (blocks > 0x7fffffff)
        return cudaErrorInvalidConfiguration;
    rope_qkv_kernel<<<(unsigned)blocks, rp::THREADS, 0, stream>>>(p);
    return cudaGetLastError();
}

} // namespace sinkattn
