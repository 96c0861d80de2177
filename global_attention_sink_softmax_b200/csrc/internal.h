// Internal host-side interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sinkattn {

// ---- prefill -------------------------------------------------------------------------------
struct PrefillParams {
    int B, L, Hq, Hkv, G; // L query rows per sequence
    int q_off;            // position of query row 0 (keys: q_off + L positions)
    int window;           // > 0 sliding window, 0 full causal
    int n_qtiles;         // ceil(L / 128)
    float scale_log2;     // scale * log2(e)
    const float *sink;    // [Hq] or nullptr
    void *o;              // bf16
    int64_t o_sb, o_sl, o_sh;
    float *lse;           // [B, Hq, L] or nullptr
    // paged prefix (paged != 0): keys at positions < q_off come from a page pool through
    // page_table [B, max_pages] (q_off and page_size multiples of 128); the K / V maps then hold
    // only the L positions of the chunk
    int paged;
    const int32_t *page_table;
    int page_size, max_pages, num_pages;
};

// Q map: dims {192, Hq, L, B}; K map: {192, Hkv, q_off + L, B}; V map: {128, Hkv, q_off + L, B}
// (paged: {.., L, B}); page maps {d, Hkv, page_size, num_pages} (the K / V maps again when not
// paged); 128-byte swizzle, 64-element inner box, 128-row boxes.
cudaError_t launch_prefill_band(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                const CUtensorMap &tmV, const CUtensorMap &tmKp,
                                const CUtensorMap &tmVp, const PrefillParams &p,
                                cudaStream_t stream);
// Full-causal prefill (window 0), same maps and parameters: two softmax warpgroups per CTA
// sharing 256-key tiles.
cudaError_t launch_prefill_wide(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                const CUtensorMap &tmV, const CUtensorMap &tmKp,
                                const CUtensorMap &tmVp, const PrefillParams &p,
                                cudaStream_t stream);

// SWA prefill, GQA-packed persistent kernel: item = (b, kv head, block of P = 128 / G positions)
// Partial RoPE applied to Q and K as they land in shared memory (rope_dim <= 64: the rotary
// dims lie in the first 64-dim region of a tile); the value scale multiplies O.
constexpr int kRopeFusedMaxHalf = 32;

struct SwaParams {
    int B, L, Hq, Hkv, G;
    int P;                // positions per item
    int W;                // window
    int NS;               // key span per item (multiple of 16, <= 256)
    int n_pblk, n_items;
    float scale_log2;
    const float *sink;
    void *o;
    int64_t o_sb, o_sl, o_sh;
    float *lse;
    // fused RoPE (rope = 0: Q, K, V taken as given): token l of sequence b at position
    // pos0 + pos_base[b] + l, pair i turning by position * inv_freq[i]
    int rope, rope_half;
    float out_mul; // the value scale (1 without RoPE)
    const int32_t *pos_base;
    int64_t pos0;
    double inv_freq[kRopeFusedMaxHalf];
};

// Q map box {64, G, P, 1}; K / V map box {64, 1, NS, 1}; K / V chunk map box {64, 1, 16, 1};
// grid = persistent CTAs. Specialised for NS = 144, P = 16 (G = 8, W <= 128).
cudaError_t launch_prefill_swa_packed(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                      const CUtensorMap &tmV, const CUtensorMap &tmKc,
                                      const CUtensorMap &tmVc, const SwaParams &p, int grid,
                                      cudaStream_t stream);
// Largest dynamic shared memory the packed SWA kernel may use on this device.
int swa_packed_smem_bytes(int ns, int P);

// ---- decode --------------------------------------------------------------------------------
struct DecodeParams {
    int kind, B, T, Hq, Hkv, G, R, MT;   // R = T * G rows per unit, MT = ceil(R / 16)
    int window;
    int splits, chunk;                  // key spans per (b, kv head) and keys per span
    float scale_log2;
    const float *sink;
    const uint16_t *q, *k_new, *v_new, *k_cache, *v_cache;
    int64_t q_sb, q_st, q_sh;
    int64_t kn_sb, kn_st, kn_sh, vn_sb, vn_st, vn_sh;
    int64_t kc_sb, kc_ss, kc_sh, vc_sb, vc_ss, vc_sh;
    const int32_t *ring_head, *ring_len;
    int ring_cap;
    const int32_t *ctx_len;
    int max_ctx;
    const int32_t *page_table;
    int page_size, max_pages, num_pages;
    uint16_t *o;
    int64_t o_sb, o_st, o_sh;
    float *lse;
    float *ws_o;    // [B, Hkv, splits, R, 128] (splits > 1)
    float *ws_ml;   // [B, Hkv, splits, R, 4]: max, sum of rounded P, sum of fp32 P, pad
    // FP8 (E4M3) cache: k8 / v8 are the caches as bytes (strides above count bytes); the new
    // tokens are quantised with k_scale / v_scale, scale_log2 includes k_scale and O is
    // multiplied by v_scale
    int fp8;
    float k_scale, v_scale;
    const uint8_t *k8, *v8;
};

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t stream);
// TMA-fed decode: cache maps {d, Hkv, rows, blocks} (rows = ring slots / positions / page rows,
// blocks = sequences or pages) and new-token maps {d, Hkv, T, B}, box {64, 1, 64, 1}.
cudaError_t launch_decode_tma(const CUtensorMap &kc, const CUtensorMap &vc, const CUtensorMap &kn,
                              const CUtensorMap &vn, const DecodeParams &p, cudaStream_t stream);
// tcgen05 decode (query blocks of 17..64 rows, and rings): q map {192, Hq, T, B} box
// {64, G, T, 1}, new-token maps with a 16-row box. max_ctas > 0 caps the grid (the CTAs then
// loop over the work items); 0 launches one CTA per item.
cudaError_t launch_decode_umma(const CUtensorMap &q, const CUtensorMap &kc, const CUtensorMap &vc,
                               const CUtensorMap &kn, const CUtensorMap &vn, const DecodeParams &p,
                               int max_ctas, cudaStream_t stream);
// Ring decode, one warp per (sequence, KV head, m16 row tile) item (one span): cache maps
// {d, Hkv, ring_cap, B} and new-token maps {d, Hkv, T, B}, box {64, 1, 32, 1}.
cudaError_t launch_decode_ring(const CUtensorMap &kc, const CUtensorMap &vc, const CUtensorMap &kn,
                               const CUtensorMap &vn, const DecodeParams &p, int sms,
                               cudaStream_t stream);
// Ring decode / verify on the tensor cores: 128-slot rings, G = 8, T <= 4; q map {192, Hq, T, B}
// box {64, 8, T, 1}, cache maps {d, Hkv, 128, B} box {64, 1, 128, 1}, new-token maps
// {d, Hkv, T, B} box {64, 1, 16, 1}. One CTA per SM (at most one per unit).
cudaError_t launch_decode_ring_umma(const CUtensorMap &q, const CUtensorMap &kc, const CUtensorMap &vc,
                                    const CUtensorMap &kn, const CUtensorMap &vn, const DecodeParams &p,
                                    int sms, cudaStream_t stream);
cudaError_t launch_decode_merge(const DecodeParams &p, cudaStream_t stream);
int decode_stages(const DecodeParams &p);

// Fused partial RoPE + value scale: rope_dim <= 2 * kRopeMaxHalf.
constexpr int kRopeMaxHalf = 64; // rope_dim <= 128

struct CommitParams {
    int kind, B, T, Hkv;
    const uint16_t *k_new, *v_new;
    int64_t kn_sb, kn_st, kn_sh, vn_sb, vn_st, vn_sh;
    uint16_t *k_cache, *v_cache;
    int64_t kc_sb, kc_ss, kc_sh, vc_sb, vc_ss, vc_sh;
    int32_t *ring_head, *ring_len;
    int ring_cap;
    int32_t *ctx_len;
    int max_ctx;
    const int32_t *page_table;
    int page_size, max_pages, num_pages;
    const int32_t *n_accept;
    int fp8;               // quantise into an E4M3 cache (strides count bytes)
    float k_scale, v_scale;
    // RoPE + value scale as the tokens are stored (rope_half = 0: store as given): pair i of the
    // first rope_half dims turns at inv_freq[i] with position pos[b] + u (pos null: the cache's
    // own count), V is multiplied by v_mul; an FP8 cache stores the codes of the results
    int rope_half;
    float v_mul;
    const int32_t *pos;
    double inv_freq[kRopeMaxHalf];
};

cudaError_t launch_commit(const CommitParams &p, cudaStream_t stream);
cudaError_t launch_decode_fp8(const DecodeParams &p, cudaStream_t stream);
// FP8-cache decode fed by TMA: code maps {d, Hkv, rows, blocks} over uint8, box {64, 1, 64, 1},
// 64-byte swizzle.
cudaError_t launch_decode_fp8_tma(const CUtensorMap &kc, const CUtensorMap &vc,
                                  const DecodeParams &p, cudaStream_t stream);
cudaError_t launch_commit_fp8(const CommitParams &p, cudaStream_t stream);

// Fused partial RoPE + value scale, in place (rope_kernels.cuh).
struct RopeParams {
    uint16_t *q, *k, *v; // any may be null (skipped)
    const int32_t *pos_base;
    int64_t pos0;
    int B, L, Hq, Hkv, half, dv;
    float v_scale;
    int64_t q_sb, q_sl, q_sh, k_sb, k_sl, k_sh, v_sb, v_sl, v_sh;
    double inv_freq[kRopeMaxHalf]; // w_i = theta^(-2i/rope_dim)
};

cudaError_t launch_rope_qkv(const RopeParams &p, cudaStream_t stream);

// ---- prefill backward ------------------------------------------------------------------------
struct BwdParams {
    int B, L, Hq, Hkv, G, window;
    float scale, scale_log2;
    const uint16_t *o, *dout;
    int64_t o_sb, o_sl, o_sh, do_sb, do_sl, do_sh;
    const float *lse, *sink;
    float *delta; // [B, Hq, L]
    float *dq, *dk, *dv, *dsink;
    int64_t dq_sb, dq_sl, dq_sh, dk_sb, dk_sl, dk_sh, dv_sb, dv_sl, dv_sh;
};

// delta and dsink (dsink, when given, must hold zeros on entry)
cudaError_t launch_bwd_delta(const BwdParams &p, cudaStream_t stream);
// q / do maps {d, Hq, L, B}, k / v maps {d, Hkv, L, B}; boxes of 64 rows (dK/dV: q, do) or
// 128 rows (dK/dV: k, v; dQ: all four)
cudaError_t launch_bwd_dkdv(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                            const CUtensorMap &dout, const BwdParams &p, cudaStream_t stream);
cudaError_t launch_bwd_dq(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                          const CUtensorMap &dout, const BwdParams &p, cudaStream_t stream);

cudaError_t read_and_clear_device_error(uint32_t *flag);
cudaError_t set_wait_limit(uint64_t ns);

} // namespace sinkattn
