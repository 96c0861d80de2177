/*
 * sinkattn.h — causal grouped-query softmax attention with a per-head sink, for NVIDIA B200
 * (sm_100a). Plain C ABI: pointers, sizes and element strides; no C++ or framework types.
 *
 * What is computed. For query position i of head h (KV head g = h / (Hq / Hkv)) and the set
 * J(i) of keys it may see:
 *
 *     a_ij = scale * <q_i, k_j>
 *     m_i  = max(sink_h, max_{j in J(i)} a_ij)
 *     D_i  = exp(sink_h - m_i) + sum_{j in J(i)} exp(a_ij - m_i)
 *     O_i  = sum_{j in J(i)} exp(a_ij - m_i) v_j / D_i
 *     LSE_i = m_i + ln D_i
 *
 * The sink adds exp(sink_h - m_i) to the denominator and contributes no value. Sources:
 * "MiMo-V2-Flash 架构 QA" Q3.7 (the max includes the sink) and Q3.8 (the formula and its
 * concat -> softmax -> drop equivalent); "MiMo-V2-Flash 模型架构深度拆解" CH3.2 (a_ij = q k^T
 * / sqrt(d)), CH10.1 (one fp32 sink per query head, appended after scaling and masking),
 * CH10.3 (scaling head_dim^-0.5; GA causal mask, SWA "only the latest 128 tokens");
 * "MiMo-V2-Flash Technical Report" paper notes §4.1, §4.3 (128 keys in the W = 128 window).
 *
 * Visible keys J(i): global attention (GA) keeps j <= i; sliding-window attention (SWA) with
 * window W keeps i - W < j <= i (exactly W keys once i >= W - 1, the query included).
 *
 * Conventions shared by every entry point.
 *   - Element types: q, k, v, o and the caches are bf16 (a decode cache may instead hold
 *     one-byte FP8 codes: see sinkattn_kv_dtype); sink and lse are fp32.
 *   - Layouts are token-major, [batch, token, head, dim], the dim contiguous; the other
 *     three dims are given as element strides (int64). Base pointers and every non-unit
 *     stride in bytes must be multiples of 16.
 *   - Head dims: dq = 192 and dv = 128 for attention and commit (the kernels are specialised
 *     for them); sinkattn_rope_qkv states its own limits.
 *     GQA group G = Hq / Hkv must be an integer; decode and commit take G in 1..16 with
 *     T * G <= 64 query rows per KV head, prefill any G.
 *   - sink: fp32 [Hq] in post-scale logit units (not multiplied by scale). NULL means no sink
 *     for any head; an entry of -inf means plain softmax for that head. NaN or +inf entries
 *     give unspecified results (not checked).
 *   - lse: natural log of the full denominator, sink included, so O = sum exp(a - LSE) v.
 *     May be NULL.
 *   - scale: finite and > 0 (1/sqrt(192) for the pages' model).
 *   - Ownership: the caller allocates and owns every buffer, host- and device-side. The
 *     library allocates nothing at run time and keeps no state between calls in the caller's
 *     memory; decode scratch is a caller workspace. Its only device state is process-wide and
 *     lives in the library's own module: the wait-timeout flag read by
 *     sinkattn_take_device_error, and the fixed scratch array of sinkattn_decode_noalloc. All
 *     device pointers must be device memory of the current device.
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream). Work is enqueued on
 *     it; nothing synchronises the host. Returns after the launch.
 *   - Errors: every entry point returns a sinkattn_status. Arguments are validated on the host
 *     before anything is enqueued; an invalid call enqueues nothing. SINKATTN_ERR_CUDA reports
 *     a launch failure (cudaGetLastError); faults during execution surface at the caller's next
 *     synchronisation. A kernel that ever waits longer than about a second on an internal
 *     barrier gives up, records it in a device flag and returns; sinkattn_take_device_error()
 *     reads and clears that flag.
 *   - Empty work (B == 0, L == 0, T == 0) is valid and enqueues nothing.
 */
#ifndef SINKATTN_H
#define SINKATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SINKATTN_VERSION 1

typedef enum sinkattn_status {
    SINKATTN_OK = 0,
    SINKATTN_ERR_INVALID_ARG = 1,          /* NULL pointer, negative size, bad stride */
    SINKATTN_ERR_UNSUPPORTED = 2,          /* head dims != 192/128, G out of range, T > 4 ... */
    SINKATTN_ERR_ALIGNMENT = 3,            /* pointer or stride not 16-byte aligned */
    SINKATTN_ERR_WORKSPACE_TOO_SMALL = 4,  /* decode workspace below the size query */
    SINKATTN_ERR_CUDA = 5                  /* a CUDA runtime call failed */
} sinkattn_status;

/* KV-cache layouts accepted by decode and commit. */
typedef enum sinkattn_kv_kind {
    SINKATTN_KV_RING = 0,    /* per-sequence ring of ring_cap slots (SWA) */
    SINKATTN_KV_CONTIG = 1,  /* per-sequence contiguous cache of max_ctx rows (GA) */
    SINKATTN_KV_PAGED = 2    /* page pool + per-sequence page table (GA) */
} sinkattn_kv_kind;

/* Element type of a KV cache (decode and commit). The new tokens' k_new / v_new are bf16 with
 * either. FP8 reading: the pages size a KV slot at one byte ("MiMo-V2-Flash Technical Report"
 * paper notes, KV-memory arithmetic) and speak of FP8 inference, naming no format; the library
 * stores E4M3 ("fn": bias 7, no infinities, largest finite 448) codes with one fp32 scale per
 * cache tensor, a code c meaning e4m3(c) * scale. */
typedef enum sinkattn_kv_dtype {
    SINKATTN_KV_BF16 = 0,     /* bf16 elements (the default of a zero-initialised struct) */
    SINKATTN_KV_FP8_E4M3 = 1  /* one-byte E4M3 codes, scaled by k_scale / v_scale */
} sinkattn_kv_dtype;

/* ---------------------------------------------------------------------------------------------
 * Prefill: every position of every sequence attends to its own sequence.
 *
 *   q   [B, L, Hq,  192]  strides q_sb, q_sl, q_sh   (read)
 *   k   [B, L, Hkv, 192]  strides k_sb, k_sl, k_sh   (read)
 *   v   [B, L, Hkv, 128]  strides v_sb, v_sl, v_sh   (read)
 *   o   [B, L, Hq,  128]  strides o_sb, o_sl, o_sh   (written; bf16, round-to-nearest-even)
 *   lse [B, Hq, L] fp32, contiguous (written; may be NULL)
 * ------------------------------------------------------------------------------------------- */
typedef struct sinkattn_prefill_args {
    const void *q;
    const void *k;
    const void *v;
    const float *sink;
    void *o;
    float *lse;
    int32_t B, L, Hq, Hkv, dq, dv;
    float scale;
    int64_t q_sb, q_sl, q_sh;
    int64_t k_sb, k_sl, k_sh;
    int64_t v_sb, v_sl, v_sh;
    int64_t o_sb, o_sl, o_sh;
} sinkattn_prefill_args;

/* Sliding-window prefill (SWA), window >= 1 keys (the pages' model uses 128). Keys outside the
 * window are never loaded: a W = 128 row touches at most two 128-key chunks ("MiMo-V2-Flash 架构
 * QA" Q3.6). */
int sinkattn_prefill_swa(const sinkattn_prefill_args *args, int32_t window, void *stream);

/* Global (full causal) prefill (GA): every position sees itself and all earlier positions
 * ("MiMo-V2-Flash 模型架构深度拆解" CH10.3, the GA layers' causal mask; CH10.1, the GA layers'
 * sink is optional and off in the model's config, so a NULL or -inf sink gives plain causal
 * softmax). Key tiles above the diagonal are skipped. */
int sinkattn_prefill_ga(const sinkattn_prefill_args *args, void *stream);

/* Chunked prefill against cached keys: a long prompt prefilled in chunks (the serving command of
 * the "MiMo-V2-Flash" model card, --chunked-prefill-size 16384), or a new turn after a cached
 * prefix ("MiMo-V2-Flash 模型架构深度拆解" §7.4, request-level prefix cache).
 *   args->q, o, lse: the L query rows, at positions prefix .. prefix + L - 1 of their sequences
 *                    ([B, L, Hq, ...] and lse [B, Hq, L], as for whole sequences);
 *   args->k, v:      all prefix + L positions of the sequences (the cached prefix followed by
 *                    the chunk's own keys), [B, prefix + L, Hkv, ...] with args' k / v strides;
 *   prefix >= 0;     window = 0: full causal (GA), window >= 1: sliding window (SWA).
 * The result equals rows prefix .. prefix + L - 1 of the whole-sequence prefill.
 * Errors: as for the whole-sequence calls; prefix < 0 or window < 0 is INVALID_ARG. */
int sinkattn_prefill_chunk(const sinkattn_prefill_args *args, int32_t prefix, int32_t window,
                           void *stream);

/* The cached prefix of a chunked prefill in a paged KV pool (the serving stack of the
 * "MiMo-V2-Flash" model card pages its KV cache): position c < prefix of sequence b is row
 * c mod page_size of page page_table[b * max_pages + c / page_size].
 *   k_pages [num_pages, page_size, Hkv, 192], v_pages [num_pages, page_size, Hkv, 128]: bf16,
 *       strides kp_sb / vp_sb (between pages), kp_ss / vp_ss (rows), kp_sh / vp_sh (heads);
 *   page_table: device int32 [B, max_pages]; every page the prefix uses must be mapped (an id
 *       outside [0, num_pages) reads as zero keys and values). */
typedef struct sinkattn_paged_kv {
    const void *k_pages;
    const void *v_pages;
    int64_t kp_sb, kp_ss, kp_sh;
    int64_t vp_sb, vp_ss, vp_sh;
    const int32_t *page_table;
    int32_t page_size, max_pages, num_pages;
} sinkattn_paged_kv;

/* Chunked prefill against a paged prefix: as sinkattn_prefill_chunk, but args->k / v hold only
 * the chunk's own L positions ([B, L, Hkv, ...]) and positions 0 .. prefix - 1 come from
 * `prefix_kv`. prefix and page_size must be multiples of 128 (whole 128-key tiles come from one
 * page, or from the chunk), and prefix <= max_pages * page_size.
 * Errors: as sinkattn_prefill_chunk; UNSUPPORTED for prefix or page_size not multiples of 128;
 * INVALID_ARG for a NULL prefix_kv or page table, non-positive page geometry or strides. */
int sinkattn_prefill_chunk_paged(const sinkattn_prefill_args *args,
                                 const sinkattn_paged_kv *prefix_kv, int32_t prefix,
                                 int32_t window, void *stream);

/* Prefill with the inputs and outputs in HOST memory (a prompt that arrives from the host and
 * whose O and LSE go back to it; the "MiMo-V2-Flash" model card's serving command prefills
 * prompts in chunks, --chunked-prefill-size 16384). The sequences pass through the device in
 * chunks of `chunk` positions: while chunk c is computed, chunk c + 1 is copied in and chunk
 * c - 1 copied out, on two internal streams, so both PCIe directions and the kernels overlap.
 * Each chunk is the chunked prefill of its rows against every earlier key (window = 0: full
 * causal, GA; window >= 1: sliding window, SWA), so the result equals sinkattn_prefill_swa / _ga
 * on the whole sequences.
 *   args->q, k, v:   HOST, dense [B, L, H, d] (the strides in args must say so), read;
 *   args->o, lse:    HOST, dense o [B, L, Hq, 128] and lse [B, Hq, L] (lse may be NULL), written;
 *   args->sink:      DEVICE fp32 [Hq] or NULL, as for the device calls;
 *   chunk:           positions per chunk, a multiple of 128;
 *   workspace:       DEVICE memory of sinkattn_prefill_host_workspace_size(args, chunk) bytes
 *                    (K and V of all positions, two chunks of Q, O and LSE), owned by the caller.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister): pageable memory works
 * but its copies do not overlap. The call returns once the work is queued; the outputs are
 * complete when `stream` reaches the end of this call's work (e.g. after cudaStreamSynchronize).
 * The two copy streams and their events are created and released by each call.
 * Errors: as sinkattn_prefill_swa; UNSUPPORTED for non-dense strides or a chunk that is not a
 * multiple of 128; INVALID_ARG for a NULL workspace, chunk <= 0 or window < 0;
 * WORKSPACE_TOO_SMALL below the size query. The size query returns 0 for invalid arguments. */
size_t sinkattn_prefill_host_workspace_size(const sinkattn_prefill_args *args, int32_t chunk);
int sinkattn_prefill_host(const sinkattn_prefill_args *args, int32_t window, int32_t chunk,
                          void *workspace, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Decode / speculative verify: T (1..4) new query tokens per sequence attend to that sequence's
 * cached tokens plus new tokens 0..t. The new tokens' K/V are passed separately and are NOT yet
 * in the cache (sinkattn_kv_commit appends the accepted ones afterwards).
 *
 * Positions: cached token c (0 = oldest of n_b) sits at c - n_b, new token u at u; new query t
 * sees keys at positions p <= t, and, when window > 0, p > t - window. For T = 1 and a full
 * ring this equals "write the new token into the ring, then attend over all its slots".
 *
 *   q     [B, T, Hq, 192]   strides q_sb, q_st, q_sh
 *   k_new [B, T, Hkv, 192], v_new [B, T, Hkv, 128]  strides kn_*, vn_*
 *   RING:   k_cache [B, ring_cap, Hkv, 192], v_cache [B, ring_cap, Hkv, 128];
 *           ring_head[B] = slot of the oldest cached token, ring_len[B] = tokens held
 *           (0..ring_cap); cached token c is in slot (ring_head + c) mod ring_cap.
 *   CONTIG: k_cache [B, max_ctx, Hkv, 192] ...; ctx_len[B] (0..max_ctx) tokens held.
 *   PAGED:  k_cache [num_pages, page_size, Hkv, 192] ...; cached token c of sequence b is row
 *           c mod page_size of page page_table[b * max_pages + c / page_size]; ctx_len[B]
 *           (0..max_ctx, max_ctx <= max_pages * page_size). Page ids outside [0, num_pages)
 *           make that page's keys invisible (no out-of-bounds read).
 *   ring_head, ring_len, ctx_len, page_table: int32 device arrays. max_ctx is a host-side
 *   upper bound on ctx_len (entries above it are clamped to it).
 *   o [B, T, Hq, 128] strides o_sb, o_st, o_sh;  lse [B, T, Hq] fp32 contiguous (may be NULL).
 *   cache strides: kc_sb = stride between sequences (RING, CONTIG) or pages (PAGED),
 *                  kc_ss = stride between slots / tokens / page rows, kc_sh = between heads.
 * ------------------------------------------------------------------------------------------- */
typedef struct sinkattn_decode_args {
    int32_t kind; /* sinkattn_kv_kind */
    int32_t B, T, Hq, Hkv, dq, dv;
    int32_t window; /* > 0: sliding window of `window` keys; 0: full causal (GA) */
    float scale;
    const float *sink;
    const void *q;
    int64_t q_sb, q_st, q_sh;
    const void *k_new;
    int64_t kn_sb, kn_st, kn_sh;
    const void *v_new;
    int64_t vn_sb, vn_st, vn_sh;
    const void *k_cache;
    int64_t kc_sb, kc_ss, kc_sh;
    const void *v_cache;
    int64_t vc_sb, vc_ss, vc_sh;
    const int32_t *ring_head;
    const int32_t *ring_len;
    int32_t ring_cap;
    const int32_t *ctx_len;
    int32_t max_ctx;
    const int32_t *page_table;
    int32_t page_size, max_pages, num_pages;
    void *o;
    int64_t o_sb, o_st, o_sh;
    float *lse;
    /* Cache element type (sinkattn_kv_dtype). With SINKATTN_KV_FP8_E4M3, k_cache / v_cache hold
     * one-byte codes in the same [.., Hkv, d] layouts, their strides count bytes and must be
     * multiples of 16, and a K (V) code c stands for e4m3(c) * k_scale (v_scale); both scales
     * must be finite and > 0. Decode then attends to the T new tokens as the commit will store
     * them: each new K / V element x becomes the E4M3 value nearest to x / scale (the division
     * in fp32, ties to even, saturating to +-448). Q is rounded to fp16 for the tensor cores, so
     * |q| must stay below 65504 on this path. */
    int32_t kv_dtype;
    float k_scale, v_scale;
    /* sinkattn_kv_commit only (decode ignores them). With commit_rope = 1 the commit applies the
     * two steps that precede attention ("MiMo-V2-Flash 模型架构深度拆解" CH10.3) as it stores each
     * accepted token, exactly as sinkattn_rope_qkv would: K's first rope_dim dims get the partial
     * rotary embedding with rope_theta at the token's absolute position, and V is multiplied by
     * commit_v_scale (0.707 for the pages' model). Accepted token u of sequence b sits at
     * position commit_pos[b] + u; commit_pos may be NULL for CONTIG and PAGED caches, where it
     * defaults to ctx_len[b] before the commit, and must be given for a RING (whose length stops
     * at ring_cap). An FP8 cache stores the codes of the rotated / scaled bf16 values.
     * commit_rope = 0 (a zero-initialised struct) stores k_new / v_new as given. */
    int32_t commit_rope;
    int32_t rope_dim;          /* a multiple of 16 in 16..128 (64 for the pages' model) */
    double rope_theta;         /* > 0 and finite: 5e6 on GA layers, 1e4 on SWA layers */
    float commit_v_scale;      /* finite */
    const int32_t *commit_pos; /* device int32 [B] or NULL */
} sinkattn_decode_args;

/* Bytes of device workspace sinkattn_decode needs for these arguments. The pages give no
 * decode algorithm, only its setting: contexts of up to 256K tokens, where decode time goes to
 * reading the KV cache ("MiMo-V2-Flash Technical Report" paper notes §1.1). A long GA context is
 * therefore split into key spans read in parallel, whose sink-free partials the merge described
 * at sinkattn_decode combines; this is the room those partials take (split-KV partials:
 * per split and query row, an unnormalised fp32 O row, its running max and two running sums,
 * one over the bf16-rounded P that multiplied V and one over fp32 P). 0 when no split is
 * needed. Depends only on kind, B, T, Hq, Hkv, dq, dv, window, ring_cap / max_ctx and the page
 * geometry; pointers and strides are not read. Returns 0 for invalid sizes too;
 * sinkattn_decode reports those. */
size_t sinkattn_decode_workspace_size(const sinkattn_decode_args *args);

/* Split-KV decode: each (sequence, KV head, key span) block computes sink-free partials; the
 * merge counts the sink exactly once: m = max(sink, max_p m_p), D = exp(sink - m) +
 * sum_p l_p exp(m_p - m), O = sum_p O_p exp(m_p - m) / D, LSE = m + ln D (derived from
 * "MiMo-V2-Flash 架构 QA" Q3.8). `workspace` is caller-owned device memory of at least
 * sinkattn_decode_workspace_size(args) bytes, 16-byte aligned (may be NULL when that is 0);
 * its contents on entry do not matter. */
int sinkattn_decode(const sinkattn_decode_args *args, void *workspace, size_t workspace_bytes,
                    void *stream);

/* Largest split-KV workspace sinkattn_decode_noalloc can provide: 16 MiB. */
#define SINKATTN_NOALLOC_WORKSPACE_BYTES (16u << 20)

/* Decode that allocates nothing and takes no workspace. The pages have no counterpart: this is
 * a service of the library, not part of the method.
 *
 * For callers that cannot allocate device memory and have no workspace to lend: a plugin host
 * that passes the library only its input and output buffers, or a serving loop whose device
 * memory is reserved up front, where a cudaMalloc on the decode path would block the device or
 * fail under memory pressure. It computes exactly what sinkattn_decode computes, with the
 * split-KV partials kept in a fixed array in the library's own device memory
 * (SINKATTN_NOALLOC_WORKSPACE_BYTES; every GPU that loads the library holds it until the process
 * exits).
 *   - Arguments, outputs and errors as for sinkattn_decode. Calls whose
 *     sinkattn_decode_workspace_size exceeds SINKATTN_NOALLOC_WORKSPACE_BYTES are rejected with
 *     SINKATTN_ERR_WORKSPACE_TOO_SMALL before anything is enqueued (e.g. B * Hkv * T * G * spans
 *     * 528 bytes above 16 MiB); use sinkattn_decode with a caller workspace for those.
 *   - The first call on a device that needs the array looks up its device address
 *     (cudaGetSymbolAddress) with that device current and remembers it; make that first call
 *     before any stream capture.
 *   - Each device has its own copy of the array; all calls on that device share it, and it
 *     keeps the last call's contents (nothing in it needs to start at zero). Calls that overlap
 *     on the GPU, for example on two streams of one device, race on it: serialise them. */
int sinkattn_decode_noalloc(const sinkattn_decode_args *args, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Commit accepted tokens to the cache (the attention module's "KV cache update" step,
 * "MiMo-V2-Flash 模型架构深度拆解" CH10.3). For each sequence b the first n_accept[b] (0..T)
 * of its T new tokens are appended oldest first:
 *   RING:   token goes to slot (ring_head + ring_len) mod ring_cap; ring_len grows to at most
 *           ring_cap, after which each new token replaces the oldest and ring_head advances.
 *   CONTIG: row ctx_len[b] + u (tokens beyond max_ctx are dropped); ctx_len grows.
 *   PAGED:  position ctx_len[b] + u through the page table (positions beyond
 *           max_pages * page_size are dropped); ctx_len grows.
 * Uses the cache, metadata, *_new and commit_* fields of `args` (q, o, lse, sink are ignored).
 * Updates k_cache, v_cache, ring_head / ring_len or ctx_len in place, in stream order. With
 * commit_rope = 1 the stored K / V are rotated and scaled first (see sinkattn_decode_args); the
 * caller's k_new / v_new are not modified. Errors: INVALID_ARG also for commit_rope not 0 / 1,
 * rope_theta <= 0 or not finite, commit_v_scale not finite, a RING without commit_pos;
 * UNSUPPORTED for rope_dim out of range.
 * ------------------------------------------------------------------------------------------- */
int sinkattn_kv_commit(const sinkattn_decode_args *args, const int32_t *n_accept, void *stream);


/* ---------------------------------------------------------------------------------------------
 * Partial rotary position embedding and the value scale, fused into one in-place pass: the
 * steps the attention module runs between the Q/K/V projection and attention ("MiMo-V2-Flash
 * 模型架构深度拆解" CH10.3: V times v_scale = 0.707, then RoPE on the first 64 of the 192 Q/K
 * dims; CH3.5 and CH8.1: partial_rotary_factor 0.334, rope_theta 5,000,000 on GA layers and
 * swa_rope_theta 10,000 on SWA layers; "MiMo-V2-Flash 架构 QA" Q2.7: angle m * theta^(-2i/d)).
 *
 * Token l of sequence b sits at position m = pos0 + pos_base[b] + l (pos_base NULL: 0), so a
 * whole prompt uses pos0 = 0, a chunk after P cached tokens pos0 = P, and decode's new tokens
 * pos_base = the tokens each sequence has seen. Dimension pair i (0 <= i < rope_dim/2) of
 * every Q and K head is dims (i, i + rope_dim/2) and turns by m * theta^(-2i/rope_dim):
 *     y_i = x_i cos - x_{i+rope_dim/2} sin,   y_{i+rope_dim/2} = x_{i+rope_dim/2} cos + x_i sin
 * (the pages leave the pairing open; this is the "rotate half" arrangement). Dims rope_dim..dq-1
 * are neither read nor written. Every V element is multiplied by v_scale. Results are rounded
 * once to bf16 (nearest even); angles are reduced in fp64, so large positions stay exact.
 *
 *   q [B, L, Hq, dq], k [B, L, Hkv, dq], v [B, L, Hkv, dv]: bf16, modified in place; any of the
 *       three may be NULL (skipped). Strides as for prefill; rows must not overlap.
 *   pos_base: device int32 [B] or NULL.
 *   rope_dim: a multiple of 16 in 16..128, <= dq (64 for the pages' model); dq a multiple of 8;
 *   dv a multiple of 16.  theta > 0 and finite; v_scale finite.
 * Errors: INVALID_ARG (negative sizes, theta <= 0, non-finite values, non-positive strides,
 * Hq / Hkv <= 0 for a given tensor), UNSUPPORTED (rope_dim / dq / dv out of range), ALIGNMENT.
 * ------------------------------------------------------------------------------------------- */
typedef struct sinkattn_rope_args {
    void *q;
    void *k;
    void *v;
    const int32_t *pos_base;
    int64_t pos0;
    int32_t B, L, Hq, Hkv, dq, dv, rope_dim;
    double theta;
    float v_scale;
    int64_t q_sb, q_sl, q_sh;
    int64_t k_sb, k_sl, k_sh;
    int64_t v_sb, v_sl, v_sh;
} sinkattn_rope_args;

int sinkattn_rope_qkv(const sinkattn_rope_args *args, void *stream);

/* Sliding-window prefill with the partial RoPE and the value scale fused into its loads: the
 * result of sinkattn_rope_qkv (same positions, rope_dim, theta and v_scale) over the sequences'
 * Q, K and V followed by sinkattn_prefill_swa, without that pass's round trip through HBM and
 * without modifying q, k, v ("MiMo-V2-Flash 模型架构深度拆解" CH10.3: V times v_scale, then RoPE
 * on the rotary part of Q and K, then attention). Each Q tile and each new K chunk is rotated in
 * shared memory as it lands, exactly as the pass rotates it (fp64-reduced angle, fp32 rotation,
 * one bf16 rounding); the value scale multiplies O instead of V (the same value in exact
 * arithmetic; bf16 rounding of v_scale * V is not reproduced).
 *   args, window: as for sinkattn_prefill_swa; token l of sequence b sits at position
 *       pos0 + pos_base[b] + l;
 *   rope_dim: a multiple of 16 in 16..64 (the rotary dims lie in the first 64 of the 192);
 *       theta > 0 and finite; v_scale finite.
 * The fused path is the GQA-packed kernel's (G = 8 query heads per KV head, window <= 128, the
 * pages' SWA layers); other shapes return UNSUPPORTED (use sinkattn_rope_qkv, then the prefill).
 * Errors: as sinkattn_prefill_swa; INVALID_ARG for window < 1, a NULL spec, theta <= 0 or
 * non-finite values; UNSUPPORTED for rope_dim out of range or a shape the fused path does not
 * take. */
typedef struct sinkattn_rope_spec {
    const int32_t *pos_base; /* device int32 [B] or NULL */
    int64_t pos0;
    int32_t rope_dim;
    double theta;
    float v_scale;
} sinkattn_rope_spec;

int sinkattn_prefill_swa_rope(const sinkattn_prefill_args *args, int32_t window,
                              const sinkattn_rope_spec *rope, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Backward of the whole-sequence prefill: the training variant. The gradients of a loss through
 * O = attention(q, k, v, sink) given dO = dLoss/dO. The sink enters the softmax the way
 * "MiMo-V2-Flash 模型架构深度拆解" CH10.1 builds it (a column of per-head logits concatenated
 * after the scaled, masked scores, softmax, then that column dropped), so its gradient is that
 * column's softmax gradient with zero value (CH10.1 creates it with requires_grad=False; it is
 * given here for a caller that does train it). With P_ij = exp(a_ij - LSE_i) and
 * p_s,i = exp(sink_h - LSE_i) (LSE of the forward, sink included), for every row i:
 *     delta_i  = <dO_i, O_i>
 *     dS_ij    = P_ij (<dO_i, v_j> - delta_i)
 *     dq_i     = scale sum_j dS_ij k_j,   dk_j = scale sum_{i, heads of the group} dS_ij q_i,
 *     dv_j     = sum_{i, heads of the group} P_ij dO_i,   dsink_h = - sum_{b, i} p_s,i delta_i.
 *
 *   q, k, v, o, dout: bf16 as in prefill (o [B, L, Hq, 128] the forward's output, dout its
 *       gradient, strides o_*, do_*); lse: fp32 [B, Hq, L] contiguous, the forward's LSE.
 *   dq [B, L, Hq, 192], dk [B, L, Hkv, 192], dv [B, L, Hkv, 128]: fp32, written (element
 *       strides dq_*, dk_*, dv_*, multiples of 4, the last dim contiguous).
 *   dsink: fp32 [Hq], written (NULL: not computed); sink NULL means no sink (dsink = 0).
 *   window = 0: full causal (GA); window >= 1: sliding window (SWA).
 *   workspace: device memory of sinkattn_prefill_backward_workspace_size bytes, 16-byte aligned
 *       (delta, B * Hq * L floats); its contents on entry do not matter.
 * Errors: as for prefill (dims 192 / 128 only), plus NULL o / dout / lse / gradient pointers,
 * SINKATTN_ERR_WORKSPACE_TOO_SMALL. The gradients do not depend on the order of any atomic sum
 * except dsink (a float sum over the batch's rows).
 * ------------------------------------------------------------------------------------------- */
typedef struct sinkattn_backward_args {
    const void *q;
    const void *k;
    const void *v;
    const void *o;
    const void *dout;
    const float *lse;
    const float *sink;
    float *dq;
    float *dk;
    float *dv;
    float *dsink;
    int32_t B, L, Hq, Hkv, d_qk, d_v;
    float scale;
    int64_t q_sb, q_sl, q_sh;
    int64_t k_sb, k_sl, k_sh;
    int64_t v_sb, v_sl, v_sh;
    int64_t o_sb, o_sl, o_sh;
    int64_t do_sb, do_sl, do_sh;
    int64_t dq_sb, dq_sl, dq_sh;
    int64_t dk_sb, dk_sl, dk_sh;
    int64_t dv_sb, dv_sl, dv_sh;
} sinkattn_backward_args;

size_t sinkattn_prefill_backward_workspace_size(const sinkattn_backward_args *args);

int sinkattn_prefill_backward(const sinkattn_backward_args *args, int32_t window,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Human-readable name of a status code (static storage). */
const char *sinkattn_status_string(int status);

/* SINKATTN_VERSION of the built library. */
int sinkattn_version(void);

/* Reads and clears the device flag that kernels set when an internal wait gives up (bit 0:
 * prefill, bit 1: decode). Synchronises the current device. Returns SINKATTN_OK and writes the
 * flag to *flag_out, or SINKATTN_ERR_CUDA. */
int sinkattn_take_device_error(uint32_t *flag_out);

/* Sets how long a kernel on the current device waits on an internal barrier before it gives
 * up, records bit 0 (prefill) or 1 (decode) in the device flag above and returns (its output
 * is then unspecified). Failure detection: a stuck copy or MMA ends the call instead of hanging
 * the GPU. Default 1 s (1e9 ns); legitimate waits last microseconds. 0 makes a wait give up as
 * soon as its first try (which suspends the thread only briefly) fails, as it does for waits
 * that span a load and an MMA step: this exercises the failure path on demand (the library's
 * tests do this). The waits a CTA makes for its own copies and MMAs before it
 * exits keep the 1 s bound. Process-wide for the current device; synchronises the device first.
 * Returns SINKATTN_OK or SINKATTN_ERR_CUDA. The pages have no counterpart: this is a service of
 * the library, not part of the method. */
int sinkattn_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* SINKATTN_H */
