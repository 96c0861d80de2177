/*
 * Sink-softmax attention: the ORACLE.
 *
 * This file is TEST INFRASTRUCTURE. It is a plain, slow, fp64 CPU restatement of what the
 * attention core of the pages computes, written so that a reader can check every line against
 * the pages by eye. Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load it. The product (the CUDA library) neither includes, links nor calls anything here,
 * and this file includes nothing from the product.
 *
 * Sources (web pages, cited by title and section):
 *   [QA]    "MiMo-V2-Flash 架构 QA", Q3.7 (why the max includes the sink) and Q3.8 (the formula
 *           s_ij = exp(a_ij - m_i) / (exp(sink - m_i) + sum_j' exp(a_ij' - m_i)), and the
 *           concat -> softmax -> drop reading of it); Q3.6 (window / chunk semantics).
 *   [ARCH]  "MiMo-V2-Flash 模型架构深度拆解", CH3.2 (a_ij = q_i k_j^T / sqrt(d)), CH10.1 (the sink
 *           is one fp32 scalar per query head, appended after scaling and masking), CH10.3
 *           (scaling = head_dim^-0.5; GA uses a causal mask, SWA only the latest 128 tokens).
 *   [NOTES] "MiMo-V2-Flash Technical Report" (paper notes), §4.1 (the sink sits in the
 *           denominator and carries no value), §4.3 (worked example: 128 keys in the W=128
 *           window).
 *
 * Readings taken where the pages are silent or ambiguous:
 *   - window W keeps keys j with i-W < j <= i (exactly W keys, the query included);
 *   - the sink is in post-scale logit units and is NOT multiplied by the scale;
 *   - GQA: query head h reads KV head h / (Hq/Hkv);
 *   - a NULL sink, or a sink of -inf, means plain softmax for that head;
 *   - LSE is the natural log of the full denominator including the sink term:
 *     LSE = m + ln(D), so that O = sum_j exp(a_j - LSE) v_j;
 *   - decode: the T new tokens are not in the cache; new token t sits right after the cached
 *     tokens and sees the cached tokens and new tokens 0..t, subject to the same causal/window
 *     rule over absolute positions.
 *
 * "Parity pinned": every function here is checked, in tests/test_oracle_pins.py, against the
 * worked example's printed numbers, a library softmax/logsumexp, a library attention routine,
 * closed-form rotation angles, and invariants the mathematics fixes.
 *
 * The last two functions restate the steps that precede the attention core (the value scale
 * and partial rotary position embedding), which the library fuses into one pass.
 *
 * Inputs are bf16 bit patterns (uint16). Each is converted exactly to fp64; all arithmetic is
 * fp64. Arrays are contiguous, token-major: [B, L, H, d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 is the top 16 bits of an IEEE-754 binary32; widening to binary64 is exact. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One query row against an explicit list of visible keys.
 *
 *   a_j  = scale * <q, k_j>                               [ARCH CH3.2, CH10.3]
 *   m    = max(sink, max_j a_j)                           [QA Q3.7]
 *   D    = exp(sink - m) + sum_j exp(a_j - m)             [QA Q3.8]
 *   O    = sum_j exp(a_j - m) * v_j / D                   [QA Q3.8; NOTES §4.1: no value for the sink]
 *   LSE  = m + ln(D)
 *   w_s  = exp(sink - m) / D                              (the sink's share, [NOTES §4.3])
 *
 * sink = -INFINITY gives exp(-inf) = 0: plain softmax. nkeys >= 1 always holds for the
 * callers below (every query sees itself), so m is finite and D > 0.
 */
static void sink_softmax_row(const uint16_t *q, const uint16_t *const *krows,
                             const uint16_t *const *vrows, int nkeys, int dq, int dv,
                             double scale, double sink, double *a, double *o, double *lse,
                             double *wsink)
{
    double m = sink;
    for (int j = 0; j < nkeys; ++j) {
        double dot = 0.0;
        for (int d = 0; d < dq; ++d)
            dot += bf16_to_f64(q[d]) * bf16_to_f64(krows[j][d]);
        a[j] = scale * dot;
        if (a[j] > m)
            m = a[j];
    }
    double D = exp(sink - m);
    for (int j = 0; j < nkeys; ++j)
        D += exp(a[j] - m);
    for (int e = 0; e < dv; ++e)
        o[e] = 0.0;
    for (int j = 0; j < nkeys; ++j) {
        double w = exp(a[j] - m) / D;
        for (int e = 0; e < dv; ++e)
            o[e] += w * bf16_to_f64(vrows[j][e]);
    }
    if (lse)
        *lse = m + log(D);
    if (wsink)
        *wsink = exp(sink - m) / D;
}

static double head_sink(const float *sink, int h)
{
    return sink ? (double)sink[h] : -INFINITY;
}

/*
 * Prefill: every query position i of every sequence b attends to the keys of its own sequence
 * at positions j with j <= i (GA, [ARCH CH10.3] causal mask) and, when window > 0, also
 * j > i - window (SWA, [ARCH CH10.3], [NOTES §4.3] "128 keys in the W=128 window").
 *
 *   q [B, L, Hq, dq], k [B, L, Hkv, dq], v [B, L, Hkv, dv]  (bf16 bits, contiguous)
 *   sink [Hq] fp32 or NULL
 *   rows: nrows (b, i) pairs to evaluate (all heads of each), or NULL for every (b, i)
 *   o    [nrows or B*L, Hq, dv] fp64;  lse, wsink [nrows or B*L, Hq] fp64 (each may be NULL)
 *
 * Returns 0, or -1 on a bad argument.
 */
int sinkattn_oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const float *sink, int B, int L, int Hq, int Hkv, int dq, int dv,
                            int window, double scale, const int32_t *rows, int64_t nrows,
                            double *o, double *lse, double *wsink)
{
    if (B < 0 || L < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || dq <= 0 || dv <= 0)
        return -1;
    const int G = Hq / Hkv;
    const int64_t n = rows ? nrows : (int64_t)B * L;

#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (L > 0 ? L : 1));
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (L > 0 ? L : 1));
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t r = 0; r < n; ++r) {
            for (int h = 0; h < Hq; ++h) {
                const int b = rows ? rows[2 * r] : (int)(r / (L > 0 ? L : 1));
                const int i = rows ? rows[2 * r + 1] : (int)(r % (L > 0 ? L : 1));
                const int g = h / G;
                const int lo = (window > 0 && i - window + 1 > 0) ? i - window + 1 : 0;
                int nk = 0;
                for (int j = lo; j <= i; ++j) {
                    kr[nk] = k + (((int64_t)b * L + j) * Hkv + g) * dq;
                    vr[nk] = v + (((int64_t)b * L + j) * Hkv + g) * dv;
                    ++nk;
                }
                const uint16_t *qr = q + (((int64_t)b * L + i) * Hq + h) * dq;
                sink_softmax_row(qr, kr, vr, nk, dq, dv, scale, head_sink(sink, h), a,
                                 o + (r * Hq + h) * dv, lse ? lse + r * Hq + h : NULL,
                                 wsink ? wsink + r * Hq + h : NULL);
            }
        }
        free(a);
        free(kr);
        free(vr);
    }
    return 0;
}

/* KV-cache kinds; the numeric values match the library's public header. */
enum { ORACLE_KV_RING = 0, ORACLE_KV_CONTIG = 1, ORACLE_KV_PAGED = 2 };

/*
 * Decode (and speculative verify): T new query tokens per sequence b attend to the cached
 * tokens of that sequence plus the new tokens 0..t (the new tokens are not in the cache).
 *
 * Positions are counted relative to the first new token: cached token c (c = 0 is the oldest
 * of n_b cached tokens) sits at position c - n_b, new token u at position u. New query t
 * sees every key at position p with p <= t and, when window > 0, p > t - window. This is the
 * prefill rule above applied to the concatenated sequence.
 *
 * Where cached token c lives:
 *   RING   (window-sized ring, capacity ring_cap): slot (ring_head[b] + c) mod ring_cap,
 *          n_b = ring_len[b];  k_cache [B, ring_cap, Hkv, dq]
 *   CONTIG k_cache [B, max_ctx, Hkv, dq], row c;  n_b = ctx_len[b]
 *   PAGED  k_cache [num_pages, page_size, Hkv, dq];
 *          page page_table[b * max_pages + c / page_size], row c % page_size;  n_b = ctx_len[b]
 * (v_cache alike with dv.)
 *
 *   q [B, T, Hq, dq], k_new [B, T, Hkv, dq], v_new [B, T, Hkv, dv]
 *   o [B, T, Hq, dv] fp64, lse / wsink [B, T, Hq] fp64 (may be NULL)
 *   seqs: nseqs sequence indices to evaluate (outputs indexed by position in seqs), or NULL
 */
int sinkattn_oracle_decode(int kind, const uint16_t *q, const uint16_t *k_new,
                           const uint16_t *v_new, const uint16_t *k_cache,
                           const uint16_t *v_cache, const int32_t *ring_head,
                           const int32_t *ring_len, int ring_cap, const int32_t *ctx_len,
                           int max_ctx, const int32_t *page_table, int page_size, int max_pages,
                           const float *sink, int B, int T, int Hq, int Hkv, int dq, int dv,
                           int window, double scale, const int32_t *seqs, int nseqs, double *o,
                           double *lse, double *wsink)
{
    if (B < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
        return -1;
    if (kind != ORACLE_KV_RING && kind != ORACLE_KV_CONTIG && kind != ORACLE_KV_PAGED)
        return -1;
    const int G = Hq / Hkv;
    const int ns = seqs ? nseqs : B;

    /* largest cache any evaluated sequence holds, for the scratch lists */
    int64_t cap = T;
    for (int s = 0; s < ns; ++s) {
        const int b = seqs ? seqs[s] : s;
        const int64_t nb = (kind == ORACLE_KV_RING) ? ring_len[b] : ctx_len[b];
        if (nb + T > cap)
            cap = nb + T;
    }
    int bad = 0;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * cap);
        const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * cap);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * cap);
#pragma omp for schedule(dynamic, 1) collapse(3)
        for (int s = 0; s < ns; ++s) {
            for (int t = 0; t < T; ++t) {
                for (int h = 0; h < Hq; ++h) {
                    const int b = seqs ? seqs[s] : s;
                    const int g = h / G;
                    const int nb = (kind == ORACLE_KV_RING) ? ring_len[b] : ctx_len[b];
                    if (nb < 0 || (kind == ORACLE_KV_RING && nb > ring_cap) ||
                        (kind == ORACLE_KV_CONTIG && nb > max_ctx)) {
#pragma omp atomic write
                        bad = 1;
                        continue;
                    }
                    int nk = 0;
                    for (int c = 0; c < nb; ++c) {
                        const int p = c - nb; /* position of cached token c */
                        if (p > t || (window > 0 && p <= t - window))
                            continue;
                        int64_t row; /* row index into the cache arrays, in units of [Hkv, d] */
                        if (kind == ORACLE_KV_RING)
                            row = (int64_t)b * ring_cap + (ring_head[b] + c) % ring_cap;
                        else if (kind == ORACLE_KV_CONTIG)
                            row = (int64_t)b * max_ctx + c;
                        else
                            row = (int64_t)page_table[(int64_t)b * max_pages + c / page_size] *
                                      page_size + c % page_size;
                        kr[nk] = k_cache + (row * Hkv + g) * dq;
                        vr[nk] = v_cache + (row * Hkv + g) * dv;
                        ++nk;
                    }
                    for (int u = 0; u <= t; ++u) {
                        if (window > 0 && u <= t - window)
                            continue;
                        kr[nk] = k_new + (((int64_t)b * T + u) * Hkv + g) * dq;
                        vr[nk] = v_new + (((int64_t)b * T + u) * Hkv + g) * dv;
                        ++nk;
                    }
                    const uint16_t *qr = q + (((int64_t)b * T + t) * Hq + h) * dq;
                    const int64_t out = ((int64_t)s * T + t) * Hq + h;
                    sink_softmax_row(qr, kr, vr, nk, dq, dv, scale, head_sink(sink, h), a,
                                     o + out * dv, lse ? lse + out : NULL,
                                     wsink ? wsink + out : NULL);
                }
            }
        }
        free(a);
        free(kr);
        free(vr);
    }
    return bad ? -1 : 0;
}

/*
 * Split-KV decomposition of one row (the decode algorithm's algebra, not on the pages; derived
 * from [QA Q3.8]). A span P of the visible keys gives, WITHOUT the sink:
 *   m_P = max_{j in P} a_j,  l_P = sum_{j in P} exp(a_j - m_P),  O_P = sum_{j in P} exp(a_j - m_P) v_j
 * (m_P = -inf, l_P = 0, O_P = 0 for an empty span). Merging the spans and counting the sink
 * exactly once:
 *   m = max(sink, max_P m_P),  D = exp(sink - m) + sum_P l_P exp(m_P - m),
 *   O = sum_P O_P exp(m_P - m) / D,  LSE = m + ln D.
 *
 * sinkattn_oracle_partial computes (O_P, m_P, l_P) of one query row over keys [j0, j1) of the
 * given key/value arrays ([n, dq] / [n, dv] bf16 bits, contiguous).
 */
void sinkattn_oracle_partial(const uint16_t *q, const uint16_t *k, const uint16_t *v, int j0,
                             int j1, int dq, int dv, double scale, double *o_p, double *m_p,
                             double *l_p)
{
    double m = -INFINITY;
    for (int j = j0; j < j1; ++j) {
        double dot = 0.0;
        for (int d = 0; d < dq; ++d)
            dot += bf16_to_f64(q[d]) * bf16_to_f64(k[(int64_t)j * dq + d]);
        if (scale * dot > m)
            m = scale * dot;
    }
    double l = 0.0;
    for (int e = 0; e < dv; ++e)
        o_p[e] = 0.0;
    for (int j = j0; j < j1; ++j) {
        double dot = 0.0;
        for (int d = 0; d < dq; ++d)
            dot += bf16_to_f64(q[d]) * bf16_to_f64(k[(int64_t)j * dq + d]);
        const double w = exp(scale * dot - m);
        l += w;
        for (int e = 0; e < dv; ++e)
            o_p[e] += w * bf16_to_f64(v[(int64_t)j * dv + e]);
    }
    *m_p = m;
    *l_p = l;
}

void sinkattn_oracle_merge(const double *o_p, const double *m_p, const double *l_p, int nparts,
                           int dv, double sink, double *o, double *lse)
{
    double m = sink;
    for (int p = 0; p < nparts; ++p)
        if (m_p[p] > m)
            m = m_p[p];
    double D = exp(sink - m);
    for (int p = 0; p < nparts; ++p)
        if (l_p[p] > 0.0)
            D += l_p[p] * exp(m_p[p] - m);
    for (int e = 0; e < dv; ++e)
        o[e] = 0.0;
    for (int p = 0; p < nparts; ++p) {
        if (l_p[p] <= 0.0)
            continue;
        const double c = exp(m_p[p] - m) / D;
        for (int e = 0; e < dv; ++e)
            o[e] += c * o_p[(int64_t)p * dv + e];
    }
    *lse = m + log(D);
}

/*
 * Committing accepted tokens to the cache (the "KV cache update" step of the attention module,
 * [ARCH CH10.3] step 6). For each sequence b the first n_accept[b] of its T new tokens are
 * appended, oldest first:
 *   RING:   while the ring holds fewer than ring_cap tokens, token goes to slot
 *           (head + len) mod cap and len grows; once full, it overwrites the oldest slot
 *           (head) and head advances by one.
 *   CONTIG: row ctx_len[b] + u; ctx_len grows.
 *   PAGED:  position ctx_len[b] + u through the page table; ctx_len grows.
 * The cache arrays and ring_head / ring_len / ctx_len are updated in place.
 */
int sinkattn_oracle_commit(int kind, const uint16_t *k_new, const uint16_t *v_new,
                           const int32_t *n_accept, uint16_t *k_cache, uint16_t *v_cache,
                           int32_t *ring_head, int32_t *ring_len, int ring_cap, int32_t *ctx_len,
                           int max_ctx, const int32_t *page_table, int page_size, int max_pages,
                           int B, int T, int Hkv, int dq, int dv)
{
    for (int b = 0; b < B; ++b) {
        if (n_accept[b] < 0 || n_accept[b] > T)
            return -1;
        for (int u = 0; u < n_accept[b]; ++u) {
            int64_t row;
            if (kind == ORACLE_KV_RING) {
                int slot;
                if (ring_len[b] < ring_cap) {
                    slot = (ring_head[b] + ring_len[b]) % ring_cap;
                    ring_len[b] += 1;
                } else {
                    slot = ring_head[b];
                    ring_head[b] = (ring_head[b] + 1) % ring_cap;
                }
                row = (int64_t)b * ring_cap + slot;
            } else if (kind == ORACLE_KV_CONTIG) {
                if (ctx_len[b] >= max_ctx)
                    return -1;
                row = (int64_t)b * max_ctx + ctx_len[b];
                ctx_len[b] += 1;
            } else if (kind == ORACLE_KV_PAGED) {
                const int c = ctx_len[b];
                if (c / page_size >= max_pages)
                    return -1;
                row = (int64_t)page_table[(int64_t)b * max_pages + c / page_size] * page_size +
                      c % page_size;
                ctx_len[b] += 1;
            } else {
                return -1;
            }
            for (int g = 0; g < Hkv; ++g) {
                memcpy(k_cache + (row * Hkv + g) * dq,
                       k_new + (((int64_t)b * T + u) * Hkv + g) * dq, sizeof(uint16_t) * dq);
                memcpy(v_cache + (row * Hkv + g) * dv,
                       v_new + (((int64_t)b * T + u) * Hkv + g) * dv, sizeof(uint16_t) * dv);
            }
        }
    }
    return 0;
}

/*
 * The two steps just before the attention core: the value scale and partial rotary position
 * embedding. [ARCH] CH10.3 lists the attention module's order: Q/K/V projection, value_states
 * times v_scale (0.707), split Q/K into 64 rotary | 128 no-pe dims, rotate the first 64,
 * concatenate, then attention. [ARCH] CH3.5 and CH8.1: partial_rotary_factor 0.334 (64 of the
 * 192 Q/K dims), rope_theta 5,000,000 on GA layers and swa_rope_theta 10,000 on SWA layers
 * ([ARCH] CH10.5; [QA] Q2.7). [QA] Q2.7: at position m, dimension i turns by m * theta^(-2i/d).
 *
 * Readings where the pages leave it open:
 *   - d in that angle is the rotated width rope_dim, and i counts dimension PAIRS,
 *     0 <= i < rope_dim/2: pair i turns at w_i = theta^(-2i/rope_dim);
 *   - pair i is dims (i, i + rope_dim/2) ("rotate half"), turned counter-clockwise:
 *         y_i              = x_i cos(m w_i) - x_{i+rope_dim/2} sin(m w_i)
 *         y_{i+rope_dim/2} = x_{i+rope_dim/2} cos(m w_i) + x_i sin(m w_i)
 *   - the rotary embedding scales nothing else (its attention scaling is 1);
 *   - dims rope_dim .. d-1 pass unchanged.
 *
 *   x [n, H, d] bf16 bits; pos [n]: the position of row n (all H heads); out [n, H, d] fp64.
 * Returns 0, or -1 on a bad argument.
 */
int sinkattn_oracle_rope(const uint16_t *x, const int64_t *pos, int64_t n, int H, int d,
                         int rope_dim, double theta, double *out)
{
    if (n < 0 || H < 0 || rope_dim < 2 || rope_dim % 2 != 0 || rope_dim > d || !(theta > 0.0))
        return -1;
    const int half = rope_dim / 2;
    for (int64_t r = 0; r < n; ++r) {
        for (int h = 0; h < H; ++h) {
            const uint16_t *xr = x + (r * H + h) * d;
            double *yr = out + (r * H + h) * d;
            for (int c = 0; c < d; ++c)
                yr[c] = bf16_to_f64(xr[c]);
            for (int i = 0; i < half; ++i) {
                const double w = pow(theta, -2.0 * i / rope_dim);
                const double angle = (double)pos[r] * w;
                const double cs = cos(angle), sn = sin(angle);
                const double a = bf16_to_f64(xr[i]), b = bf16_to_f64(xr[i + half]);
                yr[i] = a * cs - b * sn;
                yr[i + half] = b * cs + a * sn;
            }
        }
    }
    return 0;
}

/* The value scale, [ARCH] CH10.3: every value element times v_scale. v [n] bf16 bits. */
void sinkattn_oracle_vscale(const uint16_t *v, int64_t n, double v_scale, double *out)
{
    for (int64_t e = 0; e < n; ++e)
        out[e] = bf16_to_f64(v[e]) * v_scale;
}

/*
 * FP8 KV cache codes. The pages size a KV slot at one byte ([NOTES] §2 memory arithmetic) and
 * speak of FP8 inference ([BLOG]); they name no format or scaling. Readings:
 *   - the E4M3 "fn" format: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
 *     S.1111.111 is NaN; largest finite 448 = 1.75 * 2^8, smallest normal 2^-6, subnormals
 *     k * 2^-9;
 *   - one fp32 scale per cache tensor (K and V separately): a stored code c means e(c) * scale;
 *   - storing x: y = x / scale in fp32 (correctly rounded), then the nearest E4M3 value, ties
 *     to the even code, saturating to +-448 (NaN stays NaN).
 */
double sinkattn_oracle_e4m3_value(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
    const double v = (e == 0) ? ldexp((double)m, -9)        /* subnormal: m/8 * 2^-6 */
                              : ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

uint8_t sinkattn_oracle_e4m3_encode(float y)
{
    if (isnan(y))
        return 0x7f;
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    const double a = fabs((double)y);
    if (a >= 448.0)
        return sign | 0x7e;
    /* the nearest of the 127 non-negative finite values; on a tie the even code (its last
       bit is the mantissa's last bit) */
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        const double d = fabs(sinkattn_oracle_e4m3_value((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

/* codes[i] = encode(x[i] / scale), the division in fp32. x: bf16 bits. */
void sinkattn_oracle_fp8_encode(const uint16_t *x, int64_t n, float scale, uint8_t *codes)
{
    for (int64_t i = 0; i < n; ++i) {
        const float xi = (float)bf16_to_f64(x[i]);
        const float y = xi / scale;
        codes[i] = sinkattn_oracle_e4m3_encode(y);
    }
}

/* out[i] = e(codes[i]) (the scale is applied by the caller). */
void sinkattn_oracle_fp8_decode(const uint8_t *codes, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = sinkattn_oracle_e4m3_value(codes[i]);
}

/*
 * Backward of the whole-sequence prefill: the training variant. [ARCH] CH10.1 creates the sink
 * parameter with requires_grad=False (it is not trained by gradient); its gradient is given
 * here all the same, for a caller that does train it.
 *
 * With the forward of sink_softmax_row for row i of head h (p_j = exp(a_j - m) / D for the
 * visible keys, p_s = exp(sink - m) / D for the sink, O = sum_j p_j v_j), and the incoming
 * gradient dO of that row:
 *   dp_j  = <dO, v_j>
 *   delta = sum_j p_j dp_j = <dO, O>          (the sink carries no value: its dp is 0)
 *   da_j  = p_j (dp_j - delta)                (softmax backward over the keys and the sink)
 *   dsink_h += p_s (0 - delta)
 *   dq_i  = scale * sum_j da_j k_j;   dk_j += scale * da_j q_i;   dv_j += p_j dO
 * GQA: dk / dv of KV head g sum over its G query heads.
 *
 *   q, k, v, dout as prefill (bf16 bits; dout [B, L, Hq, dv]); gq [B,L,Hq,dq], gk [B,L,Hkv,dq],
 *   gv [B,L,Hkv,dv], gsink [Hq] fp64 (written). Serial: the key gradients accumulate across rows.
 */
int sinkattn_oracle_prefill_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                     const float *sink, const uint16_t *dout, int B, int L,
                                     int Hq, int Hkv, int dq, int dv, int window, double scale,
                                     double *gq, double *gk, double *gv, double *gsink)
{
    if (B < 0 || L < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || window < 0)
        return -1;
    const int G = Hq / Hkv;
    memset(gq, 0, sizeof(double) * (size_t)B * L * Hq * dq);
    memset(gk, 0, sizeof(double) * (size_t)B * L * Hkv * dq);
    memset(gv, 0, sizeof(double) * (size_t)B * L * Hkv * dv);
    memset(gsink, 0, sizeof(double) * (size_t)Hq);
    double *a = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
    double *dp = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
    double *o = (double *)malloc(sizeof(double) * dv);
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < L; ++i) {
            const int lo = (window > 0 && i - window + 1 > 0) ? i - window + 1 : 0;
            for (int h = 0; h < Hq; ++h) {
                const int g = h / G;
                const double s = head_sink(sink, h);
                const uint16_t *qi = q + (((int64_t)b * L + i) * Hq + h) * dq;
                const uint16_t *di = dout + (((int64_t)b * L + i) * Hq + h) * dv;
                /* forward of the row */
                double m = s;
                for (int j = lo; j <= i; ++j) {
                    const uint16_t *kj = k + (((int64_t)b * L + j) * Hkv + g) * dq;
                    double dot = 0.0;
                    for (int d = 0; d < dq; ++d)
                        dot += bf16_to_f64(qi[d]) * bf16_to_f64(kj[d]);
                    a[j] = scale * dot;
                    if (a[j] > m)
                        m = a[j];
                }
                double D = exp(s - m);
                for (int j = lo; j <= i; ++j)
                    D += exp(a[j] - m);
                for (int e = 0; e < dv; ++e)
                    o[e] = 0.0;
                for (int j = lo; j <= i; ++j) {
                    const uint16_t *vj = v + (((int64_t)b * L + j) * Hkv + g) * dv;
                    const double p = exp(a[j] - m) / D;
                    for (int e = 0; e < dv; ++e)
                        o[e] += p * bf16_to_f64(vj[e]);
                }
                /* backward */
                double delta = 0.0;
                for (int e = 0; e < dv; ++e)
                    delta += bf16_to_f64(di[e]) * o[e];
                for (int j = lo; j <= i; ++j) {
                    const uint16_t *vj = v + (((int64_t)b * L + j) * Hkv + g) * dv;
                    double x = 0.0;
                    for (int e = 0; e < dv; ++e)
                        x += bf16_to_f64(di[e]) * bf16_to_f64(vj[e]);
                    dp[j] = x;
                }
                const double ps = exp(s - m) / D;
                gsink[h] += ps * (0.0 - delta);
                double *gqi = gq + (((int64_t)b * L + i) * Hq + h) * dq;
                for (int j = lo; j <= i; ++j) {
                    const double p = exp(a[j] - m) / D;
                    const double da = p * (dp[j] - delta);
                    const uint16_t *kj = k + (((int64_t)b * L + j) * Hkv + g) * dq;
                    double *gkj = gk + (((int64_t)b * L + j) * Hkv + g) * dq;
                    double *gvj = gv + (((int64_t)b * L + j) * Hkv + g) * dv;
                    for (int d = 0; d < dq; ++d) {
                        gqi[d] += scale * da * bf16_to_f64(kj[d]);
                        gkj[d] += scale * da * bf16_to_f64(qi[d]);
                    }
                    for (int e = 0; e < dv; ++e)
                        gvj[e] += p * bf16_to_f64(di[e]);
                }
            }
        }
    }
    free(a);
    free(dp);
    free(o);
    return 0;
}
