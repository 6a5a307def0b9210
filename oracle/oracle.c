/*
 * Gated DSA layer: CPU ORACLE.  TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct restatement of what the Gated DeepSeek
 * Sparse Attention layer computes, in fp64.  It exists to check the CUDA
 * library; nothing in the product path may call it.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load this file.  It shares
 * no code, header, table or constant with the CUDA library: its FP8 and bf16
 * decoders are written here from the bit-format definitions.
 *
 * Sources (web pages on the method; no page prints a formula, so the score,
 * tie rule and gate form below are readings of their prose):
 *   [P2] "Open-Source LLM Architecture Evolution: How Lightweight Sparse
 *        Attention Reshapes Long-Context Modeling Efficiency",
 *        Architecture Breakdown §2 (bullets "Indexer", "Top-K selection",
 *        "Gated fusion"); Technical Deep Dive §2 ("candidate set is capped").
 *   [P5] "Fine-Grained Sparse Attention in Ultra-Large Parameter Models",
 *        §2.1 (Indexer + Top-K route), §2.2 (no RoPE in the indexer),
 *        §2.3 (multi-head screening, 32 heads x 128 dim).
 *   [P1] aiany.app item "naive-n0-5-flash", Key Capabilities (5:1 SWA(128)
 *        and DSA hybrid, 16-head indexer, top 2,048, FP8).
 *   [P4] "Open-Weight Deployment of an Ultra-Large Sparse Model:
 *        Architecture, Hardware, and Engineering Practices", §1 and §3
 *        (activations computed in MXFP8).
 *
 * Every function returns 0 on success and a negative code on bad input.
 * OpenMP spreads independent outputs (key positions, heads, rows) over the
 * host's cores; every output's own arithmetic is sequential, in the order
 * written, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EBAD (-1)   /* malformed argument (index out of range, ...) */
#define ORC_ENAN (-2)   /* non-finite input where a finite one is required */

/* ---- number formats ---------------------------------------------------- */

/* OCP 8-bit float E4M3 ("fn" variant: no infinities; S.1111.111 is NaN).
 * Layout: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 encodes subnormals m/8 * 2^-6. */
double orc_e4m3_to_f64(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 mantissa bits. */
double orc_bf16_to_f64(uint16_t b)
{
    int s = b >> 15, e = (b >> 7) & 255, m = b & 127;
    double v;
    if (e == 255) return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) v = ldexp((double)m / 128.0, -126);
    else        v = ldexp(1.0 + (double)m / 128.0, e - 127);
    return s ? -v : v;
}

/* The E4M3 code nearest to x, ties to the even mantissa, finite values of
 * magnitude 448 (the largest finite, S.1111.110) and above giving +-448 --
 * the "saturate to finite" conversion.  Steps: the exponent e with
 * 2^e <= |x| < 2^(e+1) (or the subnormal range |x| < 2^-6, quantum 2^-9);
 * |x| / 2^(e-3) rounded to an integer q in [8, 16]; q = 16 carries into the
 * next exponent; the code is (e + 7) << 3 | (q - 8).  NaN gives S.1111.111. */
uint8_t orc_e4m3_from_f64(double x)
{
    uint8_t s = signbit(x) ? 0x80 : 0;
    if (isnan(x)) return s | 0x7F;
    double a = fabs(x);
    if (a >= 448.0) return s | 0x7E;
    if (a < ldexp(1.0, -6)) {
        double m = nearbyint(a * 512.0);   /* exact: a power-of-two scaling */
        return s | (uint8_t)(m >= 8.0 ? 0x08 : (int)m);
    }
    int E;
    frexp(a, &E);                          /* a = f * 2^E, 0.5 <= f < 1 */
    int e = E - 1;
    double q = nearbyint(ldexp(a, 3 - e)); /* in [8, 16] */
    if (q >= 16.0) { q = 8.0; ++e; }
    if (e > 8 || (e == 8 && q > 14.0)) return s | 0x7E;
    return s | (uint8_t)(((e + 7) << 3) | ((int)q - 8));
}

/* ---- microscaled FP8 (MXFP8) --------------------------------------------
 * The pages name MXFP8 as the activation format ("Open-Weight Deployment of
 * an Ultra-Large Sparse Model", §1 and §3) without defining it; the reading
 * here is the OCP Microscaling (MX) format: a block of 32 consecutive
 * elements shares one E8M0 scale, and each element is an E4M3 code; an
 * element's value is its E4M3 value times the block's scale. */
#define ORC_MX_BLOCK 32

/* E8M0: 8 exponent bits, bias 127, no sign and no mantissa; code c is
 * 2^(c - 127) for c in [0, 254], and 255 is NaN. */
double orc_e8m0_to_f64(uint8_t c)
{
    if (c == 255) return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* One block of n values to MXFP8.  The shared exponent is floor(log2 of the
 * largest magnitude) minus 8 -- 8 being the exponent of the largest power of
 * two that E4M3 holds (256) -- so the largest element lands in [256, 512)
 * before rounding; it is clamped to the scale's range [-127, 127].  A block
 * of zeros takes code 0.  Each element becomes the E4M3 code nearest to
 * x / 2^shared (ties to even; magnitudes of 448 and above, which only the
 * largest elements reach, give +-448).  Non-finite input is rejected. */
int orc_mx_encode_block(const double *x, int n, uint8_t *codes, uint8_t *scale)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(x[i])) return ORC_EBAD;
        if (fabs(x[i]) > amax) amax = fabs(x[i]);
    }
    int shared = -127;
    if (amax > 0.0) {
        int E;
        frexp(amax, &E);                   /* amax = f * 2^E, 0.5 <= f < 1 */
        shared = (E - 1) - 8;              /* E - 1 = floor(log2 amax) */
        if (shared < -127) shared = -127;
        if (shared > 127) shared = 127;
    }
    *scale = (uint8_t)(shared + 127);
    for (int i = 0; i < n; ++i)
        codes[i] = orc_e4m3_from_f64(ldexp(x[i], -shared)); /* exact scaling */
    return 0;
}

/* nblocks consecutive blocks of ORC_MX_BLOCK values. */
int orc_mx_encode(const double *x, int64_t nblocks, uint8_t *codes, uint8_t *scales)
{
    for (int64_t b = 0; b < nblocks; ++b)
        if (orc_mx_encode_block(x + b * ORC_MX_BLOCK, ORC_MX_BLOCK, codes + b * ORC_MX_BLOCK, scales + b))
            return ORC_EBAD;
    return 0;
}

/* ---- paged caches ----------------------------------------------------- */

/* Byte/element offset of logical position `pos` of sequence `b` in a cache
 * laid out as [num_pages, page_size, row]: the block table maps the
 * sequence's logical page pos/page_size to a physical page. Returns -1 when
 * the position or the page id is out of range. */
static int64_t orc_row_index(const int32_t *seq_lens, const int32_t *block_table,
                             int num_seqs, int max_blocks, int page_size,
                             int num_pages, int b, int64_t pos)
{
    if (b < 0 || b >= num_seqs) return -1;
    if (pos < 0 || pos >= seq_lens[b]) return -1;
    int64_t lp = pos / page_size;
    if (lp >= max_blocks) return -1;
    int32_t page = block_table[(int64_t)b * max_blocks + lp];
    if (page < 0 || page >= num_pages) return -1;
    return (int64_t)page * page_size + pos % page_size;
}

/* ---- the step before the layer: appending new tokens to the caches ----
 * The indexer keys are FP8 ([P1] Key Capabilities: FP8; one scale per
 * tensor, read here as a multiplier applied before rounding): token j's
 * indexer key row becomes e4m3(fp32(bf16 k_new[j, d]) * k_scale) -- the
 * product rounded once, in fp32 -- at logical position tok_pos[j] of
 * sequence tok_seq[j] of the paged indexer-key cache; its latent row (when
 * latent_new is given) is stored there unchanged in the latent cache.  A
 * position outside its sequence or a page outside the cache makes the call
 * fail (nothing is defined for it). */
int orc_append_kv(const uint16_t *k_new, float k_scale, const uint16_t *latent_new,
                  const int32_t *tok_seq, const int32_t *tok_pos, int n,
                  const int32_t *seq_lens, const int32_t *block_table, int num_seqs,
                  int max_blocks, int page_size, int num_pages, int DI, int Dqk,
                  uint8_t *k_cache, uint16_t *kv_cache)
{
    for (int j = 0; j < n; ++j) {
        int64_t r = orc_row_index(seq_lens, block_table, num_seqs, max_blocks, page_size,
                                  num_pages, tok_seq[j], tok_pos[j]);
        if (r < 0) return ORC_EBAD;
        for (int d = 0; d < DI; ++d) {
            float x = (float)orc_bf16_to_f64(k_new[(int64_t)j * DI + d]) * k_scale;
            k_cache[r * DI + d] = orc_e4m3_from_f64((double)x);
        }
        if (latent_new)
            for (int d = 0; d < Dqk; ++d)
                kv_cache[r * Dqk + d] = latent_new[(int64_t)j * Dqk + d];
    }
    return 0;
}

/* The MXFP8 variant of the append step: each 32-wide block of token j's
 * bf16 key row becomes one MXFP8 block (orc_mx_encode_block, no other
 * scale), its codes stored in the token's row of the paged key cache and its
 * block scales in the same row of the paged scale cache [num_pages,
 * page_size, DI/32]; the latent row as in orc_append_kv. */
int orc_append_kv_mx(const uint16_t *k_new, const uint16_t *latent_new,
                     const int32_t *tok_seq, const int32_t *tok_pos, int n,
                     const int32_t *seq_lens, const int32_t *block_table, int num_seqs,
                     int max_blocks, int page_size, int num_pages, int DI, int Dqk,
                     uint8_t *k_cache, uint8_t *k_scales, uint16_t *kv_cache)
{
    if (DI % ORC_MX_BLOCK) return ORC_EBAD;
    const int nb = DI / ORC_MX_BLOCK;
    double x[ORC_MX_BLOCK];
    for (int j = 0; j < n; ++j) {
        int64_t r = orc_row_index(seq_lens, block_table, num_seqs, max_blocks, page_size,
                                  num_pages, tok_seq[j], tok_pos[j]);
        if (r < 0) return ORC_EBAD;
        for (int blk = 0; blk < nb; ++blk) {
            for (int i = 0; i < ORC_MX_BLOCK; ++i)
                x[i] = orc_bf16_to_f64(k_new[(int64_t)j * DI + blk * ORC_MX_BLOCK + i]);
            if (orc_mx_encode_block(x, ORC_MX_BLOCK, k_cache + r * DI + blk * ORC_MX_BLOCK,
                                    k_scales + r * nb + blk))
                return ORC_EBAD;
        }
        if (latent_new)
            for (int d = 0; d < Dqk; ++d)
                kv_cache[r * Dqk + d] = latent_new[(int64_t)j * Dqk + d];
    }
    return 0;
}

/* ---- stage 1: indexer scores ------------------------------------------ */

/* I[t,s] = sum_h w[t,h] * max(0, sum_d qI[t,h,d] * kI[s,d]) for every
 * history position s <= q_pos[t] of sequence q_seq[t] ([P2] Indexer bullet:
 * a multi-head scorer of every history position; [P5] §2.2: no rotary
 * embedding, so qI and kI enter the dot product as stored; [P5] §2.3:
 * heads x dim).  qI: e4m3 [T,HI,DI]; w: fp32 [T,HI]; kI cache: e4m3
 * [num_pages,page_size,DI].  The sum runs in fp64 and is rounded once to
 * fp32 into scores[t*ld + s].  Entries s > q_pos[t] are not written. */
int orc_indexer_scores(const uint8_t *q_idx, const float *w,
                       const uint8_t *k_cache, const int32_t *seq_lens,
                       const int32_t *block_table, int num_seqs, int max_blocks,
                       int page_size, int num_pages, const int32_t *q_seq,
                       const int32_t *q_pos, int T, int HI, int DI,
                       float *scores, int64_t ld)
{
    int bad = 0;
    double *q = (double *)malloc(sizeof(double) * (size_t)HI * DI);
    for (int t = 0; t < T; ++t) {
        int b = q_seq[t];
        int64_t p = q_pos[t];
        if (b < 0 || b >= num_seqs || p < 0 || p >= seq_lens[b] || p >= ld) { bad |= 1; continue; }
        for (int i = 0; i < HI * DI; ++i)
            q[i] = orc_e4m3_to_f64(q_idx[(int64_t)t * HI * DI + i]);
#pragma omp parallel for schedule(static) reduction(| : bad)
        for (int64_t s = 0; s <= p; ++s) {
            int64_t r = orc_row_index(seq_lens, block_table, num_seqs, max_blocks,
                                      page_size, num_pages, b, s);
            if (r < 0) { bad |= 1; continue; }
            const uint8_t *k = k_cache + r * DI;
            double I = 0.0;
            for (int h = 0; h < HI; ++h) {
                double dot = 0.0;
                for (int d = 0; d < DI; ++d)
                    dot += q[h * DI + d] * orc_e4m3_to_f64(k[d]);
                double relu = dot > 0.0 ? dot : 0.0;
                I += (double)w[(int64_t)t * HI + h] * relu;
            }
            scores[t * ld + s] = (float)I;
        }
    }
    free(q);
    return bad ? ORC_EBAD : 0;
}

/* The indexer score of orc_indexer_scores with MXFP8 operands: each qI
 * element is its E4M3 value times the scale of its 32-wide block along DI
 * (q_scales: E8M0 [T,HI,DI/32]), each cached kI element likewise (k_scales:
 * E8M0 [num_pages,page_size,DI/32], the key cache's row layout); the score
 * formula, its fp64 sum and the single rounding to fp32 are unchanged. */
int orc_indexer_scores_mx(const uint8_t *q_idx, const uint8_t *q_scales, const float *w,
                          const uint8_t *k_cache, const uint8_t *k_scales,
                          const int32_t *seq_lens, const int32_t *block_table, int num_seqs,
                          int max_blocks, int page_size, int num_pages, const int32_t *q_seq,
                          const int32_t *q_pos, int T, int HI, int DI, float *scores, int64_t ld)
{
    if (DI % ORC_MX_BLOCK) return ORC_EBAD;
    const int nb = DI / ORC_MX_BLOCK;
    int bad = 0;
    double *q = (double *)malloc(sizeof(double) * (size_t)HI * DI);
    for (int t = 0; t < T; ++t) {
        int b = q_seq[t];
        int64_t p = q_pos[t];
        if (b < 0 || b >= num_seqs || p < 0 || p >= seq_lens[b] || p >= ld) { bad |= 1; continue; }
        for (int h = 0; h < HI; ++h)
            for (int d = 0; d < DI; ++d) {
                int64_t e = ((int64_t)t * HI + h) * DI + d;
                int64_t sc = ((int64_t)t * HI + h) * nb + d / ORC_MX_BLOCK;
                q[h * DI + d] = orc_e4m3_to_f64(q_idx[e]) * orc_e8m0_to_f64(q_scales[sc]);
            }
#pragma omp parallel for schedule(static) reduction(| : bad)
        for (int64_t s = 0; s <= p; ++s) {
            int64_t r = orc_row_index(seq_lens, block_table, num_seqs, max_blocks,
                                      page_size, num_pages, b, s);
            if (r < 0) { bad |= 1; continue; }
            const uint8_t *k = k_cache + r * DI;
            const uint8_t *ks = k_scales + r * nb;
            double I = 0.0;
            for (int h = 0; h < HI; ++h) {
                double dot = 0.0;
                for (int d = 0; d < DI; ++d)
                    dot += q[h * DI + d] * (orc_e4m3_to_f64(k[d]) * orc_e8m0_to_f64(ks[d / ORC_MX_BLOCK]));
                double relu = dot > 0.0 ? dot : 0.0;
                I += (double)w[(int64_t)t * HI + h] * relu;
            }
            scores[t * ld + s] = (float)I;
        }
    }
    free(q);
    return bad ? ORC_EBAD : 0;
}

/* ---- stage 2: top-K ----------------------------------------------------- */

typedef struct { float v; int32_t pos; } orc_cand;

/* Order: higher score first; equal scores (with -0 equal to +0, as C's
 * comparison already treats them) go to the lower position. */
static int orc_cmp_desc(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int orc_cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x < y) ? -1 : (x > y);
}

/* Keep the K highest-scoring history positions of each row ([P2] Top-K
 * selection bullet, K = 2048; [P3] §2.2; [P5] §2.1).  A row with
 * row_len <= K keeps every position.  Output: the kept positions in
 * ascending order, padded with -1 to K entries.  The full row is sorted
 * (no partial selection), which is what makes this obviously correct. */
int orc_topk(const float *scores, int64_t ld, const int32_t *row_len, int R,
             int K, int32_t *idx)
{
    int bad = 0;
    if (K <= 0) return ORC_EBAD;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < R; ++r) {
        int64_t n = row_len[r];
        int32_t *out = idx + (int64_t)r * K;
        if (n < 0 || n > ld) { bad |= 1; continue; }
        if (n <= K) {
            for (int64_t j = 0; j < K; ++j) out[j] = j < n ? (int32_t)j : -1;
            continue;
        }
        orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)n);
        for (int64_t s = 0; s < n; ++s) {
            float v = scores[r * ld + s];
            if (!isfinite(v)) bad |= 2;
            c[s].v = v;
            c[s].pos = (int32_t)s;
        }
        qsort(c, (size_t)n, sizeof(orc_cand), orc_cmp_desc);
        for (int j = 0; j < K; ++j) out[j] = c[j].pos;
        qsort(out, (size_t)K, sizeof(int32_t), orc_cmp_i32);
        free(c);
    }
    if (bad & 2) return ORC_ENAN;
    return bad ? ORC_EBAD : 0;
}

/* ---- stage 3: attention over the selected rows, gated ---------------------- */

/* For query t and head h: logits l_j = sm_scale * <q[t,h,:Dqk], c_j[:Dqk]>
 * over the selected latent rows c_j = cache row idx[t,j] of sequence
 * q_seq[t] (entries < 0 are padding and skipped), softmax over j,
 * o = sum_j p_j c_j[:Dv], then out = o * sigmoid(gate[t,h])
 * ([P2] Technical Deep Dive §2: score and softmax over only the selected
 * 2048 elements; [P2] Gated fusion bullet, read as a per-head sigmoid gate
 * multiplying the sparse output).  All heads share the latent row (the
 * key is its first Dqk entries, the value its first Dv).  q, cache and
 * gate are bf16 bit patterns; out is fp64 [T,H,Dv]; lse (nullable) gets
 * log(sum_j exp(l_j)), -inf when a query selected nothing (out is then 0). */
int orc_sparse_attn(const uint16_t *q, const uint16_t *kv_cache,
                    const int32_t *seq_lens, const int32_t *block_table,
                    int num_seqs, int max_blocks, int page_size, int num_pages,
                    const int32_t *q_seq, const int32_t *idx, int K,
                    const uint16_t *gate, double sm_scale, int T, int H,
                    int Dqk, int Dv, double *out, double *lse)
{
    int bad = 0;
    if (Dv > Dqk) return ORC_EBAD;
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(K > 0 ? K : 1));
    for (int t = 0; t < T; ++t) {
        int b = q_seq[t];
        int n = 0;
        for (int j = 0; j < K; ++j) {
            int32_t pos = idx[(int64_t)t * K + j];
            if (pos < 0) continue;
            int64_t r = orc_row_index(seq_lens, block_table, num_seqs, max_blocks,
                                      page_size, num_pages, b, pos);
            if (r < 0) { bad |= 1; continue; }
            rows[n++] = r;
        }
#pragma omp parallel for schedule(dynamic, 1)
        for (int h = 0; h < H; ++h) {
            const uint16_t *qh = q + ((int64_t)t * H + h) * Dqk;
            double *o = out + ((int64_t)t * H + h) * Dv;
            if (n == 0) {
                for (int d = 0; d < Dv; ++d) o[d] = 0.0;
                if (lse) lse[(int64_t)t * H + h] = -INFINITY;
                continue;
            }
            double *qv = (double *)malloc(sizeof(double) * (size_t)Dqk);
            double *lg = (double *)malloc(sizeof(double) * (size_t)n);
            for (int d = 0; d < Dqk; ++d) qv[d] = orc_bf16_to_f64(qh[d]);
            double m = -INFINITY;
            for (int j = 0; j < n; ++j) {
                const uint16_t *c = kv_cache + rows[j] * Dqk;
                double dot = 0.0;
                for (int d = 0; d < Dqk; ++d) dot += qv[d] * orc_bf16_to_f64(c[d]);
                lg[j] = sm_scale * dot;
                if (lg[j] > m) m = lg[j];
            }
            double Z = 0.0;
            for (int j = 0; j < n; ++j) { lg[j] = exp(lg[j] - m); Z += lg[j]; }
            for (int d = 0; d < Dv; ++d) o[d] = 0.0;
            for (int j = 0; j < n; ++j) {
                const uint16_t *c = kv_cache + rows[j] * Dqk;
                double p = lg[j] / Z;
                for (int d = 0; d < Dv; ++d) o[d] += p * orc_bf16_to_f64(c[d]);
            }
            double g = orc_bf16_to_f64(gate[(int64_t)t * H + h]);
            double sig = 1.0 / (1.0 + exp(-g));
            for (int d = 0; d < Dv; ++d) o[d] *= sig;
            if (lse) lse[(int64_t)t * H + h] = m + log(Z);
            free(qv); free(lg);
        }
    }
    free(rows);
    return bad ? ORC_EBAD : 0;
}

/* ---- sliding-window attention (decode), the hybrid's local layers ------- */

/* One decode query per sequence b at position L-1 (L = seq_lens[b]) attends
 * causally to the positions [max(0, L-W), L-1] of a ring buffer that keeps
 * position p in slot p % W ([P1] Key Capabilities: SWA with a 128-token
 * window in a 5:1 layout with DSA).  Multi-head attention with as many K/V
 * heads as query heads.  q: bf16 [B,H,D]; k_ring, v_ring: bf16 [B,W,H,D];
 * out: fp64 [B,H,D]. */
int orc_swa_decode(const uint16_t *q, const uint16_t *k_ring,
                   const uint16_t *v_ring, const int32_t *seq_lens, int B,
                   int H, int D, int W, double sm_scale, double *out)
{
    int bad = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] <= 0) bad |= 1;
    if (bad) return ORC_EBAD;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int64_t L = seq_lens[b];
            int64_t p0 = L - W > 0 ? L - W : 0;
            int n = (int)(L - p0);
            double *lg = (double *)malloc(sizeof(double) * (size_t)n);
            const uint16_t *qh = q + ((int64_t)b * H + h) * D;
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                int64_t slot = (p0 + i) % W;
                const uint16_t *k = k_ring + (((int64_t)b * W + slot) * H + h) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += orc_bf16_to_f64(qh[d]) * orc_bf16_to_f64(k[d]);
                lg[i] = sm_scale * dot;
                if (lg[i] > m) m = lg[i];
            }
            double Z = 0.0;
            for (int i = 0; i < n; ++i) { lg[i] = exp(lg[i] - m); Z += lg[i]; }
            double *o = out + ((int64_t)b * H + h) * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int i = 0; i < n; ++i) {
                int64_t slot = (p0 + i) % W;
                const uint16_t *v = v_ring + (((int64_t)b * W + slot) * H + h) * D;
                for (int d = 0; d < D; ++d) o[d] += lg[i] / Z * orc_bf16_to_f64(v[d]);
            }
            free(lg);
        }
    }
    return 0;
}

/* ---- the layer: the three stages in order ---------------------------------- */

/* Indexer -> top-K -> gated attention over the selected rows ([P2]
 * Architecture Breakdown §2: the three components in this order; [P5] §2.1).
 * scores: caller-provided fp32 [T, ld] scratch; idx: int32 [T, K] output;
 * out: fp64 [T, H, Dv]. Row t's candidate count is q_pos[t] + 1. */
int orc_layer_forward(const uint8_t *q_idx, const float *w, const uint8_t *k_cache,
                      const uint16_t *q, const uint16_t *kv_cache,
                      const uint16_t *gate, const int32_t *seq_lens,
                      const int32_t *block_table, int num_seqs, int max_blocks,
                      int page_size, int num_pages, const int32_t *q_seq,
                      const int32_t *q_pos, int T, int HI, int DI, int K, int H,
                      int Dqk, int Dv, double sm_scale, float *scores, int64_t ld,
                      int32_t *idx, double *out)
{
    int rc = orc_indexer_scores(q_idx, w, k_cache, seq_lens, block_table, num_seqs,
                                max_blocks, page_size, num_pages, q_seq, q_pos, T,
                                HI, DI, scores, ld);
    if (rc) return rc;
    int32_t *row_len = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) row_len[t] = q_pos[t] + 1;
    rc = orc_topk(scores, ld, row_len, T, K, idx);
    free(row_len);
    if (rc) return rc;
    return orc_sparse_attn(q, kv_cache, seq_lens, block_table, num_seqs, max_blocks,
                           page_size, num_pages, q_seq, idx, K, gate, sm_scale, T,
                           H, Dqk, Dv, out, NULL);
}
