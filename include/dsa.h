/*
 * dsa.h -- C ABI of libdsa.so, a B200 (sm_100a) implementation of the Gated
 * DeepSeek Sparse Attention (DSA) layer.
 *
 * The layer, as the source pages describe it, has three stages, run in this
 * order for every query token:
 *   1. a lightweight multi-head indexer without rotary embedding scores every
 *      causal history position ("Open-Source LLM Architecture Evolution: How
 *      Lightweight Sparse Attention Reshapes Long-Context Modeling Efficiency",
 *      Architecture Breakdown §2, "Indexer"; "Fine-Grained Sparse Attention in
 *      Ultra-Large Parameter Models", §2.1-§2.3);
 *   2. top-K selection keeps the K = 2048 best positions (same page, "Top-K
 *      selection"; "Open-Sourcing Ultra-Large Sparse Attention Models", §2.2);
 *   3. attention and softmax over only the selected positions ("Open-Source
 *      LLM Architecture Evolution", Technical Deep Dive §2), its output scaled
 *      by a gate ("Gated fusion"; read here as a per-head sigmoid gate).
 * No page writes a formula; this library fixes the score as
 *   I[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])
 * and breaks top-K ties toward the lower position.
 *
 * Conventions (every entry point):
 *  - Pointers marked "device" are CUDA device memory allocated and owned by
 *    the caller; the library never allocates, frees or retains them.
 *  - 8-bit floats are OCP E4M3 ("e4m3fn") bytes; bf16 values travel as their
 *    16-bit patterns (uint16_t).  All arrays are dense row-major.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.  Argument checks
 *    that need only host data run first; on failure nothing is launched.
 *  - Device-side checks (positions past a sequence, page ids out of range,
 *    a pipeline wait that exceeds its time limit) skip the offending access
 *    and set bits in a per-device error word read by dsa_device_error().
 *  - Calls are thread-safe; calls on one stream run in order.
 *  - Shapes outside the supported set return DSA_ERR_UNSUPPORTED; there is no
 *    fallback path.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 2

typedef struct CUstream_st *dsa_stream_t; /* same handle as cudaStream_t */

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer */
    DSA_ERR_UNSUPPORTED = 2, /* shape outside the tuned set */
    DSA_ERR_WORKSPACE = 3,   /* workspace missing or too small */
    DSA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    DSA_ERR_TIMEOUT = 5      /* reported through dsa_device_error() only */
} dsa_status;

/* Device error word bits (dsa_device_error). */
#define DSA_DEVERR_POSITION 0x1u  /* q_pos/idx outside its sequence: row skipped */
#define DSA_DEVERR_PAGE 0x2u      /* block-table entry outside [0, num_pages) */
#define DSA_DEVERR_TIMEOUT 0x4u   /* a pipeline wait hit its time limit */
#define DSA_DEVERR_SHAPE 0x8u     /* a per-row length exceeded its host bound */

/* Paged cache geometry.  A cache is [num_pages, page_size, row] and sequence
 * b's logical position p lives in physical page block_table[b][p / page_size],
 * row p % page_size.  page_size must be 64. */
typedef struct {
    const int32_t *seq_lens;    /* device [num_seqs]: tokens in each sequence */
    const int32_t *block_table; /* device [num_seqs, max_blocks_per_seq] */
    int32_t num_seqs;
    int32_t max_blocks_per_seq;
    int32_t page_size;
    int32_t num_pages;
} dsa_paged;

/* ---- stage 1: indexer scores ------------------------------------------
 * scores[t*ld + s] = sum_h w[t*HI + h] * max(0, sum_d qI[t,h,d] * kI(q_seq[t], s)[d])
 * for 0 <= s <= q_pos[t], where kI(b, s) is row s of sequence b in the paged
 * indexer-key cache.  Scores are fp32 (FP8 products accumulate in fp32);
 * entries s > q_pos[t] are not written.
 *   q_idx       device e4m3 [T, HI, DI]
 *   w           device fp32 [T, HI]    (any sign; model scales folded in)
 *   k_idx_cache device e4m3 [num_pages, 64, DI]; base 16-byte aligned
 *   q_seq,q_pos device int32 [T]; NULL for both means decode: query t is the
 *               last token of sequence t (T == num_seqs, q_pos = seq_len-1)
 *   max_len     host bound: every q_pos[t] < max_len <= ld
 *   scores      device fp32 [T, ld]
 * Supported: HI in {4, 8, 16, 32, 64}, DI in {64, 128}.  Needs no workspace.
 * Performance: with explicit queries, T <= 64, DI = 128 and HI in {16, 32}
 * (several draft tokens per sequence), each run of up to four consecutive
 * queries of one sequence reads that sequence's keys once, so list a
 * sequence's queries next to each other.  Results do not depend on the order. */
dsa_status dsa_indexer_scores(const uint8_t *q_idx, const float *w,
                              const uint8_t *k_idx_cache, const dsa_paged *pg,
                              const int32_t *q_seq, const int32_t *q_pos,
                              int32_t T, int32_t HI, int32_t DI, int32_t max_len,
                              float *scores, int64_t ld, dsa_stream_t stream);

/* ---- stage 1 with MXFP8 operands ------------------------------------------------
 * "Open-Weight Deployment of an Ultra-Large Sparse Model", §1 and §3:
 * activations in MXFP8, read as the OCP microscaling format.  The same score
 * as dsa_indexer_scores with qI = q_idx * 2^(q_scales - 127) and kI =
 * k_idx_cache * 2^(k_scales - 127), one E8M0 scale code per 32 consecutive
 * elements along DI (code 255 is NaN and out of contract):
 *   q_scales device uint8 [T, HI, DI/32]; k_scales device uint8
 *   [num_pages, 64, DI/32] (the key cache's row layout); both 4-byte aligned.
 * Block-scaled tensor-core MMAs; fp32 accumulation.  Supported: DI == 128,
 * HI in {16, 32}, T <= 1024.  Needs no workspace. */
dsa_status dsa_indexer_scores_mx(const uint8_t *q_idx, const uint8_t *q_scales, const float *w,
                                 const uint8_t *k_idx_cache, const uint8_t *k_scales,
                                 const dsa_paged *pg, const int32_t *q_seq, const int32_t *q_pos,
                                 int32_t T, int32_t HI, int32_t DI, int32_t max_len,
                                 float *scores, int64_t ld, dsa_stream_t stream);

/* ---- stage 2: top-K --------------------------------------------------------
 * For each row r: among positions 0 <= s < row_len[r], keep the K largest
 * scores[r*ld + s] under the order (score descending, position ascending),
 * with -0.0 equal to +0.0.  A row with row_len[r] <= K keeps every position.
 * idx[r*K + j] receives the kept positions in ascending order, then -1.
 * Scores must be finite.
 *   row_len     device int32 [R]; every row_len[r] <= max_row_len <= ld
 *   idx         device int32 [R, K]
 *   ws          device scratch of dsa_topk_workspace_bytes(R, K, max_row_len)
 *               bytes, 256-byte aligned; contents need no initialisation.
 * Supported: 1 <= K <= 4096. */
size_t dsa_topk_workspace_bytes(int32_t R, int32_t K, int32_t max_row_len);
dsa_status dsa_topk(const float *scores, int64_t ld, const int32_t *row_len,
                    int32_t R, int32_t K, int32_t max_row_len, int32_t *idx,
                    void *ws, size_t ws_bytes, dsa_stream_t stream);

/* ---- top-K given each row's coarse score histogram -------------------------
 * Same result as dsa_topk, for rows whose scores the caller has already
 * counted by their top 11 key bits (the indexer does this in the layer's
 * decode path): hist[r*2048 + b] = number of positions s < row_len[r] whose
 * key(scores[r*ld + s]) >> 21 == b, where key() maps an fp32 score to an
 * order-preserving uint32 (bits flipped for negatives, sign bit set for
 * non-negatives, -0.0 taken as +0.0).  One launch: every CTA lists the keys
 * of its slice at or above the coarse bin of the K-th largest key, and the
 * last CTA of each row selects among those.  A histogram that does not match
 * the row only makes the call slower (the row is then selected in full).
 *   hist   device uint32 [R, 2048]; read, then set to zero (so a caller that
 *          counts into it again can reuse it)
 *   ws     device scratch of dsa_topk_hist_workspace_bytes(R, max_row_len)
 *          bytes, 256-byte aligned; contents need no initialisation.
 *   scores 16-byte aligned, ld a multiple of 4.
 * Supported: 1 <= K <= 4096. */
size_t dsa_topk_hist_workspace_bytes(int32_t R, int32_t max_row_len);
dsa_status dsa_topk_hist(const float *scores, int64_t ld, const int32_t *row_len,
                         int32_t R, int32_t K, int32_t max_row_len, uint32_t *hist,
                         int32_t *idx, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* ---- top-K with library-owned scratch ---------------------------------------
 * Not described by the source pages: an interface addition for callers that
 * cannot allocate device memory where the selection runs -- an engine whose
 * GPU memory is reserved up front by its own pool (a cudaMalloc would fail or
 * fragment that pool), or a latency-bound decode loop that cannot afford
 * cudaMalloc's implicit device-wide synchronisation.
 * Same result as dsa_topk (same arguments minus the workspace), computed by
 * the multi-CTA selection kernels on a scratch array the library holds in
 * each GPU's memory for the life of the process (DSA_TOPK_STATIC_SCRATCH_BYTES,
 * about 417 KB).  It allocates and frees nothing.
 *  - Limits: R <= DSA_TOPK_STATIC_MAX_ROWS and max_row_len <=
 *    DSA_TOPK_STATIC_MAX_ROW_LEN; larger calls return DSA_ERR_UNSUPPORTED
 *    before launching anything.
 *  - The first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture begins.  A lookup that fails returns
 *    DSA_ERR_CUDA and is tried again by the next call on that device.
 *  - Every call on a device shares the one array, which keeps the previous
 *    call's contents; each call clears what must start at zero.  Calls whose
 *    GPU work overlaps (different streams, no ordering between them) race on
 *    the array and give wrong results: order them on one stream or with
 *    events. */
#define DSA_TOPK_STATIC_MAX_ROWS 16
#define DSA_TOPK_STATIC_MAX_ROW_LEN 1048576
#define DSA_TOPK_STATIC_SCRATCH_BYTES 426496
dsa_status dsa_topk_static(const float *scores, int64_t ld, const int32_t *row_len,
                           int32_t R, int32_t K, int32_t max_row_len, int32_t *idx,
                           dsa_stream_t stream);

/* ---- stage 3: gated attention over the selected latent rows ----------------
 * For query t, head h, and the selected rows c_j = latent row idx[t*K + j] of
 * sequence q_seq[t] (entries < 0 are padding):
 *   l_j = sm_scale * (q[t,h,:Dqk] . c_j[:Dqk]),  p = softmax_j(l),
 *   out[t,h,:] = bf16( sigmoid(gate[t,h]) * sum_j p_j c_j[:Dv] ).
 * All H heads share the latent row (key = its first Dqk entries, value = its
 * first Dv).  A query with no valid entry gets out = 0 (and lse = -inf).
 *   q        device bf16 [T, H, Dqk]; kv_cache device bf16 [num_pages, 64, Dqk]
 *   q_seq    device int32 [T], or NULL for decode (query t -> sequence t)
 *   gate     device bf16 [T, H];  out device bf16 [T, H, Dv]
 *   lse      device fp32 [T, H] or NULL: natural-log sum of exp(l_j)
 *   ws       dsa_sparse_attn_workspace_bytes(T, H, K, Dv) bytes (may be 0)
 * Supported: (Dqk, Dv) in {(576, 512), (64, 64)}, 1 <= H <= 128,
 * K a multiple of 64, K <= 4096.  Buffers 16-byte aligned. */
size_t dsa_sparse_attn_workspace_bytes(int32_t T, int32_t H, int32_t K, int32_t Dv);
dsa_status dsa_sparse_attn(const uint16_t *q, const uint16_t *kv_cache,
                           const dsa_paged *pg, const int32_t *q_seq,
                           const int32_t *idx, int32_t K, const uint16_t *gate,
                           float sm_scale, int32_t T, int32_t H, int32_t Dqk,
                           int32_t Dv, uint16_t *out, float *lse, void *ws,
                           size_t ws_bytes, dsa_stream_t stream);

/* ---- the layer ----------------------------------------------------------------
 * Runs stage 1 -> 2 -> 3 on one stream.  Prefill: T query tokens with explicit
 * q_seq/q_pos.  Decode: one query per sequence at position seq_len-1
 * (q_seq/q_pos ignored, T == pg.num_seqs).  Row t's candidate count is
 * q_pos[t] + 1. */
enum { DSA_MODE_PREFILL = 0, DSA_MODE_DECODE = 1 };

typedef struct {
    int32_t mode;
    const uint8_t *q_idx;       /* device e4m3 [T, HI, DI] */
    const float *w;             /* device fp32 [T, HI] */
    const uint8_t *k_idx_cache; /* device e4m3 [num_pages, 64, DI] */
    const uint16_t *q;          /* device bf16 [T, H, Dqk] */
    const uint16_t *kv_cache;   /* device bf16 [num_pages, 64, Dqk] */
    const uint16_t *gate;       /* device bf16 [T, H] */
    dsa_paged pg;
    const int32_t *q_seq;       /* device int32 [T] (prefill) */
    const int32_t *q_pos;       /* device int32 [T] (prefill) */
    int32_t T, HI, DI, K, H, Dqk, Dv;
    int32_t max_len;            /* host bound on q_pos+1 (prefill) / seq_lens (decode) */
    float sm_scale;
    uint16_t *out;              /* device bf16 [T, H, Dv] */
    int32_t *idx_out;           /* device int32 [T, K] or NULL */
    float *lse;                 /* device fp32 [T, H] or NULL */
    /* MXFP8 indexer operands (dsa_indexer_scores_mx): both NULL for per-tensor
     * FP8, or both set (DI == 128, HI in {16, 32}, T <= 1024) */
    const uint8_t *q_idx_scales; /* device uint8 [T, HI, DI/32] */
    const uint8_t *k_idx_scales; /* device uint8 [num_pages, 64, DI/32] */
} dsa_layer_args;

/* Workspace: (decode, or T <= 64) a per-query histogram of the indexer scores, then the
 * fp32 scores [T, max_len] (+ idx if idx_out is NULL) + top-K scratch
 * (dsa_topk_hist_workspace_bytes when the histogram is there, else
 * dsa_topk_workspace_bytes) + split-K attention partials.  Decode calls (and calls with T <= 64, such as
 * several draft tokens per sequence) leave the histogram region zeroed and
 * take a faster top-K when they find it zeroed, so reusing one workspace
 * (zero-filled once, or simply reused after a first call) across such calls
 * is the fast arrangement; any other contents only cost a slower top-K. */
size_t dsa_layer_workspace_bytes(const dsa_layer_args *a);
dsa_status dsa_layer_forward(const dsa_layer_args *a, void *ws, size_t ws_bytes,
                             dsa_stream_t stream);

/* dsa_layer_forward that also records caller-created CUDA events (cudaEvent_t
 * handles; NULL entries are skipped) on `stream`: events[0] before the
 * indexer, events[1] after it, events[2] after top-K, events[3] after the
 * attention.  Same work, same launches; for timing the stages in place. */
dsa_status dsa_layer_forward_profiled(const dsa_layer_args *a, void *ws, size_t ws_bytes,
                                      void *const events[4], dsa_stream_t stream);

/* Number of kernels dsa_layer_forward launches for these arguments (host
 * only; the top-K scratch reset is a memset and is not counted). */
int32_t dsa_layer_kernel_launches(const dsa_layer_args *a);

/* ---- sliding-window decode (the hybrid's local layers) ------------------------
 * "aiany.app item naive-n0-5-flash", Key Capabilities: 5 sliding-window
 * layers (window 128) per DSA layer.  Sequence b's query (position
 * L-1, L = seq_lens[b]) attends causally to positions [max(0, L-window), L-1],
 * stored in ring slot p % window; multi-head with H K/V heads.
 *   q device bf16 [B, H, D]; k_ring, v_ring device bf16 [B, window, H, D];
 *   out device bf16 [B, H, D].  Supported: D == 128, window == 128, H % 8 == 0. */
dsa_status dsa_swa_decode(const uint16_t *q, const uint16_t *k_ring,
                          const uint16_t *v_ring, const int32_t *seq_lens,
                          int32_t B, int32_t H, int32_t D, int32_t window,
                          float sm_scale, uint16_t *out, dsa_stream_t stream);

/* ---- the step before the layer: new tokens into the paged caches ---------------
 * The indexer keys are stored as FP8 ("aiany.app item naive-n0-5-flash", Key
 * Capabilities: FP8; "Open-Weight Deployment of an Ultra-Large Sparse Model",
 * §1: FP8/MXFP8 activations; one scale per tensor here).  For each new token
 * j, at logical position tok_pos[j] of sequence tok_seq[j] (through the block
 * table; the position must already be counted in seq_lens):
 *   k_idx_cache row = e4m3(fp32(k_new[j, d]) * k_scale), the product rounded
 *                     once to the nearest code, ties to the even mantissa,
 *                     magnitudes of 448 and above saturating to +-448;
 *   kv_cache row    = latent_new[j, :] unchanged (skipped when latent_new is NULL).
 *   k_new       device bf16 [n, DI];  latent_new device bf16 [n, Dqk] or NULL
 *   tok_seq,tok_pos device int32 [n]
 *   k_idx_cache device e4m3 [num_pages, 64, DI]; kv_cache device bf16 [num_pages, 64, Dqk]
 * A position outside its sequence, or a page outside [0, num_pages), skips
 * that token and sets DSA_DEVERR_POSITION / DSA_DEVERR_PAGE.  Tokens must go to
 * distinct rows.  Supported: DI in {64, 128}; Dqk a multiple of 8, at most 768.  Buffers
 * 16-byte aligned.  Needs no workspace. */
dsa_status dsa_append_kv(const uint16_t *k_new, float k_scale, const uint16_t *latent_new,
                         const int32_t *tok_seq, const int32_t *tok_pos, const dsa_paged *pg,
                         int32_t n, int32_t DI, int32_t Dqk, uint8_t *k_idx_cache,
                         uint16_t *kv_cache, dsa_stream_t stream);

/* ---- context-parallel decode: one long sequence over G GPUs -----------------------
 * "Fine-Grained Sparse Attention in Ultra-Large Parameter Models", §1
 * (1,048,576-token context); "Open-Weight Deployment of an Ultra-Large Sparse
 * Model", §3 (multi-card deployment).  The pages describe no split; this one
 * deals every sequence's pages out in G contiguous runs of whole pages, rank r
 * holding positions [lo[b], hi[b]) of sequence b.  Per rank, per decode step:
 *   1. dsa_indexer_scores and dsa_topk over the rank's own pages (a paged view
 *      whose seq_lens are hi - lo and whose block table starts at page lo/64),
 *      giving local scores and local indices;
 *   2. dsa_cp_candidates: (score, global position) of each kept local index;
 *   3. the caller all-gathers the G ranks' [B, K] candidate blocks (NCCL) into
 *      [G, B, K] arrays, rank order;
 *   4. dsa_cp_select: the K best of the G*K candidates of each sequence under
 *      the top-K's order -- exactly the one-GPU selection, since a position
 *      among the K best of the history is among the K best of its own range --
 *      as global positions (ascending, -1 padded) and as this rank's local
 *      indices (position - lo, -1 where another rank holds the row);
 *   5. dsa_sparse_attn over the local indices with lse: the rank's gated
 *      partial output and log-sum-exp (-inf where it holds no kept row);
 *   6. the caller all-gathers o [G, B, H, Dv] and lse [G, B, H];
 *   7. dsa_cp_lse_merge: out = sum_r w_r o_r / sum_r w_r, w_r = exp(lse_r -
 *      max lse), over the ranks that hold a kept row.  (The gate is the same
 *      factor in every rank's term.)
 * All pointers are device memory; all calls are stream-ordered. */
/*   scores [B, ld] local scores; idx_local [B, K] dsa_topk output; lo device int32 [B];
 *   cand_score fp32 [B, K], cand_pos int32 [B, K] (padding: -inf, -1). */
dsa_status dsa_cp_candidates(const float *scores, int64_t ld, const int32_t *idx_local,
                             int32_t B, int32_t K, const int32_t *lo, float *cand_score,
                             int32_t *cand_pos, dsa_stream_t stream);
/*   cand_score, cand_pos [G, B, K] (every rank's candidates, rank order); lo, hi
 *   device int32 [B] (this rank's range); idx_global, idx_local int32 [B, K];
 *   ws of dsa_cp_select_workspace_bytes(G, B, K) bytes, 256-byte aligned.
 *   Supported: K <= 4096, G * K <= 2^24. */
size_t dsa_cp_select_workspace_bytes(int32_t G, int32_t B, int32_t K);
dsa_status dsa_cp_select(const float *cand_score, const int32_t *cand_pos, int32_t G,
                         int32_t B, int32_t K, const int32_t *lo, const int32_t *hi,
                         int32_t *idx_global, int32_t *idx_local, void *ws, size_t ws_bytes,
                         dsa_stream_t stream);
/*   o bf16 [G, B, H, Dv], lse fp32 [G, B, H]; out bf16 [B, H, Dv].  Dv % 8 == 0,
 *   o and out 16-byte aligned. */
dsa_status dsa_cp_lse_merge(const uint16_t *o, const float *lse, int32_t G, int32_t B,
                            int32_t H, int32_t Dv, uint16_t *out, dsa_stream_t stream);

/* ---- the step before the layer, MXFP8 keys -------------------------------------------
 * As dsa_append_kv, with the indexer keys stored in MXFP8 ("Open-Weight
 * Deployment of an Ultra-Large Sparse Model", §1 and §3), read as the OCP
 * microscaling format: each 32 consecutive elements x of a key row share the
 * scale code c = clamp(floor(log2 max|x|) - 8, -127, 127) + 127 (an all-zero
 * block: c = 0), stored in k_scales at the row's position; the elements
 * become e4m3(x * 2^(127 - c)), to the nearest code with ties to the even
 * mantissa, saturating to +-448.
 *   k_scales device uint8 [num_pages, 64, DI/32].  Supported: DI in {64, 128};
 *   Dqk a multiple of 8, at most 768.  Needs no workspace. */
dsa_status dsa_append_kv_mx(const uint16_t *k_new, const uint16_t *latent_new,
                            const int32_t *tok_seq, const int32_t *tok_pos, const dsa_paged *pg,
                            int32_t n, int32_t DI, int32_t Dqk, uint8_t *k_idx_cache,
                            uint8_t *k_scales, uint16_t *kv_cache, dsa_stream_t stream);

/* ---- testing the bounded waits ------------------------------------------------------
 * Every pipeline wait in the kernels gives up after a time limit (1 s),
 * records DSA_DEVERR_TIMEOUT, lets the CTA's other roles abandon their work,
 * waits (again with a limit) for its own copies in flight, frees its tensor
 * memory and returns.  For testing that path without any fault: while `tile`
 * >= 0, every later launch of the decode indexer (the layer's decode mode and
 * dsa_indexer_scores without q_seq) leaves flattened tile `tile` -- the
 * queries' 128-key tiles in order -- unfilled, so the wait on it runs out;
 * that launch's scores are then incomplete.  -1 turns it off (the default).
 * Host-side setting, all devices. */
dsa_status dsa_test_skip_indexer_tile(int64_t tile);

/* ---- housekeeping ---------------------------------------------------------------- */
const char *dsa_status_string(dsa_status s);
int32_t dsa_abi_version(void);
/* Synchronously reads (and, if reset != 0, clears) the current device's error
 * word; *code receives DSA_DEVERR_* bits, 0 when all is well. */
dsa_status dsa_device_error(uint32_t *code, int32_t reset);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
