// Host-side interfaces between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;
    uint32_t *err = nullptr;  // device address of the error word
};

// Cached per-device facts for the current device (thread-safe).
const DeviceInfo *current_device();

// Builds a 2-D tiled tensor map: `inner` elements of `elem_bytes` per row,
// `outer` rows `row_bytes` apart, box [box_inner, box_outer].
bool make_tmap_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// Builds a 3-D tiled tensor map: dims[0] elements of `elem_bytes` innermost,
// then dims[1] rows `stride1` bytes apart, then dims[2] planes `stride2` bytes
// apart; box [box0, box1, box2].
bool make_tmap_3d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, const uint64_t dims[3], uint64_t stride1,
                  uint64_t stride2, const uint32_t box[3], CUtensorMapSwizzle swz);

// Raises the dynamic shared-memory limit of `fn` once per device.
bool ensure_smem(const void *fn, int bytes);

struct PagedDev {
    const int32_t *seq_lens;
    const int32_t *block_table;
    int32_t num_seqs, max_blocks, num_pages;
};

// ---- indexer ---------------------------------------------------------------
struct IndexerArgs {
    const uint8_t *q_idx;
    const float *w;
    const uint8_t *k_cache;
    PagedDev pg;
    const int32_t *q_seq;  // NULL => decode convention
    const int32_t *q_pos;
    int32_t T, HI, DI, max_len;
    float *scores;
    int64_t ld;
    // optional (few-query kernels only): per-query histogram [T][SCORE_HIST_BINS]
    // of score_key(score) >> SCORE_HIST_SHIFT, added to (it must hold zeros)
    uint32_t *hist;
    // optional: words the kernel sets to zero before it ends (the counters
    // of the top-K that follows it)
    uint32_t *zero;
    int64_t nzero;
};
constexpr int SCORE_HIST_BINS = 2048;
constexpr int SCORE_HIST_SHIFT = 21;
dsa_status launch_indexer(const IndexerArgs &a, cudaStream_t st);
// Few explicit queries (T <= 64, 16 or 32 heads x 128): consecutive queries of
// one sequence share each key tile.  launch_indexer routes them here.
bool indexer_group_eligible(const IndexerArgs &a);
// The flattened tile (all queries' 128-key tiles in order) that later
// decode-indexer launches leave unfilled, -1 = none: dsa_test_skip_indexer_tile.
int64_t test_skip_tile();
// MXFP8 operands: E8M0 scales, q_scales [T, HI, DI/32], k_scales [pages, 64, DI/32]
// (DI = 128, HI in {16, 32}).
dsa_status launch_indexer_mx(const IndexerArgs &a, const uint8_t *q_scales, const uint8_t *k_scales,
                             cudaStream_t st);
dsa_status launch_indexer_group(const IndexerArgs &a, cudaStream_t st);

// ---- top-K ---------------------------------------------------------------------
enum RowLenMode : int32_t { ROWLEN_ARRAY = 0, ROWLEN_QPOS_PLUS_1 = 1, ROWLEN_SEQ_LENS = 2 };
struct TopkArgs {
    const float *scores;
    int64_t ld;
    const int32_t *row_len;  // meaning per mode
    int32_t mode;
    int32_t R, K, max_row_len;
    int32_t *idx;
    void *ws;
    size_t ws_bytes;
    bool pdl;  // launched as a programmatic dependent of the previous kernel
    // optional: the indexer's per-row histogram of score_key >> SCORE_HIST_SHIFT
    // ([R][SCORE_HIST_BINS]); read, then cleared to zeros for the next call
    uint32_t *hist;
};
size_t topk_workspace_bytes(int32_t R, int32_t K, int32_t max_row_len);
int topk_kernel_launches(int32_t R, int32_t K, int32_t max_row_len);
// Few rows that each fit one large thread-block cluster (10 or 16 CTAs, all
// clusters resident at once): the cluster kernel, which also reads the
// indexer's histogram, selects faster than the single-launch list-and-ticket
// kernel; longer rows and many rows go to the latter.
bool topk_prefers_cluster(int32_t R, int32_t max_row_len);
dsa_status launch_topk(const TopkArgs &a, cudaStream_t st);
dsa_status launch_topk_static(const TopkArgs &a, cudaStream_t st);
// Top-K from the indexer's per-row histogram (a.hist set): one launch, every
// CTA lists its slice's keys at or above the threshold's coarse bin, the
// last CTA of each row (atomic ticket) selects.  a.ws is its workspace, whose
// first topk_hist_zero_words(R) words (fine counts and tickets) must be zero
// at launch: the indexer zeroes them (IndexerArgs::zero), and the top-K
// leaves them zeroed.
struct HistTopkPlan {
    int S, slice;  // CTAs per row, keys per CTA
};
HistTopkPlan topk_hist_plan(int32_t R, int32_t max_row_len);
size_t topk_hist_workspace_bytes(int32_t R, int32_t max_row_len);
int64_t topk_hist_zero_words(int32_t R);
dsa_status launch_topk_hist(const TopkArgs &a, cudaStream_t st);
// Many rows (R >= 2 x SMs), each at most 32768 keys long, K <= 2048: one
// 256-thread CTA per row lists its likely candidates in shared memory and
// selects from there.  No workspace.
bool topk_rows_eligible(int32_t R, int32_t K, int32_t max_row_len);
dsa_status launch_topk_rows(const TopkArgs &a, cudaStream_t st);

// ---- gated sparse attention ----------------------------------------------------
struct AttnArgs {
    const uint16_t *q;
    const uint16_t *kv;
    PagedDev pg;
    const int32_t *q_seq;  // NULL => query t reads sequence t
    const int32_t *idx;
    int32_t K;
    const uint16_t *gate;
    float sm_scale;
    int32_t T, H, Dqk, Dv;
    uint16_t *out;
    float *lse;
    void *ws;
    size_t ws_bytes;
    bool pdl;  // launched as a programmatic dependent of the previous kernel
};
size_t attn_workspace_bytes(int32_t T, int32_t H, int32_t K, int32_t Dv);
int attn_kernel_launches(int32_t T, int32_t K, int32_t Dv);
dsa_status launch_attn(const AttnArgs &a, cudaStream_t st);

// ---- sliding-window decode -------------------------------------------------------
struct SwaArgs {
    const uint16_t *q, *k_ring, *v_ring;
    const int32_t *seq_lens;
    int32_t B, H, D, W;
    float sm_scale;
    uint16_t *out;
};
dsa_status launch_swa(const SwaArgs &a, cudaStream_t st);

// ---- the append step (new tokens into the paged caches) -----------------------------
struct AppendArgs {
    const uint16_t *k_new;       // bf16 [n, DI]
    const uint16_t *latent_new;  // bf16 [n, Dqk] or NULL
    const int32_t *tok_seq, *tok_pos;
    PagedDev pg;
    int32_t n, DI, Dqk;
    float k_scale;
    uint8_t *k_cache;
    uint16_t *kv_cache;
};
dsa_status launch_append(const AppendArgs &a, cudaStream_t st);
// MXFP8 keys: codes into k_cache, one E8M0 scale per 32 elements into k_scales [pages, 64, DI/32].
dsa_status launch_append_mx(const AppendArgs &a, uint8_t *k_scales, cudaStream_t st);

// ---- context-parallel decode: joining the ranks' partial results -----------------
dsa_status launch_cp_candidates(const float *scores, int64_t ld, const int32_t *idx, int B, int K, const int32_t *lo,
                                float *cs, int32_t *cpos, cudaStream_t st);
size_t cp_select_workspace_bytes(int G, int B, int K);
dsa_status launch_cp_select(const float *cs, const int32_t *cpos, int G, int B, int K, const int32_t *lo,
                            const int32_t *hi, int32_t *idx_g, int32_t *idx_l, void *ws, size_t ws_bytes,
                            cudaStream_t st);
dsa_status launch_cp_merge(const uint16_t *o, const float *lse, int G, int B, int H, int Dv, uint16_t *out,
                           cudaStream_t st);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace dsa
