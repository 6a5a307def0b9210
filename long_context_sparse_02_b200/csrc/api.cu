// C ABI of libdsa.so: argument checks, workspace carving and kernel choice.
// Everything that computes runs in the kernels of indexer.cu, topk.cu,
// attn.cu and swa.cu; this file only validates and launches.
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "dsa.h"
#include "dsa_internal.h"

// Per-device error word (DSA_DEVERR_* bits), set by kernels, read by
// dsa_device_error().
__device__ uint32_t g_dsa_device_error;

namespace dsa {

namespace {
constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
DeviceInfo g_dev[kMaxDevices];

std::mutex g_smem_mu;
std::vector<std::pair<const void *, int>> g_smem_done;  // (kernel, device)

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiled g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

namespace {
std::atomic<int64_t> g_test_skip_tile{-1};
}
int64_t test_skip_tile() { return g_test_skip_tile.load(std::memory_order_relaxed); }

const DeviceInfo *current_device() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return nullptr;
    std::call_once(g_dev_once[d], [d] {
        DeviceInfo &di = g_dev[d];
        void *p = nullptr;
        if (cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return;
        if (cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess)
            return;
        if (cudaGetSymbolAddress(&p, g_dsa_device_error) != cudaSuccess) return;
        di.err = static_cast<uint32_t *>(p);
        di.device = d;
    });
    return g_dev[d].device == d ? &g_dev[d] : nullptr;
}

bool ensure_smem(const void *fn, int bytes) {
    const DeviceInfo *dev = current_device();
    if (!dev || bytes > dev->max_smem_optin) return false;
    std::lock_guard<std::mutex> lk(g_smem_mu);
    for (auto &e : g_smem_done)
        if (e.first == fn && e.second == dev->device) return true;
    // Raise the limit once to the device maximum less the kernel's static
    // shared memory, so later calls with a larger request need no new
    // attribute call.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return false;
    const int limit = dev->max_smem_optin - (int)fa.sharedSizeBytes;
    if (bytes > limit || cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, limit) != cudaSuccess)
        return false;
    g_smem_done.emplace_back(fn, dev->device);
    return true;
}

bool make_tmap_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiled>(fn);
    });
    if (!g_encode || !aligned16(base) || (row_bytes & 15u) || inner == 0 || outer == 0) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, const uint64_t dims[3], uint64_t stride1,
                  uint64_t stride2, const uint32_t box[3], CUtensorMapSwizzle swz) {
    CUtensorMap probe;
    if (!make_tmap_2d(&probe, base, dt, dims[0], dims[1], stride1, box[0], box[1], swz)) return false;  // loads the encoder
    if ((stride2 & 15u) || dims[2] == 0) return false;
    cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t b[3] = {box[0], box[1], box[2]};
    cuuint32_t estr[3] = {1, 1, 1};
    return g_encode(m, dt, 3, const_cast<void *>(base), d, strides, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dsa

using namespace dsa;

namespace {

bool paged_ok(const dsa_paged *pg) {
    return pg && pg->seq_lens && pg->block_table && pg->num_seqs > 0 && pg->max_blocks_per_seq > 0 &&
           pg->page_size == 64 && pg->num_pages > 0;
}

PagedDev paged_dev(const dsa_paged *pg) {
    return PagedDev{pg->seq_lens, pg->block_table, pg->num_seqs, pg->max_blocks_per_seq, pg->num_pages};
}

bool hi_ok(int HI) { return HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64; }
bool attn_shape_ok(int Dqk, int Dv) { return (Dqk == 576 && Dv == 512) || (Dqk == 64 && Dv == 64); }

size_t ld_of(int32_t max_len) { return align_up((size_t)max_len, 4); }

struct LayerWs {
    uint32_t *score_hist;  // decode: the indexer's per-query score histogram (kept zeroed between calls)
    float *scores;
    int32_t *idx;
    void *topk_ws;
    size_t topk_bytes;
    void *attn_ws;
    size_t attn_bytes;
    size_t total;
};

// The indexer counts the scores by their top key bits for the top-K whenever
// it runs its few-query kernel: decode, or up to 64 explicit queries (several
// draft tokens per sequence, as in speculative decoding).
bool hist_mode(const dsa_layer_args *a) { return a->mode == DSA_MODE_DECODE || a->T <= 64; }

LayerWs carve_layer(const dsa_layer_args *a, void *ws) {
    LayerWs w{};
    uint8_t *p = static_cast<uint8_t *>(ws);
    size_t off = 0;
    if (hist_mode(a)) {
        w.score_hist = reinterpret_cast<uint32_t *>(p + off);
        off += align_up((size_t)a->T * SCORE_HIST_BINS * 4, 256);
    }
    w.scores = reinterpret_cast<float *>(p + off);
    off += align_up((size_t)a->T * ld_of(a->max_len) * 4, 256);
    if (!a->idx_out) {
        w.idx = reinterpret_cast<int32_t *>(p + off);
        off += align_up((size_t)a->T * a->K * 4, 256);
    } else {
        w.idx = a->idx_out;
    }
    // with the indexer's histogram the top-K lists candidates in a workspace of
    // its own (its per-row tickets first); otherwise the plain top-K's
    w.topk_bytes = hist_mode(a) ? topk_hist_workspace_bytes(a->T, a->max_len)
                                : topk_workspace_bytes(a->T, a->K, a->max_len);
    w.topk_ws = w.topk_bytes ? p + off : nullptr;
    off += w.topk_bytes;
    w.attn_bytes = attn_workspace_bytes(a->T, a->H, a->K, a->Dv);
    w.attn_ws = w.attn_bytes ? p + off : nullptr;
    off += w.attn_bytes;
    w.total = off;
    return w;
}

}  // namespace

extern "C" {

int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

dsa_status dsa_test_skip_indexer_tile(int64_t tile) {
    if (tile < -1) return DSA_ERR_INVALID_ARG;
    g_test_skip_tile.store(tile, std::memory_order_relaxed);
    return DSA_OK;
}

const char *dsa_status_string(dsa_status s) {
    switch (s) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported shape";
        case DSA_ERR_WORKSPACE: return "workspace missing or too small";
        case DSA_ERR_CUDA: return "CUDA error";
        case DSA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

dsa_status dsa_device_error(uint32_t *code, int32_t reset) {
    if (!code) return DSA_ERR_INVALID_ARG;
    if (!current_device()) return DSA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(code, g_dsa_device_error, sizeof(uint32_t)) != cudaSuccess) return DSA_ERR_CUDA;
    if (reset) {
        const uint32_t z = 0;
        if (cudaMemcpyToSymbol(g_dsa_device_error, &z, sizeof(uint32_t)) != cudaSuccess) return DSA_ERR_CUDA;
    }
    return DSA_OK;
}

dsa_status dsa_indexer_scores(const uint8_t *q_idx, const float *w, const uint8_t *k_idx_cache, const dsa_paged *pg,
                              const int32_t *q_seq, const int32_t *q_pos, int32_t T, int32_t HI, int32_t DI,
                              int32_t max_len, float *scores, int64_t ld, dsa_stream_t stream) {
    if (T < 0 || !paged_ok(pg) || max_len < 1 || ld < max_len) return DSA_ERR_INVALID_ARG;
    if ((q_seq == nullptr) != (q_pos == nullptr)) return DSA_ERR_INVALID_ARG;
    if (!q_seq && T > pg->num_seqs) return DSA_ERR_INVALID_ARG;
    if (!hi_ok(HI) || (DI != 64 && DI != 128)) return DSA_ERR_UNSUPPORTED;
    if (T == 0) return DSA_OK;
    if (!q_idx || !w || !k_idx_cache || !scores) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx_cache)) return DSA_ERR_INVALID_ARG;
    IndexerArgs a{q_idx, w, k_idx_cache, paged_dev(pg), q_seq, q_pos, T, HI, DI, max_len, scores, ld};
    return launch_indexer(a, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_indexer_scores_mx(const uint8_t *q_idx, const uint8_t *q_scales, const float *w,
                                 const uint8_t *k_idx_cache, const uint8_t *k_scales, const dsa_paged *pg,
                                 const int32_t *q_seq, const int32_t *q_pos, int32_t T, int32_t HI, int32_t DI,
                                 int32_t max_len, float *scores, int64_t ld, dsa_stream_t stream) {
    if (T < 0 || !paged_ok(pg) || max_len < 1 || ld < max_len) return DSA_ERR_INVALID_ARG;
    if ((q_seq == nullptr) != (q_pos == nullptr)) return DSA_ERR_INVALID_ARG;
    if (!q_seq && T > pg->num_seqs) return DSA_ERR_INVALID_ARG;
    if ((HI != 16 && HI != 32) || DI != 128 || T > 1024) return DSA_ERR_UNSUPPORTED;
    if (T == 0) return DSA_OK;
    if (!q_idx || !q_scales || !w || !k_idx_cache || !k_scales || !scores) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx_cache) || (reinterpret_cast<uintptr_t>(q_scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(k_scales) & 3u))
        return DSA_ERR_INVALID_ARG;
    IndexerArgs a{q_idx, w, k_idx_cache, paged_dev(pg), q_seq, q_pos, T, HI, DI, max_len, scores, ld};
    return launch_indexer_mx(a, q_scales, k_scales, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_topk_workspace_bytes(int32_t R, int32_t K, int32_t max_row_len) {
    if (R <= 0 || K <= 0 || max_row_len <= 0) return 0;
    return topk_workspace_bytes(R, K, max_row_len);
}

dsa_status dsa_topk(const float *scores, int64_t ld, const int32_t *row_len, int32_t R, int32_t K,
                    int32_t max_row_len, int32_t *idx, void *ws, size_t ws_bytes, dsa_stream_t stream) {
    if (R < 0 || K < 1 || max_row_len < 1 || ld < max_row_len) return DSA_ERR_INVALID_ARG;
    if (K > 4096) return DSA_ERR_UNSUPPORTED;
    if (R == 0) return DSA_OK;
    if (!scores || !row_len || !idx) return DSA_ERR_INVALID_ARG;
    TopkArgs a{scores, ld, row_len, ROWLEN_ARRAY, R, K, max_row_len, idx, ws, ws_bytes};
    return launch_topk(a, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk_static(const float *scores, int64_t ld, const int32_t *row_len, int32_t R, int32_t K,
                           int32_t max_row_len, int32_t *idx, dsa_stream_t stream) {
    if (R < 0 || K < 1 || max_row_len < 1 || ld < max_row_len) return DSA_ERR_INVALID_ARG;
    if (K > 4096 || R > DSA_TOPK_STATIC_MAX_ROWS || max_row_len > DSA_TOPK_STATIC_MAX_ROW_LEN)
        return DSA_ERR_UNSUPPORTED;
    if (R == 0) return DSA_OK;
    if (!scores || !row_len || !idx) return DSA_ERR_INVALID_ARG;
    TopkArgs a{scores, ld, row_len, ROWLEN_ARRAY, R, K, max_row_len, idx, nullptr, 0};
    return launch_topk_static(a, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_topk_hist_workspace_bytes(int32_t R, int32_t max_row_len) {
    if (R <= 0 || max_row_len <= 0) return 0;
    return topk_hist_workspace_bytes(R, max_row_len);
}

dsa_status dsa_topk_hist(const float *scores, int64_t ld, const int32_t *row_len, int32_t R, int32_t K,
                         int32_t max_row_len, uint32_t *hist, int32_t *idx, void *ws, size_t ws_bytes,
                         dsa_stream_t stream) {
    if (R < 0 || K < 1 || max_row_len < 1 || ld < max_row_len) return DSA_ERR_INVALID_ARG;
    if (K > 4096) return DSA_ERR_UNSUPPORTED;
    if (R == 0) return DSA_OK;
    if (!scores || !row_len || !hist || !idx || !aligned16(scores) || (ld & 3)) return DSA_ERR_INVALID_ARG;
    const size_t need = topk_hist_workspace_bytes(R, max_row_len);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return DSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the counters at the head of the workspace start at zero
    if (cudaMemsetAsync(ws, 0, (size_t)topk_hist_zero_words(R) * 4, st) != cudaSuccess) return DSA_ERR_CUDA;
    TopkArgs a{scores, ld, row_len, ROWLEN_ARRAY, R, K, max_row_len, idx, ws, ws_bytes};
    a.hist = hist;
    return launch_topk_hist(a, st);
}

size_t dsa_sparse_attn_workspace_bytes(int32_t T, int32_t H, int32_t K, int32_t Dv) {
    if (T <= 0 || H <= 0 || K < 64) return 0;
    return attn_workspace_bytes(T, H, K, Dv);
}

dsa_status dsa_sparse_attn(const uint16_t *q, const uint16_t *kv_cache, const dsa_paged *pg, const int32_t *q_seq,
                           const int32_t *idx, int32_t K, const uint16_t *gate, float sm_scale, int32_t T, int32_t H,
                           int32_t Dqk, int32_t Dv, uint16_t *out, float *lse, void *ws, size_t ws_bytes,
                           dsa_stream_t stream) {
    if (T < 0 || !paged_ok(pg) || !isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
    if (!q_seq && T > pg->num_seqs) return DSA_ERR_INVALID_ARG;
    if (!attn_shape_ok(Dqk, Dv) || H < 1 || H > 128 || K < 64 || K > 4096 || K % 64) return DSA_ERR_UNSUPPORTED;
    if (T == 0) return DSA_OK;
    if (!q || !kv_cache || !idx || !gate || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    AttnArgs a{q, kv_cache, paged_dev(pg), q_seq, idx, K, gate, sm_scale, T, H, Dqk, Dv, out, lse, ws, ws_bytes};
    return launch_attn(a, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_layer_workspace_bytes(const dsa_layer_args *a) {
    if (!a || a->T <= 0 || a->max_len < 1 || a->K < 1) return 0;
    return carve_layer(a, nullptr).total;
}

}  // extern "C"

namespace {
dsa_status layer_forward(const dsa_layer_args *a, void *ws, size_t ws_bytes, dsa_stream_t stream,
                         void *const *events) {
    auto mark = [&](int i) {
        if (events && events[i])
            return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess;
        return true;
    };
    if (!a) return DSA_ERR_INVALID_ARG;
    const bool decode = a->mode == DSA_MODE_DECODE;
    if (!decode && a->mode != DSA_MODE_PREFILL) return DSA_ERR_INVALID_ARG;
    if (a->T < 0 || a->max_len < 1 || !paged_ok(&a->pg) || !isfinite(a->sm_scale)) return DSA_ERR_INVALID_ARG;
    if (decode && a->T != a->pg.num_seqs) return DSA_ERR_INVALID_ARG;
    if (!decode && (!a->q_seq || !a->q_pos)) return DSA_ERR_INVALID_ARG;
    if (!hi_ok(a->HI) || (a->DI != 64 && a->DI != 128) || !attn_shape_ok(a->Dqk, a->Dv) || a->H < 1 || a->H > 128 ||
        a->K < 64 || a->K > 4096 || a->K % 64)
        return DSA_ERR_UNSUPPORTED;
    if (a->T == 0) return DSA_OK;
    if (!a->q_idx || !a->w || !a->k_idx_cache || !a->q || !a->kv_cache || !a->gate || !a->out)
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(a->q_idx) || !aligned16(a->k_idx_cache) || !aligned16(a->q) || !aligned16(a->kv_cache) ||
        !aligned16(a->out))
        return DSA_ERR_INVALID_ARG;
    const bool mx = a->q_idx_scales || a->k_idx_scales;
    if (mx && (!a->q_idx_scales || !a->k_idx_scales)) return DSA_ERR_INVALID_ARG;
    if (mx && (a->DI != 128 || (a->HI != 16 && a->HI != 32) || a->T > 1024)) return DSA_ERR_UNSUPPORTED;
    LayerWs lw = carve_layer(a, ws);
    if (!ws || ws_bytes < lw.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return DSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PagedDev pg = paged_dev(&a->pg);
    const int64_t ld = (int64_t)ld_of(a->max_len);
    IndexerArgs ia{a->q_idx, a->w, a->k_idx_cache, pg, decode ? nullptr : a->q_seq, decode ? nullptr : a->q_pos,
                   a->T, a->HI, a->DI, a->max_len, lw.scores, ld, hist_mode(a) ? lw.score_hist : nullptr,
                   hist_mode(a) ? static_cast<uint32_t *>(lw.topk_ws) : nullptr,
                   hist_mode(a) ? topk_hist_zero_words(a->T) : 0};
    if (!mark(0)) return DSA_ERR_CUDA;
    dsa_status s = mx ? launch_indexer_mx(ia, a->q_idx_scales, a->k_idx_scales, st) : launch_indexer(ia, st);
    if (s != DSA_OK) return s;
    if (!mark(1)) return DSA_ERR_CUDA;
    TopkArgs ta{lw.scores, ld, decode ? a->pg.seq_lens : a->q_pos,
                decode ? (int32_t)ROWLEN_SEQ_LENS : (int32_t)ROWLEN_QPOS_PLUS_1,
                a->T, a->K, a->max_len, lw.idx, lw.topk_ws, lw.topk_bytes};
    ta.pdl = true;
    if (hist_mode(a)) {
        ta.hist = lw.score_hist;
        if (topk_prefers_cluster(a->T, a->max_len)) {
            ta.ws = nullptr, ta.ws_bytes = 0;  // the cluster kernel needs none
            s = launch_topk(ta, st);
        } else {
            s = launch_topk_hist(ta, st);
        }
    } else {
        s = launch_topk(ta, st);
    }
    if (s != DSA_OK) return s;
    if (!mark(2)) return DSA_ERR_CUDA;
    AttnArgs aa{a->q, a->kv_cache, pg, decode ? nullptr : a->q_seq, lw.idx, a->K, a->gate, a->sm_scale, a->T, a->H,
                a->Dqk, a->Dv, a->out, a->lse, lw.attn_ws, lw.attn_bytes};
    aa.pdl = true;
    s = launch_attn(aa, st);
    if (s != DSA_OK) return s;
    return mark(3) ? DSA_OK : DSA_ERR_CUDA;
}
}  // namespace

extern "C" {

dsa_status dsa_layer_forward(const dsa_layer_args *a, void *ws, size_t ws_bytes, dsa_stream_t stream) {
    return layer_forward(a, ws, ws_bytes, stream, nullptr);
}

dsa_status dsa_layer_forward_profiled(const dsa_layer_args *a, void *ws, size_t ws_bytes, void *const events[4],
                                      dsa_stream_t stream) {
    return layer_forward(a, ws, ws_bytes, stream, events);
}

int32_t dsa_layer_kernel_launches(const dsa_layer_args *a) {
    if (!a || a->T <= 0 || a->max_len < 1) return 0;
    return 1 + (hist_mode(a) ? 1 : topk_kernel_launches(a->T, a->K, a->max_len)) + attn_kernel_launches(a->T, a->K, a->Dv);
}

dsa_status dsa_append_kv(const uint16_t *k_new, float k_scale, const uint16_t *latent_new, const int32_t *tok_seq,
                         const int32_t *tok_pos, const dsa_paged *pg, int32_t n, int32_t DI, int32_t Dqk,
                         uint8_t *k_idx_cache, uint16_t *kv_cache, dsa_stream_t stream) {
    if (n < 0 || !paged_ok(pg) || !isfinite(k_scale)) return DSA_ERR_INVALID_ARG;
    if ((DI != 64 && DI != 128) || (latent_new && (Dqk < 8 || Dqk % 8 || Dqk > 768))) return DSA_ERR_UNSUPPORTED;
    if (n == 0) return DSA_OK;
    if (!k_new || !tok_seq || !tok_pos || !k_idx_cache || (latent_new && !kv_cache)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(k_idx_cache) || (latent_new && (!aligned16(latent_new) || !aligned16(kv_cache))))
        return DSA_ERR_INVALID_ARG;
    AppendArgs a{k_new, latent_new, tok_seq, tok_pos, paged_dev(pg), n, DI, latent_new ? Dqk : 0, k_scale,
                 k_idx_cache, kv_cache};
    return launch_append(a, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_cp_candidates(const float *scores, int64_t ld, const int32_t *idx_local, int32_t B, int32_t K,
                             const int32_t *lo, float *cand_score, int32_t *cand_pos, dsa_stream_t stream) {
    if (B < 0 || K < 1 || ld < 1) return DSA_ERR_INVALID_ARG;
    if (B == 0) return DSA_OK;
    if (!scores || !idx_local || !lo || !cand_score || !cand_pos) return DSA_ERR_INVALID_ARG;
    return launch_cp_candidates(scores, ld, idx_local, B, K, lo, cand_score, cand_pos,
                                reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_cp_select_workspace_bytes(int32_t G, int32_t B, int32_t K) {
    if (G < 1 || B < 1 || K < 1 || (int64_t)G * K > (1 << 24)) return 0;
    return cp_select_workspace_bytes(G, B, K);
}

dsa_status dsa_cp_select(const float *cand_score, const int32_t *cand_pos, int32_t G, int32_t B, int32_t K,
                         const int32_t *lo, const int32_t *hi, int32_t *idx_global, int32_t *idx_local, void *ws,
                         size_t ws_bytes, dsa_stream_t stream) {
    if (G < 1 || B < 0 || K < 1 || (int64_t)G * K > (1 << 24)) return DSA_ERR_INVALID_ARG;
    if (K > 4096) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (!cand_score || !cand_pos || !lo || !hi || !idx_global || !idx_local) return DSA_ERR_INVALID_ARG;
    return launch_cp_select(cand_score, cand_pos, G, B, K, lo, hi, idx_global, idx_local, ws, ws_bytes,
                            reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_cp_lse_merge(const uint16_t *o, const float *lse, int32_t G, int32_t B, int32_t H, int32_t Dv,
                            uint16_t *out, dsa_stream_t stream) {
    if (G < 1 || B < 0 || H < 1 || Dv < 8 || Dv % 8) return DSA_ERR_INVALID_ARG;
    if (B == 0) return DSA_OK;
    if (!o || !lse || !out || !aligned16(o) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    return launch_cp_merge(o, lse, G, B, H, Dv, out, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_append_kv_mx(const uint16_t *k_new, const uint16_t *latent_new, const int32_t *tok_seq,
                            const int32_t *tok_pos, const dsa_paged *pg, int32_t n, int32_t DI, int32_t Dqk,
                            uint8_t *k_idx_cache, uint8_t *k_scales, uint16_t *kv_cache, dsa_stream_t stream) {
    if (n < 0 || !paged_ok(pg)) return DSA_ERR_INVALID_ARG;
    if ((DI != 64 && DI != 128) || (latent_new && (Dqk < 8 || Dqk % 8 || Dqk > 768))) return DSA_ERR_UNSUPPORTED;
    if (n == 0) return DSA_OK;
    if (!k_new || !tok_seq || !tok_pos || !k_idx_cache || !k_scales || (latent_new && !kv_cache))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(k_idx_cache) || (latent_new && (!aligned16(latent_new) || !aligned16(kv_cache))))
        return DSA_ERR_INVALID_ARG;
    AppendArgs a{k_new, latent_new, tok_seq, tok_pos, paged_dev(pg), n, DI, latent_new ? Dqk : 0, 1.f,
                 k_idx_cache, kv_cache};
    return launch_append_mx(a, k_scales, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_swa_decode(const uint16_t *q, const uint16_t *k_ring, const uint16_t *v_ring, const int32_t *seq_lens,
                          int32_t B, int32_t H, int32_t D, int32_t window, float sm_scale, uint16_t *out,
                          dsa_stream_t stream) {
    if (B < 0 || !isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
    if (D != 128 || window != 128 || H < 8 || H % 8) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (!q || !k_ring || !v_ring || !seq_lens || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    SwaArgs a{q, k_ring, v_ring, seq_lens, B, H, D, window, sm_scale, out};
    return launch_swa(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
