// Context-parallel decode of long sequences over G GPUs: the steps that
// join the ranks' partial results.
//
// Rank r holds a contiguous run of whole pages of every sequence, positions
// [lo[b], hi[b]).  It scores its own positions and selects its own top-K with
// the single-GPU calls; because a position among the K best of the whole
// history is among the K best of its own range, the union of the G local
// lists, cut back to K under the top-K's order, is exactly the one-GPU
// selection ("Open-Source LLM Architecture Evolution", Architecture
// Breakdown §2, "Top-K selection"; "Fine-Grained Sparse Attention in
// Ultra-Large Parameter Models", §1, the 1,048,576-token context).  Each
// rank then attends over the kept rows it holds and the G gated partial
// outputs merge by their log-sum-exp weights.  The exchanges between the
// steps are all-gathers the caller runs (NCCL); these kernels only read and
// write this GPU's memory.
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int CP_THREADS = 256;

// (score, global position) of each locally kept position; (-inf, -1) for padding.
__global__ void __launch_bounds__(CP_THREADS) cp_candidates_kernel(const float *scores, int64_t ld,
                                                                   const int32_t *idx, int B, int K,
                                                                   const int32_t *lo, float *cs, int32_t *cpos) {
    const int64_t i = (int64_t)blockIdx.x * CP_THREADS + threadIdx.x;
    if (i >= (int64_t)B * K) return;
    const int b = (int)(i / K);
    const int s = idx[i];
    cs[i] = s >= 0 ? scores[b * ld + s] : -INFINITY;
    cpos[i] = s >= 0 ? s + lo[b] : -1;
}

// [G][B][K] -> one row per sequence, ranks in order: [B][G*K]; every row is
// G*K long.  Ranks hold increasing ranges and each list is ascending, so the
// valid entries of a row are in ascending position order.
__global__ void __launch_bounds__(CP_THREADS) cp_rows_kernel(const float *cs, const int32_t *cpos, int G, int B,
                                                             int K, float *rs, int32_t *rp, int32_t *row_len) {
    const int64_t i = (int64_t)blockIdx.x * CP_THREADS + threadIdx.x;
    if (i < B) row_len[i] = G * K;
    if (i >= (int64_t)G * B * K) return;
    const int k = (int)(i % K);
    const int b = (int)((i / K) % B);
    const int g = (int)(i / ((int64_t)K * B));
    const int64_t o = ((int64_t)b * G + g) * K + k;
    rs[o] = cs[i];
    rp[o] = cpos[i];
}

// One CTA per sequence: the selected row indices (ascending) -> global
// positions, padding dropped and moved to the end; this rank's local indices
// (position - lo, or -1 outside [lo, hi)).
__global__ void __launch_bounds__(CP_THREADS) cp_map_kernel(const int32_t *sel, const int32_t *rp, int G, int K,
                                                            const int32_t *lo, const int32_t *hi, int32_t *idx_g,
                                                            int32_t *idx_l) {
    __shared__ uint32_t wsum[CP_THREADS / 32];
    __shared__ uint32_t base_sh;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t *row = rp + (int64_t)b * G * K;
    const int32_t *s = sel + (int64_t)b * K;
    int32_t *og = idx_g + (int64_t)b * K, *ol = idx_l + (int64_t)b * K;
    const int lob = lo[b], hib = hi[b];
    if (tid == 0) base_sh = 0;
    __syncthreads();
    for (int j0 = 0; j0 < K; j0 += CP_THREADS) {
        const int j = j0 + tid;
        const int c = j < K ? s[j] : -1;
        const int pos = c >= 0 ? row[c] : -1;
        const uint32_t v = pos >= 0;
        uint32_t x = v;  // inclusive scan over the block
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        uint32_t before = base_sh;
        for (int w = 0; w < warp; ++w) before += wsum[w];
        if (v) {
            const uint32_t slot = before + x - 1;
            og[slot] = pos;
            ol[slot] = pos >= lob && pos < hib ? pos - lob : -1;
        }
        __syncthreads();
        if (tid == 0)
            for (int w = 0; w < CP_THREADS / 32; ++w) base_sh += wsum[w];
        __syncthreads();
    }
    for (int j = base_sh + tid; j < K; j += CP_THREADS) og[j] = -1, ol[j] = -1;
}

// One thread per (sequence, head, 8 output dims):
// out = sum_r exp(lse_r - M) o_r / sum_r exp(lse_r - M), M = max_r lse_r,
// over the ranks that kept a row (lse_r > -inf).
__global__ void __launch_bounds__(CP_THREADS) cp_merge_kernel(const uint16_t *o, const float *lse, int G, int B,
                                                              int H, int Dv, uint16_t *out) {
    const int chunks = Dv / 8;
    const int64_t i = (int64_t)blockIdx.x * CP_THREADS + threadIdx.x;
    if (i >= (int64_t)B * H * chunks) return;
    const int64_t bh = i / chunks;
    const int c = (int)(i % chunks);
    const int64_t plane = (int64_t)B * H;
    float m = -INFINITY;
    for (int g = 0; g < G; ++g) m = fmaxf(m, lse[g * plane + bh]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
    if (m > -INFINITY)
        for (int g = 0; g < G; ++g) {
            const float l = lse[g * plane + bh];
            if (!(l > -INFINITY)) continue;
            const float wgt = __expf(l - m);
            wsum += wgt;
            const uint4 v = *reinterpret_cast<const uint4 *>(o + (g * plane + bh) * Dv + c * 8);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] = fmaf(wgt, __uint_as_float(u[e] << 16), acc[2 * e]);
                acc[2 * e + 1] = fmaf(wgt, __uint_as_float(u[e] & 0xFFFF0000u), acc[2 * e + 1]);
            }
        }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        r[e] = *reinterpret_cast<uint32_t *>(&p);
    }
    *reinterpret_cast<uint4 *>(out + bh * Dv + c * 8) = make_uint4(r[0], r[1], r[2], r[3]);
}

unsigned blocks_for(int64_t n) { return (unsigned)((n + CP_THREADS - 1) / CP_THREADS); }

struct CpWs {
    float *rs;
    int32_t *rp, *row_len, *sel;
    void *topk_ws;
    size_t topk_bytes, total;
};

CpWs carve_cp(void *ws, int G, int B, int K) {
    CpWs w{};
    uint8_t *p = static_cast<uint8_t *>(ws);
    size_t off = 0;
    const size_t n = (size_t)G * B * K;
    w.rs = reinterpret_cast<float *>(p + off);
    off += align_up(n * 4, 256);
    w.rp = reinterpret_cast<int32_t *>(p + off);
    off += align_up(n * 4, 256);
    w.row_len = reinterpret_cast<int32_t *>(p + off);
    off += align_up((size_t)B * 4, 256);
    w.sel = reinterpret_cast<int32_t *>(p + off);
    off += align_up((size_t)B * K * 4, 256);
    w.topk_bytes = topk_workspace_bytes(B, K, G * K);
    w.topk_ws = w.topk_bytes ? p + off : nullptr;
    off += w.topk_bytes;
    w.total = off;
    return w;
}

}  // namespace

dsa_status launch_cp_candidates(const float *scores, int64_t ld, const int32_t *idx, int B, int K, const int32_t *lo,
                                float *cs, int32_t *cpos, cudaStream_t st) {
    cp_candidates_kernel<<<blocks_for((int64_t)B * K), CP_THREADS, 0, st>>>(scores, ld, idx, B, K, lo, cs, cpos);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t cp_select_workspace_bytes(int G, int B, int K) { return carve_cp(nullptr, G, B, K).total; }

dsa_status launch_cp_select(const float *cs, const int32_t *cpos, int G, int B, int K, const int32_t *lo,
                            const int32_t *hi, int32_t *idx_g, int32_t *idx_l, void *ws, size_t ws_bytes,
                            cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    CpWs w = carve_cp(ws, G, B, K);
    if (!ws || ws_bytes < w.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return DSA_ERR_WORKSPACE;
    cp_rows_kernel<<<blocks_for((int64_t)G * B * K), CP_THREADS, 0, st>>>(cs, cpos, G, B, K, w.rs, w.rp, w.row_len);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
    TopkArgs ta{w.rs, (int64_t)G * K, w.row_len, ROWLEN_ARRAY, B, K, G * K, w.sel, w.topk_ws, w.topk_bytes};
    dsa_status s = launch_topk(ta, st);
    if (s != DSA_OK) return s;
    cp_map_kernel<<<B, CP_THREADS, 0, st>>>(w.sel, w.rp, G, K, lo, hi, idx_g, idx_l);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_cp_merge(const uint16_t *o, const float *lse, int G, int B, int H, int Dv, uint16_t *out,
                           cudaStream_t st) {
    cp_merge_kernel<<<blocks_for((int64_t)B * H * (Dv / 8)), CP_THREADS, 0, st>>>(o, lse, G, B, H, Dv, out);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
