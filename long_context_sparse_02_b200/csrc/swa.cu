// Sliding-window decode attention for the local layers of the 5:1 SWA/DSA
// hybrid ("aiany.app item naive-n0-5-flash", Key Capabilities: 128-token
// window).  Memory-bound: every step reads each sequence's whole ring
// buffer once.  One CTA = (sequence, 8 heads); a warp per head.  The ring
// rows of the CTA's 8 heads are contiguous (2 KB per slot), so each slot is
// one bulk copy into a padded shared-memory row (bank-conflict-free reads).
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int HG = 8;          // heads per CTA
constexpr int D = 128;         // head dim
constexpr int W = 128;         // window (ring slots)
constexpr int SLOTS = 32;      // slots per stage
constexpr int ROW = HG * D * 2 + 16;  // bytes per staged slot (padded)
constexpr int STAGE = SLOTS * ROW;
constexpr int NST = 2;
constexpr int SMEM = NST * STAGE + 2 * HG * W * 4 + 64;

struct SwaParams {
    const uint16_t *q, *k, *v;
    const int32_t *seq_lens;
    int32_t B, H;
    float scale;
    uint16_t *out;
    uint32_t *err;
};

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

__global__ void __launch_bounds__(256, 1) swa_decode_kernel(const SwaParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t *stages = sm;
    float *qs = reinterpret_cast<float *>(sm + NST * STAGE);  // [HG][D]
    float *ps = qs + HG * D;                                  // [HG][W]
    uint64_t *full = reinterpret_cast<uint64_t *>(ps + HG * W);
    const int warp = warp_id(), lane = lane_id();
    const int b = blockIdx.y, hg = blockIdx.x;
    const int h = hg * HG + warp;
    int L = p.seq_lens[b];
    if (L <= 0) {
        if (threadIdx.x == 0) record_error(p.err, DSA_DEVERR_POSITION);
        L = 0;
    }
    const int nv = L < W ? L : W;
    const int nchunk = (nv + SLOTS - 1) / SLOTS;
    const int nload = 2 * nchunk;

    auto issue = [&](int i) {  // thread 0 only
        const int s = i % NST;
        const bool is_v = i >= nchunk;
        const int c = is_v ? i - nchunk : i;
        const int n = min(SLOTS, nv - c * SLOTS);
        const uint16_t *base = is_v ? p.v : p.k;
        mbar_expect_tx(&full[s], n * HG * D * 2);
        for (int j = 0; j < n; ++j) {
            const int slot = c * SLOTS + j;
            bulk_load(stages + s * STAGE + j * ROW, base + (((int64_t)b * W + slot) * p.H + hg * HG) * D, HG * D * 2,
                      &full[s]);
        }
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        for (int i = 0; i < NST && i < nload; ++i) issue(i);
    {
        const uint2 qv = *reinterpret_cast<const uint2 *>(p.q + ((int64_t)b * p.H + h) * D + lane * 4);
        qs[warp * D + lane * 4 + 0] = bf_lo(qv.x);
        qs[warp * D + lane * 4 + 1] = bf_hi(qv.x);
        qs[warp * D + lane * 4 + 2] = bf_lo(qv.y);
        qs[warp * D + lane * 4 + 3] = bf_hi(qv.y);
    }
    __syncwarp();
    float sc[W / SLOTS];
    bool ok = true;
    // ---- scores: lane = slot within the chunk ----
    for (int c = 0; c < nchunk; ++c) {
        const int i = c, s = i % NST;
        ok = ok && mbar_wait(&full[s], (i / NST) & 1, p.err, nullptr);
        const int slot = c * SLOTS + lane;
        float acc = 0.f;
        if (ok && slot < nv) {
            const uint8_t *krow = stages + s * STAGE + lane * ROW + warp * D * 2;
            const float *qw = qs + warp * D;
#pragma unroll
            for (int d = 0; d < D; d += 8) {
                const uint4 kv = *reinterpret_cast<const uint4 *>(krow + d * 2);
                const float4 q0 = *reinterpret_cast<const float4 *>(qw + d);
                const float4 q1 = *reinterpret_cast<const float4 *>(qw + d + 4);
                acc = fmaf(q0.x, bf_lo(kv.x), acc);
                acc = fmaf(q0.y, bf_hi(kv.x), acc);
                acc = fmaf(q0.z, bf_lo(kv.y), acc);
                acc = fmaf(q0.w, bf_hi(kv.y), acc);
                acc = fmaf(q1.x, bf_lo(kv.z), acc);
                acc = fmaf(q1.y, bf_hi(kv.z), acc);
                acc = fmaf(q1.z, bf_lo(kv.w), acc);
                acc = fmaf(q1.w, bf_hi(kv.w), acc);
            }
        }
        sc[c] = (slot < nv) ? acc * p.scale : -INFINITY;
        __syncthreads();
        if (threadIdx.x == 0 && ok && i + NST < nload) issue(i + NST);
    }
    // ---- softmax over the window ----
    float mx = -INFINITY;
    for (int c = 0; c < nchunk; ++c) mx = fmaxf(mx, sc[c]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int c = 0; c < nchunk; ++c) {
        sc[c] = sc[c] == -INFINITY ? 0.f : __expf(sc[c] - mx);
        sum += sc[c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int c = 0; c < nchunk; ++c) ps[warp * W + c * SLOTS + lane] = sc[c] * inv;
    __syncwarp();
    // ---- output: lane = 4 value dims ----
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nchunk; ++c) {
        const int i = nchunk + c, s = i % NST;
        ok = ok && mbar_wait(&full[s], (i / NST) & 1, p.err, nullptr);
        const int n = min(SLOTS, nv - c * SLOTS);
        if (ok) {
            for (int j = 0; j < n; ++j) {
                const float pj = ps[warp * W + c * SLOTS + j];
                const uint2 vv = *reinterpret_cast<const uint2 *>(stages + s * STAGE + j * ROW + warp * D * 2 + lane * 8);
                o.x = fmaf(pj, bf_lo(vv.x), o.x);
                o.y = fmaf(pj, bf_hi(vv.x), o.y);
                o.z = fmaf(pj, bf_lo(vv.y), o.z);
                o.w = fmaf(pj, bf_hi(vv.y), o.w);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0 && ok && i + NST < nload) issue(i + NST);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t *>(&lo);
    packed.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p.out + ((int64_t)b * p.H + h) * D + lane * 4) = packed;
}

}  // namespace

dsa_status launch_swa(const SwaArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.B == 0) return DSA_OK;
    SwaParams p{a.q, a.k_ring, a.v_ring, a.seq_lens, a.B, a.H, a.sm_scale, a.out, dev->err};
    if (!ensure_smem(reinterpret_cast<const void *>(swa_decode_kernel), SMEM)) return DSA_ERR_CUDA;
    dim3 grid(a.H / HG, a.B);
    swa_decode_kernel<<<grid, 256, SMEM, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
