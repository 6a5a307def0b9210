// The step before the Gated DSA layer: new tokens' indexer keys and latent
// rows into the paged caches.
//
// The indexer keys are FP8 ("naive-n0-5-flash", Key Capabilities: FP8; one
// scale per tensor): token j's key row becomes e4m3(fp32(k_new[j, d]) *
// k_scale), the product rounded once, to the nearest code with ties to the
// even mantissa and finite magnitudes of 448 and above saturating to the
// largest finite code; its 576-wide bf16 latent row is stored unchanged.
// Both land at logical position tok_pos[j] of sequence tok_seq[j], through
// the block table.  HBM-bound: per token 2*DI + 2*Dqk bytes read and
// DI + 2*Dqk written.
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int APPEND_THREADS = 256;  // one warp per token

struct AppendParams {
    const uint16_t *k_new;       // bf16 [n, DI]
    const uint16_t *latent_new;  // bf16 [n, Dqk] or NULL
    const int32_t *tok_seq, *tok_pos;
    PagedDev pg;
    int32_t n, DI, Dqk;
    float k_scale;
    uint8_t *k_cache;    // e4m3 [num_pages, 64, DI]
    uint16_t *kv_cache;  // bf16 [num_pages, 64, Dqk]
    uint32_t *err;
};

// Two fp32 values to two e4m3 codes (round to nearest even, saturate to
// finite): lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// One warp per token.  The token's source rows are loaded first (they do
// not depend on where they go), so their latency overlaps the lookup of the
// destination row through seq_lens and the block table.
constexpr int APPEND_MAX_DI = 256;   // one 16-byte chunk of keys per lane
constexpr int APPEND_MAX_DQK = 768;  // three 16-byte chunks of latent per lane
__global__ void __launch_bounds__(APPEND_THREADS) append_kv_kernel(const AppendParams p) {
    const int j = static_cast<int>((blockIdx.x * (int64_t)APPEND_THREADS + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= p.n) return;
    const int nk = p.DI / 8, nl = p.Dqk / 8;  // 16-byte chunks of the key and latent rows
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4 kv = lane < nk ? reinterpret_cast<const uint4 *>(p.k_new + (int64_t)j * p.DI)[lane] : zero;
    uint4 lat[3];
    const uint4 *ls = reinterpret_cast<const uint4 *>(p.latent_new + (int64_t)j * p.Dqk);
#pragma unroll
    for (int i = 0; i < 3; ++i) lat[i] = p.latent_new && lane + 32 * i < nl ? ls[lane + 32 * i] : zero;
    const int b = p.tok_seq[j], pos = p.tok_pos[j];
    if (b < 0 || b >= p.pg.num_seqs || pos < 0 || pos >= p.pg.seq_lens[b]) {
        if (lane == 0) record_error(p.err, DSA_DEVERR_POSITION);
        return;
    }
    const int lp = pos >> 6;
    const int page = lp < p.pg.max_blocks ? p.pg.block_table[(int64_t)b * p.pg.max_blocks + lp] : -1;
    if (page < 0 || page >= p.pg.num_pages) {
        if (lane == 0) record_error(p.err, DSA_DEVERR_PAGE);
        return;
    }
    const int64_t row = (int64_t)page * 64 + (pos & 63);
    if (lane < nk) {  // 8 keys: fp32 products, then e4m3 (one 8-byte store)
        const float s = p.k_scale;
        const uint32_t q0 = e4m3x2(__fmul_rn(bf16_lo(kv.x), s), __fmul_rn(bf16_hi(kv.x), s));
        const uint32_t q1 = e4m3x2(__fmul_rn(bf16_lo(kv.y), s), __fmul_rn(bf16_hi(kv.y), s));
        const uint32_t q2 = e4m3x2(__fmul_rn(bf16_lo(kv.z), s), __fmul_rn(bf16_hi(kv.z), s));
        const uint32_t q3 = e4m3x2(__fmul_rn(bf16_lo(kv.w), s), __fmul_rn(bf16_hi(kv.w), s));
        reinterpret_cast<uint2 *>(p.k_cache + row * p.DI)[lane] = make_uint2(q0 | (q1 << 16), q2 | (q3 << 16));
    }
    if (p.latent_new) {
        uint4 *ld = reinterpret_cast<uint4 *>(p.kv_cache + row * p.Dqk);
#pragma unroll
        for (int i = 0; i < 3; ++i)
            if (lane + 32 * i < nl) ld[lane + 32 * i] = lat[i];
    }
}

// floor(log2 a) of a finite a > 0 (fp32, subnormals included)
__device__ __forceinline__ int floor_log2(float a) {
    const uint32_t b = __float_as_uint(a);
    const int e = static_cast<int>((b >> 23) & 0xFF);
    if (e) return e - 127;
    return -118 - __clz(b & 0x7FFFFF);  // subnormal m * 2^-149: -149 + (31 - clz(m))
}

// The MXFP8 form of the same step ("Open-Weight Deployment of an Ultra-Large
// Sparse Model", §1 and §3: activations in MXFP8; read as the OCP
// microscaling format): each 32 consecutive key elements share one E8M0
// scale 2^(c - 127) with c - 127 = floor(log2 max|x|) - 8 clamped to
// [-127, 127] (an all-zero block gets c = 0); the elements become
// e4m3(x * 2^-(c - 127)), round to nearest even, saturating.  The product
// is exact in fp32 wherever the E4M3 result is not zero.  A block is four
// consecutive lanes (8 elements each).  Scale codes go to the scale cache
// row [pages, 64, DI/32].
__global__ void __launch_bounds__(APPEND_THREADS) append_kv_mx_kernel(const AppendParams p, uint8_t *k_scales) {
    const int j = static_cast<int>((blockIdx.x * (int64_t)APPEND_THREADS + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (j >= p.n) return;
    const int nk = p.DI / 8, nl = p.Dqk / 8;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4 kv = lane < nk ? reinterpret_cast<const uint4 *>(p.k_new + (int64_t)j * p.DI)[lane] : zero;
    uint4 lat[3];
    const uint4 *ls = reinterpret_cast<const uint4 *>(p.latent_new + (int64_t)j * p.Dqk);
#pragma unroll
    for (int i = 0; i < 3; ++i) lat[i] = p.latent_new && lane + 32 * i < nl ? ls[lane + 32 * i] : zero;
    const float x[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                        bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // over the block's four lanes
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int shared = amax > 0.f ? max(-127, min(127, floor_log2(amax) - 8)) : -127;
    const float inv = scalbnf(1.0f, -shared);  // exact: 2^127 .. 2^-127
    const int b = p.tok_seq[j], pos = p.tok_pos[j];
    if (b < 0 || b >= p.pg.num_seqs || pos < 0 || pos >= p.pg.seq_lens[b]) {
        if (lane == 0) record_error(p.err, DSA_DEVERR_POSITION);
        return;
    }
    const int lp = pos >> 6;
    const int page = lp < p.pg.max_blocks ? p.pg.block_table[(int64_t)b * p.pg.max_blocks + lp] : -1;
    if (page < 0 || page >= p.pg.num_pages) {
        if (lane == 0) record_error(p.err, DSA_DEVERR_PAGE);
        return;
    }
    const int64_t row = (int64_t)page * 64 + (pos & 63);
    if (lane < nk) {
        const uint32_t q0 = e4m3x2(x[0] * inv, x[1] * inv), q1 = e4m3x2(x[2] * inv, x[3] * inv);
        const uint32_t q2 = e4m3x2(x[4] * inv, x[5] * inv), q3 = e4m3x2(x[6] * inv, x[7] * inv);
        reinterpret_cast<uint2 *>(p.k_cache + row * p.DI)[lane] = make_uint2(q0 | (q1 << 16), q2 | (q3 << 16));
        if ((lane & 3) == 0) k_scales[row * (p.DI / 32) + (lane >> 2)] = static_cast<uint8_t>(shared + 127);
    }
    if (p.latent_new) {
        uint4 *ld = reinterpret_cast<uint4 *>(p.kv_cache + row * p.Dqk);
#pragma unroll
        for (int i = 0; i < 3; ++i)
            if (lane + 32 * i < nl) ld[lane + 32 * i] = lat[i];
    }
}

}  // namespace

dsa_status launch_append_mx(const AppendArgs &a, uint8_t *k_scales, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if ((a.DI != 64 && a.DI != 128) || a.Dqk > APPEND_MAX_DQK || a.Dqk % 8) return DSA_ERR_UNSUPPORTED;
    if (a.n == 0) return DSA_OK;
    AppendParams p{a.k_new, a.latent_new, a.tok_seq, a.tok_pos, a.pg, a.n, a.DI, a.Dqk, 1.f,
                   a.k_cache, a.kv_cache, dev->err};
    const int64_t threads = (int64_t)a.n * 32;
    append_kv_mx_kernel<<<(unsigned)((threads + APPEND_THREADS - 1) / APPEND_THREADS), APPEND_THREADS, 0, st>>>(
        p, k_scales);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_append(const AppendArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.DI > APPEND_MAX_DI || a.DI % 8 || a.Dqk > APPEND_MAX_DQK || a.Dqk % 8) return DSA_ERR_UNSUPPORTED;
    if (a.n == 0) return DSA_OK;
    AppendParams p{a.k_new, a.latent_new, a.tok_seq, a.tok_pos, a.pg, a.n, a.DI, a.Dqk, a.k_scale,
                   a.k_cache, a.kv_cache, dev->err};
    const int64_t threads = (int64_t)a.n * 32;
    append_kv_kernel<<<(unsigned)((threads + APPEND_THREADS - 1) / APPEND_THREADS), APPEND_THREADS, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
