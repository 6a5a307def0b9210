// Stage 2 of the Gated DSA layer for many rows (prefill: one row per query
// token, up to 32768 keys each).  Same contract as topk.cu: per row, the K
// highest scores ("Open-Source LLM Architecture Evolution", Architecture
// Breakdown §2, "Top-K selection"; "Fine-Grained Sparse Attention in
// Ultra-Large Parameter Models", §2.1), every position when the row is not
// longer than K, ties to the lower position, -0.0 equal to +0.0, kept
// positions ascending, -1 padding.
//
// One 256-thread CTA per row, four per SM, so one row's block-wide steps
// hide behind the other rows' loads; warp w owns the w-th eighth of the row.
// Per row:
//   1. a stratified sample (64 runs of 32 scores spread over the row) gives
//      a likely lower bound tf for the K-th largest score: the lower edge of
//      the bin, in a 256-bin histogram over the sample's range, that holds
//      the sample score whose rank is the expected rank of the K-th score
//      plus four standard deviations;
//   2. the row, sent into L2 by prefetches at the CTA's start (while step 1
//      runs), is read twice from there: each warp counts its scores >= tf,
//      the counts give each warp its offset, and a second pass over the
//      warp's range lists them as (position, score) in position order into
//      shared memory;
//   3. a 1024-bin histogram of the listed scores over [tf, sample maximum]
//      gives the bin F of the K-th score; one pass over the list counts the
//      entries above F and collects F's few entries, one warp ranks those
//      (score descending, position ascending) and marks the ones kept, and
//      a second pass writes the kept positions in order.
// A row no longer than the list lists every score.  The list holds every
// score the top-K keeps when at least K scores are >= tf and no more than its
// capacity; otherwise (an unlucky sample, or heavy ties at the threshold) the
// row takes exact radix levels over its score keys instead, as does a list
// whose bin F holds more than 32 entries.  Either way the result is the exact
// top-K.
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int TR_THREADS = 256;
constexpr int TR_WARPS = TR_THREADS / 32;
constexpr int TR_MINB = 4;     // CTAs per SM
constexpr int TR_U = 8;        // loads in flight per lane: 8 steps of 64 positions, a float2 each
constexpr int TR_MAXN = 32768; // longest row
constexpr int TR_CAP = 4096;   // listed entries held in shared memory
constexpr int TR_SMEM = (TR_CAP + 32) * 8;  // and one scratch entry per lane
constexpr int TR_RUNS = 64, TR_SAMPLES = TR_RUNS * 32;
constexpr int TR_LB = 11, TR_BINS = 1 << TR_LB;  // bits and bins per radix level of the exact fallbacks
constexpr int TR_SBINS = 256;   // the sample's histogram
constexpr int TR_LBINS = 1024;  // the listed scores' histogram
constexpr int TR_CF = 32;       // entries of the threshold's bin one warp ranks
constexpr uint32_t TR_PAD = 0xFFFFFFFFu;
constexpr uint32_t TR_MARK = 0x80000000u;  // set on the position of a kept entry of bin F
constexpr uint32_t TR_POS = 0xFFFFu;       // a list entry's position bits; its bin sits at bit 16
static_assert(TR_CAP > TR_SAMPLES, "rows that skip sampling are longer than the sample");
static_assert(TR_MAXN <= (int)TR_POS + 1 && TR_LBINS <= 1 << 15, "position, bin and mark share a word");

__device__ __forceinline__ int tr_row_length(const TopkArgs &a, int r, uint32_t *err) {
    int n = a.mode == ROWLEN_QPOS_PLUS_1 ? a.row_len[r] + 1 : a.row_len[r];
    if (n < 0) {
        record_error(err, DSA_DEVERR_SHAPE);
        n = 0;
    }
    if (n > a.max_row_len) {
        record_error(err, DSA_DEVERR_SHAPE);
        n = a.max_row_len;
    }
    return n;
}

__device__ __forceinline__ uint32_t tr_warp_scan(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// The highest bin b of hist[NB] with sum(hist[b+1:]) < remaining <=
// sum(hist[b:]): res[0] = b, res[1] = keys above it, res[2] = keys in it.
// res is left as it was when no bin qualifies.  ws: TR_WARPS words.
template <int NB>
__device__ __forceinline__ void tr_pick(const uint32_t *hist, uint32_t remaining, uint32_t *ws, uint32_t *res) {
    constexpr int PER = NB / TR_THREADS;
    static_assert(PER * TR_THREADS == NB, "whole bins per thread");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t v[PER], s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        v[i] = hist[NB - 1 - PER * threadIdx.x - i];
        s += v[i];
    }
    const uint32_t x = tr_warp_scan(s);
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    uint32_t before = 0;
#pragma unroll
    for (int w = 0; w < TR_WARPS; ++w) before += w < warp ? ws[w] : 0u;
    uint32_t above = x + before - s;
    if (above < remaining && remaining <= above + s) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if (above + v[i] >= remaining) {
                res[0] = (uint32_t)(NB - 1 - PER * (int)threadIdx.x - i);
                res[1] = above;
                res[2] = v[i];
                break;
            }
            above += v[i];
        }
    }
    __syncthreads();
}

struct TrShared {
    uint32_t hist[TR_BINS];
    uint32_t ws[2 * TR_WARPS];
    uint32_t misc[8];
    float cf_x[TR_CF];
    uint32_t cf_j[TR_CF];
};

// Bins per unit score for nb bins over [lo, hi]; 0 (every score in bin 0)
// for an empty range or one too narrow for a finite factor.
__device__ __forceinline__ float tr_scale(float lo, float hi, int nb) {
    const float s = hi > lo ? (float)nb / (hi - lo) : 0.f;
    return s < INFINITY ? s : 0.f;
}

// round(min(v, cap)) for 0 <= v, cap < 2^22, on the FMA pipe: adding
// 1.5 * 2^23 leaves the rounded value in the low mantissa bits.  Monotone in v.
__device__ __forceinline__ int tr_bin(float v, float cap) {
    return __float_as_int(fminf(v, cap) + 12582912.f) - 0x4B400000;
}

// The rank-th largest (1 <= rank <= count) of the keys get(j), j < count,
// all within [base, base + span].  Histogram levels of TR_LB bits over the
// offset key - base; as soon as the chosen bin holds at most 32 keys one warp
// ranks them.  tau = that key, need = rank - #(keys > tau).
template <typename Get>
__device__ __forceinline__ void tr_select(Get get, int count, uint32_t rank, uint32_t base, uint32_t span,
                                          TrShared &sh, uint32_t &tau, uint32_t &need) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int H = 32 - __clz(span);  // offset bits still open
    uint32_t prefix = 0, rem = rank;
    for (;;) {
        if (H == 0) {
            tau = base + prefix;
            need = rem;
            return;
        }
        const int L = H > TR_LB ? H - TR_LB : 0;
        const uint32_t bmask = (1u << (H - L)) - 1u;
        for (int i = tid; i < TR_BINS; i += TR_THREADS) sh.hist[i] = 0;
        if (tid == 0) sh.misc[0] = 0, sh.misc[1] = 0, sh.misc[2] = 0, sh.misc[3] = 0, sh.misc[4] = 0, sh.misc[5] = 0;
        __syncthreads();
        for (int j = tid; j < count; j += TR_THREADS) {
            const uint32_t off = get(j) - base;
            if (H >= 32 || (off >> H) == prefix) atomicAdd(&sh.hist[(off >> L) & bmask], 1u);
        }
        __syncthreads();
        tr_pick<TR_BINS>(sh.hist, rem, sh.ws, sh.misc);
        const uint32_t F = sh.misc[0], cnt = sh.misc[2];
        rem -= sh.misc[1];
        __syncthreads();  // misc is rewritten by the next level
        prefix = (prefix << (H - L)) | F;
        H = L;
        if (H > 0 && cnt <= 32) {
            for (int j0 = warp * 32; j0 < count; j0 += TR_THREADS) {
                const int j = j0 + lane;
                const uint32_t off = j < count ? get(j) - base : 0u;
                const bool hit = j < count && (off >> H) == prefix;
                const uint32_t hm = __ballot_sync(0xffffffffu, hit);
                if (hm) {
                    uint32_t b0 = 0;
                    if (lane == 0) b0 = atomicAdd(&sh.misc[3], (uint32_t)__popc(hm));
                    b0 = __shfl_sync(0xffffffffu, b0, 0);
                    const uint32_t slot = b0 + __popc(hm & ((1u << lane) - 1u));
                    if (hit && slot < 32u) sh.cf_j[slot] = off;
                }
            }
            __syncthreads();
            if (warp == 0) {
                const uint32_t nc = min(sh.misc[3], 32u);
                const bool v = (uint32_t)lane < nc;
                const uint32_t k = v ? sh.cf_j[lane] : 0u;
                uint32_t gt = 0, eq = 0;
                for (uint32_t j = 0; j < nc; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, k, j);
                    gt += kj > k;
                    eq += kj == k;
                }
                if (v && gt < rem && rem <= gt + eq) sh.misc[4] = k, sh.misc[5] = rem - gt;
            }
            __syncthreads();
            tau = base + sh.misc[4];
            need = sh.misc[5];
            __syncthreads();
            return;
        }
    }
}

// Stable compaction of (position, key) entries given in position order:
// keeps key > tau, and key == tau while fewer than `need` came before.  Warp
// w walks its own contiguous segment (ballots order the lanes); one exchange
// of the segments' counts.
template <typename Entry>
__device__ __forceinline__ void tr_compact(Entry entry, int count, uint32_t tau, uint32_t need, int32_t *out, int K,
                                           uint32_t *ws, uint32_t *err) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int seg = (count + TR_WARPS * 32 - 1) / (TR_WARPS * 32) * 32;
    const int w0 = warp * seg, w1 = min(count, w0 + seg);
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t g = 0, e = 0;
    for (int j0 = w0; j0 < w1; j0 += 32) {
        const int j = j0 + lane;
        const uint2 v = j < w1 ? entry(j) : make_uint2(TR_PAD, 0u);
        g += __popc(__ballot_sync(0xffffffffu, v.x != TR_PAD && v.y > tau));
        e += __popc(__ballot_sync(0xffffffffu, v.x != TR_PAD && v.y == tau));
    }
    if (lane == 0) ws[warp] = g, ws[TR_WARPS + warp] = e;
    __syncthreads();
    uint32_t gcur = 0, ecur = 0;
#pragma unroll
    for (int w = 0; w < TR_WARPS; ++w) {
        gcur += w < warp ? ws[w] : 0u;
        ecur += w < warp ? ws[TR_WARPS + w] : 0u;
    }
    for (int j0 = w0; j0 < w1; j0 += 32) {
        const int j = j0 + lane;
        const uint2 v = j < w1 ? entry(j) : make_uint2(TR_PAD, 0u);
        const bool gt = v.x != TR_PAD && v.y > tau, eq = v.x != TR_PAD && v.y == tau;
        const uint32_t gm = __ballot_sync(0xffffffffu, gt), em = __ballot_sync(0xffffffffu, eq);
        const uint32_t mg = gcur + __popc(gm & lt), me = ecur + __popc(em & lt);
        if (gt || (eq && me < need)) {
            const uint32_t slot = mg + min(me, need);
            if (slot < (uint32_t)K) out[slot] = (int32_t)v.x;
            else record_error(err, DSA_DEVERR_SHAPE);
        }
        gcur += __popc(gm);
        ecur += __popc(em);
    }
}

// Positions p + 64 u + 2 lane and the next, u < TR_U, of this warp's range
// [.., hi): one coalesced 256-byte load per u (p is even, so each float2 is
// aligned).  Positions at or past hi read as NaN, which no threshold lists
// (scores are finite).
template <bool FULL>
__device__ __forceinline__ void tr_load(const float *row, int p, int hi, float2 (&x)[TR_U]) {
    const int lane = threadIdx.x & 31;
    const float nan = __int_as_float(0x7fc00000);
#pragma unroll
    for (int u = 0; u < TR_U; ++u) {
        const int q = p + 64 * u + 2 * lane;
        if (FULL || q + 1 < hi) {
            x[u] = __ldcg(reinterpret_cast<const float2 *>(row + q));
        } else {
            x[u].x = q < hi ? __ldcg(row + q) : nan;
            x[u].y = nan;
        }
    }
}

__device__ __forceinline__ void tr_load_any(const float *row, int p, int hi, float2 (&x)[TR_U]) {
    if (p + 64 * TR_U <= hi) tr_load<true>(row, p, hi, x);
    else tr_load<false>(row, p, hi, x);
}

// Top-K of the listed entries (K <= listed <= TR_CAP, every score >= lo):
// the histogram over [lo, hi] (scores above hi count in the top bin), then
// the two passes.  Returns false, having written nothing, when the
// threshold's bin holds more than TR_CF entries.
__device__ __forceinline__ bool tr_finish(uint2 *list, int listed, int K, float lo, float hi, TrShared &sh,
                                          int32_t *out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = tr_scale(lo, hi, TR_LBINS);
    for (int i = tid; i < TR_LBINS; i += TR_THREADS) sh.hist[i] = 0;
    if (tid == 0) sh.misc[0] = 0, sh.misc[1] = 0, sh.misc[2] = 0, sh.misc[3] = 0;
    __syncthreads();
    for (int j = tid; j < listed; j += TR_THREADS) {  // each entry keeps its bin for the passes below
        const uint2 e = list[j];
        const int bn = tr_bin((__uint_as_float(e.y) - lo) * scale, (float)(TR_LBINS - 1));
        atomicAdd(&sh.hist[bn], 1u);
        list[j].x = (e.x & TR_POS) | ((uint32_t)bn << 16);
    }
    __syncthreads();
    tr_pick<TR_LBINS>(sh.hist, (uint32_t)K, sh.ws, sh.misc);
    const int F = (int)sh.misc[0];
    const uint32_t above = sh.misc[1], cntF = sh.misc[2];
    if (cntF > (uint32_t)TR_CF || cntF == 0) return false;  // block-uniform
    const uint32_t need = (uint32_t)K - above;
    const uint32_t lt = (1u << lane) - 1u;
    // pass 1: entries above F per warp segment; F's entries collected
    const int seg = (listed + TR_THREADS - 1) / TR_THREADS * 32;
    const int w0 = warp * seg, w1 = min(listed, w0 + seg);
    uint32_t g = 0;
    for (int j0 = w0; j0 < w1; j0 += 32) {
        const int j = j0 + lane;
        const uint2 e = j < w1 ? list[j] : make_uint2(0u, 0u);
        const int bn = j < w1 ? (int)((e.x >> 16) & (TR_LBINS - 1)) : -1;
        g += __popc(__ballot_sync(0xffffffffu, bn > F));
        const uint32_t hm = __ballot_sync(0xffffffffu, bn == F);
        if (hm) {
            uint32_t b0 = 0;
            if (lane == 0) b0 = atomicAdd(&sh.misc[3], (uint32_t)__popc(hm));
            b0 = __shfl_sync(0xffffffffu, b0, 0);
            const uint32_t slot = b0 + __popc(hm & lt);
            if (bn == F && slot < (uint32_t)TR_CF) sh.cf_x[slot] = __uint_as_float(e.y), sh.cf_j[slot] = (uint32_t)j;
        }
    }
    if (lane == 0) sh.ws[warp] = g;
    __syncthreads();
    // one warp ranks F's entries (score descending, then position = list order) and marks the first `need`
    if (warp == 0) {
        const uint32_t nc = min(sh.misc[3], (uint32_t)TR_CF);
        const bool v = (uint32_t)lane < nc;
        const float xi = v ? sh.cf_x[lane] : 0.f;
        const uint32_t ji = v ? sh.cf_j[lane] : 0u;
        uint32_t rank = 0;
        for (uint32_t k = 0; k < nc; ++k) {
            const float xk = __shfl_sync(0xffffffffu, xi, k);
            const uint32_t jk = __shfl_sync(0xffffffffu, ji, k);
            rank += (xk > xi || (xk == xi && jk < ji)) ? 1u : 0u;
        }
        if (v && rank < need) {
            atomicAdd(&sh.ws[ji / seg], 1u);
            list[ji].x |= TR_MARK;
        }
    }
    __syncthreads();
    // pass 2: the kept entries' positions, in order
    uint32_t base = 0;
#pragma unroll
    for (int w = 0; w < TR_WARPS; ++w) base += w < warp ? sh.ws[w] : 0u;
    for (int j0 = w0; j0 < w1; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t ex = j < w1 ? list[j].x : 0u;
        const int bn = j < w1 ? (int)((ex >> 16) & (TR_LBINS - 1)) : -1;
        const bool keep = bn > F || (bn == F && (ex & TR_MARK));
        const uint32_t km = __ballot_sync(0xffffffffu, keep);
        const uint32_t slot = base + __popc(km & lt);
        st_global_if(out + slot, ex & TR_POS, keep && slot < (uint32_t)K);
        base += __popc(km);
    }
    return true;
}

// Block-wide min and max; every thread gets both.  ws: 2 * TR_WARPS words.
__device__ __forceinline__ void tr_range(float &lo, float &hi, uint32_t *ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) ws[warp] = __float_as_uint(lo), ws[TR_WARPS + warp] = __float_as_uint(hi);
    __syncthreads();
#pragma unroll
    for (int w = 0; w < TR_WARPS; ++w)
        lo = fminf(lo, __uint_as_float(ws[w])), hi = fmaxf(hi, __uint_as_float(ws[TR_WARPS + w]));
}

__global__ void __launch_bounds__(TR_THREADS, TR_MINB) topk_rows_kernel(const TopkArgs a, uint32_t *err) {
    __shared__ TrShared sh;
    extern __shared__ uint2 sh_list[];  // [TR_CAP] (position, score bits), position order; [32] scratch
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.x, K = a.K;
    pdl_trigger();
    pdl_wait();  // the scores come from the previous kernel
    const int n = tr_row_length(a, r, err);
    int32_t *out = a.idx + (int64_t)r * K;
    if (n <= K) {
        for (int j = tid; j < K; j += TR_THREADS) out[j] = j < n ? j : -1;
        return;
    }
    const float *row = a.scores + (int64_t)r * a.ld;
    uint32_t listed = 0;
    float lo = INFINITY, hi = -INFINITY;
    if (n <= TR_CAP) {
        // a short row: every score is listed, and its range found on the way
        for (int j = tid; j < n; j += TR_THREADS) {
            const float x = __ldcg(row + j);
            sh_list[j] = make_uint2((uint32_t)j, __float_as_uint(x));
            lo = fminf(lo, x);
            hi = fmaxf(hi, x);
        }
        tr_range(lo, hi, sh.ws);
        listed = (uint32_t)n;
    } else {
        // the whole row on its way into L2 while the threshold is chosen (one 128-byte line per prefetch): the
        // count pass then reads it from L2
        for (int64_t off = (int64_t)tid * 128; off < (int64_t)n * 4; off += (int64_t)TR_THREADS * 128)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(row) + off));
        // this warp's range; its first loads are in flight while the threshold is chosen
        const int span = (n + 2 * TR_THREADS - 1) / (2 * TR_THREADS) * 64;
        const int wlo = min(n, warp * span), whi = min(n, wlo + span);
        float2 x[TR_U];
        tr_load_any(row, wlo, whi, x);

        // ---- 1. the list's threshold tf from the sample
        constexpr int PER = TR_RUNS / TR_WARPS;
        float sv[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int run = warp + TR_WARPS * i;
            sv[i] = __ldcg(row + run * (n - 32) / (TR_RUNS - 1) + lane);
            lo = fminf(lo, sv[i]);
            hi = fmaxf(hi, sv[i]);
        }
        for (int i = tid; i < TR_SBINS; i += TR_THREADS) sh.hist[i] = 0;
        if (tid == 0) sh.misc[0] = 0;
        tr_range(lo, hi, sh.ws);
        const float scale = tr_scale(lo, hi, TR_SBINS);
        const float width = (hi - lo) * (1.f / TR_SBINS);
#pragma unroll
        for (int i = 0; i < PER; ++i) atomicAdd(&sh.hist[tr_bin((sv[i] - lo) * scale, (float)(TR_SBINS - 1))], 1u);
        __syncthreads();
        // the expected rank of the K-th score among the samples, plus four standard deviations
        const float q = __fdividef((float)K, (float)n), m = (float)TR_SAMPLES;
        const int s = min(TR_SAMPLES, (int)(q * m + 4.f * sqrtf(m * q * (1.f - q))) + 2);
        tr_pick<TR_SBINS>(sh.hist, (uint32_t)s, sh.ws, sh.misc);
        // any tf will do: what is listed is decided by the comparisons below alone
        const float tf = scale > 0.f ? fmaf((float)sh.misc[0], width, lo) : lo;

        // ---- 2. count this warp's scores >= tf, then list them at the warp's offset
        uint32_t cw = 0;
        for (int p = wlo;;) {
#pragma unroll
            for (int u = 0; u < TR_U; ++u) cw += (x[u].x >= tf ? 1u : 0u) + (x[u].y >= tf ? 1u : 0u);
            p += 64 * TR_U;
            if (p >= whi) break;
            tr_load_any(row, p, whi, x);
        }
        cw = __reduce_add_sync(0xffffffffu, cw);
        if (lane == 0) sh.ws[warp] = cw;
        __syncthreads();
        uint32_t o = 0;
#pragma unroll
        for (int w = 0; w < TR_WARPS; ++w) {
            listed += sh.ws[w];
            o += w < warp ? sh.ws[w] : 0u;
        }
        if (listed >= (uint32_t)K && listed <= (uint32_t)TR_CAP) {
            const uint32_t lt = (1u << lane) - 1u;
            for (int p = wlo; p < whi; p += 64 * TR_U) {
                tr_load_any(row, p, whi, x);
#pragma unroll
                for (int u = 0; u < TR_U; ++u) {
                    // order within the step: lane, then the lane's two positions
                    const bool i0 = x[u].x >= tf, i1 = x[u].y >= tf;
                    const uint32_t b0 = __ballot_sync(0xffffffffu, i0), b1 = __ballot_sync(0xffffffffu, i1);
                    const uint32_t at = o + __popc(b0 & lt) + __popc(b1 & lt);
                    const uint32_t q = (uint32_t)(p + 64 * u + 2 * lane);
                    // a lane with nothing to list writes its scratch entry: no branch
                    sh_list[i0 ? at : (uint32_t)(TR_CAP + lane)] = make_uint2(q, __float_as_uint(x[u].x));
                    sh_list[i1 ? at + (i0 ? 1u : 0u) : (uint32_t)(TR_CAP + lane)] =
                        make_uint2(q + 1, __float_as_uint(x[u].y));
                    o += __popc(b0) + __popc(b1);
                }
            }
        }
        lo = tf;  // hi stays the sample maximum: listed scores above it count in the top bin
    }
    __syncthreads();

    // ---- 3. the top-K of the list
    uint32_t tau, need;
    if (listed >= (uint32_t)K && listed <= (uint32_t)TR_CAP && tr_finish(sh_list, (int)listed, K, lo, hi, sh, out))
        return;
    __syncthreads();
    // the list missed scores or overflowed, or its threshold bin is crowded (ties): exact radix levels over the
    // row's keys
    tr_select([&](int j) { return score_key(__ldcg(row + j)); }, n, (uint32_t)K, 0u, 0xFFFFFFFFu, sh, tau, need);
    tr_compact([&](int j) { return make_uint2((uint32_t)j, score_key(__ldcg(row + j))); }, n, tau, need, out, K,
               sh.ws, err);
}

}  // namespace

bool topk_rows_eligible(int32_t R, int32_t K, int32_t max_row_len) {
    // K up to half the list: a larger K would overflow it on most rows (the radix fallback every time)
    const DeviceInfo *dev = current_device();
    return dev && R >= 2 * dev->sm_count && max_row_len <= TR_MAXN && K <= TR_CAP / 2;
}

dsa_status launch_topk_rows(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.R == 0) return DSA_OK;
    if (a.max_row_len > TR_MAXN) return DSA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(a.scores) & 15u) || (a.ld & 3)) return DSA_ERR_INVALID_ARG;
    if (!ensure_smem(reinterpret_cast<const void *>(topk_rows_kernel), TR_SMEM)) return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.R);
    cfg.blockDim = dim3(TR_THREADS);
    cfg.dynamicSmemBytes = TR_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, topk_rows_kernel, a, dev->err) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
