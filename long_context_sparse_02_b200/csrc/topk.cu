// Stage 2 of the Gated DSA layer: per-row top-K selection.
//
// Keeps the K highest indexer scores of each row ("Open-Source LLM
// Architecture Evolution", Architecture Breakdown §2, "Top-K selection",
// K = 2048; "Fine-Grained Sparse Attention in Ultra-Large Parameter Models",
// §2.1), every position when the row is not longer than K.  Ties go to the
// lower position and -0.0 equals +0.0.  The kept positions are written in
// ascending order, padded with -1.
//
// Exact radix select on order-preserving 32-bit keys: digit passes find the
// K-th largest key tau and the number `need`
// of keys equal to tau that are kept; a stable compaction in position order
// then takes every key > tau and the first `need` keys == tau.
//   * rows whose slice fits in shared memory: one thread-block cluster per
//     row (8 CTAs when rows are few, 1 when they are many), four 8-bit passes,
//     histograms merged through distributed shared memory;
//   * longer rows: CHUNK-key slices per CTA, per-row global histograms, the
//     last CTA of a pass (atomic ticket, no waiting) picks the digit; then a
//     count pass and an offset-and-write pass.
#include <mutex>
#include <vector>

#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int CHUNK = 4096;       // keys per CTA on the multi-CTA path
constexpr int MULTI_THREADS = 256;
constexpr int HBINS = 2048;

struct Pass {
    int shift, bits;
};
__device__ __constant__ Pass kPass[3] = {{21, 11}, {10, 11}, {0, 10}};

__device__ __forceinline__ int row_length(const TopkArgs &a, int r, uint32_t *err) {
    int n;
    if (a.mode == ROWLEN_ARRAY) n = a.row_len[r];
    else if (a.mode == ROWLEN_QPOS_PLUS_1) n = a.row_len[r] + 1;
    else n = a.row_len[r];  // ROWLEN_SEQ_LENS: decode, row r = sequence r
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

// Picks, from a histogram of `nb` bins, the bin b holding the remaining-th
// largest key: sum(hist[b+1:]) < remaining <= sum(hist[b:]).  Block-wide;
// returns (b, keys in bins above b) in *out (shared).
template <int NT>
__device__ void pick_bin(const uint32_t *hist, int nb, uint32_t remaining, uint32_t *scan, int2 *out) {
    const int tid = threadIdx.x;
    constexpr int PER = HBINS / NT > 0 ? HBINS / NT : 1;
    // thread tid owns bins [tid*PER, tid*PER+PER) counted from the TOP
    uint32_t local = 0;
    for (int i = 0; i < PER; ++i) {
        const int bin = nb - 1 - (tid * PER + i);
        if (bin >= 0) local += hist[bin];
    }
    scan[tid] = local;
    __syncthreads();
    // inclusive scan over threads (Hillis-Steele)
    for (int o = 1; o < NT; o <<= 1) {
        uint32_t v = tid >= o ? scan[tid - o] : 0;
        __syncthreads();
        scan[tid] += v;
        __syncthreads();
    }
    const uint32_t incl = scan[tid];
    const uint32_t excl = incl - local;
    if (excl < remaining && remaining <= incl) {
        uint32_t above = excl;
        for (int i = 0; i < PER; ++i) {
            const int bin = nb - 1 - (tid * PER + i);
            if (bin < 0) break;
            if (above + hist[bin] >= remaining) {
                *out = make_int2(bin, (int)above);
                break;
            }
            above += hist[bin];
        }
    }
    __syncthreads();
}

// Block-wide exclusive scan of two small counters packed as (hi16, lo16).
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan_packed(uint32_t v, uint32_t *wsum, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t n = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += n;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < NT / 32 ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        if (lane < NT / 32) wsum[lane] = s;
        if (lane == 31) *total = s;
    }
    __syncthreads();
    const uint32_t base = warp > 0 ? wsum[warp - 1] : 0;
    const uint32_t res = base + x - v;
    __syncthreads();
    return res;
}

// Writes the kept positions of [s0, s1) in order.  gt_before/eq_before count
// keys > tau / == tau before s0 in the row.
template <int NT, typename KeyAt>
__device__ void compact(KeyAt key_at, int s0, int s1, uint32_t tau, uint32_t need, uint32_t gt_before,
                        uint32_t eq_before, int32_t *out, int K, uint32_t *wsum, uint32_t *total, uint32_t *err) {
    for (int base = s0; base < s1; base += NT) {
        const int s = base + threadIdx.x;
        uint32_t gt = 0, eq = 0;
        if (s < s1) {
            const uint32_t k = key_at(s);
            gt = k > tau;
            eq = k == tau;
        }
        const uint32_t pk = block_excl_scan_packed<NT>((gt << 16) | eq, wsum, total);
        const uint32_t tot = *total;
        const uint32_t e_before = eq_before + (pk & 0xFFFFu);
        const uint32_t g_before = gt_before + (pk >> 16);
        if (gt || (eq && e_before < need)) {
            const uint32_t slot = g_before + min(e_before, need);
            if (slot < (uint32_t)K) out[slot] = s;
            else record_error(err, DSA_DEVERR_SHAPE);
        }
        gt_before += tot >> 16;
        eq_before += tot & 0xFFFFu;
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// One thread-block cluster per row (CL CTAs; CL = 1 for many short rows).
// Each CTA holds its contiguous slice of the row (raw fp32 scores) in shared
// memory.
//
//   1. load the slice (16-byte loads); the row's key range [min, max] over
//      the cluster (barrier 1);
//   2. a histogram of LBINS equal-width bins over [min, max] in score space.
//      The bin of a score x is floor((x - min) * LBINS / (max - min)) in
//      fp32 with every rounding monotone, so the bins split the row into
//      consecutive key intervals.  Each CTA bins its slice, then adds its
//      counts into the CTA that owns each bin (LBINS / CL bins per CTA;
//      barrier 2);
//   3. every CTA reads the totals (one 8-byte remote load per thread) and
//      finds the bin b holding the K-th largest key.  One sweep of the slice
//      lists, per warp and in position order, the positions whose bin is
//      >= b, and collects the keys of bin b (barrier 3).  Every key in a bin
//      above b is kept; an exact select on the cluster's keys of bin b (few
//      unless the row is degenerate) gives the threshold key tau and how
//      many keys equal to tau are kept;
//   4. stable compaction of the listed positions (the whole slice when a
//      warp's list overflows) in position order.
// Rows whose bin b holds more than CAND_CAP keys (heavy ties, an outlier
// that squeezes the rest into one bin) or whose range is not finite fall
// back to 8-bit radix passes over the whole slice.  Counts and candidates
// move through distributed shared memory.
// ---------------------------------------------------------------------------
constexpr int CT_THREADS = 1024;
constexpr int CT_WARPS = CT_THREADS / 32;
constexpr int LBINS = 2048;
constexpr int CAND_CAP = 4096;  // keys of the threshold bin, whole cluster
constexpr int WCAP = 128;       // listed positions per warp
constexpr int RANK_MAX = 128;   // at most this many candidates: select by counting ranks
// shared memory, in 32-bit words
constexpr int CT_W_WORDS = CT_WARPS * 256;  // radix warp histograms | candidate lists
constexpr int OWN_WORDS = LBINS / 2;        // bins owned by one CTA (CL >= 2)
static_assert(2 * ((LBINS / 2 + 2 - 1) / 2) <= OWN_WORDS, "owned bins fit");
constexpr int CT_FIXED_WORDS =
    CT_W_WORDS + LBINS + OWN_WORDS + 2 * CT_WARPS * WCAP + 2 * 256 + 256 + CT_WARPS * 4 + 64 + 4;
constexpr int CT_FIXED_SMEM = CT_FIXED_WORDS * 4;
static_assert(CT_W_WORDS >= 2 * CAND_CAP, "candidate lists alias the radix histograms");
static_assert(CT_FIXED_WORDS % 4 == 0, "the slice starts 16-byte aligned");
static_assert(LBINS == 2 * CT_THREADS, "two bins per thread");
// misc words: 0,1 digit/bin pick; 2 candidate counter; 3 keys in bin b (cluster);
// 4,5 CTA totals (radix path) / tau, need; 6,7 offsets; 8,9 CTA key range;
// 10,11 row key range; 12,13 sums; 20,21 this CTA's keys above b / in b;
// 22 list overflow; 24,25 above-b keys / bin-b keys of earlier CTAs;
// 32..47 bin-b keys of earlier CTAs, per CTA rank

__device__ __forceinline__ int linear_bin(float x, float lo, float scale) {
    const float y = __fmul_rn(__fsub_rn(x, lo), scale);
    return min(LBINS - 1, __float2int_rz(y));
}
__device__ __forceinline__ float key_score(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Block-wide (CT_THREADS) inclusive scan; ws holds CT_WARPS words.
__device__ __forceinline__ uint32_t ct_incl_scan(uint32_t v, uint32_t *ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t t = ws[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        ws[lane] = t;
    }
    __syncthreads();
    return x + (warp > 0 ? ws[warp - 1] : 0u);
}

// Block-wide sums of two counters; ws holds 2 * CT_WARPS words, out 2 words.
__device__ __forceinline__ void ct_sum2(uint32_t a, uint32_t b, uint32_t *ws, uint32_t *out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
        ws[2 * warp] = a;
        ws[2 * warp + 1] = b;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t x = ws[2 * lane], y = ws[2 * lane + 1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            x += __shfl_xor_sync(0xffffffffu, x, o);
            y += __shfl_xor_sync(0xffffffffu, y, o);
        }
        if (lane == 0) {
            out[0] = x;
            out[1] = y;
        }
    }
    __syncthreads();
}

// Warp 0: from a 256-bin digit histogram (tot), the digit holding the
// remaining-th largest key and the count of keys in higher digits -> res[0..1].
__device__ __forceinline__ void pick_digit256(const uint32_t *tot, uint32_t remaining, uint32_t *res) {
    const int lane = threadIdx.x & 31;
    uint32_t v[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // lane l owns digits 255-8l .. 248-8l (from the top)
        v[i] = tot[255 - 8 * lane - i];
        sum += v[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    const uint32_t excl = incl - sum;
    if (excl < remaining && remaining <= incl) {
        uint32_t above = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (above + v[i] >= remaining) {
                res[0] = 255 - 8 * lane - i;
                res[1] = above;
                break;
            }
            above += v[i];
        }
    }
}

template <int CL>
__device__ __forceinline__ void ct_cluster_or_block_sync() {
    if (CL > 1) cluster_sync();
    else __syncthreads();
}

// Exact select among C keys (block-wide): the rem-th largest key -> res[0]
// and how many keys equal to it are among the rem largest -> res[1].
__device__ void select_among(const uint32_t *cand, int C, uint32_t rem, uint32_t *hist, uint32_t *wcnt,
                             uint32_t *res) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (C <= RANK_MAX) {
        // rank of key j in the order (key descending, index ascending)
        if (tid < C) {
            const uint32_t kj = cand[tid];
            uint32_t g = 0, e = 0;
            for (int i = 0; i < C; ++i) {
                const uint32_t ki = cand[i];
                g += ki > kj;
                e += (ki == kj) & (i < tid);
            }
            if (g + e == rem - 1) {
                res[0] = kj;
                res[1] = rem - g;
            }
        }
        __syncthreads();
        return;
    }
    uint32_t cmn = 0xFFFFFFFFu, cmx = 0u;
    for (int j = tid; j < C; j += CT_THREADS) {
        cmn = min(cmn, cand[j]);
        cmx = max(cmx, cand[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        cmn = min(cmn, __shfl_xor_sync(0xffffffffu, cmn, o));
        cmx = max(cmx, __shfl_xor_sync(0xffffffffu, cmx, o));
    }
    if (lane == 0) {
        wcnt[warp * 4 + 2] = cmn;
        wcnt[warp * 4 + 3] = cmx;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t a0 = wcnt[lane * 4 + 2], a1 = wcnt[lane * 4 + 3];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a0 = min(a0, __shfl_xor_sync(0xffffffffu, a0, o));
            a1 = max(a1, __shfl_xor_sync(0xffffffffu, a1, o));
        }
        if (lane == 0) {
            res[2] = a0;
            res[3] = a1;
        }
    }
    __syncthreads();
    const uint32_t c0 = res[2], c1 = res[3];
    int bits = c0 == c1 ? 0 : 32 - __clz(c0 ^ c1);
    uint32_t prefix = bits >= 32 ? 0u : (c1 >> bits), remaining = rem;
    while (bits > 0) {
        const int d = bits < 8 ? bits : 8;
        const int shift = bits - d, hs = shift + d;
        if (tid < 256) hist[tid] = 0;
        __syncthreads();
        for (int j = tid; j < C; j += CT_THREADS) {
            const uint32_t k = cand[j];
            if (hs >= 32 || (k >> hs) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) pick_digit256(hist, remaining, res);
        __syncthreads();
        prefix = (prefix << d) | res[0];
        remaining -= res[1];
        bits = shift;
        __syncthreads();  // res[0..1] read by every thread before the next pick
    }
    __syncthreads();
    if (tid == 0) {
        res[0] = prefix;
        res[1] = remaining;
    }
    __syncthreads();
}

template <int CL>
__global__ void __launch_bounds__(CT_THREADS, 1) topk_cluster_kernel(const TopkArgs a, uint32_t *err) {
    extern __shared__ __align__(16) uint32_t sm[];
    uint32_t *whist = sm;                  // radix path: [32][256] warp-private histograms
    uint32_t *cand_local = sm;             // binned path: this CTA's keys of bin b (read by the cluster)
    uint32_t *cand_all = sm + CAND_CAP;    // binned path: the cluster's keys of bin b, CTA order
    uint32_t *lhist = sm + CT_W_WORDS;     // [LBINS] this CTA's linear histogram
    uint32_t *own = lhist + LBINS;         // [LBINS / CL] cluster totals of the bins this CTA owns
    uint32_t *wlist = own + OWN_WORDS;     // [32][WCAP] per-warp listed positions
    uint32_t *wkey = wlist + CT_WARPS * WCAP;  // [32][WCAP] their keys (histogram path)
    uint32_t *chist = wkey + CT_WARPS * WCAP;  // [2][256] radix path: this CTA's digit histogram
    uint32_t *lcnt = chist;                // [32] binned path: listed positions per warp
    uint32_t *tot = chist + 2 * 256;       // [256] digit histogram
    uint32_t *wcnt = tot + 256;            // [32][4] per-warp scratch
    uint32_t *misc = wcnt + CT_WARPS * 4;  // [64] scalars (see above)
    uint64_t *sbar = reinterpret_cast<uint64_t *>(misc + 64);  // the slice's bulk copy
    float *xs = reinterpret_cast<float *>(misc + 68);          // [slice] the scores
    constexpr int W = 2 * ((LBINS / 2 + CL - 1) / CL);  // bins owned per CTA (even: bin pairs share an owner)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t crank = CL > 1 ? cluster_ctarank() : 0;
    const int r = blockIdx.x / CL;
    const int n = row_length(a, r, crank == 0 ? err : nullptr);
    int32_t *out = a.idx + (int64_t)r * a.K;
    // This CTA's share of the row's score histogram is cleared for the next
    // call once every CTA of the cluster has read it.
    auto clear_hist_share = [&]() {
        uint32_t *hr = a.hist + (int64_t)r * SCORE_HIST_BINS;
        for (int i = (int)crank * SCORE_HIST_BINS / CL + tid; i < ((int)crank + 1) * SCORE_HIST_BINS / CL; i += CT_THREADS)
            hr[i] = 0;
    };
    if (n <= a.K) {  // uniform across the cluster: every CTA returns here
        const int per = (a.K + CL - 1) / CL;
        for (int j = crank * per + tid; j < min(a.K, (int)(crank + 1) * per); j += CT_THREADS) out[j] = j < n ? j : -1;
        if (a.hist) {
            pdl_wait();  // the histogram is complete
            clear_hist_share();
        }
        return;
    }
    const int len = ((n + CL - 1) / CL + 3) & ~3;  // slices start 4 keys apart
    const int s0 = min(n, (int)crank * len);
    const int m = min(n, s0 + len) - s0;
    const float *row = a.scores + (int64_t)r * a.ld + s0;
    // Histogram path: the slice arrives in one bulk copy (the copy engine keeps
    // more of it in flight than per-thread loads do).
    const bool bulk = a.hist != nullptr && m > 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0 &&
                      (a.ld & 3) == 0;
    if (bulk && tid == 0) {
        mbar_init(sbar, 1);
        fence_mbar_init();
    }
    if (bulk) __syncthreads();  // the barrier is initialised before anyone waits on it
    pdl_trigger();
    pdl_wait();  // the scores come from the previous kernel
    if (bulk && tid == 0) {
        const uint32_t bytes = (uint32_t)((m + 3) & ~3) * 4u;
        mbar_expect_tx(sbar, bytes);
        bulk_load(xs, row, bytes, sbar);
    }

    bool fast_done = false, final_wait = CL > 1;
    if (a.hist) {
        // ---- histogram path.  The indexer counted the row's keys by their
        // top bits (coarse bins).  Every CTA finds the coarse bin B of the
        // K-th largest key from those counts; one pass over the slice lists,
        // per warp and in position order, every position whose coarse bin is
        // >= B with its key, and bins the keys of B into LBINS equal-width
        // fine bins over B's score range; the fine counts meet in their owner
        // CTAs (barrier 2); every CTA picks the fine bin of the K-th largest
        // key; each CTA then stores its counts and its keys of that fine bin
        // into every CTA of the cluster (barrier 3), after which all the rest
        // is local: an exact select among those few keys and the compaction.
        // Counts that do not add up to the row length (a workspace not
        // cleared yet), a non-finite bin range or a full list take the full
        // path below.
        constexpr int CPR = CAND_CAP / 16;  // keys of the fine bin per CTA, stored at [rank][CPR]
        const uint32_t *hr = a.hist + (int64_t)r * SCORE_HIST_BINS;
        const int hb0 = SCORE_HIST_BINS - 1 - 2 * tid, hb1 = hb0 - 1;
        const uint2 hv = *reinterpret_cast<const uint2 *>(hr + hb1);  // first: its latency hides behind the slice's
        if (CL > 1) {
            for (int i = tid; i < W; i += CT_THREADS) own[i] = 0;
            cluster_arrive();  // own[] is clear before any CTA adds into it (paired wait below)
        }
        for (int i = tid; i < LBINS; i += CT_THREADS) lhist[i] = 0;
        // the slice, 128 keys per warp step, loaded before anything waits on it
        constexpr int NSTEP = 4;
        const int per4 = ((m + CT_WARPS - 1) / CT_WARPS + 127) & ~127;
        const int w0 = warp * per4, w1 = min(m, w0 + per4);
        // uniform across the cluster: decided on the common slice length, not this CTA's m
        // (and on the alignment of the score rows, which is common to every slice)
        const bool fits = (((len + CT_WARPS - 1) / CT_WARPS + 127) & ~127) <= NSTEP * 128 &&
                          (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0 && (a.ld & 3) == 0;
        float xv[NSTEP][4];
        // the copy is waited for on every path: nothing else may write xs while it is in flight
        if (bulk) mbar_wait(sbar, 0, err, nullptr);
        if (fits) {
#pragma unroll
            for (int st = 0; st < NSTEP; ++st) {
                const int i0 = w0 + st * 128 + 4 * lane;
                if (i0 + 3 < w1) {
                    const float4 v = *reinterpret_cast<const float4 *>(xs + i0);
                    xv[st][0] = v.x, xv[st][1] = v.y, xv[st][2] = v.z, xv[st][3] = v.w;
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) xv[st][k] = i0 + k < w1 ? xs[i0 + k] : -INFINITY;
                }
            }
        }
        const uint32_t v0 = hv.y, v1 = hv.x, Ku = (uint32_t)a.K;
        const bool sane = __syncthreads_and(v0 <= (uint32_t)n && v1 <= (uint32_t)n) != 0;
        const uint32_t incl = ct_incl_scan(v0 + v1, wcnt);
        const uint32_t total = wcnt[CT_WARPS - 1];
        const uint32_t excl = incl - v0 - v1;
        if (sane && total == (uint32_t)n && excl < Ku && Ku <= incl) {
            const bool first = excl + v0 >= Ku;
            misc[0] = first ? hb0 : hb1;
            misc[1] = first ? excl : excl + v0;
        }
        if (tid == 0) misc[22] = 0;
        __syncthreads();
        const uint32_t B = misc[0], aboveB = misc[1];
        const float xlo = key_score(B << SCORE_HIST_SHIFT), xhi = key_score(((B + 1) << SCORE_HIST_SHIFT) - 1u);
        const float fscale = __fdiv_rn((float)LBINS, __fsub_rn(xhi, xlo));
        // uniform across the cluster: the same counts and bin everywhere
        const bool go = fits && sane && total == (uint32_t)n && isfinite(xlo) && isfinite(xhi) && xhi > xlo &&
                        isfinite(fscale);
        if (!go) {
            if (CL > 1) cluster_wait();
        } else {
            uint32_t *wl = wlist + warp * WCAP, *wk = wkey + warp * WCAP;
            uint32_t cnt = 0;
            const uint32_t lt = (1u << lane) - 1u;
            // A key is listed when its coarse bin is >= B, that is when its score is
            // >= xlo (keys are monotone in the score, xlo is finite here, and entries
            // past the slice hold -inf).  Listed keys are a few percent of the row, so
            // each key costs one compare; the list bookkeeping runs only in the warps
            // that found some, and usually with one ballot (at most one listed key
            // per lane).
#pragma unroll
            for (int st = 0; st < NSTEP; ++st) {
                const int i0 = w0 + st * 128 + 4 * lane;
                uint32_t selm = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) selm |= (xv[st][k] >= xlo ? 1u : 0u) << k;
                const uint32_t anyl = __ballot_sync(0xffffffffu, selm != 0);
                if (anyl == 0) continue;
                // list slot of this lane's first key: every listed key of the lower lanes comes first
                uint32_t before, stot;
                if (__any_sync(0xffffffffu, (selm & (selm - 1u)) != 0)) {
                    before = 0, stot = 0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t bk = __ballot_sync(0xffffffffu, (selm >> k) & 1u);
                        before += __popc(bk & lt);
                        stot += __popc(bk);
                    }
                } else {
                    before = __popc(anyl & lt);
                    stot = __popc(anyl);
                }
                uint32_t so = cnt + before;
#pragma unroll
                for (int k = 0; k < 4; ++k) {  // predicated, not branched: most warps list a key of some lane
                    const bool b = ((selm >> k) & 1u) != 0;
                    const float x = xv[st][k];
                    const uint32_t key = score_key(x);
                    const int fbn = linear_bin(x, xlo, fscale);  // meaningful only for keys of bin B
                    inc_shared_if(lhist + (fbn > 0 ? fbn : 0), b && (key >> SCORE_HIST_SHIFT) == B);
                    st_shared_if(wl + (so < (uint32_t)WCAP ? so : 0u), (uint32_t)(i0 + k), b && so < (uint32_t)WCAP);
                    st_shared_if(wk + (so < (uint32_t)WCAP ? so : 0u), key, b && so < (uint32_t)WCAP);
                    so += b ? 1u : 0u;
                }
                cnt += stot;
            }
            if (lane == 0) {
                lcnt[warp] = cnt;
                if (cnt > (uint32_t)WCAP) misc[22] = 1;
            }
            __syncthreads();  // the fine histogram of this CTA is complete
            if (CL > 1) {
                cluster_wait();  // every CTA's own[] is clear
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int bin = tid + h * CT_THREADS;
                    const uint32_t v = lhist[bin];
                    if (v) dsmem_red_add(dsmem_addr(own + bin % W, bin / W), v);
                }
            }
            ct_cluster_or_block_sync<CL>();  // barrier 2: every fine total and overflow flag is in place
            // the fine bin of the K-th largest key among bin B's keys (thread t: fine bins LBINS-1-2t, LBINS-2-2t)
            const int fb0 = LBINS - 1 - 2 * tid, fb1 = fb0 - 1;
            uint2 t2;
            if (CL > 1) t2 = dsmem_ld_v2(dsmem_addr(own + fb1 % W, fb1 / W));
            else t2 = make_uint2(lhist[fb1], lhist[fb0]);
            const uint32_t f0 = t2.y, f1 = t2.x, rem = Ku - aboveB;
            uint32_t ovf = 0;
            if (warp == 0 && lane < CL) ovf = CL > 1 ? ld_dsmem_u32(misc + 22, lane) : misc[22];
            const uint32_t fincl = ct_incl_scan(f0 + f1, wcnt);
            const uint32_t fexcl = fincl - f0 - f1;
            if (fexcl < rem && rem <= fincl) {
                const bool first = fexcl + f0 >= rem;
                misc[8] = first ? fb0 : fb1;
                misc[9] = first ? fexcl : fexcl + f0;
                misc[10] = first ? f0 : f1;
            }
            if (warp == 0) {
                const bool any_ovf = __any_sync(0xffffffffu, ovf != 0);
                if (lane == 0) misc[26] = any_ovf;
            }
            if (tid == 0) {
                misc[2] = 0;   // candidates of this CTA
                misc[20] = 0;  // keys of this CTA above the threshold fine bin
            }
            __syncthreads();
            if (misc[26] == 0) {  // uniform across the cluster; else every CTA takes the full path
                const int fb = (int)misc[8];
                const uint32_t abovef = misc[9], Cf = misc[10];
                // this CTA's candidates (fine bin fb of B), stored into every CTA at [crank][CPR]
                const int wn = (int)lcnt[warp];
                uint32_t nab = 0;
                for (int j0 = 0; j0 < wn; j0 += 32) {
                    const int j = j0 + lane;
                    const uint32_t k = j < wn ? wk[j] : 0u;
                    int f = -1;
                    bool ab = false;
                    if (j < wn) {
                        if ((k >> SCORE_HIST_SHIFT) > B) ab = true;
                        else {
                            f = linear_bin(key_score(k), xlo, fscale);
                            ab = f > fb;
                        }
                    }
                    nab += __popc(__ballot_sync(0xffffffffu, ab));
                    const bool isc = f == fb;
                    const uint32_t cm = __ballot_sync(0xffffffffu, isc);
                    if (cm) {
                        uint32_t base = 0;
                        if (lane == 0) base = atomicAdd(&misc[2], (uint32_t)__popc(cm));
                        base = __shfl_sync(0xffffffffu, base, 0);
                        const uint32_t slot = base + __popc(cm & lt);
                        if (isc && slot < (uint32_t)CPR)
                            for (int q = 0; q < CL; ++q) {
                                uint32_t *dst = cand_all + crank * CPR + slot;
                                if (CL > 1) dsmem_st(dsmem_addr(dst, q), k);
                                else *dst = k;
                            }
                    }
                }
                if (lane == 0) atomicAdd(&misc[20], nab);
                __syncthreads();  // this CTA's counts are final
                if (tid < CL) {   // (keys above, candidates) of this CTA into slot crank of every CTA
                    if (CL > 1) {
                        dsmem_st(dsmem_addr(misc + 32 + crank, tid), misc[20]);
                        dsmem_st(dsmem_addr(misc + 48 + crank, tid), misc[2]);
                    } else {
                        misc[32] = misc[20];
                        misc[48] = misc[2];
                    }
                }
                ct_cluster_or_block_sync<CL>();  // barrier 3: every count and key is stored everywhere
                if (warp == 0) {
                    // the candidates in rank order, contiguous; the counts of the earlier ranks
                    uint32_t hq = lane < CL ? misc[32 + lane] : 0u, cq = lane < CL ? misc[48 + lane] : 0u;
                    const bool ovc = __any_sync(0xffffffffu, cq > (uint32_t)CPR);
                    uint32_t hx = hq, cx = cq;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y0 = __shfl_up_sync(0xffffffffu, hx, o), y1 = __shfl_up_sync(0xffffffffu, cx, o);
                        if (lane >= o) hx += y0, cx += y1;
                    }
                    const uint32_t ctot = __shfl_sync(0xffffffffu, cx, 31), htot = __shfl_sync(0xffffffffu, hx, 31);
                    const uint32_t cbefore = __shfl_sync(0xffffffffu, cx - cq, crank);
                    const uint32_t hbefore = __shfl_sync(0xffffffffu, hx - hq, crank);
                    if (lane == 0) {
                        misc[24] = hbefore;
                        misc[25] = cbefore;
                        misc[27] = ctot;
                        // more keys in a CTA's fine bin than its slots, or counts that disagree
                        // with the histograms: the full path (identical copies: uniform)
                        misc[28] = ovc || ctot != Cf || htot != aboveB + abovef;
                    }
                    if (!ovc) for (int q = 0; q < CL; ++q) {
                        const uint32_t cn = min(__shfl_sync(0xffffffffu, cq, q), (uint32_t)CPR);
                        const uint32_t o = __shfl_sync(0xffffffffu, cx - cq, q);
                        for (uint32_t i = lane; i < cn; i += 32) cand_local[o + i] = cand_all[q * CPR + i];
                    }
                }
                __syncthreads();
              if (misc[28] == 0) {
                final_wait = false;  // no CTA reads or writes another's shared memory from here on
                clear_hist_share();
                const uint32_t C = misc[27];
                select_among(cand_local, (int)C, rem - abovef, tot, wcnt, misc + 4);
                const uint32_t tau = misc[4], need = misc[5];
                const uint32_t hi_before = misc[24], c_before = misc[25];
                uint32_t g = 0, e = 0;
                for (int j = tid; j < (int)c_before; j += CT_THREADS) {
                    g += cand_local[j] > tau;
                    e += cand_local[j] == tau;
                }
                ct_sum2(g, e, wcnt, misc + 12);
                const uint32_t gt_before = hi_before + misc[12], eq_before = misc[13];
                // compaction of the listed positions, in position order
                g = 0, e = 0;
                for (int j0 = 0; j0 < wn; j0 += 32) {
                    const int j = j0 + lane;
                    const uint32_t k = j < wn ? wk[j] : 0u;
                    g += __popc(__ballot_sync(0xffffffffu, j < wn && k > tau));
                    e += __popc(__ballot_sync(0xffffffffu, j < wn && k == tau));
                }
                if (lane == 0) {
                    wcnt[warp * 4 + 0] = g;
                    wcnt[warp * 4 + 1] = e;
                }
                __syncthreads();
                if (warp == 0) {
                    const uint32_t gv = wcnt[lane * 4 + 0], ev = wcnt[lane * 4 + 1];
                    uint32_t gi = gv, ei = ev;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t xg = __shfl_up_sync(0xffffffffu, gi, o), xe = __shfl_up_sync(0xffffffffu, ei, o);
                        if (lane >= o) gi += xg, ei += xe;
                    }
                    wcnt[lane * 4 + 2] = gi - gv;
                    wcnt[lane * 4 + 3] = ei - ev;
                }
                __syncthreads();
                uint32_t gcur = gt_before + wcnt[warp * 4 + 2], ecur = eq_before + wcnt[warp * 4 + 3];
                for (int j0 = 0; j0 < wn; j0 += 32) {
                    const int j = j0 + lane;
                    const uint32_t k = j < wn ? wk[j] : 0u;
                    const bool gt = j < wn && k > tau, eq = j < wn && k == tau;
                    const uint32_t gm = __ballot_sync(0xffffffffu, gt), em = __ballot_sync(0xffffffffu, eq);
                    const uint32_t mg = gcur + __popc(gm & lt), me = ecur + __popc(em & lt);
                    const bool keep = gt || (eq && me < need);
                    const uint32_t slot = mg + min(me, need);
                    st_global_if(out + slot, (uint32_t)(s0 + (int)(j < wn ? wl[j] : 0u)), keep && slot < Ku);
                    if (keep && slot >= Ku) record_error(err, DSA_DEVERR_SHAPE);
                    gcur += __popc(gm);
                    ecur += __popc(em);
                }
                fast_done = true;
              }
            }
        }
    }

    if (!fast_done) {
    // ---- 1. load the slice; its key range.  Histograms and counters are
    // cleared here: barrier 1 orders that before any CTA adds into them.
    for (int i = tid; i < LBINS; i += CT_THREADS) lhist[i] = 0;
    if (CL > 1)
        for (int i = tid; i < W; i += CT_THREADS) own[i] = 0;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    {
        int done = 0;
        if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
            const int m4 = m >> 2;
            const float4 *r4 = reinterpret_cast<const float4 *>(row);
            float4 *x4 = reinterpret_cast<float4 *>(xs);
            constexpr int U = 4;
            for (int base = 0; base < m4; base += U * CT_THREADS) {
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = base + u * CT_THREADS + tid;
                    if (i < m4) v[u] = r4[i];
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int i = base + u * CT_THREADS + tid;
                    if (i < m4) {
                        x4[i] = v[u];
                        const uint32_t k0 = score_key(v[u].x), k1 = score_key(v[u].y), k2 = score_key(v[u].z),
                                       k3 = score_key(v[u].w);
                        kmin = min(kmin, min(min(k0, k1), min(k2, k3)));
                        kmax = max(kmax, max(max(k0, k1), max(k2, k3)));
                    }
                }
            }
            done = m4 * 4;
        }
#pragma unroll 4
        for (int i = done + tid; i < m; i += CT_THREADS) {
            const float x = row[i];
            xs[i] = x;
            const uint32_t k = score_key(x);
            kmin = min(kmin, k);
            kmax = max(kmax, k);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        wcnt[warp * 4 + 0] = kmin;
        wcnt[warp * 4 + 1] = kmax;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t a0 = wcnt[lane * 4 + 0], a1 = wcnt[lane * 4 + 1];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a0 = min(a0, __shfl_xor_sync(0xffffffffu, a0, o));
            a1 = max(a1, __shfl_xor_sync(0xffffffffu, a1, o));
        }
        if (lane == 0) {
            misc[8] = a0;
            misc[9] = a1;
        }
    }
    ct_cluster_or_block_sync<CL>();  // cluster barrier 1: every CTA's range is published
    if (a.hist) clear_hist_share();  // every CTA has read the histogram
    if (tid == 0) misc[2] = 0;  // candidate counter: the histogram path's remote reads of it end before barrier 1
    if (warp == 0) {
        uint32_t g0 = 0xFFFFFFFFu, g1 = 0u;
        if (lane < CL) {
            g0 = CL > 1 ? ld_dsmem_u32(misc + 8, lane) : misc[8];
            g1 = CL > 1 ? ld_dsmem_u32(misc + 9, lane) : misc[9];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g0 = min(g0, __shfl_xor_sync(0xffffffffu, g0, o));
            g1 = max(g1, __shfl_xor_sync(0xffffffffu, g1, o));
        }
        if (lane == 0) {
            misc[10] = g0;
            misc[11] = g1;
        }
    }
    __syncthreads();
    const uint32_t gmin = misc[10], gmax = misc[11];

    if (gmin == gmax) {  // every key equal: the first K positions (uniform across the cluster)
        if (CL > 1) cluster_arrive();  // the range reads above were the last remote reads
        for (int i = tid; i < m && s0 + i < a.K; i += CT_THREADS) {
            out[s0 + i] = s0 + i;
        }
        if (CL > 1) cluster_wait();
        return;
    }

    uint32_t tau = 0, need = 0, gt_before = 0, eq_before = 0;
    bool binned = false, use_list = false;  // binned: uniform across the cluster
    const float lo = key_score(gmin), hi = key_score(gmax);
    const float width = __fsub_rn(hi, lo);
    const float scale = __fdiv_rn((float)LBINS, width);
    if (isfinite(lo) && isfinite(hi) && isfinite(width) && width > 0.f && isfinite(scale)) {
        // ---- 2. linear histogram over [lo, hi]; counts into the owning CTAs
        for (int i = tid; i < m; i += CT_THREADS) atomicAdd(&lhist[linear_bin(xs[i], lo, scale)], 1u);
        __syncthreads();
        if (CL > 1) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int bin = tid + h * CT_THREADS;
                const uint32_t v = lhist[bin];
                if (v) dsmem_red_add(dsmem_addr(own + bin % W, bin / W), v);
            }
        }
        ct_cluster_or_block_sync<CL>();  // cluster barrier 2: every total is complete
        // ---- 3. the bin of the K-th largest key (thread t: bins LBINS-1-2t, LBINS-2-2t)
        const int hb0 = LBINS - 1 - 2 * tid, hb1 = hb0 - 1;
        uint2 t2;
        if (CL > 1) t2 = dsmem_ld_v2(dsmem_addr(own + hb1 % W, hb1 / W));
        else t2 = make_uint2(lhist[hb1], lhist[hb0]);
        const uint32_t v0 = t2.y, v1 = t2.x;
        const uint32_t incl = ct_incl_scan(v0 + v1, wcnt);
        const uint32_t excl = incl - v0 - v1, Ku = (uint32_t)a.K;
        if (excl < Ku && Ku <= incl) {
            const bool first = excl + v0 >= Ku;
            misc[0] = first ? hb0 : hb1;
            misc[1] = first ? excl : excl + v0;
            misc[3] = first ? v0 : v1;
        }
        __syncthreads();
        const int b = (int)misc[0];
        const uint32_t above = misc[1], C = misc[3];
        if (C <= (uint32_t)CAND_CAP) {
            binned = true;
            // one sweep: per-warp lists of positions with bin >= b (position
            // order) and this CTA's keys of bin b
            const int per = (((m + CT_WARPS - 1) / CT_WARPS) + 31) & ~31;
            const int w0 = warp * per, w1 = min(m, w0 + per);
            uint32_t cnt = 0;
            uint32_t *wl = wlist + warp * WCAP;
            const uint32_t lt = (1u << lane) - 1u;
            for (int i0 = w0; i0 < w1; i0 += 32) {
                const int i = i0 + lane;
                const float x = i < w1 ? xs[i] : 0.f;
                const int bn = i < w1 ? linear_bin(x, lo, scale) : -1;
                const uint32_t sel = __ballot_sync(0xffffffffu, bn >= b);
                const uint32_t inb = __ballot_sync(0xffffffffu, bn == b);
                if (bn >= b) {
                    const uint32_t slot = cnt + __popc(sel & lt);
                    if (slot < (uint32_t)WCAP) wl[slot] = (uint32_t)i;
                }
                cnt += __popc(sel);
                if (inb) {
                    uint32_t base = 0;
                    if (lane == 0) base = atomicAdd(&misc[2], (uint32_t)__popc(inb));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (bn == b) cand_local[base + __popc(inb & lt)] = score_key(x);
                }
            }
            if (lane == 0) lcnt[warp] = cnt;
            __syncthreads();
            if (warp == 0) {
                const uint32_t c = lcnt[lane];
                uint32_t s = c;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                const bool ovf = __any_sync(0xffffffffu, c > (uint32_t)WCAP);
                if (lane == 0) {
                    misc[20] = s - lhist[b];  // keys above b in this CTA
                    misc[21] = lhist[b];      // keys in b in this CTA
                    misc[22] = ovf;
                }
            }
            ct_cluster_or_block_sync<CL>();  // cluster barrier 3: every candidate list is complete
            use_list = misc[22] == 0;
            if (warp == 0) {
                uint32_t hq = 0, cq = 0;
                if (lane < CL) {
                    hq = CL > 1 ? ld_dsmem_u32(misc + 20, lane) : misc[20];
                    cq = CL > 1 ? ld_dsmem_u32(misc + 21, lane) : misc[21];
                }
                uint32_t hx = hq, cx = cq;  // inclusive prefix over CTA ranks
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y0 = __shfl_up_sync(0xffffffffu, hx, o), y1 = __shfl_up_sync(0xffffffffu, cx, o);
                    if (lane >= o) hx += y0, cx += y1;
                }
                if (lane < CL) misc[32 + lane] = cx - cq;  // bin-b keys of earlier CTAs
                if (lane == (int)crank) {
                    misc[24] = hx - hq;
                    misc[25] = cx - cq;
                }
            }
            __syncthreads();
            const uint32_t *cand = cand_local;
            if (CL > 1) {
                for (int j = tid; j < (int)C; j += CT_THREADS) {
                    int q = 0;
                    while (q < CL - 1 && (uint32_t)j >= misc[32 + q + 1]) ++q;
                    cand_all[j] = ld_dsmem_u32(cand_local + (j - misc[32 + q]), q);
                }
                cluster_arrive();  // no more reads of other CTAs' shared memory
                cand = cand_all;
                __syncthreads();
            }
            select_among(cand, (int)C, Ku - above, tot, wcnt, misc + 4);
            tau = misc[4];
            need = misc[5];
            const uint32_t hi_before = misc[24], c_before = misc[25];
            uint32_t g = 0, e = 0;
            for (int j = tid; j < (int)c_before; j += CT_THREADS) {
                g += cand[j] > tau;
                e += cand[j] == tau;
            }
            ct_sum2(g, e, wcnt, misc + 12);
            gt_before = hi_before + misc[12];
            eq_before = misc[13];
        }
    }

    if (!binned) {
        // ---- fallback: 8-bit radix passes over the whole slice
        int bits = 32 - __clz(gmin ^ gmax);
        uint32_t prefix = bits >= 32 ? 0u : (gmax >> bits), remaining = (uint32_t)a.K;
        for (int ps = 0; bits > 0; ++ps) {
            const int d = bits < 8 ? bits : 8;
            const int shift = bits - d;
            const int hs = shift + d;
            uint32_t *wh = whist + warp * 256;
            for (int b = lane; b < 256; b += 32) wh[b] = 0;
            __syncthreads();  // every warp's histogram cleared
            for (int i = tid; i < m; i += CT_THREADS) {
                const uint32_t k = score_key(xs[i]);
                if (hs >= 32 || (k >> hs) == prefix) atomicAdd(&wh[(k >> shift) & 255u], 1u);
            }
            __syncthreads();
            uint32_t *ch = chist + (ps & 1) * 256;
            if (tid < 256) {
                uint32_t c = 0;
#pragma unroll 8
                for (int w = 0; w < CT_WARPS; ++w) c += whist[w * 256 + tid];
                ch[tid] = c;
            }
            ct_cluster_or_block_sync<CL>();
            if (tid < 256) {
                uint32_t c = 0;
                for (int q = 0; q < CL; ++q) c += CL > 1 ? ld_dsmem_u32(ch + tid, q) : ch[tid];
                tot[tid] = c;
            }
            __syncthreads();
            if (warp == 0) pick_digit256(tot, remaining, misc);
            __syncthreads();
            prefix = (prefix << d) | misc[0];
            remaining -= misc[1];
            bits = shift;
        }
        tau = prefix;
        need = remaining;
        // this CTA's counts, then the cluster's earlier CTAs' totals
        uint32_t g = 0, e = 0;
        for (int i = tid; i < m; i += CT_THREADS) {
            const uint32_t k = score_key(xs[i]);
            g += k > tau;
            e += k == tau;
        }
        ct_sum2(g, e, wcnt, misc + 4);
        ct_cluster_or_block_sync<CL>();
        if (warp == 0) {
            uint32_t gb = 0, eb = 0;
            if (lane < (int)crank) {
                gb = ld_dsmem_u32(misc + 4, lane);
                eb = ld_dsmem_u32(misc + 5, lane);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                gb += __shfl_xor_sync(0xffffffffu, gb, o);
                eb += __shfl_xor_sync(0xffffffffu, eb, o);
            }
            if (lane == 0) {
                misc[6] = gb;
                misc[7] = eb;
            }
        }
        __syncthreads();
        gt_before = misc[6];
        eq_before = misc[7];
        if (CL > 1) cluster_arrive();
    }

    // ---- 4. compaction in position order: warp w walks its listed positions
    // (or all of [w*per, (w+1)*per) of the slice)
    const int per = (((m + CT_WARPS - 1) / CT_WARPS) + 31) & ~31;
    const int w0 = warp * per;
    const int wn = use_list ? (int)lcnt[warp] : max(0, min(m, w0 + per) - w0);
    const uint32_t *wl = wlist + warp * WCAP;
    auto pos_at = [&](int j) -> int { return use_list ? (int)wl[j] : w0 + j; };
    uint32_t g = 0, e = 0;
    for (int j0 = 0; j0 < wn; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t k = j < wn ? score_key(xs[pos_at(j)]) : 0u;
        g += __popc(__ballot_sync(0xffffffffu, j < wn && k > tau));
        e += __popc(__ballot_sync(0xffffffffu, j < wn && k == tau));
    }
    if (lane == 0) {
        wcnt[warp * 4 + 0] = g;
        wcnt[warp * 4 + 1] = e;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t gv = wcnt[lane * 4 + 0], ev = wcnt[lane * 4 + 1];
        uint32_t gi = gv, ei = ev;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t xg = __shfl_up_sync(0xffffffffu, gi, o), xe = __shfl_up_sync(0xffffffffu, ei, o);
            if (lane >= o) gi += xg, ei += xe;
        }
        wcnt[lane * 4 + 2] = gi - gv;
        wcnt[lane * 4 + 3] = ei - ev;
    }
    __syncthreads();
    uint32_t gcur = gt_before + wcnt[warp * 4 + 2], ecur = eq_before + wcnt[warp * 4 + 3];
    const uint32_t lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < wn; j0 += 32) {
        const int j = j0 + lane;
        const int i = j < wn ? pos_at(j) : 0;
        const uint32_t k = j < wn ? score_key(xs[i]) : 0u;
        const bool gt = j < wn && k > tau, eq = j < wn && k == tau;
        const uint32_t gm = __ballot_sync(0xffffffffu, gt), em = __ballot_sync(0xffffffffu, eq);
        const uint32_t mg = gcur + __popc(gm & lt), me = ecur + __popc(em & lt);
        if (gt || (eq && me < need)) {
            const uint32_t slot = mg + min(me, need);
            if (slot < (uint32_t)a.K) out[slot] = s0 + i;
            else record_error(err, DSA_DEVERR_SHAPE);
        }
        gcur += __popc(gm);
        ecur += __popc(em);
    }
    }  // full path
    if (final_wait) cluster_wait();  // no CTA leaves while another may still read its shared memory
}

// ---------------------------------------------------------------------------
// long rows: several CTAs per row
// ---------------------------------------------------------------------------
struct RowState {
    uint32_t prefix, remaining;
    uint32_t ticket[3];
    uint32_t pad[3];
};

struct MultiWs {
    uint32_t *hist;    // [R][3][HBINS]
    RowState *state;   // [R]
    uint32_t *counts;  // [R][nchunks][2]
    int nchunks;
};

__host__ __device__ inline MultiWs carve_multi(void *ws, int R, int max_row_len) {
    MultiWs m;
    uint8_t *p = static_cast<uint8_t *>(ws);
    m.hist = reinterpret_cast<uint32_t *>(p);
    p += (size_t)R * 3 * HBINS * 4;
    m.state = reinterpret_cast<RowState *>(p);
    p += (size_t)R * sizeof(RowState);
    m.counts = reinterpret_cast<uint32_t *>(p);
    m.nchunks = (max_row_len + CHUNK - 1) / CHUNK;
    return m;
}
__host__ inline size_t multi_zero_bytes(int R) { return (size_t)R * (3 * HBINS * 4 + sizeof(RowState)); }

__device__ __forceinline__ uint32_t key_at_global(const float *row, int s) { return score_key(__ldg(row + s)); }

__global__ void __launch_bounds__(MULTI_THREADS) topk_pass_kernel(const TopkArgs a, MultiWs m, int ps,
                                                                 uint32_t *err) {
    __shared__ uint32_t hist[HBINS];
    __shared__ uint32_t scan[MULTI_THREADS];
    __shared__ int2 res;
    __shared__ uint32_t is_last;
    const int r = blockIdx.y, c = blockIdx.x;
    const int n = row_length(a, r, ps == 0 ? err : nullptr);
    if (n <= a.K) return;
    const int nch = (n + CHUNK - 1) / CHUNK;
    if (c >= nch) return;
    RowState *st = m.state + r;
    const uint32_t prefix = ps == 0 ? 0u : st->prefix;
    const uint32_t remaining = ps == 0 ? (uint32_t)a.K : st->remaining;
    const int shift = kPass[ps].shift, bits = kPass[ps].bits, nb = 1 << bits, hs = shift + bits;
    for (int i = threadIdx.x; i < nb; i += MULTI_THREADS) hist[i] = 0;
    __syncthreads();
    const float *row = a.scores + (int64_t)r * a.ld;
    const int s1 = min(n, (c + 1) * CHUNK);
    for (int s = c * CHUNK + threadIdx.x; s < s1; s += MULTI_THREADS) {
        const uint32_t k = key_at_global(row, s);
        if (hs == 32 || (k >> hs) == prefix) atomicAdd(&hist[(k >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    uint32_t *gh = m.hist + ((size_t)r * 3 + ps) * HBINS;
    for (int i = threadIdx.x; i < nb; i += MULTI_THREADS)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(&st->ticket[ps], 1u) == (uint32_t)(nch - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < nb; i += MULTI_THREADS) hist[i] = __ldcg(&gh[i]);
    __syncthreads();
    pick_bin<MULTI_THREADS>(hist, nb, remaining, scan, &res);
    if (threadIdx.x == 0) {
        st->prefix = (prefix << bits) | (uint32_t)res.x;
        st->remaining = remaining - (uint32_t)res.y;
    }
}

__global__ void __launch_bounds__(MULTI_THREADS) topk_count_kernel(const TopkArgs a, MultiWs m) {
    __shared__ uint32_t wsum[32];
    const int r = blockIdx.y, c = blockIdx.x;
    const int n = row_length(a, r, nullptr);
    if (n <= a.K) return;
    const int nch = (n + CHUNK - 1) / CHUNK;
    if (c >= nch) return;
    const uint32_t tau = m.state[r].prefix;
    const float *row = a.scores + (int64_t)r * a.ld;
    const int s1 = min(n, (c + 1) * CHUNK);
    uint32_t gt = 0, eq = 0;
    for (int s = c * CHUNK + threadIdx.x; s < s1; s += MULTI_THREADS) {
        const uint32_t k = key_at_global(row, s);
        gt += k > tau;
        eq += k == tau;
    }
    uint32_t v = (gt << 16) | eq;  // <= CHUNK each: fits in 16 bits
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) wsum[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (int w = 0; w < MULTI_THREADS / 32; ++w) t += wsum[w];
        m.counts[((size_t)r * m.nchunks + c) * 2 + 0] = t >> 16;
        m.counts[((size_t)r * m.nchunks + c) * 2 + 1] = t & 0xFFFFu;
    }
}

__global__ void __launch_bounds__(MULTI_THREADS) topk_write_kernel(const TopkArgs a, MultiWs m, uint32_t *err) {
    __shared__ uint32_t wsum[32];
    __shared__ uint32_t tot[2];
    __shared__ uint32_t before[2];
    const int r = blockIdx.y, c = blockIdx.x;
    const int n = row_length(a, r, nullptr);
    int32_t *out = a.idx + (int64_t)r * a.K;
    if (n <= a.K) {
        for (int j = c * CHUNK + threadIdx.x; j < min(a.K, (c + 1) * CHUNK); j += MULTI_THREADS)
            out[j] = j < n ? j : -1;
        return;
    }
    const int nch = (n + CHUNK - 1) / CHUNK;
    if (c >= nch) return;
    const uint32_t tau = m.state[r].prefix, need = m.state[r].remaining;
    if (threadIdx.x < 32) {
        uint32_t g = 0, e = 0;
        for (int i = threadIdx.x; i < c; i += 32) {
            g += m.counts[((size_t)r * m.nchunks + i) * 2 + 0];
            e += m.counts[((size_t)r * m.nchunks + i) * 2 + 1];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (threadIdx.x == 0) {
            before[0] = g;
            before[1] = e;
        }
    }
    __syncthreads();
    const float *row = a.scores + (int64_t)r * a.ld;
    compact<MULTI_THREADS>([&](int s) { return key_at_global(row, s); }, c * CHUNK, min(n, (c + 1) * CHUNK), tau,
                           need, before[0], before[1], out, a.K, wsum, tot, err);
}

struct ClusterPlan {
    int cl;  // CTAs per row (0: use the multi-launch path)
    int smem;
};

int cluster_smem(int max_row_len, int cl) {
    const int slice = ((max_row_len + cl - 1) / cl + 3) & ~3;
    return CT_FIXED_SMEM + slice * 4;
}

template <int CL>
cudaLaunchConfig_t cluster_cfg(int R, int smem, cudaStream_t st, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(R * CL);
    cfg.blockDim = dim3(CT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// How many clusters of CL CTAs of this kernel the device runs at once (0
// when it cannot), cached per device, size and shared-memory size.
template <int CL>
int max_active_clusters(const DeviceInfo *dev, int smem) {
    static std::mutex mu;
    static std::vector<std::pair<std::pair<int, int>, int>> memo;
    std::lock_guard<std::mutex> lk(mu);
    for (auto &e : memo)
        if (e.first.first == dev->device && e.first.second == smem) return e.second;
    int num = 0;
    auto fn = topk_cluster_kernel<CL>;
    if (ensure_smem(reinterpret_cast<const void *>(fn), smem) &&
        (CL <= 8 || cudaFuncSetAttribute(reinterpret_cast<const void *>(fn),
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = cluster_cfg<CL>(1, smem, 0, attr);
        if (cudaOccupancyMaxActiveClusters(&num, fn, &cfg) != cudaSuccess) num = 0;
    }
    cudaGetLastError();
    memo.push_back({{dev->device, smem}, num});
    return num;
}

// Few rows: 16 or 10 CTAs per row when every row's cluster runs at once
// (the graphics-processing-cluster layout decides how many large clusters
// fit), else 8.  Many rows (prefill): one CTA per row.  A row whose slice
// does not fit in shared memory is split over more CTAs (up to 8); longer
// rows go to the multi-launch path.
ClusterPlan cluster_plan(int R, int max_row_len, const DeviceInfo *dev) {
    if (R * 16 <= dev->sm_count) {
        const int smem = cluster_smem(max_row_len, 16);
        if (smem <= dev->max_smem_optin && max_active_clusters<16>(dev, smem) >= R) return ClusterPlan{16, smem};
    }
    if (R * 10 <= dev->sm_count) {
        const int smem = cluster_smem(max_row_len, 10);
        if (smem <= dev->max_smem_optin && max_active_clusters<10>(dev, smem) >= R) return ClusterPlan{10, smem};
    }
    for (int cl = (R >= dev->sm_count / 2) ? 1 : 8; cl <= 8; cl *= 2) {
        const int smem = cluster_smem(max_row_len, cl);
        if (smem <= dev->max_smem_optin) return ClusterPlan{cl, smem};
    }
    return ClusterPlan{0, 0};
}

template <int CL>
dsa_status launch_cluster_t(const TopkArgs &a, int smem, cudaStream_t st, uint32_t *err) {
    auto fn = topk_cluster_kernel<CL>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), smem)) return DSA_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = cluster_cfg<CL>(a.R, smem, st, attr);
    if (a.pdl) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, fn, a, err) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_cluster(const TopkArgs &a, const ClusterPlan &cp, cudaStream_t st, uint32_t *err) {
    switch (cp.cl) {
        case 1: return launch_cluster_t<1>(a, cp.smem, st, err);
        case 2: return launch_cluster_t<2>(a, cp.smem, st, err);
        case 4: return launch_cluster_t<4>(a, cp.smem, st, err);
        case 8: return launch_cluster_t<8>(a, cp.smem, st, err);
        case 10: return launch_cluster_t<10>(a, cp.smem, st, err);
        default: return launch_cluster_t<16>(a, cp.smem, st, err);
    }
}

}  // namespace

size_t topk_workspace_bytes(int32_t R, int32_t K, int32_t max_row_len) {
    (void)K;
    const DeviceInfo *dev = current_device();
    if (dev && (topk_rows_eligible(R, K, max_row_len) || cluster_plan(R, max_row_len, dev).cl > 0)) return 0;
    const int nch = (max_row_len + CHUNK - 1) / CHUNK;
    return align_up(multi_zero_bytes(R) + (size_t)R * nch * 2 * 4, 256);
}

bool topk_prefers_cluster(int32_t R, int32_t max_row_len) {
    const DeviceInfo *dev = current_device();
    return dev && cluster_plan(R, max_row_len, dev).cl >= 10;
}

int topk_kernel_launches(int32_t R, int32_t K, int32_t max_row_len) {
    const DeviceInfo *dev = current_device();
    return (dev && (topk_rows_eligible(R, K, max_row_len) || cluster_plan(R, max_row_len, dev).cl > 0)) ? 1 : 5;
}

dsa_status launch_topk(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.R == 0) return DSA_OK;
    if (!a.hist && topk_rows_eligible(a.R, a.K, a.max_row_len) && !(reinterpret_cast<uintptr_t>(a.scores) & 15u) &&
        !(a.ld & 3))
        return launch_topk_rows(a, st);
    const ClusterPlan cp = cluster_plan(a.R, a.max_row_len, dev);
    if (cp.cl > 0) return launch_cluster(a, cp, st, dev->err);
    const size_t need = topk_workspace_bytes(a.R, a.K, a.max_row_len);
    if (a.ws == nullptr || a.ws_bytes < need) return DSA_ERR_WORKSPACE;
    MultiWs m = carve_multi(a.ws, a.R, a.max_row_len);
    if (cudaMemsetAsync(a.ws, 0, multi_zero_bytes(a.R), st) != cudaSuccess) return DSA_ERR_CUDA;
    dim3 grid(m.nchunks, a.R);
    for (int ps = 0; ps < 3; ++ps) topk_pass_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, ps, dev->err);
    topk_count_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m);
    topk_write_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, dev->err);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Top-K without caller-provided scratch.
//
// Some callers cannot allocate device memory on the path that selects
// positions: an engine whose GPU memory is reserved up front by its own pool
// (so a cudaMalloc would fail or fragment that pool), or a latency-bound
// decode loop that cannot afford cudaMalloc's implicit device-wide
// synchronisation.  For them the multi-CTA selection above runs on a scratch
// area that lives in this library's own device memory: a file-scope array
// every GPU that loads the library holds until the process exits.  Host code
// cannot use the array's name as a device address, so its address is looked
// up once per device with cudaGetSymbolAddress (with that device current) on
// the first call.
// ---------------------------------------------------------------------------
namespace {
constexpr int STATIC_MAX_ROWS = DSA_TOPK_STATIC_MAX_ROWS;
constexpr int STATIC_MAX_ROW_LEN = DSA_TOPK_STATIC_MAX_ROW_LEN;
constexpr size_t STATIC_SCRATCH_BYTES =
    (size_t)STATIC_MAX_ROWS * (3 * HBINS * 4 + sizeof(RowState)) +
    (size_t)STATIC_MAX_ROWS * ((STATIC_MAX_ROW_LEN + CHUNK - 1) / CHUNK) * 2 * 4;
static_assert(STATIC_SCRATCH_BYTES == DSA_TOPK_STATIC_SCRATCH_BYTES, "header states the scratch size");

static __device__ __align__(256) uint8_t g_topk_static_scratch[STATIC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
std::mutex g_static_mu;
void *g_static_ptr[kMaxDev];  // set once a lookup on that device has succeeded
}  // namespace

dsa_status launch_topk_static(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev || dev->device >= kMaxDev) return DSA_ERR_CUDA;
    if (a.R > STATIC_MAX_ROWS || a.max_row_len > STATIC_MAX_ROW_LEN) return DSA_ERR_UNSUPPORTED;
    if (a.R == 0) return DSA_OK;
    const int d = dev->device;
    void *scratch = nullptr;
    {
        // Only a successful lookup is kept: a call that failed (made during a
        // stream capture, say) returns DSA_ERR_CUDA and the next call tries again.
        std::lock_guard<std::mutex> lk(g_static_mu);
        if (!g_static_ptr[d]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_topk_static_scratch) != cudaSuccess || !p) {
                cudaGetLastError();
                return DSA_ERR_CUDA;
            }
            g_static_ptr[d] = p;
        }
        scratch = g_static_ptr[d];
    }
    MultiWs m = carve_multi(scratch, a.R, a.max_row_len);
    // Histograms, tickets and row state must start at zero; the array keeps
    // whatever the previous call left.
    if (cudaMemsetAsync(scratch, 0, multi_zero_bytes(a.R), st) != cudaSuccess) return DSA_ERR_CUDA;
    dim3 grid(m.nchunks, a.R);
    for (int ps = 0; ps < 3; ++ps) topk_pass_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, ps, dev->err);
    topk_count_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m);
    topk_write_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, dev->err);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
