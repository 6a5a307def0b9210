// Stage 2 of the Gated DSA layer when the indexer has already counted each
// query's scores by their top key bits: decode, and up to 64 explicit
// queries (draft tokens).  Same contract as topk.cu: per row, the K highest
// scores ("Open-Source LLM Architecture Evolution", Architecture Breakdown
// §2, "Top-K selection", K = 2048; "Fine-Grained Sparse Attention in
// Ultra-Large Parameter Models", §2.1), every position when the row is not
// longer than K, ties to the lower position, -0.0 equal to +0.0, kept
// positions in ascending order, -1 padding.
//
// One launch, no CTA ever waits for another:
//   * every CTA (row r, slice c) reads the row's coarse histogram (counts of
//     key >> 21 written by the indexer), finds the coarse bin B that holds
//     the K-th largest key, and lists -- in position order, into its own
//     region of the workspace -- every key of its slice whose coarse bin is
//     >= B, with its position.  Those are a few percent of the row (the K
//     kept ones plus the rest of bin B);
//   * the CTA that finishes the row last (an atomic ticket) loads the list
//     into shared memory and selects from it alone: histograms of key bits 20..10 over bin B's entries, then of
//     bits 9..0 over the chosen fine bin, give the exact threshold key tau
//     and how many keys equal to it are kept; a stable compaction of the
//     list, which is already in position order, writes the row's output.
// It also clears the row's coarse histogram and ticket for the next call.
// When the histogram does not describe the row (a workspace never cleared,
// or scores that do not match it), the listed keys do not hold the K largest
// and the last CTA selects from the whole row instead (three radix passes
// and a compaction over its scores): slower, same result.
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int HT_THREADS = 1024;
constexpr int HT_WARPS = HT_THREADS / 32;
constexpr int HT_STEP = HT_THREADS * 4;  // keys per step: one float4 per thread
constexpr int HT_MAX_SLICES = 256;
constexpr int HT_CAP = 12288;            // listed entries the last CTA holds in shared memory
constexpr int HT_CF_CAP = 1024;          // keys of the threshold's fine bin held apart
constexpr int HT_SMEM = HT_CAP * 8;      // dynamic shared memory per CTA
constexpr int FINE_BINS = 2048;          // key bits 20..10
constexpr int LOW_BINS = 1024;           // key bits 9..0
constexpr uint32_t PAD = 0xFFFFFFFFu;    // position of an entry to skip
static_assert(SCORE_HIST_BINS == 2048 && SCORE_HIST_SHIFT == 21, "coarse bins are key bits 31..21");
static_assert(HT_WARPS == 32, "one warp's lanes cover the block's warps");

struct HistWs {
    uint32_t *fine;    // [R][FINE_BINS] counts of bin B's keys by key bits 20..10
    uint32_t *ticket;  // [R] CTAs of the row that have finished listing
    uint4 *cnt;        // [R][S] per slice: (listed, above bin B, in bin B, 0)
    uint2 *cand;       // [R][S][slice] (position, key) of every listed key
    int S, slice;
};

__device__ __forceinline__ int ht_row_length(const TopkArgs &a, int r, uint32_t *err) {
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

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// Block-wide inclusive scan; *total gets the sum.  ws: HT_WARPS words.
__device__ __forceinline__ uint32_t ht_incl_scan(uint32_t v, uint32_t *ws, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t x = warp_incl_scan(v);
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    if (warp == 0) ws[lane] = warp_incl_scan(ws[lane]);
    __syncthreads();
    const uint32_t r = x + (warp > 0 ? ws[warp - 1] : 0u);
    *total = ws[HT_WARPS - 1];
    __syncthreads();  // ws may be reused at once
    return r;
}

// From PER bins per thread given top-down (v[0] is bin NB-1-PER*t), the bin
// b holding the remaining-th largest key: sum(hist[b+1:]) < remaining <=
// sum(hist[b:]).  Block-wide; res[0] = b, res[1] = keys in bins above b,
// res[2] = keys in b.  res is left as it was when no bin qualifies.
template <int PER>
__device__ __forceinline__ void ht_pick(const uint32_t (&v)[PER], uint32_t remaining, uint32_t *ws, uint32_t *res) {
    constexpr int NB = PER * HT_THREADS;
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) s += v[i];
    uint32_t tot;
    const uint32_t incl = ht_incl_scan(s, ws, &tot);
    uint32_t above = incl - s;
    if (above < remaining && remaining <= incl) {
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
template <int NB>
__device__ __forceinline__ void ht_pick_smem(const uint32_t *hist, uint32_t remaining, uint32_t *ws, uint32_t *res) {
    constexpr int PER = NB / HT_THREADS;
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = hist[NB - 1 - PER * threadIdx.x - i];
    ht_pick<PER>(v, remaining, ws, res);
}

// Stable compaction of a sequence of (position, key) entries given in
// position order: keeps key > tau, and key == tau while fewer than `need`
// equal keys came before.  Warp w walks its own contiguous segment, E
// consecutive entries per lane per step (ballots order the lanes); a first
// pass counts each segment's kept candidates, one exchange gives every
// segment its offsets, a second pass writes.  entry(j) returns (position,
// key); position PAD marks an entry to skip.  ws: 2 * HT_WARPS words.
template <int E, typename Entry>
__device__ __forceinline__ void ht_compact(Entry entry, int64_t count, uint32_t tau, uint32_t need, int32_t *out,
                                           int K, uint32_t *ws, uint32_t *err) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int W = 32 * E;  // entries per warp step
    const int64_t seg = (count + HT_WARPS * W - 1) / (HT_WARPS * W) * W;
    const int64_t w0 = warp * seg, w1 = w0 + seg < count ? w0 + seg : count;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t g = 0, e = 0;
    for (int64_t j0 = w0; j0 < w1; j0 += W) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const int64_t j = j0 + E * lane + i;
            const uint2 v = j < w1 ? entry(j) : make_uint2(PAD, 0u);
            g += __popc(__ballot_sync(0xffffffffu, v.x != PAD && v.y > tau));
            e += __popc(__ballot_sync(0xffffffffu, v.x != PAD && v.y == tau));
        }
    }
    if (lane == 0) ws[warp] = g, ws[HT_WARPS + warp] = e;
    __syncthreads();
    if (warp == 0) {
        const uint32_t gv = ws[lane], ev = ws[HT_WARPS + lane];
        const uint32_t gi = warp_incl_scan(gv), ei = warp_incl_scan(ev);
        ws[lane] = gi - gv, ws[HT_WARPS + lane] = ei - ev;
    }
    __syncthreads();
    uint32_t gcur = ws[warp], ecur = ws[HT_WARPS + warp];
    for (int64_t j0 = w0; j0 < w1; j0 += W) {
        uint2 v[E];
        bool gt[E], eq[E];
        uint32_t gb = 0, eb = 0, gs = 0, es = 0;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const int64_t j = j0 + E * lane + i;
            v[i] = j < w1 ? entry(j) : make_uint2(PAD, 0u);
            gt[i] = v[i].x != PAD && v[i].y > tau;
            eq[i] = v[i].x != PAD && v[i].y == tau;
            const uint32_t gm = __ballot_sync(0xffffffffu, gt[i]), em = __ballot_sync(0xffffffffu, eq[i]);
            gb += __popc(gm & lt), eb += __popc(em & lt);  // in lower lanes (they come first)
            gs += __popc(gm), es += __popc(em);
        }
        uint32_t mg = gcur + gb, me = ecur + eb;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const bool keep = gt[i] || (eq[i] && me < need);
            const uint32_t slot = mg + min(me, need);
            st_global_if(out + slot, v[i].x, keep && slot < (uint32_t)K);
            if (keep && slot >= (uint32_t)K) record_error(err, DSA_DEVERR_SHAPE);
            mg += gt[i], me += eq[i];
        }
        gcur += gs, ecur += es;
    }
    __syncthreads();  // ws may be reused
}

// The whole row, without the list: three radix passes (key bits 31..21,
// 20..10, 9..0) over its scores, then a compaction over every position.
// Used only when the listed keys cannot hold the K largest.
__device__ void ht_select_row(const float *row, int n, int K, int32_t *out, uint32_t *hist, uint32_t *ws,
                              uint32_t *ws2, uint32_t *res, uint32_t *err) {
    const int tid = threadIdx.x;
    uint32_t prefix = 0, remaining = (uint32_t)K;
    constexpr int SH[3] = {21, 10, 0}, BITS[3] = {11, 11, 10};
#pragma unroll
    for (int ps = 0; ps < 3; ++ps) {
        const int shift = SH[ps], bits = BITS[ps], hs = shift + bits;
        const uint32_t mask = (1u << bits) - 1u;
        for (int i = tid; i < FINE_BINS; i += HT_THREADS) hist[i] = 0;
        __syncthreads();
        for (int s = tid; s < n; s += HT_THREADS) {
            const uint32_t k = score_key(__ldcg(row + s));
            if (hs >= 32 || (k >> hs) == prefix) atomicAdd(&hist[(k >> shift) & mask], 1u);
        }
        __syncthreads();
        if (tid == 0) res[0] = 0, res[1] = 0;
        __syncthreads();
        if (bits == 11) ht_pick_smem<FINE_BINS>(hist, remaining, ws, res);
        else ht_pick_smem<LOW_BINS>(hist, remaining, ws, res);
        prefix = (prefix << bits) | res[0];
        remaining -= res[1];
        __syncthreads();
    }
    ht_compact<1>([&](int64_t j) { return make_uint2((uint32_t)j, score_key(__ldcg(row + j))); }, n, prefix,
                  remaining, out, K, ws2, err);
}

__global__ void __launch_bounds__(HT_THREADS, 1) topk_hist_kernel(const TopkArgs a, const HistWs w, uint32_t *err) {
    __shared__ uint32_t sh_hist[FINE_BINS];  // low histogram, or the whole-row select's histograms (last CTA)
    __shared__ uint32_t sh_off[HT_MAX_SLICES + 1];
    __shared__ uint32_t sh_cf[HT_CF_CAP];   // keys of the threshold's fine bin (last CTA)
    __shared__ uint32_t sh_ws[HT_WARPS];
    __shared__ uint32_t sh_ws2[2 * HT_WARPS];
    __shared__ uint32_t sh_wt[2 * HT_WARPS];
    __shared__ uint32_t sh_misc[16];
    extern __shared__ __align__(16) uint2 sh_ent[];  // [HT_CAP] the row's listed entries (last CTA)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.y, c = blockIdx.x;
    const int S = w.S, slice = w.slice, K = a.K;
    pdl_trigger();
    pdl_wait();  // the scores and the histogram come from the indexer
    const int n = ht_row_length(a, r, c == 0 ? err : nullptr);
    int32_t *out = a.idx + (int64_t)r * K;
    uint32_t *hrow = a.hist + (int64_t)r * SCORE_HIST_BINS;
    uint32_t *frow = w.fine + (int64_t)r * FINE_BINS;
    if (n <= K) {  // every position is kept; each CTA writes its share and clears its share of the counts
        const int per = (K + S - 1) / S;
        for (int j = c * per + tid; j < min(K, (c + 1) * per); j += HT_THREADS) out[j] = j < n ? j : -1;
        for (int i = c * SCORE_HIST_BINS / S + tid; i < (c + 1) * SCORE_HIST_BINS / S; i += HT_THREADS) hrow[i] = 0;
        return;
    }
    const int S_r = (n + slice - 1) / slice;
    if (c >= S_r) return;
    const int64_t s_begin = (int64_t)c * slice;
    const int s_end = (int)(s_begin + slice < (int64_t)n ? s_begin + slice : (int64_t)n);
    const float *row = a.scores + (int64_t)r * a.ld;

    // two steps of the slice at a time: thread t holds keys p0 .. p0+3 of
    // each (warps in position order)
    constexpr int G = 2;
    float x[G][4];
    auto load_steps = [&](int st0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int p0 = (int)s_begin + (st0 + g) * HT_STEP + 4 * tid;
            if (p0 + 3 < s_end) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(row + p0));
                x[g][0] = v.x, x[g][1] = v.y, x[g][2] = v.z, x[g][3] = v.w;
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) x[g][k] = p0 + k < s_end ? __ldcg(row + p0 + k) : -INFINITY;
            }
        }
    };
    // the first keys and the row's coarse counts, loaded together
    load_steps(0);
    const uint2 hv = __ldcg(reinterpret_cast<const uint2 *>(hrow + SCORE_HIST_BINS - 2 - 2 * tid));

    // ---- the coarse bin B of the K-th largest key (every CTA of the row alike)
    const uint32_t hb[2] = {hv.y, hv.x};  // bins 2047-2t, 2046-2t
    if (tid == 0) sh_misc[0] = SCORE_HIST_BINS, sh_misc[9] = 0, sh_misc[10] = 0;  // B = 2048 lists nothing
    const bool sane = __syncthreads_and(hb[0] <= (uint32_t)n && hb[1] <= (uint32_t)n) != 0;
    uint32_t htot;
    const uint32_t s2 = hb[0] + hb[1];
    const uint32_t hincl = ht_incl_scan(s2, sh_ws, &htot);
    if (sane && htot == (uint32_t)n) {
        const uint32_t above = hincl - s2;
        if (above < (uint32_t)K && (uint32_t)K <= hincl)
            sh_misc[0] = (uint32_t)(SCORE_HIST_BINS - 1 - 2 * tid - (above + hb[0] >= (uint32_t)K ? 0 : 1));
    }
    __syncthreads();
    const uint32_t B = sh_misc[0];

    // ---- list this slice's keys of coarse bin >= B, in position order
    // (absolute positions); count bin B's keys by their fine bin (key bits
    // 20..10) into the row's fine histogram
    uint2 *region = w.cand + ((int64_t)r * S + c) * slice;
    uint32_t listed = 0, n_above = 0, n_in = 0;
    const int nsteps = slice / HT_STEP;
    static_assert(G * HT_WARPS == 64, "two (step, warp) entries per lane");
    for (int st0 = 0; st0 < nsteps; st0 += G) {
        if (st0 > 0) load_steps(st0);
        uint32_t m[G], ex[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int p0 = (int)s_begin + (st0 + g) * HT_STEP + 4 * tid;
            m[g] = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t key = score_key(x[g][k]);
                const uint32_t cb = key >> SCORE_HIST_SHIFT;
                const bool in = st0 + g < nsteps && p0 + k < s_end && cb >= B;
                m[g] |= (in ? 1u : 0u) << k;
                n_above += in && cb > B;
                n_in += in && cb == B;
                inc_global_if(frow + ((key >> 10) & (FINE_BINS - 1)), in && cb == B);
            }
            const uint32_t cnt = __popc(m[g]);
            const uint32_t incl = warp_incl_scan(cnt);
            ex[g] = incl - cnt;
            if (lane == 31) sh_wt[g * HT_WARPS + warp] = incl;
        }
        __syncthreads();
        if (warp == 0) {  // exclusive prefix over (step, warp) in position order; the steps' total
            const uint32_t v0 = sh_wt[2 * lane], v1 = sh_wt[2 * lane + 1];
            const uint32_t t = warp_incl_scan(v0 + v1);
            sh_wt[2 * lane] = t - v0 - v1;
            sh_wt[2 * lane + 1] = t - v1;
            if (lane == 31) sh_misc[2] = t;
        }
        __syncthreads();
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int p0 = (int)s_begin + (st0 + g) * HT_STEP + 4 * tid;
            uint32_t o = listed + sh_wt[g * HT_WARPS + warp] + ex[g];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const bool b = ((m[g] >> k) & 1u) != 0;
                st_global_if(region + o, make_uint2((uint32_t)(p0 + k), score_key(x[g][k])), b);
                o += b ? 1u : 0u;
            }
        }
        listed += sh_misc[2];
        __syncthreads();  // sh_wt and sh_misc[2] are rewritten by the next steps
    }
    // an even count keeps every slice's part of the list 16-byte aligned for
    // the last CTA's copy; the pad entry (key 0) lies below every listed key
    if ((listed & 1u) && tid == 0) region[listed] = make_uint2(PAD, 0u);
    const uint32_t listed2 = (listed + 1u) & ~1u;
    // per-CTA totals: warp sums, then one shared add per warp
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        n_above += __shfl_xor_sync(0xffffffffu, n_above, o);
        n_in += __shfl_xor_sync(0xffffffffu, n_in, o);
    }
    if (lane == 0 && (n_above | n_in)) {
        atomicAdd(&sh_misc[9], n_above);
        atomicAdd(&sh_misc[10], n_in);
    }
    __syncthreads();  // every thread's entries and fine counts are issued
    if (tid == 0) {
        w.cnt[(int64_t)r * S + c] = make_uint4(listed2, sh_misc[9], sh_misc[10], 0u);
        // the CTA's entries, fine counts and counts are visible device-wide
        // before the ticket (cumulative over the barrier above)
        __threadfence();
        sh_misc[3] = atomicAdd(&w.ticket[r], 1u) == (uint32_t)(S_r - 1);
    }
    __syncthreads();
    if (!sh_misc[3]) return;

    // ================= the last CTA of the row =================
    __threadfence();
    // per-slice counts -> list offsets; the row's totals above and in B; the fine counts
    uint4 cv = make_uint4(0, 0, 0, 0);
    if (tid < S_r) cv = __ldcg(w.cnt + (int64_t)r * S + tid);
    static_assert(HT_MAX_SLICES <= HT_THREADS, "one slice per thread");
    const uint2 fv = __ldcg(reinterpret_cast<const uint2 *>(frow + FINE_BINS - 2 - 2 * tid));
    if (tid == 0) {
        w.ticket[r] = 0;
        sh_misc[9] = 0, sh_misc[10] = 0;
    }
    __syncthreads();
    // every CTA of the row has read the coarse counts and added its fine ones: clear both for the next call
    *reinterpret_cast<uint2 *>(frow + FINE_BINS - 2 - 2 * tid) = make_uint2(0, 0);
    *reinterpret_cast<uint2 *>(hrow + SCORE_HIST_BINS - 2 - 2 * tid) = make_uint2(0, 0);
    uint32_t ltot;
    const uint32_t loff = ht_incl_scan(cv.x, sh_ws, &ltot);
    if (tid < S_r) sh_off[tid] = loff - cv.x;
    if (tid == 0) sh_off[S_r] = ltot;
    uint32_t ya = cv.y, yb = cv.z;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ya += __shfl_xor_sync(0xffffffffu, ya, o);
        yb += __shfl_xor_sync(0xffffffffu, yb, o);
    }
    if (lane == 0 && (ya | yb)) {
        atomicAdd(&sh_misc[9], ya);
        atomicAdd(&sh_misc[10], yb);
    }
    __syncthreads();
    const uint32_t atot = sh_misc[9], btot = sh_misc[10];
    // the list holds the K largest keys exactly when fewer than K lie above B
    // and at least K lie at or above it; it must also fit in shared memory
    const bool listed_ok = B < (uint32_t)SCORE_HIST_BINS && atot < (uint32_t)K && (uint32_t)K <= atot + btot &&
                           ltot <= (uint32_t)HT_CAP;
    if (!listed_ok) {
        ht_select_row(row, n, K, out, sh_hist, sh_ws, sh_ws2, sh_misc + 12, err);
        return;
    }
    // copy the list into shared memory: every 16-byte piece in flight at once
    {
        const uint2 *rbase = w.cand + (int64_t)r * S * slice;
        for (int q = warp; q < S_r; q += HT_WARPS) {
            const uint32_t o = sh_off[q], np = (sh_off[q + 1] - o) >> 1;
            const uint2 *src = rbase + (int64_t)q * slice;
            for (uint32_t i = lane; i < np; i += 32) cp_async_16(sh_ent + o + 2 * i, src + 2 * i);
        }
        cp_async_commit();
    }
    // meanwhile: the fine bin F of the rem-th largest key of bin B
    const uint32_t rem = (uint32_t)K - atot;  // 1 <= rem <= btot
    if (tid == 0) sh_misc[4] = 0, sh_misc[5] = 0, sh_misc[6] = 0, sh_misc[7] = 0, sh_misc[11] = 0;
    if (tid == 0) sh_misc[12] = 0xFFFFFFFFu, sh_misc[13] = 0;
    {
        const uint32_t f[2] = {fv.y, fv.x};  // fine bins 2047-2t, 2046-2t
        uint32_t fs = f[0] <= btot && f[1] <= btot ? f[0] + f[1] : btot + 1u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) fs += __shfl_xor_sync(0xffffffffu, fs, o);
        __syncthreads();
        if (lane == 0) atomicAdd(&sh_misc[11], fs);
        ht_pick<2>(f, rem, sh_ws, sh_misc + 4);
    }
    cp_async_wait<0>();
    __syncthreads();
    const uint32_t F = sh_misc[4], rem2 = rem - sh_misc[5], CF = sh_misc[6];
    if (sh_misc[11] != btot || CF == 0) {  // fine counts that do not add up (a workspace not zeroed as documented)
        ht_select_row(row, n, K, out, sh_hist, sh_ws, sh_ws2, sh_misc + 12, err);
        return;
    }
    const uint32_t BF = (B << 11) | F;
    // the keys of fine bin F (few unless the row is degenerate) -> the exact
    // threshold key tau and how many keys equal to it are kept
    for (uint32_t j0 = warp * 64; j0 < ltot; j0 += HT_THREADS * 2) {  // a warp reads 64 consecutive entries
        const uint32_t j = j0 + 2 * lane;
        const uint4 e2 = j < ltot ? *reinterpret_cast<const uint4 *>(sh_ent + j) : make_uint4(PAD, 0u, PAD, 0u);
        const bool h0 = (e2.y >> 10) == BF, h1 = (e2.w >> 10) == BF;  // pads (key 0) never match: B >= 3
        const uint32_t m0 = __ballot_sync(0xffffffffu, h0), m1 = __ballot_sync(0xffffffffu, h1);
        if (m0 | m1) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(&sh_misc[7], (uint32_t)(__popc(m0) + __popc(m1)));
            base = __shfl_sync(0xffffffffu, base, 0);
            const uint32_t lt = (1u << lane) - 1u;
            uint32_t slot = base + __popc(m0 & lt) + __popc(m1 & lt);
            if (h0 && slot < (uint32_t)HT_CF_CAP) sh_cf[slot] = e2.y;
            slot += h0;
            if (h1 && slot < (uint32_t)HT_CF_CAP) sh_cf[slot] = e2.w;
        }
    }
    __syncthreads();
    const uint32_t ncf = sh_misc[7];
    if (ncf != CF) {  // the list and the fine counts disagree: select from the whole row
        ht_select_row(row, n, K, out, sh_hist, sh_ws, sh_ws2, sh_misc + 12, err);
        return;
    }
    if (ncf <= 32) {
        // one warp ranks the few keys: the rem2-th largest is tau
        if (warp == 0) {
            const bool v = lane < (int)ncf;
            const uint32_t k = v ? sh_cf[lane] : 0u;
            uint32_t gt = 0, eq = 0;
            for (int j = 0; j < (int)ncf; ++j) {
                const uint32_t kj = __shfl_sync(0xffffffffu, k, j);
                gt += kj > k;
                eq += kj == k;
            }
            if (v && gt < rem2 && rem2 <= gt + eq) {
                sh_misc[12] = k;
                sh_misc[13] = rem2 - gt;
            }
        }
    } else {
        // a crowded fine bin: a histogram of its keys' low bits (key bits 9..0)
        for (int i = tid; i < LOW_BINS; i += HT_THREADS) sh_hist[i] = 0;
        __syncthreads();
        if (ncf <= (uint32_t)HT_CF_CAP) {
            for (uint32_t i = tid; i < ncf; i += HT_THREADS) atomicAdd(&sh_hist[sh_cf[i] & (LOW_BINS - 1)], 1u);
        } else {
            for (uint32_t j = tid; j < ltot; j += HT_THREADS) {
                const uint32_t k = sh_ent[j].y;
                if ((k >> 10) == BF) atomicAdd(&sh_hist[k & (LOW_BINS - 1)], 1u);
            }
        }
        __syncthreads();
        ht_pick_smem<LOW_BINS>(sh_hist, rem2, sh_ws, sh_misc + 4);  // sh_misc[4..6]: low bin, above, in it
        if (tid == 0) {
            sh_misc[12] = (BF << 10) | sh_misc[4];
            sh_misc[13] = rem2 - sh_misc[5];
        }
    }
    __syncthreads();
    const uint32_t tau = sh_misc[12], need = sh_misc[13];
    ht_compact<2>([&](int64_t j) { return sh_ent[j]; }, (int64_t)ltot, tau, need, out, K, sh_ws2, err);
}

}  // namespace

HistTopkPlan topk_hist_plan(int32_t R, int32_t max_row_len) {
    HistTopkPlan pl{0, 0};
    if (R <= 0 || max_row_len <= 0) return pl;
    // about one CTA per SM of a B200 (148 SMs) over the whole launch -- fixed,
    // so the workspace size needs no device query -- slices a multiple of one
    // step, at most HT_MAX_SLICES per row
    const int64_t target = 148;
    const int64_t s_target = (target + R - 1) / R;
    int64_t slice = (max_row_len + s_target - 1) / s_target;
    slice = (slice + HT_STEP - 1) / HT_STEP * HT_STEP;
    const int64_t min_slice = ((int64_t)max_row_len + HT_MAX_SLICES - 1) / HT_MAX_SLICES;
    if (slice < min_slice) slice = (min_slice + HT_STEP - 1) / HT_STEP * HT_STEP;
    if (slice < HT_STEP) slice = HT_STEP;
    pl.slice = (int)slice;
    pl.S = (int)((max_row_len + slice - 1) / slice);
    return pl;
}

size_t topk_hist_workspace_bytes(int32_t R, int32_t max_row_len) {
    const HistTopkPlan pl = topk_hist_plan(R, max_row_len);
    if (pl.S == 0) return 0;
    return align_up((size_t)topk_hist_zero_words(R) * 4, 256) + align_up((size_t)R * pl.S * 16, 256) +
           align_up((size_t)R * pl.S * pl.slice * 8, 256);
}

int64_t topk_hist_zero_words(int32_t R) { return (int64_t)R * (FINE_BINS + 1); }

dsa_status launch_topk_hist(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.R == 0) return DSA_OK;
    const HistTopkPlan pl = topk_hist_plan(a.R, a.max_row_len);
    if (!a.hist || pl.S == 0 || pl.S > HT_MAX_SLICES || a.R > 65535) return DSA_ERR_UNSUPPORTED;
    // whole float4 loads of every row: 16-byte aligned rows
    if ((reinterpret_cast<uintptr_t>(a.scores) & 15u) || (a.ld & 3)) return DSA_ERR_INVALID_ARG;
    if (!a.ws || a.ws_bytes < topk_hist_workspace_bytes(a.R, a.max_row_len) ||
        (reinterpret_cast<uintptr_t>(a.ws) & 255u))
        return DSA_ERR_WORKSPACE;
    uint8_t *p = static_cast<uint8_t *>(a.ws);
    HistWs w;
    w.fine = reinterpret_cast<uint32_t *>(p);  // then the tickets: the words that start at zero
    w.ticket = w.fine + (size_t)a.R * FINE_BINS;
    p += align_up((size_t)topk_hist_zero_words(a.R) * 4, 256);
    w.cnt = reinterpret_cast<uint4 *>(p);
    p += align_up((size_t)a.R * pl.S * 16, 256);
    w.cand = reinterpret_cast<uint2 *>(p);
    w.S = pl.S;
    w.slice = pl.slice;
    if (!ensure_smem(reinterpret_cast<const void *>(topk_hist_kernel), HT_SMEM)) return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.S, (unsigned)a.R);
    cfg.blockDim = dim3(HT_THREADS);
    cfg.dynamicSmemBytes = HT_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, topk_hist_kernel, a, w, dev->err) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
