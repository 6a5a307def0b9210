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
// Each CTA holds its contiguous slice of the row as keys in shared memory
// (RESIDENT) or re-reads it from global memory (L2) every pass.  The row's
// key range is found first; 8-bit radix passes then run below the bits all
// keys share, with warp-private histograms summed across the cluster through
// distributed shared memory after one hardware cluster barrier per pass.  Compaction: warp ballots in position order, one
// cluster exchange of per-CTA counts for the offsets.
// ---------------------------------------------------------------------------
constexpr int CT_THREADS = 1024;
constexpr int CT_WARPS = CT_THREADS / 32;
constexpr int CT_FIXED_SMEM = (CT_WARPS * 256 + 2 * 256 + 256 + CT_WARPS * 4 + 16) * 4;

template <int CL, bool RESIDENT>
__global__ void __launch_bounds__(CT_THREADS, 1) topk_cluster_kernel(const TopkArgs a, uint32_t *err) {
    extern __shared__ __align__(16) uint32_t sm[];
    uint32_t *whist = sm;                      // [32][256] warp-private histograms
    uint32_t *chist = whist + CT_WARPS * 256;  // [2][256] this CTA's histogram (read by the cluster)
    uint32_t *tot = chist + 2 * 256;           // [256] the cluster's histogram
    uint32_t *wcnt = tot + 256;                // [32][4] per-warp (gt, eq) counts and prefixes
    uint32_t *misc = wcnt + CT_WARPS * 4;      // [16] (8..11: key range)
    uint32_t *keys = misc + 16;                // [slice] (RESIDENT)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t crank = CL > 1 ? cluster_ctarank() : 0;
    const int r = blockIdx.x / CL;
    const int n = row_length(a, r, crank == 0 ? err : nullptr);
    int32_t *out = a.idx + (int64_t)r * a.K;
    if (n <= a.K) {  // uniform across the cluster: every CTA returns here
        const int per = (a.K + CL - 1) / CL;
        for (int j = crank * per + tid; j < min(a.K, (int)(crank + 1) * per); j += CT_THREADS) out[j] = j < n ? j : -1;
        return;
    }
    const int len = (n + CL - 1) / CL;
    const int s0 = crank * len;
    const int m = max(0, min(n, s0 + len) - s0);
    const float *row = a.scores + (int64_t)r * a.ld + s0;
    auto key_at = [&](int i) -> uint32_t { return RESIDENT ? keys[i] : score_key(__ldg(row + i)); };
    // ---- the row's key range: bits above the highest bit where min and max
    // differ are shared by every key, so the digit passes start below them.
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = tid; i < m; i += CT_THREADS) {
        const uint32_t k = score_key(row[i]);
        if (RESIDENT) keys[i] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
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
    if (CL > 1) cluster_sync(); else __syncthreads();
    if (tid == 0) {
        uint32_t g0 = misc[8], g1 = misc[9];
        for (int q = 0; q < CL; ++q) {
            if (q == (int)crank) continue;
            g0 = min(g0, ld_dsmem_u32(misc + 8, q));
            g1 = max(g1, ld_dsmem_u32(misc + 9, q));
        }
        misc[10] = g0;
        misc[11] = g1;
    }
    __syncthreads();
    const uint32_t gmin = misc[10], gmax = misc[11];
    int bits = gmin == gmax ? 0 : 32 - __clz(gmin ^ gmax);
    uint32_t prefix = bits >= 32 ? 0u : (gmax >> bits), remaining = (uint32_t)a.K;
    for (int ps = 0; bits > 0; ++ps) {
        const int d = bits < 8 ? bits : 8;
        const int shift = bits - d;
        const int hs = shift + d;
        uint32_t *wh = whist + warp * 256;
        for (int b = lane; b < 256; b += 32) wh[b] = 0;
        __syncthreads();  // keys loaded; every warp's histogram cleared
        for (int i = tid; i < m; i += CT_THREADS) {
            const uint32_t k = key_at(i);
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
        if (CL > 1) cluster_sync(); else __syncthreads();
        if (tid < 256) {
            uint32_t c = 0;
            for (int q = 0; q < CL; ++q) c += CL > 1 ? ld_dsmem_u32(ch + tid, q) : ch[tid];
            tot[tid] = c;
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns bins 255-8l .. 248-8l (from the top)
            uint32_t v[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
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
                        misc[0] = 255 - 8 * lane - i;
                        misc[1] = above;
                        break;
                    }
                    above += v[i];
                }
            }
        }
        __syncthreads();
        prefix = (prefix << d) | misc[0];
        remaining -= misc[1];
        bits = shift;
    }
    const uint32_t tau = prefix, need = remaining;

    // ---- compaction: warp w owns positions [w*per, (w+1)*per) of the slice
    const int per = (((m + CT_WARPS - 1) / CT_WARPS) + 31) & ~31;
    const int w0 = warp * per, w1 = min(m, w0 + per);
    uint32_t g = 0, e = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < w1 ? key_at(i) : 0u;
        g += __popc(__ballot_sync(0xffffffffu, i < w1 && k > tau));
        e += __popc(__ballot_sync(0xffffffffu, i < w1 && k == tau));
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
        if (lane == 31) {
            misc[4] = gi;  // this CTA's totals, read by later CTAs of the cluster
            misc[5] = ei;
        }
    }
    if (CL > 1) cluster_sync(); else __syncthreads();
    if (tid == 0) {
        uint32_t gb = 0, eb = 0;
        for (int q = 0; q < (int)crank; ++q) {
            gb += ld_dsmem_u32(misc + 4, q);
            eb += ld_dsmem_u32(misc + 5, q);
        }
        misc[6] = gb;
        misc[7] = eb;
    }
    __syncthreads();
    uint32_t gcur = misc[6] + wcnt[warp * 4 + 2], ecur = misc[7] + wcnt[warp * 4 + 3];
    const uint32_t lt = (1u << lane) - 1u;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t k = i < w1 ? key_at(i) : 0u;
        const bool gt = i < w1 && k > tau, eq = i < w1 && k == tau;
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
    if (CL > 1) cluster_sync();  // no CTA leaves while another may still read its shared memory
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
    int cl;         // CTAs per row (0: use the multi-launch path)
    bool resident;  // slice kept in shared memory
    int smem;
};

// Short rows are many (prefill): one CTA per row.  Few rows: 8 CTAs per row.
// The slice must fit in shared memory; longer rows go to the multi-launch path.
ClusterPlan cluster_plan(int R, int max_row_len, const DeviceInfo *dev) {
    ClusterPlan cp{0, true, 0};
    const int cl = (R >= dev->sm_count / 2) ? 1 : 8;
    const int slice = (max_row_len + cl - 1) / cl;
    const int smem = CT_FIXED_SMEM + slice * 4;
    if (smem <= dev->max_smem_optin) cp = ClusterPlan{cl, true, smem};
    return cp;
}

template <int CL, bool RES>
dsa_status launch_cluster_t(const TopkArgs &a, int smem, cudaStream_t st, uint32_t *err) {
    auto fn = topk_cluster_kernel<CL, RES>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), smem)) return DSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.R * CL);
    cfg.blockDim = dim3(CT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, a, err) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_cluster(const TopkArgs &a, const ClusterPlan &cp, cudaStream_t st, uint32_t *err) {
    if (cp.cl == 1) return launch_cluster_t<1, true>(a, cp.smem, st, err);
    return launch_cluster_t<8, true>(a, cp.smem, st, err);
}

}  // namespace

size_t topk_workspace_bytes(int32_t R, int32_t K, int32_t max_row_len) {
    (void)K;
    const DeviceInfo *dev = current_device();
    if (dev && cluster_plan(R, max_row_len, dev).cl > 0) return 0;
    const int nch = (max_row_len + CHUNK - 1) / CHUNK;
    return align_up(multi_zero_bytes(R) + (size_t)R * nch * 2 * 4, 256);
}

int topk_kernel_launches(int32_t R, int32_t max_row_len) {
    const DeviceInfo *dev = current_device();
    return (dev && cluster_plan(R, max_row_len, dev).cl > 0) ? 1 : 5;
}

dsa_status launch_topk(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.R == 0) return DSA_OK;
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
std::once_flag g_static_once[kMaxDev];
void *g_static_ptr[kMaxDev];
cudaError_t g_static_rc[kMaxDev];
}  // namespace

dsa_status launch_topk_static(const TopkArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev || dev->device >= kMaxDev) return DSA_ERR_CUDA;
    if (a.R > STATIC_MAX_ROWS || a.max_row_len > STATIC_MAX_ROW_LEN) return DSA_ERR_UNSUPPORTED;
    if (a.R == 0) return DSA_OK;
    const int d = dev->device;
    std::call_once(g_static_once[d], [d] {
        void *p = nullptr;
        g_static_rc[d] = cudaGetSymbolAddress(&p, g_topk_static_scratch);
        g_static_ptr[d] = p;
    });
    if (g_static_rc[d] != cudaSuccess || !g_static_ptr[d]) return DSA_ERR_CUDA;
    MultiWs m = carve_multi(g_static_ptr[d], a.R, a.max_row_len);
    // Histograms, tickets and row state must start at zero; the array keeps
    // whatever the previous call left.
    if (cudaMemsetAsync(g_static_ptr[d], 0, multi_zero_bytes(a.R), st) != cudaSuccess) return DSA_ERR_CUDA;
    dim3 grid(m.nchunks, a.R);
    for (int ps = 0; ps < 3; ++ps) topk_pass_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, ps, dev->err);
    topk_count_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m);
    topk_write_kernel<<<grid, MULTI_THREADS, 0, st>>>(a, m, dev->err);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
