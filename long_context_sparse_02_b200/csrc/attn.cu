// Stage 3 of the Gated DSA layer: attention over only the selected latent
// rows, multiplied by a per-head sigmoid gate.
//
// ("Open-Source LLM Architecture Evolution", Technical Deep Dive §2: scores
// and softmax over only the 2048 selected elements; Architecture Breakdown
// §2, "Gated fusion", read as out = sigmoid(g) * attention output.)  All
// heads share the selected latent row: the key is its first Dqk entries and
// the value its first Dv.
//
// One CTA = (query token, a 256-wide slice of the value dims, a split of the
// selected rows).  The selected rows are gathered 64 at a time through the
// block table with 16-byte async copies straight into the 128-byte-swizzled
// layout the tensor core reads; Q arrives by TMA.  tcgen05 bf16 MMAs compute
// S = Q C^T (M = 128 heads, N = 64 rows, fp32 in TMEM, double-buffered) and
// O += P V (V read as an MN-major operand from the same gathered tile); the
// softmax warps keep the running max in the exp2 domain and rescale O in
// TMEM only when the max grows by more than 2^8.  With one split the gate is
// applied in the epilogue; otherwise normalised partials and (max, sum) go
// to the workspace and attn_combine_kernel merges them and applies the gate.
//
// Warps 0-3: softmax/epilogue (one TMEM lane quarter each, a thread per
// head); warp 4: MMA issuer and TMEM owner; warps 5-8: gather producers.
#include <utility>

#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int ATT_THREADS = 288;

template <int DQK, int DVP>
struct AttnCfg {
    static constexpr int KQ = DQK / 64;   // 128-byte k-blocks of a latent row used by S
    static constexpr int NVB = DVP / 64;  // 64-dim value blocks per CTA
    static constexpr int NC = 64;         // selected rows per chunk
    static constexpr int NST = 8;         // gather ring stages
    static constexpr int LAG = 4;         // copies a producer keeps in flight before signalling
    static constexpr int STAGE_BYTES = NC * 128;
    static constexpr int Q_BYTES = KQ * 128 * 128;
    static constexpr int P_BYTES = 128 * 128;
    static constexpr int S_COL = 0;
    static constexpr int O_COL = 128;
    static constexpr int TMEM_COLS = (O_COL + DVP) <= 256 ? 256 : 512;
    static constexpr int NBAR = 2 * NST + 8;
    static constexpr int SMEM = 1024 + Q_BYTES + NST * STAGE_BYTES + P_BYTES + 8 * NBAR + 64;
    static_assert(DQK % 64 == 0 && DVP % 64 == 0 && DVP <= DQK, "shape");
};

struct AttnParams {
    const uint16_t *kv;
    PagedDev pg;
    const int32_t *q_seq;
    const int32_t *idx;
    int32_t K;
    const uint16_t *gate;
    float scale_log2;
    int32_t T, H, Dv, nparts, splits, rows_per_split;
    uint16_t *out;
    float *lse;
    float *part_o;   // [T, splits, H, Dv] normalised partial outputs
    float *part_ml;  // [T, splits, H, 2]   (running max in log2 units, sum)
    uint32_t *err;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Latent-cache row of selected entry g of token t, or -1 when the entry is
// padding, past the split, or invalid (recorded when `report`).
__device__ __forceinline__ int64_t latent_row(const AttnParams &p, int b, int L, int t, int g, int row_end,
                                              bool report) {
    if (g >= row_end) return -1;
    const int pos = p.idx[(int64_t)t * p.K + g];
    if (pos < 0) return -1;
    if (pos >= L) {
        if (report) record_error(p.err, DSA_DEVERR_POSITION);
        return -1;
    }
    const int lp = pos >> 6;
    if (lp >= p.pg.max_blocks) {
        if (report) record_error(p.err, DSA_DEVERR_PAGE);
        return -1;
    }
    const int pg = p.pg.block_table[(int64_t)b * p.pg.max_blocks + lp];
    if (pg < 0 || pg >= p.pg.num_pages) {
        if (report) record_error(p.err, DSA_DEVERR_PAGE);
        return -1;
    }
    return (int64_t)pg * 64 + (pos & 63);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int DQK, int DVP>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap qmap, const AttnParams p) {
    using C = AttnCfg<DQK, DVP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *Qs = smem;
    uint8_t *ring = Qs + C::Q_BYTES;
    uint8_t *Ps = ring + C::NST * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(Ps + C::P_BYTES);
    uint64_t *empty = full + C::NST;
    uint64_t *q_full = empty + C::NST;
    uint64_t *s_full = q_full + 1;   // [2]
    uint64_t *s_empty = s_full + 2;  // [2]
    uint64_t *p_full = s_empty + 2;
    uint64_t *o_done = p_full + 1;
    uint64_t *drain = o_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *last_sh = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *abort_flag = last_sh + 1;

    const int warp = warp_id(), lane = lane_id();
    const int t = blockIdx.y;
    const int part = blockIdx.x % p.nparts;
    const int split = blockIdx.x / p.nparts;
    const int row0 = split * p.rows_per_split;
    const int row_end = min(p.K, row0 + p.rows_per_split);

    int b = p.q_seq ? p.q_seq[t] : t;
    bool tok_ok = b >= 0 && b < p.pg.num_seqs;
    const int L = tok_ok ? p.pg.seq_lens[b] : 0;
    if (!tok_ok) b = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&full[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *last_sh = -1;
        *abort_flag = 0;
        if (!tok_ok) record_error(p.err, DSA_DEVERR_POSITION);
        fence_mbar_init();
        tma_prefetch_desc(&qmap);
    }
    if (warp == 4) tmem_alloc(tmem_slot, C::TMEM_COLS);
    __syncthreads();
    pdl_trigger();
    pdl_wait();  // the selection comes from the previous kernel
    if (tok_ok)
        for (int g = row0 + threadIdx.x; g < row_end; g += ATT_THREADS)
            if (p.idx[(int64_t)t * p.K + g] >= 0) atomicMax(last_sh, g);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nc = *last_sh < 0 ? 0 : (*last_sh - row0) / C::NC + 1;

    if (warp >= 5) {
        // ---------------- gather producers ----------------
        const int pi = threadIdx.x - 160;
        const int r = pi >> 1, half = pi & 1;
        if (pi == 0 && nc > 0) {
            mbar_expect_tx(q_full, C::Q_BYTES);
            for (int kb = 0; kb < C::KQ; ++kb) tma_load_2d(Qs + kb * 128 * 128, &qmap, q_full, kb * 64, t * p.H);
        }
        int ld = 0;
        bool ok = true;
        int64_t src_cur = -1, src_prev = -1;
        auto load_block = [&](int bi, int64_t src) -> bool {
            const int s = ld % C::NST;
            if (!mbar_wait(&empty[s], ((ld / C::NST) & 1) ^ 1, p.err, abort_flag)) return false;
            uint8_t *dst = ring + s * C::STAGE_BYTES + r * 128;
            const uint16_t *g = p.kv + src * DQK + bi * 64;
#pragma unroll
            for (int cc = half * 4; cc < half * 4 + 4; ++cc) {
                uint8_t *d = dst + ((cc ^ (r & 7)) << 4);
                if (src >= 0) cp_async_16(d, g + cc * 8);
                else *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
            }
            cp_async_commit();
            if (ld >= C::LAG) {
                cp_async_wait<C::LAG>();
                fence_proxy_async_smem();
                mbar_arrive(&full[(ld - C::LAG) % C::NST]);
            }
            ++ld;
            return true;
        };
        for (int c = 0; ok && c <= nc; ++c) {
            if (c < nc) {
                src_cur = latent_row(p, b, L, t, row0 + c * C::NC + r, row_end, half == 0);
                for (int kb = 0; ok && kb < C::KQ; ++kb) ok = load_block(kb, src_cur);
            }
            if (c >= 1)
                for (int db = 0; ok && db < C::NVB; ++db) ok = load_block(part * C::NVB + db, src_prev);
            src_prev = src_cur;
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        if (ok)
            for (int i = ld - C::LAG < 0 ? 0 : ld - C::LAG; i < ld; ++i) mbar_arrive(&full[i % C::NST]);
        if (pi == 0 && nc > 0) mbar_wait(q_full, 0, p.err, nullptr);
    } else if (warp == 4) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && nc > 0) {
            constexpr uint32_t ID_S = idesc(1, 1, 0, 0, C::NC, 128);
            constexpr uint32_t ID_PV = idesc(1, 1, 0, 1, 64, 128);
            bool ok = mbar_wait(q_full, 0, p.err, abort_flag);
            tc_fence_after();
            const uint32_t qa0 = smem_u32(Qs), ring0 = smem_u32(ring), pa = smem_u32(Ps);
            int ld = 0;
            for (int c = 0; ok && c <= nc; ++c) {
                if (c < nc) {
                    const int sb = c & 1;
                    if (!mbar_wait(&s_empty[sb], ((c >> 1) & 1) ^ 1, p.err, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t dS = tmem + C::S_COL + sb * C::NC;
                    for (int kb = 0; ok && kb < C::KQ; ++kb) {
                        const int s = ld % C::NST;
                        if (!mbar_wait(&full[s], (ld / C::NST) & 1, p.err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t qa = qa0 + kb * 128 * 128, ca = ring0 + s * C::STAGE_BYTES;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(dS, sdesc(qa + 32 * k, 16, 1024, SWZ_128B), sdesc(ca + 32 * k, 16, 1024, SWZ_128B),
                                     ID_S, (kb | k) != 0);
                        mma_commit(&empty[s]);
                        ++ld;
                    }
                    if (!ok) break;
                    mma_commit(&s_full[sb]);
                }
                if (c >= 1) {
                    const int j = c - 1;
                    if (!mbar_wait(p_full, j & 1, p.err, abort_flag)) break;
                    tc_fence_after();
                    for (int db = 0; ok && db < C::NVB; ++db) {
                        const int s = ld % C::NST;
                        if (!mbar_wait(&full[s], (ld / C::NST) & 1, p.err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ca = ring0 + s * C::STAGE_BYTES;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_bf16(tmem + C::O_COL + db * 64, sdesc(pa + 32 * k, 16, 1024, SWZ_128B),
                                     sdesc(ca + 2048 * k, C::STAGE_BYTES, 1024, SWZ_128B), ID_PV, (j > 0 || k > 0));
                        mma_commit(&empty[s]);
                        ++ld;
                    }
                    if (!ok) break;
                    mma_commit(o_done);
                }
            }
            mma_commit(drain);
            mbar_wait(drain, 0, p.err, nullptr);
        }
    } else {
        // ---------------- softmax + epilogue (warps 0..3, thread = head) ----------------
        const int row = threadIdx.x;  // 0..127
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int c = 0; c < nc; ++c) {
            const int sb = c & 1;
            if (!mbar_wait(&s_full[sb], (c >> 1) & 1, p.err, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[C::NC];
            tmem_ld32(tmem + C::S_COL + sb * C::NC + lane_off, sr);
            tmem_ld32(tmem + C::S_COL + sb * C::NC + 32 + lane_off, sr + 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[sb]);
            const int gbase = row0 + c * C::NC;
            const uint32_t vlo = __ballot_sync(0xffffffffu, latent_row(p, b, L, t, gbase + lane, row_end, false) >= 0);
            const uint32_t vhi =
                __ballot_sync(0xffffffffu, latent_row(p, b, L, t, gbase + 32 + lane, row_end, false) >= 0);
            float x[C::NC];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < C::NC; ++i) {
                const bool v = ((i < 32 ? vlo >> i : vhi >> (i - 32)) & 1u) != 0;
                x[i] = v ? __uint_as_float(sr[i]) * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, x[i]);
            }
            const float m_new = fmaxf(m, mx);
            const bool resc = m_new > m + 8.f;
            float alpha = 1.f;
            if (resc) {
                alpha = ex2_approx(m - m_new);
                l *= alpha;
                m = m_new;
            }
            uint32_t pk[C::NC / 2];
            float lsum = 0.f;
#pragma unroll
            for (int i = 0; i < C::NC; i += 2) {
                const float p0 = x[i] == -INFINITY ? 0.f : ex2_approx(x[i] - m);
                const float p1 = x[i + 1] == -INFINITY ? 0.f : ex2_approx(x[i + 1] - m);
                pk[i / 2] = pack_bf16(p0, p1);
                const __nv_bfloat162 bv = *reinterpret_cast<__nv_bfloat162 *>(&pk[i / 2]);
                lsum += __bfloat162float(bv.x) + __bfloat162float(bv.y);
            }
            l += lsum;
            if (c >= 1) {
                if (!mbar_wait(o_done, (c - 1) & 1, p.err, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (resc) {
#pragma unroll 1
                    for (int cc = 0; cc < DVP / 32; ++cc) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + C::O_COL + cc * 32 + lane_off;
                        tmem_ld32(ta, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(ta, o);
                    }
                    tmem_wait_st();
                }
            }
            uint8_t *prow = Ps + row * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                *reinterpret_cast<uint4 *>(prow + ((cc ^ (row & 7)) << 4)) =
                    make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && nc > 0) ok = mbar_wait(o_done, (nc - 1) & 1, p.err, abort_flag);
        tc_fence_after();
        const bool have_o = ok && nc > 0;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool live = row < p.H;
        if (p.splits == 1) {
            const float g = live ? __bfloat162float(__ushort_as_bfloat16(p.gate[(int64_t)t * p.H + row])) : 0.f;
            const float sig = 1.f / (1.f + __expf(-g));
            const float scale = inv * sig;
            uint16_t *orow = p.out + ((int64_t)t * p.H + row) * p.Dv + part * DVP;
#pragma unroll 1
            for (int cc = 0; cc < DVP / 32; ++cc) {
                uint32_t o[32];
                if (have_o) {
                    tmem_ld32(tmem + C::O_COL + cc * 32 + lane_off, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (live) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(o[i]) * scale, __uint_as_float(o[i + 1]) * scale);
                        v.y = pack_bf16(__uint_as_float(o[i + 2]) * scale, __uint_as_float(o[i + 3]) * scale);
                        v.z = pack_bf16(__uint_as_float(o[i + 4]) * scale, __uint_as_float(o[i + 5]) * scale);
                        v.w = pack_bf16(__uint_as_float(o[i + 6]) * scale, __uint_as_float(o[i + 7]) * scale);
                        *reinterpret_cast<uint4 *>(orow + cc * 32 + i) = v;
                    }
                }
            }
            if (live && part == 0 && p.lse)
                p.lse[(int64_t)t * p.H + row] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else {
            const int64_t prow = ((int64_t)t * p.splits + split) * p.H + row;
            float *po = p.part_o + prow * p.Dv + part * DVP;
#pragma unroll 1
            for (int cc = 0; cc < DVP / 32; ++cc) {
                uint32_t o[32];
                if (have_o) {
                    tmem_ld32(tmem + C::O_COL + cc * 32 + lane_off, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (live) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4 *>(po + cc * 32 + i) =
                            make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                        __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                }
            }
            if (live && part == 0) {
                p.part_ml[prow * 2 + 0] = m;
                p.part_ml[prow * 2 + 1] = have_o ? l : 0.f;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ============================================================================
// Decode: one CTA = (query token, 128 selected rows).  The 128 gathered
// latent rows stay resident in shared memory (all copies in flight at once);
// Q streams from L2 through a small TMA ring.  S = Q C^T fills 128 TMEM
// columns; the softmax over the 128 rows is exact (no running max); after S
// has been read, O = P V overwrites TMEM columns [0, Dv) with V read MN-major
// from the same resident rows.  Output: bf16 partial o/l plus (max, sum) per
// (token, split, head), merged by attn_decode_combine_kernel.
// ============================================================================
constexpr int DEC_NR = 128;      // rows per CTA
constexpr int DEC_WORKERS = 16;  // warps 0..15: gather, then softmax and epilogue
constexpr int DEC_MMA_WARP = 16;
constexpr int DEC_Q_WARP = 17;
constexpr int DEC_THREADS = 18 * 32;
constexpr int DEC_WORKER_THREADS = DEC_WORKERS * 32;

template <int DQK, int DV>
struct DecAttnCfg {
    static constexpr int NKB = DQK / 64;           // 128-byte k-blocks per row
    static constexpr int NVB = DV / 64;
    static constexpr int KB_BYTES = DEC_NR * 128;  // one k-block of 128 rows
    static constexpr int C_BYTES = NKB * KB_BYTES;
    static constexpr int QS = NKB >= 4 ? 4 : NKB;  // Q ring stages
    static constexpr int Q_STAGE = 128 * 128;      // [128 heads x 64 dims] bf16
    static constexpr int Q_BYTES = QS * Q_STAGE;
    static constexpr int P_BYTES = 2 * 128 * 128;  // [128 heads x 128 rows] bf16, two atoms
    static constexpr int RING = Q_BYTES > P_BYTES ? Q_BYTES : P_BYTES;
    static constexpr int TMEM_COLS = DV <= 128 ? 128 : DV <= 256 ? 256 : 512;
    static constexpr int NBAR = NKB + 2 * QS + 5;
    // the output is staged in the rows region once PV has consumed it: one
    // [128 heads x 64 dims] 128-byte-swizzled box per 64 value dims
    static_assert(NVB * KB_BYTES <= C_BYTES, "output staging fits in the rows region");
    static constexpr int DPW = DV / 4;            // value dims per worker warp in the epilogue
    static constexpr bool DV_HALF_SPLIT = DV == 512;  // the epilogue halves: warps 0-7 dims < 256, 8-15 the rest
    static constexpr int SMEM = 1024 + C_BYTES + RING + 8 * NBAR + 8 * DEC_NR + 2 * 4 * 128 * 4 + 64;
    static_assert(DV >= 64 && DV % 64 == 0 && DV <= 512, "value width");
};

struct DecAttnParams {
    const uint16_t *kv;
    PagedDev pg;
    const int32_t *q_seq;
    const int32_t *idx;
    int32_t K;
    float scale_log2;
    int32_t T, H, Dv, splits;
    uint16_t *part_o;  // [T, splits, H, Dv] bf16, normalised by the split's sum
    float *part_ml;    // [T, splits, H, 2]  (max in log2 units, sum)
    uint32_t *err;
};

// Warps 0..15 first gather the 128 rows (every copy in flight at once), then
// share the softmax (warp w: heads 32(w%4).., rows 32(w/4)..) and the
// epilogue (heads 32(w%4).., value dims DV/4 * (w/4)..).  Warp 16 issues the
// MMAs and owns TMEM; warp 17 streams Q.
template <int DQK, int DV>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap omap,
                       const DecAttnParams p) {
    using C = DecAttnCfg<DQK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *Cs = smem;              // [NKB][128 rows][128 B]
    uint8_t *ring = Cs + C::C_BYTES;  // Q stages, later P
    uint64_t *c_full = reinterpret_cast<uint64_t *>(ring + C::RING);  // [NKB]
    uint64_t *q_full = c_full + C::NKB;                                 // [QS]
    uint64_t *q_empty = q_full + C::QS;                                 // [QS]
    uint64_t *s_full = q_empty + C::QS;
    uint64_t *p_full = s_full + 1;
    uint64_t *o_full = p_full + 1;  // [2]: O columns [0, 256) and [256, DV)
    uint64_t *drain = o_full + 2;
    int64_t *rowid = reinterpret_cast<int64_t *>(drain + 1);  // [128] cache row of each selected entry, -1 = none
    float *red_m = reinterpret_cast<float *>(rowid + DEC_NR);  // [4][128] partial row maxima
    float *red_l = red_m + 4 * 128;                            // [4][128] partial sums
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(red_l + 4 * 128);
    int *any_valid = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *abort_flag = any_valid + 1;

    const int warp = warp_id(), lane = lane_id();
    const int t = blockIdx.y, split = blockIdx.x;
    const int row0 = split * DEC_NR;
    const int row_end = min(p.K, row0 + DEC_NR);
    int b = p.q_seq ? p.q_seq[t] : t;
    const bool tok_ok = b >= 0 && b < p.pg.num_seqs;
    const int L = tok_ok ? p.pg.seq_lens[b] : 0;
    if (!tok_ok) b = 0;
    AttnParams ap{};  // for latent_row()
    ap.pg = p.pg;
    ap.idx = p.idx;
    ap.K = p.K;
    ap.err = p.err;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NKB; ++i) mbar_init(&c_full[i], DEC_WORKER_THREADS);
        for (int i = 0; i < C::QS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, 1);
        mbar_init(&o_full[0], 1);
        mbar_init(&o_full[1], 1);
        mbar_init(drain, 1);
        *any_valid = 0;
        *abort_flag = 0;
        if (!tok_ok) record_error(p.err, DSA_DEVERR_POSITION);
        fence_mbar_init();
        tma_prefetch_desc(&qmap);
        tma_prefetch_desc(&omap);
    }
    if (warp == DEC_MMA_WARP) tmem_alloc(tmem_slot, C::TMEM_COLS);
    __syncthreads();
    // Q does not depend on the selection: start it while the rows are resolved.
    if (warp == DEC_Q_WARP && lane == 0)
        for (int kb = 0; kb < C::QS; ++kb) {
            mbar_expect_tx(&q_full[kb], C::Q_STAGE);
            tma_load_2d(ring + kb * C::Q_STAGE, &qmap, &q_full[kb], kb * 64, t * p.H);
        }
    pdl_trigger();
    pdl_wait();  // the selection comes from the previous kernel
    if (threadIdx.x < DEC_NR) {  // resolve every selected row once, through the block table
        const int64_t rid = tok_ok ? latent_row(ap, b, L, t, row0 + threadIdx.x, row_end, true) : -1;
        rowid[threadIdx.x] = rid;
        if (rid >= 0) *any_valid = 1;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool work = *any_valid != 0;

    if (warp < DEC_WORKERS) {
        const int wt = threadIdx.x;  // 0..511
        // ---------------- gather: all 128 rows, every k-block, in flight at once ----------------
        // Eight consecutive lanes copy one row's 128-byte k-block segment (a
        // full line per 8 lanes); a thread serves rows rg and rg + 64.
        {
            const int c8 = wt & 7, rg = wt >> 3;
            if (work) {
                const int64_t src0 = rowid[rg], src1 = rowid[rg + 64];
#pragma unroll 1
                for (int kb = 0; kb < C::NKB; ++kb) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int r = rg + 64 * q;
                        const int64_t src = q ? src1 : src0;
                        uint8_t *d = Cs + kb * C::KB_BYTES + r * 128 + ((c8 ^ (r & 7)) << 4);
                        if (src >= 0) cp_async_16(d, p.kv + src * DQK + kb * 64 + c8 * 8);
                        else *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
                    }
                    cp_async_commit();
                }
                // signal each k-block as its copies land (groups complete in order)
#define DSA_DEC_SIGNAL(KB)                                                    \
    if (KB < C::NKB) {                                                         \
        cp_async_wait<(C::NKB - 1 - (KB)) < 0 ? 0 : (C::NKB - 1 - (KB))>();    \
        fence_proxy_async_smem();                                              \
        mbar_arrive(&c_full[KB]);                                              \
    }
                DSA_DEC_SIGNAL(0) DSA_DEC_SIGNAL(1) DSA_DEC_SIGNAL(2) DSA_DEC_SIGNAL(3) DSA_DEC_SIGNAL(4)
                DSA_DEC_SIGNAL(5) DSA_DEC_SIGNAL(6) DSA_DEC_SIGNAL(7) DSA_DEC_SIGNAL(8)
#undef DSA_DEC_SIGNAL
            }
        }
        // ---------------- softmax: warp w = (head quarter w%4, row block w/4) ----------------
        const int qr = warp & 3, cb = warp >> 2;
        const int head = 32 * qr + lane;
        // value dims of this warp's epilogue: [DV/4 * cb, DV/4 * (cb + 1)), in O half ohalf;
        // warps 0-7 / 8-15 (threads 0-255 / 256-511) are the two halves when DV > 256
        const int ohalf = C::DPW * cb >= 256 ? 1 : 0;
        static_assert(C::DV_HALF_SPLIT || DV <= 256, "halves");
        const uint32_t lane_off = static_cast<uint32_t>(32 * qr) << 16;
        float m = -INFINITY;
        bool have_o = false;
        // Every worker passes the same named barriers whatever happens; a
        // timed-out wait in any warp turns the whole softmax off for all.
        const bool s_ok = work && mbar_wait(s_full, 0, p.err, abort_flag);
        const bool go = !named_bar_or(1, DEC_WORKER_THREADS, !s_ok) && work;
        uint32_t sr[32];
        uint32_t vm = 0;
        if (go) {
            tc_fence_after();
            vm = __ballot_sync(0xffffffffu, rowid[32 * cb + lane] >= 0);
            tmem_ld32(tmem + 32 * cb + lane_off, sr);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if ((vm >> i) & 1u) mx = fmaxf(mx, __uint_as_float(sr[i]) * p.scale_log2);
            red_m[cb * 128 + head] = mx;
        }
        named_bar_sync(1, DEC_WORKER_THREADS);
        if (go) {
            m = fmaxf(fmaxf(red_m[head], red_m[128 + head]), fmaxf(red_m[256 + head], red_m[384 + head]));
            uint32_t pk[16];
            float ls = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float p0 = ((vm >> i) & 1u) ? ex2_approx(__uint_as_float(sr[i]) * p.scale_log2 - m) : 0.f;
                const float p1 = ((vm >> (i + 1)) & 1u) ? ex2_approx(__uint_as_float(sr[i + 1]) * p.scale_log2 - m) : 0.f;
                pk[i / 2] = pack_bf16(p0, p1);
                const __nv_bfloat162 bv = *reinterpret_cast<__nv_bfloat162 *>(&pk[i / 2]);
                ls += __bfloat162float(bv.x) + __bfloat162float(bv.y);
            }
            red_l[cb * 128 + head] = ls;
            // P columns 32cb..32cb+31 -> atom cb/2, 16-byte chunks 4*(cb%2) .. 4*(cb%2)+3
            uint8_t *atom = ring + (cb >> 1) * 16384 + head * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int cc = 4 * (cb & 1) + q;
                *reinterpret_cast<uint4 *>(atom + ((cc ^ (head & 7)) << 4)) =
                    make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, DEC_WORKER_THREADS);  // P and every partial sum are written
            if (threadIdx.x == 0) mbar_arrive(p_full);
            have_o = mbar_wait(&o_full[ohalf], 0, p.err, abort_flag);
            tc_fence_after();
        }
        // ---------------- epilogue: warp w = (head quarter w%4, value dims DV/4 * (w/4)..) ----------------
        // every partial sum written; S, P and the rows are consumed; O is read by all or by none.
        // O/l goes to the rows region as bf16 in the 128-byte-swizzled layout of
        // the output map's [64 dims x 128 heads] boxes, then one tensor store per box.
        // (per O half: the half's 256 worker threads agree; the halves do not wait for each other)
        const uint32_t hbar = C::DV_HALF_SPLIT ? 2 + ohalf : 1;
        const uint32_t hthreads = C::DV_HALF_SPLIT ? DEC_WORKER_THREADS / 2 : DEC_WORKER_THREADS;
        have_o = !named_bar_or(hbar, hthreads, go && !have_o) && go;
        const float l = have_o ? red_l[head] + red_l[128 + head] + red_l[256 + head] + red_l[384 + head] : 0.f;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int d0 = cb * C::DPW;
        constexpr int STEP = C::DPW % 32 == 0 ? 32 : 16;  // TMEM columns read per wait
#pragma unroll 1
        for (int c0 = 0; c0 < C::DPW; c0 += STEP) {
            uint32_t o[STEP];
            if (have_o) {
#pragma unroll
                for (int h = 0; h < STEP; h += 16) tmem_ld16(tmem + d0 + c0 + h + lane_off, o + h);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < STEP; ++i) o[i] = 0u;
            }
#pragma unroll
            for (int i = 0; i < STEP; i += 8) {
                const int d = d0 + c0 + i;
                uint4 v;
                v.x = pack_bf16(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv);
                v.y = pack_bf16(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                v.z = pack_bf16(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                v.w = pack_bf16(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                *reinterpret_cast<uint4 *>(Cs + (d >> 6) * C::KB_BYTES + head * 128 +
                                           ((((d & 63) >> 3) ^ (head & 7)) << 4)) = v;
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(hbar, hthreads);  // every box of this half is staged
        const bool issuer = threadIdx.x == (C::DV_HALF_SPLIT ? ohalf * (DEC_WORKER_THREADS / 2) : 0);
        if (issuer) {  // heads >= H lie outside the map and are not written
            const int b0 = C::DV_HALF_SPLIT ? ohalf * (C::NVB / 2) : 0;
            const int b1 = C::DV_HALF_SPLIT ? b0 + C::NVB / 2 : C::NVB;
            for (int bx = b0; bx < b1; ++bx) tma_store_3d(&omap, Cs + bx * C::KB_BYTES, bx * 64, 0, t * p.splits + split);
            bulk_commit();
        }
        if (cb == 0 && head < p.H) {
            const int64_t prow = ((int64_t)t * p.splits + split) * p.H + head;
            p.part_ml[prow * 2 + 0] = m;
            p.part_ml[prow * 2 + 1] = l;
        }
        if (issuer) bulk_wait_read_all();  // the staged boxes stay until the stores have read them
    } else if (warp == DEC_Q_WARP) {
        // ---------------- rest of the Q stream (TMA, from L2) ----------------
        if (lane == 0) {
            int issued = C::QS;
            if (work)
                for (int kb = C::QS; kb < C::NKB; ++kb) {
                    const int s = kb % C::QS;
                    if (!mbar_wait(&q_empty[s], ((kb / C::QS) & 1) ^ 1, p.err, abort_flag)) break;
                    mbar_expect_tx(&q_full[s], C::Q_STAGE);
                    tma_load_2d(ring + s * C::Q_STAGE, &qmap, &q_full[s], kb * 64, t * p.H);
                    ++issued;
                }
            if (!work)  // never leave a copy in flight behind
                for (int kb = 0; kb < C::QS; ++kb) mbar_wait(&q_full[kb], 0, p.err, nullptr);
        }
    } else {
        // ---------------- MMA issuer (warp 16) ----------------
        if (lane == 0 && work) {
            constexpr uint32_t ID_S = idesc(1, 1, 0, 0, DEC_NR, 128);
            bool ok = true;
            const uint32_t c0 = smem_u32(Cs), r0 = smem_u32(ring);
            for (int kb = 0; ok && kb < C::NKB; ++kb) {
                const int s = kb % C::QS;
                if (!mbar_wait(&c_full[kb], 0, p.err, abort_flag) ||
                    !mbar_wait(&q_full[s], (kb / C::QS) & 1, p.err, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tmem, sdesc(r0 + s * C::Q_STAGE + 32 * k, 16, 1024, SWZ_128B),
                             sdesc(c0 + kb * C::KB_BYTES + 32 * k, 16, 1024, SWZ_128B), ID_S, (kb | k) != 0);
                mma_commit(&q_empty[s]);
            }
            if (ok) mma_commit(s_full);
            if (ok && mbar_wait(p_full, 0, p.err, abort_flag)) {
                tc_fence_after();
                for (int nb = 0; nb < C::NVB; nb += 4) {
                    const int nblk = (C::NVB - nb) < 4 ? (C::NVB - nb) : 4;
                    const uint32_t id_pv = idesc(1, 1, 0, 1, 64 * nblk, 128);
#pragma unroll
                    for (int k = 0; k < DEC_NR / 16; ++k)
                        mma_bf16(tmem + nb * 64, sdesc(r0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024, SWZ_128B),
                                 sdesc(c0 + nb * C::KB_BYTES + k * 2048, C::KB_BYTES, 1024, SWZ_128B), id_pv, k != 0);
                    mma_commit(&o_full[nb / 4]);  // this half of O is complete
                }
                if (C::NVB <= 4) mma_commit(&o_full[1]);
            }
            mma_commit(drain);
            mbar_wait(drain, 0, p.err, nullptr);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == DEC_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// One thread per (token, head, 16-byte chunk of the value row):
// out = sigmoid(g) * sum_s w_s o_s with w_s = l_s 2^(m_s - M) / sum l 2^(m - M).
// Every load of a thread (split maxima and sums, gate, partial chunks) is
// independent of the others and issued before any is used.
constexpr int CMB_THREADS = 256;
constexpr int CMB_BATCH = 8;  // splits in flight per thread
__global__ void __launch_bounds__(CMB_THREADS) attn_decode_combine_kernel(const DecAttnParams p, const uint16_t *gate,
                                                                          uint16_t *out, float *lse) {
    pdl_wait();  // the partials come from the previous kernel
    const int nch = p.Dv / 8;
    const int64_t gid = (int64_t)blockIdx.x * CMB_THREADS + threadIdx.x;
    if (gid >= (int64_t)p.T * p.H * nch) return;
    const int c = (int)(gid % nch);
    const int th = (int)(gid / nch);  // t * H + h
    const int t = th / p.H, h = th % p.H;
    const int S = p.splits;
    const float g = __bfloat162float(__ushort_as_bfloat16(gate[th]));
    const uint16_t *base = p.part_o + ((int64_t)t * S * p.H + h) * p.Dv + c * 8;
    const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml) + (int64_t)t * S * p.H + h;
    const int64_t sstride = (int64_t)p.H * p.Dv;
    float M = -INFINITY, W = 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // running merge over batches of splits: acc and W are kept relative to M
    for (int s0 = 0; s0 < S; s0 += CMB_BATCH) {
        float2 v[CMB_BATCH];
        uint4 o[CMB_BATCH];
#pragma unroll
        for (int u = 0; u < CMB_BATCH; ++u) {
            const bool in = s0 + u < S;
            v[u] = in ? ml[(int64_t)(s0 + u) * p.H] : make_float2(-INFINITY, 0.f);
            o[u] = in ? *reinterpret_cast<const uint4 *>(base + (s0 + u) * sstride) : make_uint4(0, 0, 0, 0);
        }
        float Mb = M;
#pragma unroll
        for (int u = 0; u < CMB_BATCH; ++u)
            if (v[u].y > 0.f) Mb = fmaxf(Mb, v[u].x);
        if (Mb == -INFINITY) continue;  // nothing selected so far
        const float r = M == -INFINITY ? 0.f : ex2_approx(M - Mb);
        W *= r;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= r;
        M = Mb;
#pragma unroll
        for (int u = 0; u < CMB_BATCH; ++u) {
            const float w = v[u].y > 0.f ? v[u].y * ex2_approx(v[u].x - M) : 0.f;
            W += w;
            const uint32_t w4[4] = {o[u].x, o[u].y, o[u].z, o[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = fmaf(w, __uint_as_float(w4[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = fmaf(w, __uint_as_float(w4[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
    }
    const float sc = W > 0.f ? (1.f / (1.f + __expf(-g))) / W : 0.f;
    uint4 r;
    r.x = pack_bf16(acc[0] * sc, acc[1] * sc);
    r.y = pack_bf16(acc[2] * sc, acc[3] * sc);
    r.z = pack_bf16(acc[4] * sc, acc[5] * sc);
    r.w = pack_bf16(acc[6] * sc, acc[7] * sc);
    *reinterpret_cast<uint4 *>(out + (int64_t)th * p.Dv + c * 8) = r;
    if (c == 0 && lse) lse[th] = W > 0.f ? (M + __log2f(W)) * 0.69314718055994531f : -INFINITY;
}

// Merges split partials: out = sigmoid(g) * sum_s w_s o_s with
// w_s = l_s 2^(m_s - M) / sum_s' l_s' 2^(m_s' - M).
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p) {
    pdl_wait();  // the partials come from the previous kernel
    const int t = blockIdx.x;
    const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (h >= p.H) return;
    const int S = p.splits;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) {
        const float *ml = p.part_ml + (((int64_t)t * S + s) * p.H + h) * 2;
        if (ml[1] > 0.f) M = fmaxf(M, ml[0]);
    }
    float wsum = 0.f;
    for (int s = 0; s < S; ++s) {
        const float *ml = p.part_ml + (((int64_t)t * S + s) * p.H + h) * 2;
        if (ml[1] > 0.f) wsum += ml[1] * ex2_approx(ml[0] - M);
    }
    const float g = __bfloat162float(__ushort_as_bfloat16(p.gate[(int64_t)t * p.H + h]));
    const float sig = 1.f / (1.f + __expf(-g));
    const float inv = wsum > 0.f ? sig / wsum : 0.f;
    uint16_t *orow = p.out + ((int64_t)t * p.H + h) * p.Dv;
    for (int d0 = lane * 4; d0 < p.Dv; d0 += 128) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
            const int64_t prow = ((int64_t)t * S + s) * p.H + h;
            const float *ml = p.part_ml + prow * 2;
            if (!(ml[1] > 0.f)) continue;
            const float c = ml[1] * ex2_approx(ml[0] - M);
            const float4 v = *reinterpret_cast<const float4 *>(p.part_o + prow * p.Dv + d0);
            acc.x = fmaf(c, v.x, acc.x);
            acc.y = fmaf(c, v.y, acc.y);
            acc.z = fmaf(c, v.z, acc.z);
            acc.w = fmaf(c, v.w, acc.w);
        }
        uint2 o;
        o.x = pack_bf16(acc.x * inv, acc.y * inv);
        o.y = pack_bf16(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(orow + d0) = o;
    }
    if (lane == 0 && p.lse)
        p.lse[(int64_t)t * p.H + h] = wsum > 0.f ? (M + __log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

struct Plan {
    int nparts, splits, rows_per_split;
};

Plan plan_for(int T, int K, int Dv, int sm_count) {
    Plan pl;
    pl.nparts = Dv == 512 ? 2 : 1;
    const int nchunks = K / 64;
    int splits = 1;
    const int base = T * pl.nparts;
    if (base < sm_count) splits = sm_count / base;
    if (splits > nchunks) splits = nchunks;
    if (splits < 1) splits = 1;
    const int cps = (nchunks + splits - 1) / splits;
    pl.rows_per_split = cps * 64;
    pl.splits = (nchunks + cps - 1) / cps;
    return pl;
}

// Launches fn<<<grid, block, smem, st>>>(args...), as a programmatic
// dependent of the previous kernel in the stream when pdl is set.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*fn)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t st, bool pdl,
                     Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, fn, std::forward<Args>(args)...);
}

template <int DQK, int DVP>
dsa_status run_attn(const CUtensorMap &qm, const AttnParams &p, bool pdl, cudaStream_t st) {
    using C = AttnCfg<DQK, DVP>;
    auto fn = attn_kernel<DQK, DVP>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    dim3 grid(p.nparts * p.splits, p.T);
    if (launch_k(fn, grid, dim3(ATT_THREADS), C::SMEM, st, pdl, qm, p) != cudaSuccess) return DSA_ERR_CUDA;
    if (p.splits > 1) {
        dim3 cg(p.T, (p.H + 7) / 8);
        if (launch_k(attn_combine_kernel, cg, dim3(256), 0, st, pdl, p) != cudaSuccess) return DSA_ERR_CUDA;
    }
    return DSA_OK;
}

}  // namespace

// Few queries (decode): one CTA per (token, 128 selected rows) plus a
// combine.  Many queries (prefill): the row-looping kernel above.
constexpr int DEC_MAX_T = 64;
bool use_decode(int T) { return T <= DEC_MAX_T; }
int dec_splits(int K) { return (K + DEC_NR - 1) / DEC_NR; }
size_t dec_ws_bytes(int T, int H, int K, int Dv) {
    const size_t rows = (size_t)T * dec_splits(K) * H;
    return align_up(rows * Dv * 2, 256) + align_up(rows * 2 * 4, 256);
}

size_t attn_workspace_bytes(int32_t T, int32_t H, int32_t K, int32_t Dv) {
    const DeviceInfo *dev = current_device();
    if (!dev || T <= 0 || K < 64) return 0;
    if (use_decode(T)) return dec_ws_bytes(T, H, K, Dv);
    Plan pl = plan_for(T, K, Dv, dev->sm_count);
    if (pl.splits == 1) return 0;
    const size_t rows = (size_t)T * pl.splits * H;
    return align_up(rows * Dv * 4, 256) + align_up(rows * 2 * 4, 256);
}

int attn_kernel_launches(int32_t T, int32_t K, int32_t Dv) {
    const DeviceInfo *dev = current_device();
    if (!dev || T <= 0) return 0;
    if (use_decode(T)) return 2;
    return plan_for(T, K, Dv, dev->sm_count).splits > 1 ? 2 : 1;
}

template <int DQK, int DV>
dsa_status run_attn_decode(const CUtensorMap &qm, const DecAttnParams &p, const uint16_t *gate, uint16_t *out,
                           float *lse, bool pdl, cudaStream_t st) {
    using C = DecAttnCfg<DQK, DV>;
    auto fn = attn_decode_kernel<DQK, DV>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    // partials [T * splits][H][Dv] bf16, stored one [64 dims x H heads] box at a time
    CUtensorMap om;
    const uint64_t odims[3] = {(uint64_t)p.Dv, (uint64_t)p.H, (uint64_t)p.T * p.splits};
    const uint32_t obox[3] = {64, (uint32_t)p.H, 1};
    if (p.H > 128 || !make_tmap_3d(&om, p.part_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, odims, (uint64_t)p.Dv * 2,
                                   (uint64_t)p.H * p.Dv * 2, obox, CU_TENSOR_MAP_SWIZZLE_128B))
        return DSA_ERR_INVALID_ARG;
    if (launch_k(fn, dim3(p.splits, p.T), dim3(DEC_THREADS), C::SMEM, st, pdl, qm, om, p) != cudaSuccess)
        return DSA_ERR_CUDA;
    const int64_t threads = (int64_t)p.T * p.H * (p.Dv / 8);
    return launch_k(attn_decode_combine_kernel, dim3((unsigned)((threads + CMB_THREADS - 1) / CMB_THREADS)),
                    dim3(CMB_THREADS), 0, st, pdl, p, gate, out, lse) == cudaSuccess
               ? DSA_OK
               : DSA_ERR_CUDA;
}

dsa_status launch_attn(const AttnArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.T == 0) return DSA_OK;
    CUtensorMap qm;
    if (!make_tmap_2d(&qm, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Dqk, (uint64_t)a.T * a.H, (uint64_t)a.Dqk * 2,
                      64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return DSA_ERR_INVALID_ARG;
    if (use_decode(a.T)) {
        DecAttnParams dp{};
        dp.kv = a.kv;
        dp.pg = a.pg;
        dp.q_seq = a.q_seq;
        dp.idx = a.idx;
        dp.K = a.K;
        dp.scale_log2 = a.sm_scale * 1.4426950408889634f;
        dp.T = a.T;
        dp.H = a.H;
        dp.Dv = a.Dv;
        dp.splits = dec_splits(a.K);
        dp.err = dev->err;
        const size_t rows = (size_t)a.T * dp.splits * a.H;
        if (!a.ws || a.ws_bytes < dec_ws_bytes(a.T, a.H, a.K, a.Dv)) return DSA_ERR_WORKSPACE;
        dp.part_o = static_cast<uint16_t *>(a.ws);
        dp.part_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + align_up(rows * a.Dv * 2, 256));
        if (a.Dqk == 576 && a.Dv == 512) return run_attn_decode<576, 512>(qm, dp, a.gate, a.out, a.lse, a.pdl, st);
        if (a.Dqk == 64 && a.Dv == 64) return run_attn_decode<64, 64>(qm, dp, a.gate, a.out, a.lse, a.pdl, st);
        return DSA_ERR_UNSUPPORTED;
    }
    Plan pl = plan_for(a.T, a.K, a.Dv, dev->sm_count);
    AttnParams p{};
    p.kv = a.kv;
    p.pg = a.pg;
    p.q_seq = a.q_seq;
    p.idx = a.idx;
    p.K = a.K;
    p.gate = a.gate;
    p.scale_log2 = a.sm_scale * 1.4426950408889634f;
    p.T = a.T;
    p.H = a.H;
    p.Dv = a.Dv;
    p.nparts = pl.nparts;
    p.splits = pl.splits;
    p.rows_per_split = pl.rows_per_split;
    p.out = a.out;
    p.lse = a.lse;
    p.err = dev->err;
    if (pl.splits > 1) {
        const size_t rows = (size_t)a.T * pl.splits * a.H;
        const size_t need = align_up(rows * a.Dv * 4, 256) + align_up(rows * 2 * 4, 256);
        if (!a.ws || a.ws_bytes < need) return DSA_ERR_WORKSPACE;
        p.part_o = static_cast<float *>(a.ws);
        p.part_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + align_up(rows * a.Dv * 4, 256));
    }
    if (a.Dqk == 576 && a.Dv == 512) return run_attn<576, 256>(qm, p, a.pdl, st);
    if (a.Dqk == 64 && a.Dv == 64) return run_attn<64, 64>(qm, p, a.pdl, st);
    return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
