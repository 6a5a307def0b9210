// Stage 1 of the Gated DSA layer: the lightweight FP8 indexer.
//
//   I[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])     for s <= q_pos[t]
//
// ("Open-Source LLM Architecture Evolution: How Lightweight Sparse Attention
// Reshapes Long-Context Modeling Efficiency", Architecture Breakdown §2,
// "Indexer"; "Fine-Grained Sparse Attention in Ultra-Large Parameter Models",
// §2.2 -- no rotary embedding, so the stored keys are used as they are -- and
// §2.3 -- heads x 128 dims.)
//
// Both kernels put 128 keys on the M side of a tcgen05 e4m3 MMA (two 64-row
// pages of the paged key cache, fetched by TMA with the 128- or 64-byte
// swizzle the MMA reads), accumulate in fp32 in tensor memory and apply the
// ReLU and the w-weighted head reduction in the epilogue warps:
//   * decode: N = the query's heads (padded to 16); one query per tile; the
//     tiles of all queries are spread evenly over a persistent grid, so even
//     one 1M-token query keeps every SM streaming its own slice of keys.
//   * prefill: N = 256 = a group of 256/HI consecutive queries x HI heads; a
//     persistent CTA takes whole query groups (snake order, costliest first)
//     and streams the key tiles of the group's causal range.
// Up to 64 explicit queries of 16 or 32 heads x 128 go to the grouped kernel
// of indexer_group.cu instead, where a sequence's draft queries share keys.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM owner),
// then two epilogue warpgroups that take alternate tiles (each warp reads
// one TMEM lane quarter), so one tile's TMEM read latency overlaps another's
// arithmetic.
#include "indexer_common.cuh"

namespace dsa {
namespace {

// ============================================================================
// decode: keys x heads, one query per tile
// ============================================================================

// Two CTAs share each SM (two TMA-issuing producers keep more of HBM busy
// than one producer with a deeper ring), each with its own TMEM slice.
template <int DI, int NH>
struct DecCfg {
    static constexpr int CTAS_PER_SM = 2;
    static constexpr int STAGES = DI == 128 ? 5 : 10;  // key tiles in flight per CTA
    static constexpr int EPI_GROUPS = 2;  // epilogue warpgroups, alternate tiles
    static constexpr int ACC = NH <= 32 ? 8 : 4;  // TMEM: ACC * NH <= 256 columns per CTA
    static constexpr int THREADS = 64 + 128 * EPI_GROUPS;
    static constexpr int A_BYTES = 128 * DI;      // one key tile (two pages)
    static constexpr int B_BYTES = NH * DI;       // one query's heads
    static constexpr int TMEM_COLS = pow2_cols(ACC * NH);
    static constexpr uint32_t SWZ = DI == 128 ? SWZ_128B : SWZ_64B;
    static constexpr uint32_t SBO = 8 * DI;
    static constexpr int MAXT = 1024;
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * ACC + 4 + 1);
    static constexpr int HIST_WORDS = SCORE_HIST_BINS / 2;  // per epilogue warpgroup: packed 16-bit counts
    static constexpr int HIST_FLUSH_TILES = 256;            // a count stays below 2^16
    static constexpr int SMEM =
        1024 + STAGES * A_BYTES + 2 * B_BYTES + BAR_BYTES + 4 * (MAXT + 1) + 16 + 4 * EPI_GROUPS * HIST_WORDS;
    static_assert(HIST_FLUSH_TILES * 128 < 65536, "packed counts do not carry");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tile alignment");
};

template <int DI, int NH>
__global__ void __launch_bounds__(DecCfg<DI, NH>::THREADS, DecCfg<DI, NH>::CTAS_PER_SM)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                          const IdxParams p) {
    using C = DecCfg<DI, NH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                                  // [STAGES][A_BYTES]
    uint8_t *qbuf = smem + C::STAGES * C::A_BYTES;            // [2][B_BYTES]
    uint64_t *full = reinterpret_cast<uint64_t *>(qbuf + 2 * C::B_BYTES);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + C::ACC;
    uint64_t *qfull = tempty + C::ACC;   // [2]
    uint64_t *qempty = qfull + 2;        // [2]
    uint64_t *drain = qempty + 2;
    int32_t *tstart = reinterpret_cast<int32_t *>(drain + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tstart + C::MAXT + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *hist_sm = reinterpret_cast<uint32_t *>(tmem_slot + 4);  // [EPI_GROUPS][HIST_WORDS]

    const int warp = warp_id(), lane = lane_id();
    const int T = p.T;
    if (threadIdx.x == 64 && p.q_seq == nullptr) {
        // Warm L2 with what the producer's first lookups read (inputs of the
        // layer, cold at launch): the sequence lengths, and the block-table
        // lines of this CTA's share of the tiles as if every query had max_len
        // keys (exact when the lengths are equal; a prefetch that misses costs nothing).
        for (int i = 0; i < T; i += 32) prefetch_l2(p.pg.seq_lens + i);
        const int64_t tq = (p.max_len + 127) >> 7;  // tiles per query at max_len
        const int64_t tb = (int64_t)T * tq;
        const int64_t k0 = tb * blockIdx.x / gridDim.x, k1 = tb * (blockIdx.x + 1) / gridDim.x;
        for (int64_t k = k0; k < k1 + 16; k += 16) {  // 16 tiles = 32 pages = one 128-byte line of the table
            const int64_t kk = k < k1 ? k : k1 - 1;
            const int64_t q = kk / tq, j = kk % tq;
            if (kk < k0 || q >= p.pg.num_seqs || 2 * j >= p.pg.max_blocks) break;
            prefetch_l2(p.pg.block_table + q * p.pg.max_blocks + 2 * j);
        }
    }
    if (p.hist)
        for (int i = threadIdx.x; i < C::EPI_GROUPS * C::HIST_WORDS; i += blockDim.x) hist_sm[i] = 0;
    clear_words(p);

    if (threadIdx.x == 32) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&qmap);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    // Per-query tile counts -> their inclusive scan tstart -> this CTA's share
    // [lo, hi) of the flattened (query, tile) space.  With up to 64 queries
    // warp 0 does it alone and goes on to look up the pages of its first 32
    // tiles while the other warps set up barriers and TMEM, so the first key
    // tile is issued right after set-up.
    const bool early = T <= 64;
    auto scan_counts = [&](int base, int v, int &running) {  // warp 0: tstart[base+1..] from counts v
        const int i = base + lane;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += x;
        }
        if (i < T) tstart[i + 1] = running + v;
        running += __shfl_sync(0xffffffffu, v, 31);
    };
    int w0_tq = -1, w0_p0 = -1, w0_p1 = -1;  // early: lane's tile of the producer's first window
    if (early) {
        if (warp == 0) {
            int cnt[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = lane + 32 * h;
                cnt[h] = t < T ? (query_info(t, p.q_seq, p.q_pos, p.pg, p.max_len, nullptr).last + 1 + 127) >> 7 : 0;
            }
            if (lane == 0) tstart[0] = 0;
            int running = 0;
            scan_counts(0, cnt[0], running);
            if (T > 32) scan_counts(32, cnt[1], running);
            __syncwarp();
            const int64_t tot = tstart[T];
            const int64_t lo0 = tot * blockIdx.x / gridDim.x, hi0 = tot * (blockIdx.x + 1) / gridDim.x;
            if (lane < hi0 - lo0) {
                const int64_t g = lo0 + lane;
                w0_tq = locate(tstart, T, g);
                const int j = static_cast<int>(g - tstart[w0_tq]);
                const QInfo qi = query_info(w0_tq, p.q_seq, p.q_pos, p.pg, p.max_len, p.err);
                w0_p0 = page_of(p.pg, qi.b, 2 * j, p.err);
                w0_p1 = (2 * j + 1) * 64 <= qi.last ? page_of(p.pg, qi.b, 2 * j + 1, p.err) : -1;
            }
        }
    } else {
        for (int t = threadIdx.x; t < T; t += blockDim.x) {
            QInfo qi = query_info(t, p.q_seq, p.q_pos, p.pg, p.max_len, nullptr);
            tstart[t + 1] = (qi.last + 1 + 127) >> 7;
        }
        if (threadIdx.x == 0) tstart[0] = 0;
        __syncthreads();
        if (warp == 0) {
            int running = 0;
            for (int base = 0; base < T; base += 32) scan_counts(base, base + lane < T ? tstart[base + lane + 1] : 0,
                                                                 running);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();
    const uint32_t tmem = *tmem_slot;
    const int64_t total = tstart[T];
    const int64_t lo = total * blockIdx.x / gridDim.x;
    const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
    const int n = static_cast<int>(hi - lo);

    if (warp == 0 && n > 0) {
        // ---------------- producer ----------------
        // The warp looks up the next 32 tiles' (query, pages) in parallel, one
        // tile per lane, a window ahead of the tiles lane 0 is issuing, so no
        // block-table load sits on the issue path.
        auto lookup = [&](int i, int &tq, int &p0, int &p1) {
            tq = -1, p0 = -1, p1 = -1;
            if (i < n) {
                const int64_t g = lo + i;
                tq = locate(tstart, T, g);
                const int j = static_cast<int>(g - tstart[tq]);
                const QInfo qi = query_info(tq, p.q_seq, p.q_pos, p.pg, p.max_len, p.err);
                p0 = page_of(p.pg, qi.b, 2 * j, p.err);
                p1 = (2 * j + 1) * 64 <= qi.last ? page_of(p.pg, qi.b, 2 * j + 1, p.err) : -1;
            }
        };
        int tq = w0_tq, p0 = w0_p0, p1 = w0_p1;
        if (!early) lookup(lane, tq, p0, p1);
        // keys are read once: let them leave L2 first, so the scores written
        // meanwhile are still there for the top-K that follows
        const uint64_t kpol = l2_policy_evict_first();
        int issued = 0, qo = -1, tprev = -1;
        bool ok = true;
        for (int base = 0; ok && base < n; base += 32) {
            int tq_n, p0_n, p1_n;
            lookup(base + 32 + lane, tq_n, p0_n, p1_n);
            const int cnt = min(32, n - base);
            for (int k = 0; k < cnt; ++k) {
                const int t = __shfl_sync(0xffffffffu, tq, k);
                const int pg0 = __shfl_sync(0xffffffffu, p0, k);
                const int pg1 = __shfl_sync(0xffffffffu, p1, k);
                if (lane == 0) {
                    const int i = base + k;
                    if (t != tprev) {  // a new query: its heads go to the next q buffer
                        tprev = t;
                        ++qo;
                        const int qb = qo & 1;
                        if (mbar_wait(&qempty[qb], ((qo >> 1) & 1) ^ 1, p.err, abort_flag)) {
                            mbar_expect_tx(&qfull[qb], C::B_BYTES);
                            tma_load_2d(qbuf + qb * C::B_BYTES, &qmap, &qfull[qb], 0, t * p.HI);
                        } else {
                            ok = false;
                        }
                    }
                    const int s = i % C::STAGES;
                    const uint32_t ph = (i / C::STAGES) & 1;
                    if (ok && mbar_wait(&empty[s], ph ^ 1, p.err, abort_flag)) {
                        uint8_t *A = stages + s * C::A_BYTES;
                        const uint32_t bytes = (pg0 >= 0 ? 64 * DI : 0) + (pg1 >= 0 ? 64 * DI : 0);
                        if (lo + i + 1 == p.test_skip_tile_plus1) {
                            // testing the bounded waits: this tile is never filled, so the
                            // MMA's wait on it runs out and the CTA abandons its work
                        } else if (bytes) {
                            mbar_expect_tx(&full[s], bytes);
                            if (pg0 >= 0) tma_load_2d_hint(A, &kmap, &full[s], 0, pg0 * 64, kpol);
                            if (pg1 >= 0) tma_load_2d_hint(A + 64 * DI, &kmap, &full[s], 0, pg1 * 64, kpol);
                        } else {
                            mbar_arrive(&full[s]);
                        }
                        ++issued;
                    } else {
                        ok = false;
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                    ok = false;
                    break;
                }
            }
            tq = tq_n, p0 = p0_n, p1 = p1_n;
        }
        // never leave a copy in flight behind
        if (lane == 0) {
            for (int i = issued - 1; i >= 0 && i >= issued - C::STAGES; --i)
                mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1, p.err, nullptr);
            if (qo >= 0) mbar_wait(&qfull[qo & 1], (qo >> 1) & 1, p.err, nullptr);
        }
    } else if (warp == 1 && lane == 0 && n > 0) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t ID = idesc(0, 0, 0, 0, NH, 128);
        int t = locate(tstart, T, lo);
        int j = static_cast<int>(lo - tstart[t]);
        int qo = -1, tprev = -1;
        for (int i = 0; i < n; ++i) {
            if (t != tprev) {  // the query changes: release the old heads, wait for the new
                if (qo >= 0) mma_commit(&qempty[qo & 1]);
                tprev = t;
                ++qo;
                if (!mbar_wait(&qfull[qo & 1], (qo >> 1) & 1, p.err, abort_flag)) break;
            }
            const int s = i % C::STAGES;
            const uint32_t ph = (i / C::STAGES) & 1;
            const int a = i % C::ACC;
            const uint32_t aph = (i / C::ACC) & 1;
            if (!mbar_wait(&full[s], ph, p.err, abort_flag)) break;
            if (!mbar_wait(&tempty[a], aph ^ 1, p.err, abort_flag)) break;
            tc_fence_after();
            const uint32_t A = smem_u32(stages + s * C::A_BYTES);
            const uint32_t B = smem_u32(qbuf + (qo & 1) * C::B_BYTES);
            const uint32_t d = tmem + a * NH;
#pragma unroll
            for (int k = 0; k < DI / 32; ++k)
                mma_e4m3(d, sdesc(A + 32 * k, 16, C::SBO, C::SWZ), sdesc(B + 32 * k, 16, C::SBO, C::SWZ), ID,
                         k > 0);
            mma_commit(&empty[s]);
            mma_commit(&tfull[a]);
            if (++j == tstart[t + 1] - tstart[t]) {
                j = 0;
                do { ++t; } while (t < T && tstart[t + 1] == tstart[t]);
            }
        }
        mma_commit(drain);
        mbar_wait(drain, 0, p.err, nullptr);
    } else if (warp >= 2 && n > 0) {
        // ---------------- epilogue: warpgroup eg takes tiles i with i % EPI_GROUPS == eg ----------------
        // Every thread of a warpgroup walks the same tiles (a failed wait only
        // turns the work off), so the warpgroup's named barriers stay uniform.
        const int eg = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        int t = locate(tstart, T, lo);
        int j = static_cast<int>(lo - tstart[t]);
        int tw = -1;  // query whose w is in registers
        QInfo qi{0, -1};
        float wr[NH];
        bool alive = true;
        // score histogram of this warpgroup's tiles of query hq (packed 16-bit counts)
        uint32_t *hw = hist_sm + eg * C::HIST_WORDS;
        int hq = -1, htiles = 0;
        auto hflush = [&]() {
            named_bar_sync(1 + eg, 128);  // every add of the warpgroup has landed
            if (hq >= 0 && alive)
                for (int wi = row; wi < C::HIST_WORDS; wi += 128) {
                    const uint32_t v = hw[wi];
                    if (v) {
                        uint32_t *g = p.hist + (int64_t)hq * SCORE_HIST_BINS + 2 * wi;
                        if (v & 0xFFFFu) red_add_global(g, v & 0xFFFFu);
                        if (v >> 16) red_add_global(g + 1, v >> 16);
                        hw[wi] = 0;
                    }
                }
            htiles = 0;
            named_bar_sync(1 + eg, 128);  // cleared before the next adds
        };
        for (int i = 0; i < n; ++i) {
            if (i % C::EPI_GROUPS == eg) {
                if (t != tw) {
                    tw = t;
                    qi = query_info(t, p.q_seq, p.q_pos, p.pg, p.max_len, p.err);
#pragma unroll
                    for (int h = 0; h < NH; ++h) wr[h] = h < p.HI ? p.w[(int64_t)t * p.HI + h] : 0.f;
                }
                if (p.hist && (t != hq || htiles == C::HIST_FLUSH_TILES)) {
                    hflush();
                    hq = t;
                }
                ++htiles;
                const int a = i % C::ACC;
                const uint32_t aph = (i / C::ACC) & 1;
                if (alive && !mbar_wait(&tfull[a], aph, p.err, abort_flag)) alive = false;
            }
            if (i % C::EPI_GROUPS == eg && alive) {
                const int a = i % C::ACC;
                tc_fence_after();
                uint32_t r[NH];
                const uint32_t ta = tmem + a * NH + lane_off;
                if constexpr (NH == 16) {
                    tmem_ld16(ta, r);
                } else {
#pragma unroll
                    for (int c = 0; c < NH / 32; ++c) tmem_ld32(ta + 32 * c, r + 32 * c);
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[a]);
                float sc = 0.f;
#pragma unroll
                for (int h = 0; h < NH; ++h)
                    if (h < p.HI) sc = fmaf(wr[h], fmaxf(__uint_as_float(r[h]), 0.f), sc);
                const int spos = j * 128 + row;
                if (spos <= qi.last) {
                    p.scores[(int64_t)t * p.ld + spos] = sc;
                    if (p.hist) {
                        const uint32_t bin = score_key(sc) >> SCORE_HIST_SHIFT;
                        atomicAdd(&hw[bin >> 1], 1u << ((bin & 1u) << 4));
                    }
                }
            }
            if (++j == tstart[t + 1] - tstart[t]) {
                j = 0;
                do { ++t; } while (t < T && tstart[t + 1] == tstart[t]);
            }
        }
        if (p.hist) hflush();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ============================================================================
// prefill: keys x (query group x heads), N = 256
// ============================================================================

template <int DI, int HI>
struct PreCfg {
    static constexpr int N = 256;
    static constexpr int G = N / HI;  // queries per group
    static constexpr int A_BYTES = 128 * DI;
    static constexpr int B_BYTES = N * DI;
    static constexpr int ASTAGES = DI == 128 ? 6 : 10;
    static constexpr int TMEM_COLS = 512;  // two 256-column accumulators
    static constexpr int EPI_WG = 4;       // epilogue warpgroups: each reduces one column quarter of every tile
    static constexpr int THREADS = 64 + 128 * EPI_WG;
    static constexpr uint32_t SWZ = DI == 128 ? SWZ_128B : SWZ_64B;
    static constexpr uint32_t SBO = 8 * DI;
    static constexpr int BAR_BYTES = 8 * (2 * ASTAGES + 4 + 4 + 1);
    static constexpr int TBL = 3 * G;  // three per-role copies of the group table
    // + 16: up to 8 bytes to align the weights, then the TMEM slot and abort flag
    static constexpr int SMEM = 1024 + 2 * B_BYTES + ASTAGES * A_BYTES + BAR_BYTES + 4 * N + 8 * TBL + 16;
    static_assert(N % 4 == 0 && (4 * N) % 8 == 0, "weights are read as float4; the tables stay 8-byte aligned");
};

// One role's view of a query group: token u's (sequence, last position).
__device__ __forceinline__ void load_group_tbl(int2 *tbl, int g, int G, const IdxParams &p, bool report, int lane,
                                               int nthr) {
    for (int u = lane; u < G; u += nthr) {
        const int t = g * G + u;
        int2 v = make_int2(-1, -1);
        if (t < p.T) {
            QInfo qi = query_info(t, p.q_seq, p.q_pos, p.pg, p.max_len, report ? p.err : nullptr);
            v = make_int2(qi.last >= 0 ? qi.b : -1, qi.last);
        }
        tbl[u] = v;
    }
}

// Next run of consecutive tokens [u, *u1) of one sequence; returns its key
// tile count.
__device__ __forceinline__ int next_run(const int2 *tbl, int G, int u, int *u1, int *b) {
    const int bb = tbl[u].x;
    int mx = tbl[u].y, v = u + 1;
    while (v < G && tbl[v].x == bb) {
        mx = max(mx, tbl[v].y);
        ++v;
    }
    *u1 = v;
    *b = bb;
    return bb < 0 ? 0 : (mx + 1 + 127) >> 7;
}

__device__ __forceinline__ int group_of(int r, int c, int grid, int ngroups) {
    const int k = r * grid + ((r & 1) ? grid - 1 - c : c);
    return k < ngroups ? ngroups - 1 - k : -1;
}

template <int DI, int HI>
__global__ void __launch_bounds__(PreCfg<DI, HI>::THREADS, 1)
    indexer_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                           const IdxParams p) {
    using C = PreCfg<DI, HI>;
    constexpr int G = C::G;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *Bbuf = smem;                     // [2][B_BYTES]
    uint8_t *Abuf = smem + 2 * C::B_BYTES;    // [ASTAGES][A_BYTES]
    uint64_t *afull = reinterpret_cast<uint64_t *>(Abuf + C::ASTAGES * C::A_BYTES);
    uint64_t *aempty = afull + C::ASTAGES;
    uint64_t *bfull = aempty + C::ASTAGES;
    uint64_t *bempty = bfull + 2;
    uint64_t *tfull = bempty + 2;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    float *wbuf = reinterpret_cast<float *>(  // [N], 16-byte aligned: read as float4
        (reinterpret_cast<uintptr_t>(drain + 1) + 15) & ~uintptr_t(15));
    int2 *tbl_p = reinterpret_cast<int2 *>(wbuf + C::N);
    int2 *tbl_m = tbl_p + G;
    int2 *tbl_e = tbl_m + G;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tbl_e + G);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const int ngroups = (p.T + G - 1) / G;
    const int grid = gridDim.x, cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::ASTAGES; ++s) {
            mbar_init(&afull[s], 1);
            mbar_init(&aempty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4 * C::EPI_WG);  // every epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&qmap);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- producer ----------------
        // The warp loads the group table and, per run, looks up the pages of
        // 32 key tiles at a time (one per lane, the next window in flight while
        // lane 0 issues the current one).
        int ac = 0, issued_a = 0, gi = 0;
        bool ok = true;
        for (int r = 0; ok; ++r, ++gi) {
            const int g = group_of(r, cta, grid, ngroups);
            if (g < 0) break;
            load_group_tbl(tbl_p, g, G, p, false, lane, 32);
            __syncwarp();
            const int bst = gi & 1;
            if (lane == 0) {
                if (!mbar_wait(&bempty[bst], ((gi >> 1) & 1) ^ 1, p.err, abort_flag)) ok = false;
                if (ok) {
                    mbar_expect_tx(&bfull[bst], C::B_BYTES);
                    tma_load_2d(Bbuf + bst * C::B_BYTES, &qmap, &bfull[bst], 0, g * G * HI);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            for (int u = 0; ok && u < G;) {
                int u1, b;
                const int nt = next_run(tbl_p, G, u, &u1, &b);
                int mx = -1;
                for (int v = u; v < u1; ++v) mx = max(mx, tbl_p[v].y);
                auto lookup = [&](int kt, int &q0, int &q1) {
                    q0 = -1, q1 = -1;
                    if (kt < nt) {
                        q0 = page_of(p.pg, b, 2 * kt, p.err);
                        q1 = (2 * kt + 1) * 64 <= mx ? page_of(p.pg, b, 2 * kt + 1, p.err) : -1;
                    }
                };
                int q0, q1;
                lookup(lane, q0, q1);
                for (int base = 0; ok && base < nt; base += 32) {
                    int q0n, q1n;
                    lookup(base + 32 + lane, q0n, q1n);
                    const int cnt = min(32, nt - base);
                    for (int k = 0; k < cnt; ++k) {
                        const int pg0 = __shfl_sync(0xffffffffu, q0, k);
                        const int pg1 = __shfl_sync(0xffffffffu, q1, k);
                        if (lane == 0) {
                            const int s = ac % C::ASTAGES;
                            if (mbar_wait(&aempty[s], ((ac / C::ASTAGES) & 1) ^ 1, p.err, abort_flag)) {
                                uint8_t *A = Abuf + s * C::A_BYTES;
                                const uint32_t bytes = (pg0 >= 0 ? 64 * DI : 0) + (pg1 >= 0 ? 64 * DI : 0);
                                if (bytes) {
                                    mbar_expect_tx(&afull[s], bytes);
                                    if (pg0 >= 0) tma_load_2d(A, &kmap, &afull[s], 0, pg0 * 64);
                                    if (pg1 >= 0) tma_load_2d(A + 64 * DI, &kmap, &afull[s], 0, pg1 * 64);
                                } else {
                                    mbar_arrive(&afull[s]);
                                }
                                ++ac;
                                issued_a = ac;
                            } else {
                                ok = false;
                            }
                        }
                        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                            ok = false;
                            break;
                        }
                    }
                    q0 = q0n, q1 = q1n;
                }
                u = u1;
            }
        }
        if (lane == 0) {
            for (int i = issued_a - 1; i >= 0 && i >= issued_a - C::ASTAGES; --i)
                mbar_wait(&afull[i % C::ASTAGES], (i / C::ASTAGES) & 1, p.err, nullptr);
            if (gi > 0) mbar_wait(&bfull[(gi - 1) & 1], ((gi - 1) >> 1) & 1, p.err, nullptr);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t ID = idesc(0, 0, 0, 0, C::N, 128);
        int ac = 0, tc = 0, gi = 0;
        bool ok = true;
        for (int r = 0; ok; ++r, ++gi) {
            const int g = group_of(r, cta, grid, ngroups);
            if (g < 0) break;
            load_group_tbl(tbl_m, g, G, p, false, lane, 32);
            __syncwarp();
            if (lane == 0) {
                const int bst = gi & 1;
                if (!mbar_wait(&bfull[bst], (gi >> 1) & 1, p.err, abort_flag)) ok = false;
                const uint32_t B = smem_u32(Bbuf + bst * C::B_BYTES);
                for (int u = 0; ok && u < G;) {
                    int u1, b;
                    const int nt = next_run(tbl_m, G, u, &u1, &b);
                    for (int kt = 0; kt < nt; ++kt) {
                        const int s = ac % C::ASTAGES;
                        const int a = tc & 1;
                        if (!mbar_wait(&afull[s], (ac / C::ASTAGES) & 1, p.err, abort_flag) ||
                            !mbar_wait(&tempty[a], ((tc >> 1) & 1) ^ 1, p.err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t A = smem_u32(Abuf + s * C::A_BYTES);
#pragma unroll
                        for (int k = 0; k < DI / 32; ++k)
                            mma_e4m3(tmem + a * C::N, sdesc(A + 32 * k, 16, C::SBO, C::SWZ),
                                     sdesc(B + 32 * k, 16, C::SBO, C::SWZ), ID, k > 0);
                        mma_commit(&aempty[s]);
                        mma_commit(&tfull[a]);
                        ++ac;
                        ++tc;
                    }
                    u = u1;
                }
                if (ok) mma_commit(&bempty[bst]);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        if (lane == 0) {
            mma_commit(drain);
            mbar_wait(drain, 0, p.err, nullptr);
        }
    } else {
        // ---------------- epilogue: four warpgroups (warps 2..17) ----------------
        // Tile tc lives in TMEM buffer a = tc % 2; warpgroup eg reduces column
        // quarter eg of every tile (warp w reads TMEM lane quarter w % 4), so
        // while the MMA refills one buffer every epilogue warp works on the
        // other one.
        constexpr int NT = C::EPI_WG * 128;
        const int et = threadIdx.x - 64;  // 0..NT-1
        const int eg = et >> 7;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        constexpr int HALF = C::N / C::EPI_WG;  // columns per warpgroup
        const int ch = eg;
        int tc = 0;
        bool ok = true;
        for (int r = 0; ok; ++r) {
            const int g = group_of(r, cta, grid, ngroups);
            if (g < 0) break;
            named_bar_sync(1, NT);
            load_group_tbl(tbl_e, g, G, p, true, et, NT);
            // halved weights: w * max(x, 0) = (w / 2) * (x + |x|) exactly (x + |x| is 2x or 0), so the
            // ReLU runs on the FMA pipe as an add with an absolute-value operand
            for (int i = et; i < C::N; i += NT) {
                const int t = g * G + i / HI;
                wbuf[i] = t < p.T ? 0.5f * p.w[(int64_t)t * HI + (i % HI)] : 0.f;
            }
            named_bar_sync(1, NT);
            for (int u = 0; ok && u < G;) {
                int u1, b;
                const int nt = next_run(tbl_e, G, u, &u1, &b);
                for (int kt = 0; kt < nt; ++kt, ++tc) {
                    const int a = tc & 1;
                    if (!mbar_wait(&tfull[a], (tc >> 1) & 1, p.err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int spos = kt * 128 + row;
                    const uint32_t ta = tmem + a * C::N + ch * HALF + lane_off;
                    // 32 columns at a time, the next chunk's TMEM load in flight while
                    // this one is reduced; independent partial sums keep the FMA chains
                    // short (sums of exact products: the order does not matter)
                    uint32_t rr[2][32];
                    tmem_ld32(ta, rr[0]);
                    tmem_wait_ld();
                    float acc = 0.f;
#pragma unroll
                    for (int cc = 0; cc < HALF / 32; ++cc) {
                        if (cc + 1 < HALF / 32) tmem_ld32(ta + 32 * (cc + 1), rr[(cc + 1) & 1]);
                        const uint32_t *x = rr[cc & 1];
                        const int col0 = ch * HALF + 32 * cc;  // first column of the chunk
                        if constexpr (HI >= 32) {
                            float wv[32];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float4 w4 = *reinterpret_cast<const float4 *>(wbuf + col0 + 4 * i);
                                wv[4 * i] = w4.x, wv[4 * i + 1] = w4.y, wv[4 * i + 2] = w4.z, wv[4 * i + 3] = w4.w;
                            }
                            const int tok = col0 / HI;
                            const int h0 = col0 % HI;
                            float2 ps[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                            for (int h = 0; h < 32; h += 2) {
                                const float x0 = __uint_as_float(x[h]), x1 = __uint_as_float(x[h + 1]);
                                ps[(h >> 1) & 3].x = fmaf(wv[h], x0 + fabsf(x0), ps[(h >> 1) & 3].x);
                                ps[(h >> 1) & 3].y = fmaf(wv[h + 1], x1 + fabsf(x1), ps[(h >> 1) & 3].y);
                            }
                            acc += ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) + ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
                            if (h0 + 32 == HI) {
                                const int2 info = tbl_e[tok];
                                st_global_if(p.scores + (int64_t)(g * G + tok) * p.ld + spos, acc,
                                             tok >= u && tok < u1 && spos <= info.y);
                                acc = 0.f;
                            }
                        } else {
                            constexpr int NA = HI >= 8 ? 2 : 1;  // partial sums per token
#pragma unroll
                            for (int uu = 0; uu < 32 / HI; ++uu) {
                                const int tok = col0 / HI + uu;
                                float2 ps[NA];
#pragma unroll
                                for (int i = 0; i < NA; ++i) ps[i] = make_float2(0.f, 0.f);
#pragma unroll
                                for (int h = 0; h < HI; h += 4) {
                                    const float4 w4 = *reinterpret_cast<const float4 *>(wbuf + col0 + uu * HI + h);
                                    const float x0 = __uint_as_float(x[uu * HI + h]), x1 = __uint_as_float(x[uu * HI + h + 1]);
                                    const float x2 = __uint_as_float(x[uu * HI + h + 2]), x3 = __uint_as_float(x[uu * HI + h + 3]);
                                    float2 &q0 = ps[(h >> 1) % NA], &q1 = ps[((h >> 1) + 1) % NA];
                                    q0.x = fmaf(w4.x, x0 + fabsf(x0), q0.x);
                                    q0.y = fmaf(w4.y, x1 + fabsf(x1), q0.y);
                                    q1.x = fmaf(w4.z, x2 + fabsf(x2), q1.x);
                                    q1.y = fmaf(w4.w, x3 + fabsf(x3), q1.y);
                                }
                                float sc = ps[0].x + ps[0].y;
                                if constexpr (NA == 2) sc += ps[1].x + ps[1].y;
                                const int2 info = tbl_e[tok];
                                st_global_if(p.scores + (int64_t)(g * G + tok) * p.ld + spos, sc,
                                             tok >= u && tok < u1 && spos <= info.y);
                            }
                        }
                        if (cc + 1 < HALF / 32) tmem_wait_ld();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[a]);
                }
                u = u1;
            }
            // the epilogue warpgroups leave the group loop together
            ok = !named_bar_or(1, NT, !ok || *abort_flag);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int DI, int NH>
dsa_status run_decode(const CUtensorMap &km, const CUtensorMap &qm, const IdxParams &p, int grid, cudaStream_t st) {
    using C = DecCfg<DI, NH>;
    auto fn = indexer_decode_kernel<DI, NH>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    fn<<<grid, C::THREADS, C::SMEM, st>>>(km, qm, p);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

template <int DI, int HI>
dsa_status run_prefill(const CUtensorMap &km, const CUtensorMap &qm, const IdxParams &p, int grid,
                       cudaStream_t st) {
    using C = PreCfg<DI, HI>;
    auto fn = indexer_prefill_kernel<DI, HI>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    fn<<<grid, C::THREADS, C::SMEM, st>>>(km, qm, p);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

dsa_status launch_indexer(const IndexerArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.T == 0) return DSA_OK;
    if (indexer_group_eligible(a)) return launch_indexer_group(a, st);
    IdxParams p{a.w, a.q_seq, a.q_pos, a.pg, a.T, a.HI, a.max_len, a.scores, a.ld, dev->err,
                (a.q_seq == nullptr || a.T <= 64) ? a.hist : nullptr,  // the few-query kernel counts
                a.zero, a.nzero, test_skip_tile() + 1};
    const CUtensorMapSwizzle swz = a.DI == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUtensorMap km, qm;
    if (!make_tmap_2d(&km, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.pg.num_pages * 64, a.DI,
                      a.DI, 64, swz))
        return DSA_ERR_INVALID_ARG;
    const bool decode = a.q_seq == nullptr || a.T <= 64;
    if (decode) {
        if (a.T > DecCfg<128, 32>::MAXT) return DSA_ERR_UNSUPPORTED;
        const int NH = a.HI <= 16 ? 16 : a.HI <= 32 ? 32 : 64;
        if (!make_tmap_2d(&qm, a.q_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.T * a.HI, a.DI, a.DI, NH,
                          swz))
            return DSA_ERR_INVALID_ARG;
        const int64_t tiles_bound = (int64_t)a.T * ((a.max_len + 127) / 128);
        const int64_t slots = (int64_t)dev->sm_count * DecCfg<128, 32>::CTAS_PER_SM;
        const int grid = (int)(tiles_bound < slots ? tiles_bound : slots);
        if (grid <= 0) return DSA_OK;
        if (a.DI == 128) {
            if (NH == 16) return run_decode<128, 16>(km, qm, p, grid, st);
            if (NH == 32) return run_decode<128, 32>(km, qm, p, grid, st);
            return run_decode<128, 64>(km, qm, p, grid, st);
        }
        if (NH == 16) return run_decode<64, 16>(km, qm, p, grid, st);
        if (NH == 32) return run_decode<64, 32>(km, qm, p, grid, st);
        return run_decode<64, 64>(km, qm, p, grid, st);
    }
    if (!make_tmap_2d(&qm, a.q_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.T * a.HI, a.DI, a.DI, 256, swz))
        return DSA_ERR_INVALID_ARG;
    const int G = 256 / a.HI;
    const int ngroups = (a.T + G - 1) / G;
    const int grid = ngroups < dev->sm_count ? ngroups : dev->sm_count;
#define DSA_PRE(DIV, HIV) \
    if (a.DI == DIV && a.HI == HIV) return run_prefill<DIV, HIV>(km, qm, p, grid, st);
    DSA_PRE(128, 4) DSA_PRE(128, 8) DSA_PRE(128, 16) DSA_PRE(128, 32) DSA_PRE(128, 64)
    DSA_PRE(64, 4) DSA_PRE(64, 8) DSA_PRE(64, 16) DSA_PRE(64, 32) DSA_PRE(64, 64)
#undef DSA_PRE
    return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
