// Stage 1 of the Gated DSA layer for a few explicit queries (several draft
// tokens per sequence, as in speculative decoding): the indexer score
//
//   I[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])     for s <= q_pos[t]
//
// ("Open-Source LLM Architecture Evolution: How Lightweight Sparse Attention
// Reshapes Long-Context Modeling Efficiency", Architecture Breakdown §2,
// "Indexer"), with up to four consecutive queries of one sequence in one
// tcgen05 e4m3 MMA (N = queries x heads), so that sequence's keys cross HBM
// once rather than once per query.  Warp 0 issues TMA, warp 1 the MMAs,
// four epilogue warpgroups take alternate tiles; each query's scores are
// also counted into its score histogram for the top-K that follows.
#include "indexer_common.cuh"

namespace dsa {
namespace {

// ============================================================================
// few explicit queries, grouped: up to GQ consecutive queries of one sequence
// (several draft tokens per sequence, as in speculative decoding) share every
// key tile -- one MMA of N = GQ x heads per tile and one key stream per group
// instead of one per query
// ============================================================================

template <int NH>
struct GrpCfg {
    static constexpr int DI = 128;
    static constexpr int GQ = 4;          // queries per group
    static constexpr int N = GQ * NH;     // MMA columns: the group's queries x heads
    static constexpr int STAGES = 7;      // key tiles in flight (one CTA per SM)
    static constexpr int EPI_GROUPS = 4;  // epilogue warpgroups, alternate tiles
    static constexpr int ACC = 512 / N;   // tiles in TMEM
    static constexpr int THREADS = 64 + 128 * EPI_GROUPS;
    static constexpr int A_BYTES = 128 * DI;
    static constexpr int B_BYTES = N * DI;
    static constexpr int TMEM_COLS = 512;
    static constexpr int MAXQ = 64;
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * ACC + 4 + 1);
    static constexpr int HIST_WORDS = SCORE_HIST_BINS / 2;  // packed 16-bit counts per query
    static constexpr int HIST_FLUSH_TILES = 256;
    // tables: gstart [MAXQ+1], gfirst/gsize/gseq/glast [MAXQ], qlast [MAXQ], weights [MAXQ*NH]
    // byte offsets from the 1024-aligned base; the weights are read as float4
    static constexpr int OFF_BAR = STAGES * A_BYTES + 2 * B_BYTES;
    static constexpr int OFF_TBL = OFF_BAR + BAR_BYTES;
    static constexpr int OFF_W = (OFF_TBL + 4 * (MAXQ + 1) + 4 * 5 * MAXQ + 15) / 16 * 16;
    static constexpr int OFF_MISC = OFF_W + 4 * MAXQ * NH;
    static constexpr int SMEM = 1024 + OFF_MISC + 16 + 4 * EPI_GROUPS * GQ * HIST_WORDS;
    static_assert(OFF_W % 16 == 0 && OFF_MISC % 16 == 0, "float4 weight rows");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tile alignment");
    static_assert(N <= 256 && ACC * N <= 512, "TMEM");
};

template <int NH>
__global__ void __launch_bounds__(GrpCfg<NH>::THREADS, 1)
    indexer_group_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                         const IdxParams p) {
    using C = GrpCfg<NH>;
    constexpr int DI = C::DI, GQ = C::GQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                            // [STAGES][A_BYTES]
    uint8_t *qbuf = smem + C::STAGES * C::A_BYTES;     // [2][B_BYTES]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + C::ACC;
    uint64_t *qfull = tempty + C::ACC;  // [2]
    uint64_t *qempty = qfull + 2;       // [2]
    uint64_t *drain = qempty + 2;
    int32_t *gstart = reinterpret_cast<int32_t *>(smem + C::OFF_TBL);  // [NG + 1] first tile of each group
    int32_t *gfirst = gstart + C::MAXQ + 1;  // [NG] first query of the group
    int32_t *gsize = gfirst + C::MAXQ;       // [NG] queries in it
    int32_t *gseq = gsize + C::MAXQ;         // [NG] its sequence
    int32_t *glast = gseq + C::MAXQ;         // [NG] its largest position scored
    int32_t *qlast = glast + C::MAXQ;        // [T] each query's last position (-1: none)
    float *wsm = reinterpret_cast<float *>(smem + C::OFF_W);  // [T][NH] the queries' weights (0 past HI)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *ngroups = reinterpret_cast<int *>(tmem_slot + 2);
    uint32_t *hist_sm = tmem_slot + 4;  // [EPI_GROUPS][GQ][HIST_WORDS]

    const int warp = warp_id(), lane = lane_id();
    const int T = p.T;
    if (p.hist)
        for (int i = threadIdx.x; i < C::EPI_GROUPS * GQ * C::HIST_WORDS; i += blockDim.x) hist_sm[i] = 0;
    for (int i = threadIdx.x; i < T * NH; i += blockDim.x)
        wsm[i] = (i % NH) < p.HI ? p.w[(int64_t)(i / NH) * p.HI + (i % NH)] : 0.f;
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
    if (warp == 0) {
        // each query's (sequence, last position); groups = runs of consecutive
        // queries of one sequence, at most GQ long; a group's tiles cover its
        // largest position
        int qbv[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int t = lane + 32 * h;
            qbv[h] = -1;
            if (t < T) {
                const QInfo qi = query_info(t, p.q_seq, p.q_pos, p.pg, p.max_len, nullptr);
                qlast[t] = qi.last;
                qbv[h] = qi.last >= 0 ? qi.b : -1 - t;  // a query with nothing to score forms its own group
            }
            if (t < T) gseq[t] = qbv[h];  // (scratch: the sequence of query t, read by lane 0 below)
        }
        __syncwarp();
        if (lane == 0) {
            int ng = 0, run = 0;
            for (int t = 0; t < T; ++t) {
                const int b = gseq[t];  // query t's sequence (the groups' own entries are written behind t)
                if (t == 0 || b != gseq[ng - 1] || run == GQ) {
                    gfirst[ng] = t;
                    gsize[ng] = 0;
                    glast[ng] = -1;
                    ++ng;
                    run = 0;
                }
                gseq[ng - 1] = b;
                ++gsize[ng - 1];
                glast[ng - 1] = max(glast[ng - 1], qlast[t]);
                ++run;
            }
            *ngroups = ng;
            gstart[0] = 0;
            for (int g = 0; g < ng; ++g) gstart[g + 1] = gstart[g] + ((glast[g] + 1 + 127) >> 7);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();
    const uint32_t tmem = *tmem_slot;
    const int NG = *ngroups;
    const int64_t total = gstart[NG];
    const int64_t lo = total * blockIdx.x / gridDim.x;
    const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
    const int n = static_cast<int>(hi - lo);

    if (warp == 0 && n > 0) {
        // ---------------- producer: 32 tiles' pages looked up a window ahead ----------------
        auto lookup = [&](int i, int &tg, int &p0, int &p1) {
            tg = -1, p0 = -1, p1 = -1;
            if (i < n) {
                const int64_t g = lo + i;
                tg = locate(gstart, NG, g);
                const int j = static_cast<int>(g - gstart[tg]);
                p0 = page_of(p.pg, gseq[tg], 2 * j, p.err);
                p1 = (2 * j + 1) * 64 <= glast[tg] ? page_of(p.pg, gseq[tg], 2 * j + 1, p.err) : -1;
            }
        };
        int tg, p0, p1;
        lookup(lane, tg, p0, p1);
        const uint64_t kpol = l2_policy_evict_first();
        int issued = 0, qo = -1, gprev = -1;
        bool ok = true;
        for (int base = 0; ok && base < n; base += 32) {
            int tg_n, p0_n, p1_n;
            lookup(base + 32 + lane, tg_n, p0_n, p1_n);
            const int cnt = min(32, n - base);
            for (int k = 0; k < cnt; ++k) {
                const int grp = __shfl_sync(0xffffffffu, tg, k);
                const int pg0 = __shfl_sync(0xffffffffu, p0, k);
                const int pg1 = __shfl_sync(0xffffffffu, p1, k);
                if (lane == 0) {
                    const int i = base + k;
                    if (grp != gprev) {  // a new group: its queries' heads go to the next q buffer
                        gprev = grp;
                        ++qo;
                        const int qb = qo & 1;
                        if (mbar_wait(&qempty[qb], ((qo >> 1) & 1) ^ 1, p.err, abort_flag)) {
                            mbar_expect_tx(&qfull[qb], C::B_BYTES);
                            tma_load_2d(qbuf + qb * C::B_BYTES, &qmap, &qfull[qb], 0, gfirst[grp] * p.HI);
                        } else {
                            ok = false;
                        }
                    }
                    const int s = i % C::STAGES;
                    if (ok && mbar_wait(&empty[s], ((i / C::STAGES) & 1) ^ 1, p.err, abort_flag)) {
                        uint8_t *A = stages + s * C::A_BYTES;
                        const uint32_t bytes = (pg0 >= 0 ? 64 * DI : 0) + (pg1 >= 0 ? 64 * DI : 0);
                        if (bytes) {
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
            tg = tg_n, p0 = p0_n, p1 = p1_n;
        }
        if (lane == 0) {  // never leave a copy in flight behind
            for (int i = issued - 1; i >= 0 && i >= issued - C::STAGES; --i)
                mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1, p.err, nullptr);
            if (qo >= 0) mbar_wait(&qfull[qo & 1], (qo >> 1) & 1, p.err, nullptr);
        }
    } else if (warp == 1 && lane == 0 && n > 0) {
        // ---------------- MMA issuer: keys x (group queries x heads) ----------------
        constexpr uint32_t ID = idesc(0, 0, 0, 0, C::N, 128);
        int grp = locate(gstart, NG, lo);
        int j = static_cast<int>(lo - gstart[grp]);
        int qo = -1, gprev = -1;
        for (int i = 0; i < n; ++i) {
            if (grp != gprev) {
                if (qo >= 0) mma_commit(&qempty[qo & 1]);
                gprev = grp;
                ++qo;
                if (!mbar_wait(&qfull[qo & 1], (qo >> 1) & 1, p.err, abort_flag)) break;
            }
            const int s = i % C::STAGES;
            const int a = i % C::ACC;
            if (!mbar_wait(&full[s], (i / C::STAGES) & 1, p.err, abort_flag)) break;
            if (!mbar_wait(&tempty[a], ((i / C::ACC) & 1) ^ 1, p.err, abort_flag)) break;
            tc_fence_after();
            const uint32_t A = smem_u32(stages + s * C::A_BYTES);
            const uint32_t B = smem_u32(qbuf + (qo & 1) * C::B_BYTES);
#pragma unroll
            for (int k = 0; k < DI / 32; ++k)
                mma_e4m3(tmem + a * C::N, sdesc(A + 32 * k, 16, 8 * DI, SWZ_128B), sdesc(B + 32 * k, 16, 8 * DI, SWZ_128B),
                         ID, k > 0);
            mma_commit(&empty[s]);
            mma_commit(&tfull[a]);
            if (++j == gstart[grp + 1] - gstart[grp]) {
                j = 0;
                do { ++grp; } while (grp < NG && gstart[grp + 1] == gstart[grp]);
            }
        }
        mma_commit(drain);
        mbar_wait(drain, 0, p.err, nullptr);
    } else if (warp >= 2 && n > 0) {
        // ---------------- epilogue: warpgroup eg takes tiles i with i % EPI_GROUPS == eg ----------------
        // For each query u of the tile's group: ReLU and the w-weighted sum
        // over its NH accumulator columns, the score stored and counted.
        const int eg = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        int grp = locate(gstart, NG, lo);
        int j = static_cast<int>(lo - gstart[grp]);
        bool alive = true;
        uint32_t *hw = hist_sm + eg * GQ * C::HIST_WORDS;  // [GQ][HIST_WORDS] of group hg
        int hg = -1, htiles = 0;
        auto hflush = [&]() {
            named_bar_sync(1 + eg, 128);  // every add of the warpgroup has landed
            if (hg >= 0 && alive)
                for (int u = 0; u < gsize[hg]; ++u)
                    for (int wi = row; wi < C::HIST_WORDS; wi += 128) {
                        const uint32_t v = hw[u * C::HIST_WORDS + wi];
                        if (v) {
                            uint32_t *g = p.hist + (int64_t)(gfirst[hg] + u) * SCORE_HIST_BINS + 2 * wi;
                            if (v & 0xFFFFu) red_add_global(g, v & 0xFFFFu);
                            if (v >> 16) red_add_global(g + 1, v >> 16);
                            hw[u * C::HIST_WORDS + wi] = 0;
                        }
                    }
            htiles = 0;
            named_bar_sync(1 + eg, 128);  // cleared before the next adds
        };
        for (int i = 0; i < n; ++i) {
            if (i % C::EPI_GROUPS == eg) {
                if (p.hist && (grp != hg || htiles == C::HIST_FLUSH_TILES)) {
                    hflush();
                    hg = grp;
                }
                ++htiles;
                const int a = i % C::ACC;
                if (alive && !mbar_wait(&tfull[a], (i / C::ACC) & 1, p.err, abort_flag)) alive = false;
                if (alive) {
                    tc_fence_after();
                    const int q0 = gfirst[grp], gs = gsize[grp];
                    const int spos = j * 128 + row;
                    float sc[GQ];
#pragma unroll
                    for (int u = 0; u < GQ; ++u) {
                        uint32_t r[NH];
                        const uint32_t ta = tmem + a * C::N + u * NH + lane_off;
                        if constexpr (NH == 16) {
                            tmem_ld16(ta, r);
                        } else {
#pragma unroll
                            for (int c = 0; c < NH / 32; ++c) tmem_ld32(ta + 32 * c, r + 32 * c);
                        }
                        tmem_wait_ld();
                        float acc = 0.f;
                        const float *wq = wsm + (q0 + min(u, gs - 1)) * NH;
#pragma unroll
                        for (int h = 0; h < NH; h += 4) {
                            const float4 w4 = *reinterpret_cast<const float4 *>(wq + h);
                            acc = fmaf(w4.x, fmaxf(__uint_as_float(r[h]), 0.f), acc);
                            acc = fmaf(w4.y, fmaxf(__uint_as_float(r[h + 1]), 0.f), acc);
                            acc = fmaf(w4.z, fmaxf(__uint_as_float(r[h + 2]), 0.f), acc);
                            acc = fmaf(w4.w, fmaxf(__uint_as_float(r[h + 3]), 0.f), acc);
                        }
                        sc[u] = acc;
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
                    for (int u = 0; u < GQ; ++u) {
                        if (u < gs && spos <= qlast[q0 + u]) {
                            p.scores[(int64_t)(q0 + u) * p.ld + spos] = sc[u];
                            if (p.hist) {
                                const uint32_t bin = score_key(sc[u]) >> SCORE_HIST_SHIFT;
                                atomicAdd(&hw[u * C::HIST_WORDS + (bin >> 1)], 1u << ((bin & 1u) << 4));
                            }
                        }
                    }
                }
            }
            if (++j == gstart[grp + 1] - gstart[grp]) {
                j = 0;
                do { ++grp; } while (grp < NG && gstart[grp + 1] == gstart[grp]);
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

template <int NH>
dsa_status run_group(const CUtensorMap &km, const CUtensorMap &qm, const IdxParams &p, int grid, cudaStream_t st) {
    using C = GrpCfg<NH>;
    auto fn = indexer_group_kernel<NH>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    fn<<<grid, C::THREADS, C::SMEM, st>>>(km, qm, p);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

bool indexer_group_eligible(const IndexerArgs &a) {
    return a.q_seq != nullptr && a.T > 0 && a.T <= GrpCfg<32>::MAXQ && a.DI == 128 && (a.HI == 16 || a.HI == 32);
}

dsa_status launch_indexer_group(const IndexerArgs &a, cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (!indexer_group_eligible(a)) return DSA_ERR_UNSUPPORTED;
    IdxParams p{a.w, a.q_seq, a.q_pos, a.pg, a.T, a.HI, a.max_len, a.scores, a.ld, dev->err, a.hist, a.zero, a.nzero};
    CUtensorMap km, qm;
    if (!make_tmap_2d(&km, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.pg.num_pages * 64, a.DI,
                      a.DI, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return DSA_ERR_INVALID_ARG;
    const int NH = a.HI;
    if (!make_tmap_2d(&qm, a.q_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.T * a.HI, a.DI, a.DI,
                      GrpCfg<32>::GQ * NH, CU_TENSOR_MAP_SWIZZLE_128B))
        return DSA_ERR_INVALID_ARG;
    const int64_t tiles_bound = (int64_t)a.T * ((a.max_len + 127) / 128);
    const int grid = (int)(tiles_bound < dev->sm_count ? tiles_bound : dev->sm_count);
    if (grid <= 0) return DSA_OK;
    return NH == 32 ? run_group<32>(km, qm, p, grid, st) : run_group<16>(km, qm, p, grid, st);
}

}  // namespace dsa
