// Stage 1 of the Gated DSA layer with MXFP8 indexer operands: the same score
//
//   I[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])
//
// ("Open-Source LLM Architecture Evolution", Architecture Breakdown §2,
// "Indexer"), where qI and kI are MXFP8 ("Open-Weight Deployment of an
// Ultra-Large Sparse Model", §1 and §3: activations in MXFP8; read as the
// OCP microscaling format): E4M3 elements, one E8M0 scale 2^(c-127) per 32
// consecutive elements along DI.  The decode indexer's design (keys on the
// M side of the MMA, queries' heads on N, persistent grid, ReLU-w epilogue
// and score histogram) with block-scaled tensor-core MMAs
// (tcgen05.mma kind::mxf8f6f4.block_scale, four K=32 steps per 128-key tile,
// each selecting its scale byte): the producer warp's lanes bring each
// tile's 128 x 4 key scales and each query's heads x 4 scales into shared
// memory by 4-byte cp.async, in the 128-row atom the MMA reads (row r =
// r0 + 32 r1 at byte 16 r0 + 4 r1), and the MMA warp moves them to tensor
// memory with tcgen05.cp before the tile's MMAs.  DI = 128, HI in {16, 32}.
#include "indexer_common.cuh"

namespace dsa {
namespace {

__device__ __forceinline__ void cp_async_4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t d) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}
__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t sfa, uint32_t sfb,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::
            "r"(d), "l"(a), "l"(b), "r"(id), "r"(sfa), "r"(sfb), "r"(acc)
        : "memory");
}
__host__ __device__ constexpr uint32_t idesc_mx(uint32_t a_sf_id, uint32_t b_sf_id, uint32_t n, uint32_t m) {
    return (b_sf_id << 4) | ((n >> 3) << 17) | (1u << 23) | ((m >> 4) << 24) | (a_sf_id << 29);
}

template <int DI, int NH>
struct MxCfg {
    static constexpr int CTAS_PER_SM = 2;
    static constexpr int STAGES = DI == 128 ? 5 : 10;  // key tiles in flight per CTA
    static constexpr int EPI_GROUPS = 2;  // epilogue warpgroups, alternate tiles
    static constexpr int ACC = NH <= 16 ? 8 : 7;  // TMEM: ACC * NH + 16 scale columns <= 256 per CTA
    static constexpr int SF_BYTES = 512;          // one 128-row x 4-block E8M0 scale atom
    static constexpr int THREADS = 64 + 128 * EPI_GROUPS;
    static constexpr int A_BYTES = 128 * DI;      // one key tile (two pages)
    static constexpr int B_BYTES = NH * DI;       // one query's heads
    static constexpr int TMEM_COLS = 256;
    static constexpr int SFA_COL = (ACC * NH + 7) / 8 * 8;  // keys' scales (one slot, refilled per tile)
    static constexpr int SFB_COL = SFA_COL + 8;             // queries' scales, two slots of 4 columns
    static_assert(DI == 128 && SFB_COL + 8 <= TMEM_COLS, "scale columns");
    static constexpr uint32_t SWZ = DI == 128 ? SWZ_128B : SWZ_64B;
    static constexpr uint32_t SBO = 8 * DI;
    static constexpr int MAXT = 1024;
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * ACC + 4 + 1);
    static constexpr int HIST_WORDS = SCORE_HIST_BINS / 2;  // per epilogue warpgroup: packed 16-bit counts
    static constexpr int HIST_FLUSH_TILES = 256;            // a count stays below 2^16
    static constexpr int SMEM =
        1024 + STAGES * A_BYTES + 2 * B_BYTES + (STAGES + 2) * SF_BYTES + BAR_BYTES + 4 * (MAXT + 1) + 16 + 4 * EPI_GROUPS * HIST_WORDS;
    static_assert(HIST_FLUSH_TILES * 128 < 65536, "packed counts do not carry");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tile alignment");
};

template <int DI, int NH>
__global__ void __launch_bounds__(MxCfg<DI, NH>::THREADS, MxCfg<DI, NH>::CTAS_PER_SM)
    indexer_mx_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                          const IdxParams p, const uint8_t *q_scales, const uint8_t *k_scales) {
    using C = MxCfg<DI, NH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                                  // [STAGES][A_BYTES]
    uint8_t *qbuf = smem + C::STAGES * C::A_BYTES;            // [2][B_BYTES]
    uint8_t *sfa = qbuf + 2 * C::B_BYTES;                     // [STAGES][SF_BYTES]
    uint8_t *sfb = sfa + C::STAGES * C::SF_BYTES;             // [2][SF_BYTES]
    uint64_t *full = reinterpret_cast<uint64_t *>(sfb + 2 * C::SF_BYTES);
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
            mbar_init(&full[s], 33);  // lane 0's copy or arrival + 32 lanes' scale copies
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 33);
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
                const bool newq = t != tprev;
                if (newq) {
                    tprev = t;
                    ++qo;
                }
                if (lane == 0) {
                    const int i = base + k;
                    if (newq) {  // a new query: its heads go to the next q buffer
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
                // every lane: the scales, 4 bytes per row, into the 128-row x 4-block atom
                // (row r = r0 + 32 * r1 at byte r0 * 16 + r1 * 4); the buffers were freed by lane 0's waits
                const int s = (base + k) % C::STAGES;
                if (newq) {
                    const int qb = qo & 1;
                    if (lane < NH) cp_async_4(sfb + qb * C::SF_BYTES + lane * 16, q_scales + ((int64_t)t * NH + lane) * 4);
                    cp_async_arrive_noinc(&qfull[qb]);
                }
#pragma unroll
                for (int r1 = 0; r1 < 4; ++r1) {
                    const int pg = r1 < 2 ? pg0 : pg1;
                    if (pg >= 0)
                        cp_async_4(sfa + s * C::SF_BYTES + lane * 16 + r1 * 4,
                                   k_scales + ((int64_t)pg * 64 + lane + 32 * (r1 & 1)) * 4);
                }
                cp_async_arrive_noinc(&full[s]);
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
        int t = locate(tstart, T, lo);
        int j = static_cast<int>(lo - tstart[t]);
        int qo = -1, tprev = -1;
        for (int i = 0; i < n; ++i) {
            if (t != tprev) {  // the query changes: release the old heads, wait for the new
                if (qo >= 0) mma_commit(&qempty[qo & 1]);
                tprev = t;
                ++qo;
                if (!mbar_wait(&qfull[qo & 1], (qo >> 1) & 1, p.err, abort_flag)) break;
                fence_proxy_async_smem();  // the scales came by cp.async: make them visible to tcgen05.cp
                tmem_cp_32x128b_x4(tmem + C::SFB_COL + 4 * (qo & 1),
                                   sdesc(smem_u32(sfb + (qo & 1) * C::SF_BYTES), 0, 128, SWZ_NONE));
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
            fence_proxy_async_smem();
            tmem_cp_32x128b_x4(tmem + C::SFA_COL, sdesc(smem_u32(sfa + s * C::SF_BYTES), 0, 128, SWZ_NONE));
            const uint32_t sfb_col = tmem + C::SFB_COL + 4 * (qo & 1);
#pragma unroll
            for (int k = 0; k < DI / 32; ++k)
                mma_mx(d, sdesc(A + 32 * k, 16, C::SBO, C::SWZ), sdesc(B + 32 * k, 16, C::SBO, C::SWZ),
                       idesc_mx(k, k, NH, 128), (tmem + C::SFA_COL) | (uint32_t(k) << 30),
                       sfb_col | (uint32_t(k) << 30), k > 0);
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


template <int NH>
dsa_status run_mx_decode(const CUtensorMap &km, const CUtensorMap &qm, const IdxParams &p, const uint8_t *qs,
                         const uint8_t *ks, int grid, cudaStream_t st) {
    using C = MxCfg<128, NH>;
    auto fn = indexer_mx_decode_kernel<128, NH>;
    if (!ensure_smem(reinterpret_cast<const void *>(fn), C::SMEM)) return DSA_ERR_CUDA;
    fn<<<grid, C::THREADS, C::SMEM, st>>>(km, qm, p, qs, ks);
    return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

dsa_status launch_indexer_mx(const IndexerArgs &a, const uint8_t *q_scales, const uint8_t *k_scales,
                             cudaStream_t st) {
    const DeviceInfo *dev = current_device();
    if (!dev) return DSA_ERR_CUDA;
    if (a.T == 0) return DSA_OK;
    if (a.DI != 128 || (a.HI != 16 && a.HI != 32) || a.T > MxCfg<128, 32>::MAXT) return DSA_ERR_UNSUPPORTED;
    IdxParams p{a.w, a.q_seq, a.q_pos, a.pg, a.T, a.HI, a.max_len, a.scores, a.ld, dev->err,
                (a.q_seq == nullptr || a.T <= 64) ? a.hist : nullptr, a.zero, a.nzero};
    CUtensorMap km, qm;
    if (!make_tmap_2d(&km, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.pg.num_pages * 64, a.DI,
                      a.DI, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&qm, a.q_idx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.DI, (uint64_t)a.T * a.HI, a.DI, a.DI, a.HI,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return DSA_ERR_INVALID_ARG;
    const int64_t tiles_bound = (int64_t)a.T * ((a.max_len + 127) / 128);
    const int64_t slots = (int64_t)dev->sm_count * MxCfg<128, 32>::CTAS_PER_SM;
    const int grid = (int)(tiles_bound < slots ? tiles_bound : slots);
    if (grid <= 0) return DSA_OK;
    return a.HI == 32 ? run_mx_decode<32>(km, qm, p, q_scales, k_scales, grid, st)
                      : run_mx_decode<16>(km, qm, p, q_scales, k_scales, grid, st);
}

}  // namespace dsa
