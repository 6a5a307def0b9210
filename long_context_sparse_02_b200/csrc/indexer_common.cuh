// Shared by the indexer kernels: where a query's scores end (its sequence
// and last position), the block-table lookup, the kernels' parameters and
// the tile-to-query search.
#pragma once
#include "dsa_device.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

struct QInfo {
    int32_t b;     // sequence
    int32_t last;  // last history position scored (inclusive); -1 = none
};

__device__ __forceinline__ QInfo query_info(int t, const int32_t *q_seq, const int32_t *q_pos, const PagedDev &pg,
                                            int max_len, uint32_t *err) {
    int b, last;
    if (q_seq == nullptr) {
        b = t;
        if (b >= pg.num_seqs) {
            record_error(err, DSA_DEVERR_POSITION);
            return {0, -1};
        }
        last = pg.seq_lens[b] - 1;
    } else {
        b = q_seq[t];
        last = q_pos[t];
        if (b < 0 || b >= pg.num_seqs || last < 0) {
            record_error(err, DSA_DEVERR_POSITION);
            return {0, -1};
        }
    }
    const int L = pg.seq_lens[b];
    if (last >= L) {
        record_error(err, DSA_DEVERR_POSITION);
        last = L - 1;
    }
    if (last >= max_len) {
        record_error(err, DSA_DEVERR_SHAPE);
        last = max_len - 1;
    }
    return {b, last};
}

// Physical page of logical page lp of sequence b, or -1 (recorded) if the
// table entry is out of range.
__device__ __forceinline__ int page_of(const PagedDev &pg, int b, int lp, uint32_t *err) {
    if (lp >= pg.max_blocks) {
        record_error(err, DSA_DEVERR_PAGE);
        return -1;
    }
    const int p = pg.block_table[(int64_t)b * pg.max_blocks + lp];
    if (p < 0 || p >= pg.num_pages) {
        record_error(err, DSA_DEVERR_PAGE);
        return -1;
    }
    return p;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

constexpr int pow2_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

struct IdxParams {
    const float *w;
    const int32_t *q_seq, *q_pos;
    PagedDev pg;
    int32_t T, HI, max_len;
    float *scores;
    int64_t ld;
    uint32_t *err;
    uint32_t *hist;  // [T][SCORE_HIST_BINS] or NULL (few-query kernels only)
    uint32_t *zero;  // nzero words the grid sets to zero (or NULL)
    int64_t nzero;
    // testing the bounded waits (decode kernel): flattened tile
    // test_skip_tile_plus1 - 1 (queries' 128-key tiles in order) is never
    // filled; 0 = off
    int64_t test_skip_tile_plus1;
};

// The grid clears the words the next kernel expects at zero, each CTA a share.
__device__ __forceinline__ void clear_words(const IdxParams &p) {
    if (p.zero)
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.nzero; i += (int64_t)gridDim.x * blockDim.x)
            p.zero[i] = 0;
}

// Index t with tstart[t] <= g < tstart[t+1] (tstart non-decreasing, g < tstart[T]).
__device__ __forceinline__ int locate(const int32_t *tstart, int T, int64_t g) {
    int lo = 0, hi = T;  // answer in [lo, hi)
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (tstart[mid] <= g) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace
}  // namespace dsa
