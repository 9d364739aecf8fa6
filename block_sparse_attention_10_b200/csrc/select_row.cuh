// select_row.cuh — top-16 block selection of one (sequence, query token) row by one warp.
//
// "Main attention then runs exactly, but only over the top 16 blocks, and the most recent
// block is always kept" ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash",
// ainewsbites.com, "A model built for efficient inference").  Reading: the query's own
// block r plus the best min(15, r) other blocks under the total order (score desc,
// index asc), written ascending and padded with -1.
//
// Each candidate becomes a 64-bit key (order-preserving bits of the fp32 score, then the
// inverted block index), so "best" is a plain maximum and ties go to the lower index.
// Lane i holds candidates i, i + 32, ... in registers; every round takes, per lane, the
// largest key below the previous winner with a depth-log2(PER) tree, then the warp
// maximum with two 32-bit redux.sync.  Deterministic.  A key of 0 marks an empty slot
// (scores are never NaN, so every real key is non-zero).
#pragma once

#include "common.cuh"

namespace msa {

__device__ __forceinline__ uint64_t rank_key(float s, int64_t n) {
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)n);
}

__device__ __forceinline__ uint64_t max64(uint64_t a, uint64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint64_t warp_max64(uint64_t v) {
    const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32));
    const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(v >> 32) == hi ? (uint32_t)v : 0u);
    return ((uint64_t)hi << 32) | lo;
}

// Selection of row `s` (nvis visible blocks, forced block r = nvis - 1).  Rows longer than
// 32 * PER blocks are taken in chunks of that size, the best keys so far carried along.
// kCoherent: the scores were written by other warps of the same launch (read through L2).
// Returns, in lane i < 16, the i-th selected block id in ascending order (or -1).
template <int PER, bool kCoherent = false>
__device__ __forceinline__ int select_row_warp(const float* __restrict__ s, int64_t nvis, int64_t r, int lane) {
    const int want = (int)min64(kTopK - 1, nvis - 1);
    uint64_t best = 0ull;  // lane k < want: the k-th best key among the blocks seen so far
    for (int64_t base = 0; base < nvis; base += 32 * PER) {
        uint64_t k0[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int64_t n = base + (int64_t)j * 32 + lane;
            k0[j] = (n < nvis && n != r) ? rank_key(kCoherent ? __ldcg(s + n) : __ldg(s + n), n) : 0ull;
        }
        const uint64_t carry = best;
        uint64_t prev = ~0ull;
        for (int k = 0; k < want; ++k) {
            uint64_t cand[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j) cand[j] = k0[j] < prev ? k0[j] : 0ull;
#pragma unroll
            for (int w = PER / 2; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) cand[j] = max64(cand[j], cand[j + w]);
            prev = warp_max64(max64(cand[0], carry < prev ? carry : 0ull));
            if (lane == k) best = prev;
        }
    }
    int mine = lane < want ? (int)(0xFFFFFFFFu - (uint32_t)best) : -1;  // lane k < want holds the k-th best
    if (lane == want) mine = (int)r;
    const int nsel = want + 1;
    int rank = 0;
    for (int i = 0; i < nsel; ++i) rank += (__shfl_sync(0xffffffffu, mine, i) < mine) ? 1 : 0;
    // scatter to ascending order: lane `rank` receives the id
    int out = -1;
#pragma unroll
    for (int i = 0; i < kTopK; ++i) {
        const int id = __shfl_sync(0xffffffffu, mine, i);
        const int rk = __shfl_sync(0xffffffffu, rank, i);
        if (i < nsel && rk == lane) out = id;
    }
    return out;
}

}  // namespace msa
