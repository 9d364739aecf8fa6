// select_row.cuh — top-16 block selection of one (sequence, query token) row by one warp.
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com, section
// "A model built for efficient inference"): exact attention is restricted to 16 blocks
// per query, and the block holding the query itself is never dropped.  Reading: the
// query's own block r plus the best min(15, r) other blocks under the total order
// (score desc, index asc), written ascending and padded with -1.  r = nvis - 1 is the last visible
// block, so it always comes last in the ascending list.
//
// Threshold selection (select_row_warp): every candidate becomes a 32-bit key whose
// unsigned order is the order of the fp32 scores (-0 ranks below +0; 0 marks an empty
// slot: scores are never NaN).  Lane i holds candidates i, i + 32, ... in registers.
// Rounds of "largest key below the previous one, and how many candidates hold it"
// (two redux.sync each) find T, the want-th best key counted with multiplicity; then
// one ballot pass in ascending block order writes every block with key > T and, of
// the blocks with key == T, the lowest-indexed ones still needed — the index tie-break.
// Rows longer than 32 * PER blocks take select_row_warp_long: 64-bit keys (score key,
// inverted index) and 15 rounds of "largest key below the previous winner" per chunk
// of 32 * PER blocks, the best keys so far carried along.  Both are deterministic.
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

// Unsigned key with the order of the fp32 score.
__device__ __forceinline__ uint32_t score_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// T = the want-th largest of the warp's non-zero keys counted with multiplicity, and
// n_gt = how many keys exceed it.  Needs 1 <= want <= the number of non-zero keys.
// Each round's multiplicity count and the next round's maximum are independent, so both
// reductions are in flight together (the last round computes one maximum it does not use).
template <int PER>
__device__ __forceinline__ uint32_t warp_kth_key(const uint32_t (&k)[PER], int want, int& n_gt) {
    auto max_below = [&](uint32_t prev) -> uint32_t {
        uint32_t m[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) m[j] = k[j] < prev ? k[j] : 0u;
#pragma unroll
        for (int w = PER / 2; w >= 1; w >>= 1)
#pragma unroll
            for (int j = 0; j < w; ++j) m[j] = max(m[j], m[j + w]);
        return __reduce_max_sync(0xffffffffu, m[0]);
    };
    auto count_eq = [&](uint32_t v) -> int {
        int c = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) c += k[j] == v ? 1 : 0;
        return (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
    };
    int taken = 0;
    uint32_t v = max_below(0xFFFFFFFFu);  // above every finite score's key
    for (;;) {
        const int c = count_eq(v);
        const uint32_t next = max_below(v);
        if (taken + c >= want) {
            n_gt = taken;
            return v;
        }
        taken += c;
        v = next;
    }
}

// Calls put(slot, j) for the lane holding candidate j of the selected ones, slots
// ascending in candidate order (j-th register of lane l is candidate 32 j + l): every key
// above T, and the first need_eq keys equal to T.
template <int PER, class Put>
__device__ __forceinline__ void warp_compact(const uint32_t (&k)[PER], uint32_t T, int need_eq, int lane, Put&& put) {
    const uint32_t below = (1u << lane) - 1u;
    int base = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const uint32_t gt = __ballot_sync(0xffffffffu, k[j] > T);
        uint32_t eq = __ballot_sync(0xffffffffu, k[j] == T);
        uint32_t keep = 0u;
        while (need_eq > 0 && eq != 0u) {  // warp-uniform
            const uint32_t low = eq & (0u - eq);
            keep |= low;
            eq ^= low;
            --need_eq;
        }
        const uint32_t sel = gt | keep;
        if ((sel >> lane) & 1u) put(base + __popc(sel & below), j);
        base += __popc(sel);
    }
}

// Selection of row `s` (nvis <= 32 * PER visible blocks, forced block r = nvis - 1),
// written to out[0..15] (shared or global memory) by the warp.  kCoherent: the scores
// were written by other warps of the same launch (read through L2).
template <int PER, bool kCoherent = false>
__device__ __forceinline__ void select_row_warp(const float* __restrict__ s, int64_t nvis, int64_t r, int lane,
                                                int32_t* out) {
    const int want = (int)min64(kTopK - 1, nvis - 1);
    if (want > 0) {
        uint32_t k[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int64_t n = (int64_t)j * 32 + lane;
            k[j] = (n < nvis && n != r) ? score_key(kCoherent ? __ldcg(s + n) : __ldg(s + n)) : 0u;
        }
        int n_gt;
        const uint32_t T = warp_kth_key(k, want, n_gt);
        warp_compact(k, T, want - n_gt, lane, [&](int slot, int j) { out[slot] = j * 32 + lane; });
    }
    if (lane == want) out[want] = (int32_t)r;
    if (lane > want && lane < kTopK) out[lane] = -1;
}

// Rows of <= WARPS * 32 * PER blocks, selected by the WARPS warps of a CTA: warp w keeps the
// best 15 of blocks [32 PER w, 32 PER (w + 1)) in shared memory (ckey/cid, WARPS * 15
// entries each), in ascending block order; then warp 0 selects the row's best 15 from those
// candidates (they contain it), which sit in ascending block order, so the index tie-break
// carries over, and writes out[0..15].  Every thread of the CTA calls it (one barrier).
template <int WARPS, int PER, bool kCoherent = false>
__device__ __forceinline__ void select_row_cta(const float* __restrict__ s, int64_t nvis, int64_t r, int warp,
                                               int lane, uint32_t* ckey, int32_t* cid, int32_t* out) {
    constexpr int kCand = kTopK - 1;
    const int base = warp * 32 * PER;
    uint32_t k[PER];
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int64_t n = base + j * 32 + lane;
        k[j] = (n < nvis && n != r) ? score_key(kCoherent ? __ldcg(s + n) : __ldg(s + n)) : 0u;
        cnt += k[j] != 0u ? 1 : 0;
    }
    cnt = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
    const int want_w = min(kCand, cnt);
    if (want_w > 0) {
        int n_gt;
        const uint32_t T = warp_kth_key(k, want_w, n_gt);
        warp_compact(k, T, want_w - n_gt, lane, [&](int slot, int j) {
            ckey[warp * kCand + slot] = k[j];
            cid[warp * kCand + slot] = base + j * 32 + lane;
        });
    }
    if (lane >= want_w && lane < kCand) ckey[warp * kCand + lane] = 0u;
    __syncthreads();
    if (warp != 0) return;
    constexpr int kC = WARPS * kCand;
    constexpr int kPer2 = (kC + 31) / 32;
    const int want = (int)min64(kCand, nvis - 1);
    if (want > 0) {
        uint32_t kk[kPer2];
#pragma unroll
        for (int j = 0; j < kPer2; ++j) {
            const int cc = j * 32 + lane;
            kk[j] = cc < kC ? ckey[cc] : 0u;
        }
        int n_gt;
        const uint32_t T = warp_kth_key(kk, want, n_gt);
        warp_compact(kk, T, want - n_gt, lane, [&](int slot, int j) { out[slot] = cid[j * 32 + lane]; });
    }
    if (lane == want) out[want] = (int32_t)r;
    if (lane > want && lane < kTopK) out[lane] = -1;
}

// Any row length: chunks of 32 * PER blocks, the best keys so far carried along.  Returns,
// in lane i < 16, the i-th selected block id in ascending order (or -1).
template <int PER, bool kCoherent = false>
__device__ __forceinline__ int select_row_warp_long(const float* __restrict__ s, int64_t nvis, int64_t r, int lane) {
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
