// select.cu — top-16 block selection with the most recent block forced.
//
// "Main attention then runs exactly, but only over the top 16 blocks, and the
// most recent block is always kept" ("vLLM Adds Day-0 Support for
// MiniMax-M3.1-Flash", ainewsbites.com, "A model built for efficient
// inference").  Reading: the query's own block r = pos div 128 plus the best
// min(15, r) other blocks under the total order (score desc, index asc); the
// list is written ascending and padded with -1.
//
// One warp per (sequence, query token).  Each candidate becomes a 64-bit key
// (order-preserving bits of the fp32 score, then the inverted block index),
// so "best" is a plain maximum and ties go to the lower index; 15 rounds of
// "largest key below the previous winner" with two 32-bit warp reductions
// (redux.sync) each.  The first 512 candidates of a row live in registers.
// Deterministic and independent of the warp layout.
#include "internal.h"

namespace msa {
namespace {

constexpr int kSelWarps = 4;

__device__ __forceinline__ uint64_t rank_key(float s, int64_t n) {
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)n);
}

__global__ void __launch_bounds__(32 * kSelWarps)
    select_kernel(const Problem p, const float* __restrict__ block_scores, int32_t* __restrict__ sel,
                  int32_t* __restrict__ sel_copy) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kSelWarps + warp;
    if (row >= (int64_t)p.B * p.Tq) return;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t pos = L - p.Tq + t;
    const int64_t r = pos / kBlock;  // forced block
    const int64_t nvis = r + 1;
    const float* s = block_scores + row * p.nbmax;
    const int want = (int)min64(kTopK - 1, nvis - 1);

    // The first 512 candidates stay in registers (16 per lane, loads issued together);
    // longer rows stream the rest from L1/L2 in chunks of 512 every round.
    constexpr int kPer = 16;
    uint64_t k0[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t n = j * 32 + lane;
        k0[j] = (n < nvis && n != r) ? rank_key(__ldg(s + n), n) : 0ull;
    }
    uint64_t prev = ~0ull;
    int mine = -1;  // lane i < want holds the i-th best
    for (int k = 0; k < want; ++k) {
        uint64_t best = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (k0[j] < prev && k0[j] > best) best = k0[j];
        for (int64_t base = 32 * kPer; base < nvis; base += 32 * kPer) {
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int64_t n = base + j * 32 + lane;
                const uint64_t key = (n < nvis && n != r) ? rank_key(__ldg(s + n), n) : 0ull;
                if (key < prev && key > best) best = key;
            }
        }
        const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
        const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hi ? (uint32_t)best : 0u);
        prev = ((uint64_t)hi << 32) | lo;
        if (lane == k) mine = (int)(0xFFFFFFFFu - lo);
    }
    if (lane == want) mine = (int)r;
    const int nsel = want + 1;
    // ascending order: rank = number of smaller ids
    int rank = 0;
    for (int i = 0; i < nsel; ++i) {
        const int other = __shfl_sync(0xffffffffu, mine, i);
        rank += (other < mine) ? 1 : 0;
    }
    int32_t* out = sel + row * kTopK;
    if (lane < nsel) out[rank] = mine;
    else if (lane < kTopK) out[lane] = -1;
    if (sel_copy != nullptr) {
        int32_t* o2 = sel_copy + row * kTopK;
        if (lane < nsel) o2[rank] = mine;
        else if (lane < kTopK) o2[lane] = -1;
    }
}

}  // namespace

int launch_select(const Problem& p, const float* block_scores, int32_t* sel, int32_t* sel_copy, bool pdl,
                  cudaStream_t st) {
    const int64_t rows = (int64_t)p.B * p.Tq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows + kSelWarps - 1) / kSelWarps));
    cfg.blockDim = dim3(32 * kSelWarps);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, select_kernel, p, block_scores, sel, sel_copy) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace msa
