// select.cu — top-16 block selection with the most recent block forced.
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com,
// section "A model built for efficient inference"): 16 blocks per query are
// attended, and the block that holds the query is always among them.
// Reading: the query's own block r = pos div 128 plus the best
// min(15, r) other blocks under the total order (score desc, index asc); the
// list is written ascending and padded with -1.
//
// Rows of <= 1,024 blocks: one warp per (sequence, query token), the threshold
// selection of select_row.cuh.  Rows of <= 4,096 blocks: one CTA of 8 warps per
// row; each warp selects the best 15 of its 256-block (rows of <= 2,048 blocks) or
// 512-block chunk (the row's best 15
// are among those 120), then one warp selects from the 120 candidates, which
// sit in ascending block order so the index tie-break carries over.  Longer
// rows: 64-bit keys (score key, inverted index) and 15 rounds of "largest key
// below the previous winner" over the whole CTA.  All deterministic.
#include "internal.h"
#include "select_row.cuh"

namespace msa {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kPer = 16;  // candidates per thread held in registers (rows of <= 4,096 blocks)

// Rows of <= 4,096 blocks: one CTA of 8 warps per (sequence, query token), two levels; each
// lane holds PER candidates (16: rows of <= 4,096 blocks, 8: rows of <= 2,048 blocks).
constexpr int kCtaPer = 16;  // 8 warps x 32 lanes x 16 candidates
constexpr int kCtaMaxBlocks = kSelWarps * 32 * kCtaPer;

template <int PER>
__global__ void __launch_bounds__(kSelThreads)
    select_cta_kernel(const Problem p, const float* __restrict__ block_scores, int32_t* __restrict__ sel,
                      int32_t* __restrict__ sel_copy) {
    __shared__ uint32_t ckey[kSelWarps * (kTopK - 1)];
    __shared__ int32_t cid[kSelWarps * (kTopK - 1)];
    __shared__ int32_t res[kTopK];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t r = (L - p.Tq + t) / kBlock;  // forced block
    select_row_cta<kSelWarps, PER>(block_scores + row * p.nbmax, r + 1, r, warp, lane, ckey, cid, res);
    if (warp != 0) return;
    __syncwarp();
    if (lane < kTopK) {
        sel[row * kTopK + lane] = res[lane];
        if (sel_copy) sel_copy[row * kTopK + lane] = res[lane];
    }
}

// Rows of more than 4,096 blocks: one CTA per (sequence, query token).  Thread i holds
// candidates i, i + 256, ... of the row's first 4,096 blocks in registers (the rest are
// re-read each round); each of the 15 rounds takes the largest key below the previous
// winner with a warp reduction (redux.sync) and one exchange of 8 warp maxima through
// shared memory (double-buffered, one __syncthreads per round).
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const Problem p, const float* __restrict__ block_scores, int32_t* __restrict__ sel,
                  int32_t* __restrict__ sel_copy) {
    __shared__ uint64_t wmax[2][kSelWarps];
    __shared__ int chosen[kTopK];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t pos = L - p.Tq + t;
    const int64_t r = pos / kBlock;  // forced block
    const int64_t nvis = r + 1;
    const float* s = block_scores + row * p.nbmax;
    const int want = (int)min64(kTopK - 1, nvis - 1);

    uint64_t k0[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t n = (int64_t)j * kSelThreads + threadIdx.x;
        k0[j] = (n < nvis && n != r) ? rank_key(__ldg(s + n), n) : 0ull;
    }
    uint64_t prev = ~0ull;
    for (int k = 0; k < want; ++k) {
        uint64_t best = 0;
#pragma unroll
        for (int j = 0; j < kPer; ++j)
            if (k0[j] < prev && k0[j] > best) best = k0[j];
        for (int64_t base = (int64_t)kPer * kSelThreads; base < nvis; base += (int64_t)kPer * kSelThreads) {
#pragma unroll 4
            for (int j = 0; j < kPer; ++j) {
                const int64_t n = base + (int64_t)j * kSelThreads + threadIdx.x;
                const uint64_t key = (n < nvis && n != r) ? rank_key(__ldg(s + n), n) : 0ull;
                if (key < prev && key > best) best = key;
            }
        }
        best = warp_max64(best);
        if (lane == 0) wmax[k & 1][warp] = best;
        __syncthreads();
        uint64_t m = 0;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) m = wmax[k & 1][w] > m ? wmax[k & 1][w] : m;
        prev = m;
        if (threadIdx.x == 0) chosen[k] = (int)(0xFFFFFFFFu - (uint32_t)m);
    }
    if (threadIdx.x == 0) chosen[want] = (int)r;
    __syncthreads();
    // ascending order: rank = number of smaller ids
    const int nsel = want + 1;
    if (threadIdx.x < kTopK) {
        int32_t* out = sel + row * kTopK;
        int32_t* o2 = sel_copy ? sel_copy + row * kTopK : nullptr;
        if (threadIdx.x < nsel) {
            const int mine = chosen[threadIdx.x];
            int rank = 0;
            for (int i = 0; i < nsel; ++i) rank += chosen[i] < mine ? 1 : 0;
            out[rank] = mine;
            if (o2) o2[rank] = mine;
        } else {
            out[threadIdx.x] = -1;
            if (o2) o2[threadIdx.x] = -1;
        }
    }
}

// Short rows (<= 1,024 blocks): one warp per (sequence, query token), up to 32
// candidates per lane in registers.
constexpr int kWarpRows = 4;
constexpr int kWarpPer = 32;  // rows of up to 32 * kWarpPer blocks take the warp kernel

template <int PER>
__global__ void __launch_bounds__(32 * kWarpRows)
    select_warp_kernel(const Problem p, const float* __restrict__ block_scores, int32_t* __restrict__ sel,
                       int32_t* __restrict__ sel_copy) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kWarpRows + warp;
    if (row >= (int64_t)p.B * p.Tq) return;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t r = (L - p.Tq + t) / kBlock;
    __shared__ int32_t res[kWarpRows][kTopK];
    select_row_warp<PER>(block_scores + row * p.nbmax, r + 1, r, lane, res[warp]);
    __syncwarp();
    if (lane < kTopK) {
        sel[row * kTopK + lane] = res[warp][lane];
        if (sel_copy) sel_copy[row * kTopK + lane] = res[warp][lane];
    }
}

}  // namespace

int launch_select(const Problem& p, const float* block_scores, int32_t* sel, int32_t* sel_copy, bool pdl,
                  cudaStream_t st) {
    const int64_t rows = (int64_t)p.B * p.Tq;
    if (rows > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    const bool short_rows = p.nbmax <= 32 * kWarpPer;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(short_rows ? (unsigned)((rows + kWarpRows - 1) / kWarpRows) : (unsigned)rows);
    cfg.blockDim = dim3(short_rows ? 32 * kWarpRows : kSelThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (!short_rows && p.nbmax <= kCtaMaxBlocks / 2)
        e = cudaLaunchKernelEx(&cfg, select_cta_kernel<kCtaPer / 2>, p, block_scores, sel, sel_copy);
    else if (!short_rows && p.nbmax <= kCtaMaxBlocks)
        e = cudaLaunchKernelEx(&cfg, select_cta_kernel<kCtaPer>, p, block_scores, sel, sel_copy);
    else if (!short_rows) e = cudaLaunchKernelEx(&cfg, select_kernel, p, block_scores, sel, sel_copy);
    else if (p.nbmax <= 32 * 4) e = cudaLaunchKernelEx(&cfg, select_warp_kernel<4>, p, block_scores, sel, sel_copy);
    else if (p.nbmax <= 32 * 16) e = cudaLaunchKernelEx(&cfg, select_warp_kernel<16>, p, block_scores, sel, sel_copy);
    else e = cudaLaunchKernelEx(&cfg, select_warp_kernel<32>, p, block_scores, sel, sel_copy);
    if (e != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace msa
