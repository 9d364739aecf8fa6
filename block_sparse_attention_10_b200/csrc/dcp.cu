// dcp.cu — indexer decode context parallelism: the kernels that let G ranks, each
// holding one contiguous range of every sequence's blocks, produce the single-rank
// decode result with one exchange of selection candidates and one of attention partials.
//
// Prior art: the pages report context parallelism of the indexer for decode, each GPU
// indexing its own share of a long context ("vLLM delivers day-0 support for
// MiniMax-M3.1-Flash", readmex.ai, TL;DR; "vLLM Adds Day-0 Support for
// MiniMax-M3.1-Flash on NVIDIA and AMD GPUs", ainewsbites.com, "Kernel and serving
// optimizations").  The pages give no algorithm; the steps here follow from the method
// of "A model built for efficient inference" on the same page (a per-block score, the
// query's own block plus the best 15 others, exact softmax attention over them):
//   1. rank g scores the blocks [n0, n1) it holds (the decode indexer restricted to the
//      range) and keeps its best min(15, count) blocks other than the query's own block,
//      by (score desc, index asc): dcp_candidates_cta_kernel (threshold selection, ranges of
//      up to 4,096 blocks) or dcp_candidates_kernel (rounds of a warp maximum, any range);
//   2. the G lists are exchanged; every rank merges the G x 16 (score, id) pairs the same
//      way: the query's own block plus the best min(15, r) of the pairs.  The best 15
//      blocks of the whole context are among the ranks' best 15, so this is the
//      single-rank selection exactly: dcp_merge_kernel;
//   3. each rank attends over the selected blocks it holds (attend.cu with the range),
//      giving an output normalised over its own keys and its log-sum-exp;
//   4. the G partials are exchanged and combined in rank order:
//      lse = log sum_g exp(lse_g), out = sum_g exp(lse_g - lse) out_g: dcp_combine_kernel.
// All three kernels are small and latency-bound (one warp per query row for 1-2, one
// thread per four output elements for 4); the range indexer carries the HBM traffic.
#include "internal.h"
#include "select_row.cuh"

namespace msa {
namespace {

constexpr int kDcpWarps = 4;
constexpr int kDcpCandPer = 8;  // range blocks per lane per chunk of the candidate scan

// Lane k < want receives the k-th best rank key (score desc, index asc) among blocks n in
// [lo, hi), n != skip, of score row s; other lanes receive 0.  Chunks of 32 * PER blocks;
// the best keys of the earlier chunks are carried into each chunk's rounds.
template <int PER>
__device__ __forceinline__ uint64_t warp_best_keys(const float* __restrict__ s, int64_t lo, int64_t hi,
                                                   int64_t skip, int want, int lane) {
    uint64_t best = 0ull;
    for (int64_t base = lo; base < hi; base += 32 * PER) {
        uint64_t k0[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int64_t n = base + (int64_t)j * 32 + lane;
            k0[j] = (n < hi && n != skip) ? rank_key(__ldg(s + n), n) : 0ull;
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
    return best;
}

__device__ __forceinline__ int32_t key_index(uint64_t key) { return (int32_t)(0xFFFFFFFFu - (uint32_t)key); }

// Step 1 for any range: block_scores (written by the range indexer) -> this rank's candidates
// per row: slots 0..want-1 in (score desc, index asc) order, the rest (-inf, -1).
__global__ void __launch_bounds__(32 * kDcpWarps)
    dcp_candidates_kernel(const Problem p, const float* __restrict__ block_scores, float* __restrict__ cand_score,
                          int32_t* __restrict__ cand_id) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kDcpWarps + warp;
    if (row >= (int64_t)p.B * p.Tq) return;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t r = (L - p.Tq + t) / kBlock;  // the query's own block
    const int64_t lo = p.blk_lo, hi = min64(p.blk_hi, r + 1);
    const int64_t count = max64(0, hi - lo) - ((r >= lo && r < hi) ? 1 : 0);
    const int want = (int)min64(kTopK - 1, count);
    const float* s = block_scores + row * p.nbmax;
    const uint64_t key = warp_best_keys<kDcpCandPer>(s, lo, hi, r, want, lane);
    if (lane < kTopK) {
        const bool have = lane < want;
        const int32_t id = have ? key_index(key) : -1;
        cand_id[row * kTopK + lane] = id;
        cand_score[row * kTopK + lane] = have ? __ldg(s + id) : -INFINITY;
    }
}

// Step 1 for ranges of up to 8 * 32 * PER blocks: one CTA of 8 warps per row.  Warp w finds
// the best min(15, c_w) blocks of its 32 * PER blocks of the range by threshold (the k-th best
// 32-bit score key, then an ordered pass that keeps the lowest-indexed ties), writing them in
// ascending block order; warp 0 then does the same over the warps' candidates, which are in
// ascending block order, so the index tie-break carries over.  Output ascending by block.
constexpr int kDcpCtaWarps = 8;
template <int PER>
__global__ void __launch_bounds__(32 * kDcpCtaWarps)
    dcp_candidates_cta_kernel(const Problem p, const float* __restrict__ block_scores, float* __restrict__ cand_score,
                              int32_t* __restrict__ cand_id) {
    constexpr int kCand = kTopK - 1;
    __shared__ uint32_t ckey[kDcpCtaWarps * kCand];
    __shared__ int32_t cid[kDcpCtaWarps * kCand];
    __shared__ int32_t res[kTopK];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t r = (L - p.Tq + t) / kBlock;  // the query's own block
    const int64_t lo = p.blk_lo, hi = min64(p.blk_hi, r + 1);
    const float* s = block_scores + row * p.nbmax;
    const int64_t base = lo + (int64_t)warp * 32 * PER;
    uint32_t k[PER];
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int64_t n = base + (int64_t)j * 32 + lane;
        k[j] = (n < hi && n != r) ? score_key(__ldg(s + n)) : 0u;
        cnt += k[j] != 0u ? 1 : 0;
    }
    cnt = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
    const int want_w = min(kCand, cnt);
    if (want_w > 0) {
        int n_gt;
        const uint32_t T = warp_kth_key(k, want_w, n_gt);
        warp_compact(k, T, want_w - n_gt, lane, [&](int slot, int j) {
            ckey[warp * kCand + slot] = k[j];
            cid[warp * kCand + slot] = (int32_t)(base + j * 32 + lane);
        });
    }
    if (lane >= want_w && lane < kCand) ckey[warp * kCand + lane] = 0u;
    __syncthreads();
    if (warp != 0) return;
    constexpr int kC = kDcpCtaWarps * kCand;
    constexpr int kPer2 = (kC + 31) / 32;
    uint32_t kk[kPer2];
    int c2 = 0;
#pragma unroll
    for (int j = 0; j < kPer2; ++j) {
        const int cc = j * 32 + lane;
        kk[j] = cc < kC ? ckey[cc] : 0u;
        c2 += kk[j] != 0u ? 1 : 0;
    }
    c2 = (int)__reduce_add_sync(0xffffffffu, (unsigned)c2);
    const int want = min(kCand, c2);
    if (want > 0) {
        int n_gt;
        const uint32_t T = warp_kth_key(kk, want, n_gt);
        warp_compact(kk, T, want - n_gt, lane, [&](int slot, int j) { res[slot] = cid[j * 32 + lane]; });
    }
    __syncwarp();
    if (lane < kTopK) {
        const int32_t id = lane < want ? res[lane] : -1;
        cand_id[row * kTopK + lane] = id;
        cand_score[row * kTopK + lane] = id >= 0 ? __ldg(s + id) : -INFINITY;
    }
}

// Step 2: G ranks' candidates [G][rows][16] -> the selection [rows][16] (ascending, -1
// padded), the query's own block forced.  Pairs with an id outside the visible blocks or
// equal to the forced block are ignored; a pair sent twice counts once (its rank key is
// the same), so overlapping ranges cannot duplicate a block.
template <int PER>
__global__ void __launch_bounds__(32 * kDcpWarps)
    dcp_merge_kernel(const Problem p, int G, const float* __restrict__ cand_score,
                     const int32_t* __restrict__ cand_id, int32_t* __restrict__ sel) {
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)p.B * p.Tq;
    const int64_t row = (int64_t)blockIdx.x * kDcpWarps + warp;
    if (row >= rows) return;
    const int b = (int)(row / p.Tq), t = (int)(row % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t r = (L - p.Tq + t) / kBlock;
    const int64_t nvis = r + 1;
    uint64_t k0[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const int e = j * 32 + lane;  // pair e: rank e / 16, slot e % 16
        k0[j] = 0ull;
        if (e < G * kTopK) {
            const int64_t at = ((int64_t)(e / kTopK) * rows + row) * kTopK + (e % kTopK);
            const int32_t id = __ldg(cand_id + at);
            if (id >= 0 && id < nvis && id != r) k0[j] = rank_key(__ldg(cand_score + at), id);
        }
    }
    const int want = (int)min64(kTopK - 1, nvis - 1);
    uint64_t best = 0ull, prev = ~0ull;
    int found = 0;
    for (int k = 0; k < want; ++k) {
        uint64_t m = 0ull;
#pragma unroll
        for (int j = 0; j < PER; ++j) m = (k0[j] < prev && k0[j] > m) ? k0[j] : m;
        prev = warp_max64(m);
        if (prev == 0ull) break;  // fewer pairs than wanted (ranges that do not cover the context)
        if (lane == k) best = prev;
        ++found;
    }
    int mine = lane < found ? key_index(best) : -1;
    if (lane == found) mine = (int)r;
    const int nsel = found + 1;
    int rank = 0;
    for (int i = 0; i < nsel; ++i) rank += (__shfl_sync(0xffffffffu, mine, i) < mine) ? 1 : 0;
    int out = -1;
#pragma unroll
    for (int i = 0; i < kTopK; ++i) {
        const int id = __shfl_sync(0xffffffffu, mine, i);
        const int rk = __shfl_sync(0xffffffffu, rank, i);
        if (i < nsel && rk == lane) out = id;
    }
    if (lane < kTopK) sel[row * kTopK + lane] = out;
}

// Step 4: G partial outputs [G][rows][Hq][D] (each normalised over its rank's keys) and
// their log-sum-exps [G][rows][Hq] -> out [rows][Hq][D] (fp32 or bf16) and lse [rows][Hq].
// One thread per four consecutive output elements; ranks are combined in rank order.
__global__ void __launch_bounds__(256)
    dcp_combine_kernel(const Problem p, int G, const float* __restrict__ part_out, const float* __restrict__ part_lse,
                       float* __restrict__ out, float* __restrict__ lse) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t heads = (int64_t)p.B * p.Tq * p.Hq;  // (row, head) pairs
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= heads * (p.D / 4)) return;
    const int64_t rh = i / (p.D / 4);
    const int d = (int)(i % (p.D / 4)) * 4;
    float M = -INFINITY;
    for (int g = 0; g < G; ++g) M = fmaxf(M, __ldg(part_lse + g * heads + rh));
    float Ls = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (M != -INFINITY) {
        for (int g = 0; g < G; ++g) {
            const float l = __ldg(part_lse + g * heads + rh);
            if (l == -INFINITY) continue;  // the rank holds none of the row's selected keys
            const float w = expf(l - M);
            const float4 o = __ldg(reinterpret_cast<const float4*>(part_out + (g * heads + rh) * p.D + d));
            Ls += w;
            acc.x += w * o.x;
            acc.y += w * o.y;
            acc.z += w * o.z;
            acc.w += w * o.w;
        }
    }
    const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
    store_out2(p, out, rh * p.D + d, acc.x * inv, acc.y * inv);
    store_out2(p, out, rh * p.D + d + 2, acc.z * inv, acc.w * inv);
    if (d == 0 && lse != nullptr) lse[rh] = Ls > 0.0f ? M + logf(Ls) : -INFINITY;
}

cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, bool pdl, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <int PER>
int launch_merge_per(const Problem& p, int G, const float* cs, const int32_t* ci, int32_t* sel, bool pdl,
                     cudaStream_t st) {
    const int64_t rows = (int64_t)p.B * p.Tq;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg =
        pdl_config(dim3((unsigned)((rows + kDcpWarps - 1) / kDcpWarps)), dim3(32 * kDcpWarps), pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, dcp_merge_kernel<PER>, p, G, cs, ci, sel) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace

int launch_dcp_candidates(const Problem& p, const float* block_scores, float* cand_score, int32_t* cand_id, bool pdl,
                          cudaStream_t st) {
    const int64_t rows = (int64_t)p.B * p.Tq;
    const int64_t span = p.blk_hi - p.blk_lo;
    if (span <= 8 * 32 * 16 && rows <= 0x7FFFFFFFll) {  // one CTA per row, threshold selection
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = pdl_config(dim3((unsigned)rows), dim3(32 * kDcpCtaWarps), pdl, st, attr);
        cudaError_t e = span <= 8 * 32 * 4 ? cudaLaunchKernelEx(&cfg, dcp_candidates_cta_kernel<4>, p, block_scores,
                                                                cand_score, cand_id)
                        : span <= 8 * 32 * 8 ? cudaLaunchKernelEx(&cfg, dcp_candidates_cta_kernel<8>, p, block_scores,
                                                                  cand_score, cand_id)
                                             : cudaLaunchKernelEx(&cfg, dcp_candidates_cta_kernel<16>, p, block_scores,
                                                                  cand_score, cand_id);
        return e == cudaSuccess ? MSA_OK : MSA_ECUDA;
    }
    if ((rows + kDcpWarps - 1) / kDcpWarps > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg =
        pdl_config(dim3((unsigned)((rows + kDcpWarps - 1) / kDcpWarps)), dim3(32 * kDcpWarps), pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, dcp_candidates_kernel, p, block_scores, cand_score, cand_id) != cudaSuccess)
        return MSA_ECUDA;
    return MSA_OK;
}

int launch_dcp_merge(const Problem& p, int G, const float* cand_score, const int32_t* cand_id, int32_t* sel,
                     bool pdl, cudaStream_t st) {
    if ((int64_t)p.B * p.Tq > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    if (G <= 2) return launch_merge_per<1>(p, G, cand_score, cand_id, sel, pdl, st);
    if (G <= 4) return launch_merge_per<2>(p, G, cand_score, cand_id, sel, pdl, st);
    if (G <= 8) return launch_merge_per<4>(p, G, cand_score, cand_id, sel, pdl, st);
    if (G <= 16) return launch_merge_per<8>(p, G, cand_score, cand_id, sel, pdl, st);
    if (G <= kDcpMaxRanks) return launch_merge_per<16>(p, G, cand_score, cand_id, sel, pdl, st);
    return MSA_EUNSUPPORTED;
}

int launch_dcp_combine(const Problem& p, int G, const float* part_out, const float* part_lse, float* out, float* lse,
                       bool pdl, cudaStream_t st) {
    const int64_t n = (int64_t)p.B * p.Tq * p.Hq * (p.D / 4);
    if ((n + 255) / 256 > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(dim3((unsigned)((n + 255) / 256)), dim3(256), pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, dcp_combine_kernel, p, G, part_out, part_lse, out, lse) != cudaSuccess)
        return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace msa
