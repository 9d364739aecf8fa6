// internal.h — launchers and argument blocks shared between the entry points
// (msa_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "common.cuh"
#include "msa.h"

namespace msa {

struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    size_t smem_optin = 0;
};
// Cached per current device (queried once per device).
const DeviceInfo& device_info();

// Kernel-side view of an NVFP4 cache.
struct Cache {
    const uint8_t* data;
    const uint8_t* scale;
    float s_t;
};

// Arguments shared by the decode kernels.
struct Problem {
    int B, Tq, Hq, Hkv, D, HI, DI;
    int64_t lmax;
    int64_t nbmax;  // lmax / 128
    const int32_t* seq_lens;
    Cache k, v, ik;
    const __nv_bfloat16* q;
    const __nv_bfloat16* q_idx;
    const float* w_idx;
    float softmax_scale;
    int pool_mode;
    uint32_t* status;
    const int32_t* block_table;  // [B][nbmax] page of each block, or nullptr (contiguous caches)
    int64_t num_pages;
    int out_bf16;                // attention output as bf16 (else fp32)
    // Blocks [blk_lo, blk_hi) of every sequence are the ones this call covers (the whole
    // context, [0, nbmax), except for the context-parallel entry points, where each rank
    // holds one contiguous range): the indexer scores only these blocks and attention
    // skips selected blocks outside them.
    int64_t blk_lo, blk_hi;
};

// First cache vector of block n of sequence b, head h of H: contiguous caches hold
// [B][H][lmax][...]; paged caches hold pages [num_pages][H][128][...] found through the
// block table.  A page id outside the pool is flagged and replaced by page 0, so every
// copy stays inside the pool.  PAGED is a compile-time choice in the indexers' stream
// loops (the contiguous path then carries no table lookup); block_vec_any decides at run
// time where it is called once per warp.
template <bool PAGED>
__device__ __forceinline__ int64_t block_vec(const Problem& p, int b, int64_t n, int h, int H) {
    if constexpr (!PAGED) {
        return ((int64_t)b * H + h) * p.lmax + n * kBlock;
    } else {
        int64_t page = __ldg(p.block_table + (int64_t)b * p.nbmax + n);
        if (page < 0 || page >= p.num_pages) {
            set_status(p.status, MSA_STATUS_PAGE);
            page = 0;
        }
        return (page * H + h) * kBlock;
    }
}
__device__ __forceinline__ int64_t block_vec_any(const Problem& p, int b, int64_t n, int h, int H) {
    return p.block_table != nullptr ? block_vec<true>(p, b, n, h, H) : block_vec<false>(p, b, n, h, H);
}

// Stores two adjacent output elements (index i, i + 1) as fp32 or, with out_bf16, bf16 (RNE).
__device__ __forceinline__ void store_out2(const Problem& p, float* out, int64_t i, float a, float b) {
    if (p.out_bf16)
        *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(out) + i) = __floats2bfloat162_rn(a, b);
    else
        *reinterpret_cast<float2*>(out + i) = make_float2(a, b);
}

int launch_nvfp4_encode(const float* x, int64_t nvec, int dim, float s_t, uint8_t* data, uint8_t* scale,
                        cudaStream_t st);
int launch_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim, float s_t, float* out,
                        cudaStream_t st);
int launch_nvfp4_amax(const float* x, int64_t n, float* amax_out, cudaStream_t st);

// Indexer + pooling over every visible key (decode: Tq * HI <= 32).
int launch_index_decode(const Problem& p, float* block_scores, float* token_scores, bool pdl, cudaStream_t st);
// Indexer + pooling for many query tokens (chunked prefill, tcgen05; mean pooling).
int launch_index_prefill(const Problem& p, float* block_scores, bool pdl, cudaStream_t st);
// Picks the decode or the prefill indexer for the problem's Tq * HI.
int launch_index(const Problem& p, float* block_scores, float* token_scores, bool pdl, cudaStream_t st);
// Top-16 selection, recent block forced.
int launch_select(const Problem& p, const float* block_scores, int32_t* sel, int32_t* sel_copy, bool pdl,
                  cudaStream_t st);
// Sparse attention over the selected blocks.
int launch_attend(const Problem& p, const int32_t* sel, float* out, float* lse, bool pdl, cudaStream_t st);
// Selection fused into the attention kernel (rows of <= 1,024 blocks; else MSA_EUNSUPPORTED).
int launch_select_attend(const Problem& p, const float* block_scores, int32_t* sel_out, float* out, float* lse,
                         bool pdl, cudaStream_t st);

// Sparse attention for chunked prefill (attend_prefill.cu): block-major tensor-core tiles.
// Used by msa_decode when attend_prefill_supported(p) (Tq * HI > 32, Hq / Hkv = 8); its
// workspace (selection inversion lists and per-slot partials) follows msa_decode's own.
bool attend_prefill_supported(const Problem& p);
size_t attend_prefill_ws_bytes(const Problem& p);
int launch_attend_prefill(const Problem& p, const int32_t* sel, void* ws, float* out, float* lse, bool pdl,
                          cudaStream_t st);
// cuTensorMapEncodeTiled from the driver (nullptr if unavailable), looked up once.
void* tensor_map_encode_entry();

// Context-parallel decode (dcp.cu).  Candidates: this rank's best 15 blocks of [blk_lo,
// blk_hi) per row, from block scores written by the range indexer; merge: G ranks'
// candidates -> the selection; combine: G attention partials -> the output.
constexpr int kDcpMaxRanks = 32;
int launch_dcp_candidates(const Problem& p, const float* block_scores, float* cand_score, int32_t* cand_id, bool pdl,
                          cudaStream_t st);
int launch_dcp_merge(const Problem& p, int G, const float* cand_score, const int32_t* cand_id, int32_t* sel,
                     bool pdl, cudaStream_t st);
int launch_dcp_combine(const Problem& p, int G, const float* part_out, const float* part_lse, float* out, float* lse,
                       bool pdl, cudaStream_t st);

// The whole decode step in one persistent launch (decode_fused.cu).  Workspace: byte
// offsets of its regions; the counter region [0, ctr_bytes) is cleared by the launcher.
struct FusedLayout {
    size_t ctr_bytes, bscores, sel, part, total;
};
FusedLayout fused_layout(const Problem& p);
bool fused_supported(const Problem& p);
int launch_decode_fused(const Problem& p, void* ws, float* out, float* lse, int32_t* sel_out, bool pdl,
                        cudaStream_t st);

}  // namespace msa
