// index_block.cuh — the decode indexer's work on one 128-token block: dequantise the
// block's NVFP4 index keys, score them against the query tokens' indexer heads on the
// tensor cores, and pool the scores into one value per (query token, block).
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com, "A model
// built for efficient inference"): a lightweight indexer scores every key and the scores
// are pooled per 128-token block.  Reading: s_j = sum_h w_h * max(0, q_h . k_j), one
// index key per token, pooled = mean (or max) over the visible tokens of the block.
//
// Shared by the stand-alone indexer (index_decode.cu) and the single-launch decode
// kernel (decode_fused.cu).  Both stream the keys through per-warp rings of
// shared-memory stages; a stage holds 4 KB of key nibbles followed by their 512 B of
// E4M3 scales: 64 keys at DI = 128, a whole block at DI = 64.
#pragma once

#include "internal.h"
#include "nvfp4_mma.cuh"

namespace msa {

constexpr int kIdxStageData = 4096;
constexpr int kIdxStageBytes = kIdxStageData + 512;
template <int DI>
constexpr int idx_stage_keys() {
    return kIdxStageData / (DI / 2);
}

// Query token of accumulator column (n-tile nt, thread column c, element e) when the
// 8 columns of an n-tile hold HI consecutive heads of 8 / HI tokens.
template <int HI>
__device__ __forceinline__ int token_of(int nt, int c, int e) {
    if constexpr (HI == 1) return 8 * nt + 2 * c + e;
    else if constexpr (HI == 2) return 4 * nt + c;
    else if constexpr (HI == 4) return 2 * nt + (c >> 1);
    else return nt;
}
// The thread that holds a token's head sum after the shuffles over its heads.
template <int HI>
__device__ __forceinline__ bool token_owner(int c) {
    if constexpr (HI <= 2) return true;
    else if constexpr (HI == 4) return (c & 1) == 0;
    else return c == 0;
}

// The Tq * HI indexer query rows of one sequence as mma B fragments (fp16, head dim
// permuted as the key rows) and their head weights.
template <int DI, int NT>
struct IdxQuery {
    uint32_t qf[NT][DI / 16][2];
    float wq[NT][2];
};

template <int DI, int HI, int NT>
__device__ __forceinline__ void idx_load_query(const Problem& p, int b, int g, int c, IdxQuery<DI, NT>& q) {
    constexpr int kPairs = DI / 8;
    const int NQ = p.Tq * HI;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int qn = 8 * nt + g;
        uint32_t pr[kPairs];
        if (qn < NQ) {
            const __nv_bfloat16* row = p.q_idx + ((int64_t)b * NQ + qn) * DI + c * (DI / 4);
#pragma unroll
            for (int v = 0; v < kPairs / 4; ++v) {
                const uint4 w4 = *reinterpret_cast<const uint4*>(row + 8 * v);
                pr[4 * v + 0] = bf16x2_to_f16x2(w4.x);
                pr[4 * v + 1] = bf16x2_to_f16x2(w4.y);
                pr[4 * v + 2] = bf16x2_to_f16x2(w4.z);
                pr[4 * v + 3] = bf16x2_to_f16x2(w4.w);
            }
        } else {
#pragma unroll
            for (int v = 0; v < kPairs; ++v) pr[v] = 0u;
        }
#pragma unroll
        for (int i = 0; i < DI / 16; ++i) {
            q.qf[nt][i][0] = pr[2 * i];
            q.qf[nt][i][1] = pr[2 * i + 1];
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int qq = 8 * nt + 2 * c + e;
            q.wq[nt][e] = qq < NQ ? (p.w_idx ? p.w_idx[(int64_t)b * NQ + qq] : 1.0f) : 0.0f;
        }
    }
}

// Shared-memory stages that block n of a sequence of length L occupies in the stream.
template <int DI>
__device__ __forceinline__ int idx_block_stages(int64_t n, int64_t L) {
    const int valid = (int)min64(kBlock, L - n * kBlock);
    return (valid + idx_stage_keys<DI>() - 1) / idx_stage_keys<DI>();
}

// Scores block n of sequence b (length L) and writes its pooled score for every query
// token (and, if token_scores != nullptr, every visible key's score).  acquire() hands
// out the warp's next stage in stream order (nullptr after a timeout, which is returned
// as false).  Full, fully visible blocks under mean pooling take a fast path: the pooled
// mean is linear, so ReLU'd products are summed per accumulator element over all tiles
// and reduced over heads and rows once per block.
template <int DI, int HI, int NT, class Acquire>
__device__ __forceinline__ bool idx_block(const Problem& p, int b, int64_t n, int64_t L, const IdxQuery<DI, NT>& q,
                                          Acquire&& acquire, float* __restrict__ block_scores,
                                          float* __restrict__ token_scores, int g, int c) {
    constexpr int KPS = idx_stage_keys<DI>();
    constexpr int TPN = HI == 1 ? 2 : 1;  // tokens per thread per n-tile
    const int Tq = p.Tq;
    const int valid = (int)min64(kBlock, L - n * kBlock);
    const int64_t kbase = n * kBlock;
    const float s_t = p.ik.s_t;

    const bool fast = valid == kBlock && kbase + (kBlock - 1) <= L - Tq && p.pool_mode == 0 && token_scores == nullptr;
    if (fast) {
        float colsum[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) colsum[nt][0] = colsum[nt][1] = colsum[nt][2] = colsum[nt][3] = 0.0f;
        for (int st = 0; st < kBlock / KPS; ++st) {
            const uint8_t* sd = acquire();
            if (sd == nullptr) return false;
            const uint8_t* ss = sd + kIdxStageData;
#pragma unroll
            for (int ti = 0; ti < KPS / 16; ++ti) {
                float acc[NT][4];
                nvfp4_tile_mma<DI, NT>(sd, ss, ti * 16 + g, c, q.qf, acc);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) colsum[nt][e] += fmaxf(acc[nt][e], 0.0f);
            }
            __syncwarp();  // every lane is done reading the stage before it is refilled
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            // rows g and g+8 of the same column, then the head weights
            const float x0 = (colsum[nt][0] + colsum[nt][2]) * q.wq[nt][0];
            const float x1 = (colsum[nt][1] + colsum[nt][3]) * q.wq[nt][1];
            float tsum[TPN];
            if constexpr (HI == 1) {
                tsum[0] = x0;
                tsum[TPN - 1] = x1;
            } else {
                float x = x0 + x1;
                if constexpr (HI >= 4) x += __shfl_xor_sync(0xffffffffu, x, 1);
                if constexpr (HI >= 8) x += __shfl_xor_sync(0xffffffffu, x, 2);
                tsum[0] = x;
            }
#pragma unroll
            for (int e = 0; e < TPN; ++e) {
                float x = tsum[e];
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                const int t = token_of<HI>(nt, c, e);
                if (g == 0 && token_owner<HI>(c) && t < Tq)
                    block_scores[((int64_t)b * Tq + t) * p.nbmax + n] = (x * (1.0f / kBlock)) * s_t;
            }
        }
        return true;
    }

    float pool[NT][TPN];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < TPN; ++e) pool[nt][e] = p.pool_mode == 1 ? -INFINITY : 0.0f;
    for (int st = 0; st < kBlock / KPS; ++st) {
        const int svalid = min(valid - st * KPS, KPS);
        if (svalid <= 0) break;
        const uint8_t* sd = acquire();
        if (sd == nullptr) return false;
        const uint8_t* ss = sd + kIdxStageData;
        const int64_t sbase = kbase + st * KPS;
        const int ntiles = (svalid + 15) >> 4;
        for (int ti = 0; ti < ntiles; ++ti) {
            const int r0 = ti * 16 + g, r1 = r0 + 8;
            float acc[NT][4];
            nvfp4_tile_mma<DI, NT>(sd, ss, r0, c, q.qf, acc);
            // epilogue: ReLU * w, sum over heads, mask, pool
            const int64_t j0 = sbase + r0, j1 = sbase + r1;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float v[2][2];  // [row][col]
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    v[0][e] = fmaxf(acc[nt][e], 0.0f) * q.wq[nt][e];
                    v[1][e] = fmaxf(acc[nt][2 + e], 0.0f) * q.wq[nt][e];
                }
                float tsum[2][TPN];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    if constexpr (HI == 1) {
                        tsum[rr][0] = v[rr][0];
                        tsum[rr][TPN - 1] = v[rr][1];
                    } else {
                        float x = v[rr][0] + v[rr][1];
                        if constexpr (HI >= 4) x += __shfl_xor_sync(0xffffffffu, x, 1);
                        if constexpr (HI >= 8) x += __shfl_xor_sync(0xffffffffu, x, 2);
                        tsum[rr][0] = x;
                    }
                }
#pragma unroll
                for (int e = 0; e < TPN; ++e) {
                    const int t = token_of<HI>(nt, c, e);
                    const int64_t pos = L - Tq + t;
                    const bool vis0 = t < Tq && j0 <= pos, vis1 = t < Tq && j1 <= pos;
                    const float x0 = vis0 ? tsum[0][e] : 0.0f, x1 = vis1 ? tsum[1][e] : 0.0f;
                    if (p.pool_mode == 1) {
                        if (vis0) pool[nt][e] = fmaxf(pool[nt][e], x0);
                        if (vis1) pool[nt][e] = fmaxf(pool[nt][e], x1);
                    } else {
                        pool[nt][e] += x0 + x1;
                    }
                    if (token_scores != nullptr && token_owner<HI>(c)) {
                        float* ts = token_scores + ((int64_t)b * Tq + t) * p.lmax;
                        if (vis0) ts[j0] = x0 * s_t;
                        if (vis1) ts[j1] = x1 * s_t;
                    }
                }
            }
        }
        __syncwarp();  // every lane is done reading the stage before it is refilled
    }

    // pool across the 8 row groups and store one score per (token, block)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < TPN; ++e) {
            float x = pool[nt][e];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const float y = __shfl_xor_sync(0xffffffffu, x, o);
                x = p.pool_mode == 1 ? fmaxf(x, y) : x + y;
            }
            const int t = token_of<HI>(nt, c, e);
            if (g == 0 && token_owner<HI>(c) && t < Tq) {
                const int64_t pos = L - Tq + t;
                const int64_t cnt = min64(kBlock, max64(0, pos + 1 - kbase));
                float outv = -INFINITY;
                if (cnt > 0) outv = p.pool_mode == 1 ? x * s_t : (x / (float)cnt) * s_t;
                block_scores[((int64_t)b * Tq + t) * p.nbmax + n] = outv;
            }
        }
    }
    return true;
}

}  // namespace msa
