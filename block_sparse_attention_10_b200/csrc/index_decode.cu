// index_decode.cu — MSA indexer + per-block pooling for decode (Tq * HI <= 32).
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com,
// "A model built for efficient inference"): a lightweight indexer scores every
// key of the context and the scores are pooled into one score per 128-token
// block.  Reading taken here: s_j = sum_h w_h * max(0, q_h . k_j) with one
// NVFP4 index key per token; pooled = mean (or max) over visible tokens.
//
// Design (B200): the kernel is HBM-bound — it must stream every index key
// (DI/2 + DI/16 bytes per token) exactly once for all Tq query tokens.
//   * 2 CTAs of 8 warps per SM; each warp owns a contiguous range of
//     (sequence, block) units and streams them itself: its lane 0 issues
//     untiled bulk copies (cp.async.bulk, no multicast) of 64-key half-blocks
//     (4.5 KB at DI = 128) into the warp's private ring of shared-memory
//     stages, two half-blocks ahead of the one being computed, each stage with
//     its own mbarrier.  A warp only ever waits on its own stages, in order, so
//     ~150 KB per SM are in flight while every warp computes.
//   * Dequantisation in registers with the sm_100a converters (E2M1x2 ->
//     f16x2, E4M3 -> f16; e2m1*e4m3 is exact in f16) feeding tensor-core
//     mma.sync m16n8k16 ([16 keys x DI] x [DI x 8 queries], f32 accumulate).
//     The per-tensor fp32 scale is applied once, after pooling (ReLU and both
//     pools commute with a positive scale).
//   * Each thread reads the 16 (DI = 128) or 8 (DI = 64) contiguous bytes of
//     a key that its A-fragment needs: the head dim is permuted identically
//     on the key and query side, so every shared-memory read is one 128/64-bit
//     load.
//   * Epilogue in registers: ReLU, head weights, sum over heads with warp
//     shuffles, causal / length masking, block pooling, one store per
//     (token, block).  Full, fully visible blocks under mean pooling take a
//     fast path that sums ReLU'd accumulators and reduces heads/rows once.
#include "internal.h"
#include "nvfp4_mma.cuh"

namespace msa {
namespace {

constexpr int kIdxWarps = 8;
constexpr int kIdxThreads = 32 * kIdxWarps;
constexpr int kMaxB = 4096;
constexpr int kHalf = 64;  // keys per shared-memory stage

template <int DI>
struct IdxGeom {
    static constexpr int kRowBytes = DI / 2;
    static constexpr int kSclBytes = DI / 16;
    static constexpr int kDataBytes = kHalf * kRowBytes;
    static constexpr int kStageBytes = kHalf * (kRowBytes + kSclBytes);
    static constexpr int kStages = DI == 128 ? 3 : 6;  // per warp: 13.5 KB either way
    static constexpr int kKSteps = DI / 16;
    static constexpr int kPairs = DI / 8;  // f16x2 pairs of q per thread
};

template <int DI>
constexpr size_t idx_smem_bytes(int B) {
    return (size_t)kIdxWarps * IdxGeom<DI>::kStages * (IdxGeom<DI>::kStageBytes + sizeof(uint64_t)) +
           (size_t)(2 * B + 2) * sizeof(int);
}

template <int HI>
__device__ __forceinline__ int token_of(int nt, int c, int e) {
    if constexpr (HI == 1) return 8 * nt + 2 * c + e;
    else if constexpr (HI == 2) return 4 * nt + c;
    else if constexpr (HI == 4) return 2 * nt + (c >> 1);
    else return nt;
}
template <int HI>
__device__ __forceinline__ bool token_owner(int c) {
    if constexpr (HI <= 2) return true;
    else if constexpr (HI == 4) return (c & 1) == 0;
    else return c == 0;
}

template <int DI, int HI, int NT>
__global__ void __launch_bounds__(kIdxThreads, 2)
    index_decode_kernel(const Problem p, float* __restrict__ block_scores, float* __restrict__ token_scores) {
    using G = IdxGeom<DI>;
    constexpr int R = G::kStages;
    constexpr int KS = G::kKSteps;
    constexpr int TPN = HI == 1 ? 2 : 1;  // tokens per thread per n-tile

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kIdxWarps * R * G::kStageBytes);
    int* prefix = reinterpret_cast<int*>(bars + kIdxWarps * R);  // [B + 1] units before sequence b
    int* lens = prefix + (p.B + 1);                               // [B] clamped lengths

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int B = p.B, Tq = p.Tq;
    const int NQ = Tq * HI;
    uint8_t* my_stages = smem + warp * R * G::kStageBytes;
    uint64_t* my_bars = bars + warp * R;

    pdl_wait();
    if (warp == 0) {
        int carry = 0;
        if (lane == 0) prefix[0] = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            int nb = 0;
            if (b < B) {
                const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, blockIdx.x == 0 ? p.status : nullptr);
                lens[b] = (int)L;
                nb = (int)((L + kBlock - 1) / kBlock);
            }
            int x = nb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < B) prefix[b + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    if (lane == 0) {
        for (int s = 0; s < R; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    const float s_t = p.ik.s_t;
    // blocks past a sequence's length score -inf (no unit covers them)
    {
        const int64_t total = (int64_t)B * Tq * p.nbmax;
        const int64_t stride = (int64_t)gridDim.x * kIdxThreads;
        for (int64_t i = (int64_t)blockIdx.x * kIdxThreads + threadIdx.x; i < total; i += stride) {
            const int64_t n = i % p.nbmax;
            const int b = (int)(i / (p.nbmax * Tq));
            if (n >= prefix[b + 1] - prefix[b]) block_scores[i] = -INFINITY;
        }
    }

    // this warp's contiguous range of units
    const int64_t U = prefix[B];
    const int64_t Wt = (int64_t)gridDim.x * kIdxWarps;
    const int64_t gw = (int64_t)blockIdx.x * kIdxWarps + warp;
    const int64_t u_begin = U * gw / Wt, u_end = U * (gw + 1) / Wt;

    // issue side: walks the same (unit, half) sequence as the compute side, R halves ahead
    int64_t iu = u_begin;
    int ih = 0, ib = 0;
    uint32_t slot_issued = 0;
    auto issue_upto = [&](uint32_t limit) {
        while (slot_issued < limit && iu < u_end) {
            while (prefix[ib + 1] <= iu) ++ib;
            const int64_t n = iu - prefix[ib];
            const int valid = (int)min64(kBlock, lens[ib] - n * kBlock) - ih * kHalf;
            if (valid > 0) {
                if (lane == 0) {
                    const int rows = (min(valid, kHalf) + 15) & ~15;
                    const int s = (int)(slot_issued % R);
                    const int64_t row0 = (int64_t)ib * p.lmax + n * kBlock + ih * kHalf;
                    uint8_t* st = my_stages + s * G::kStageBytes;
                    const uint32_t db = (uint32_t)(rows * G::kRowBytes), sb = (uint32_t)(rows * G::kSclBytes);
                    mbar_arrive_expect_tx(&my_bars[s], db + sb);
                    bulk_g2s(st, p.ik.data + row0 * G::kRowBytes, db, &my_bars[s]);
                    bulk_g2s(st + G::kDataBytes, p.ik.scale + row0 * G::kSclBytes, sb, &my_bars[s]);
                }
                ++slot_issued;
            }
            if (++ih == 2) {
                ih = 0;
                ++iu;
            }
        }
    };

    uint32_t qf[NT][KS][2];
    float wq[NT][2];
    int cur_b = -1;
    int b = 0;
    uint32_t slot = 0;
    bool failed = false;

    for (int64_t u = u_begin; u < u_end && !failed; ++u) {
        while (prefix[b + 1] <= u) ++b;
        const int64_t n = u - prefix[b];
        const int L = lens[b];
        const int valid = (int)min64(kBlock, L - n * kBlock);
        const int64_t kbase = n * kBlock;

        if (b != cur_b) {
            cur_b = b;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int qn = 8 * nt + g;
                uint32_t pr[G::kPairs];
                if (qn < NQ) {
                    const __nv_bfloat16* row = p.q_idx + ((int64_t)b * Tq * HI + qn) * DI + c * (DI / 4);
#pragma unroll
                    for (int v = 0; v < G::kPairs / 4; ++v) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(row + 8 * v);
                        pr[4 * v + 0] = bf16x2_to_f16x2(w4.x);
                        pr[4 * v + 1] = bf16x2_to_f16x2(w4.y);
                        pr[4 * v + 2] = bf16x2_to_f16x2(w4.z);
                        pr[4 * v + 3] = bf16x2_to_f16x2(w4.w);
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < G::kPairs; ++v) pr[v] = 0u;
                }
#pragma unroll
                for (int i = 0; i < KS; ++i) {
                    qf[nt][i][0] = pr[2 * i];
                    qf[nt][i][1] = pr[2 * i + 1];
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int qq = 8 * nt + 2 * c + e;
                    wq[nt][e] = qq < NQ ? (p.w_idx ? p.w_idx[(int64_t)b * Tq * HI + qq] : 1.0f) : 0.0f;
                }
            }
        }

        // fast path: a full block that every query token sees entirely, mean pooling, no
        // per-token output.  The pooled mean is linear, so ReLU'd products are summed per
        // accumulator element over all tiles and reduced over heads and rows once per block.
        const bool fast = valid == kBlock && kbase + (kBlock - 1) <= (int64_t)L - Tq && p.pool_mode == 0 &&
                          token_scores == nullptr;
        // acquire the next half-block of this warp's stream (in order), or flag a timeout
        auto acquire = [&](int& s_out) -> bool {
            issue_upto(slot + R);
            const int s = (int)(slot % R);
            if (!mbar_wait(&my_bars[s], (slot / R) & 1u)) {
                if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_CONSUMER);
                failed = true;
                return false;
            }
            ++slot;
            s_out = s;
            return true;
        };

        if (fast) {
            float colsum[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) colsum[nt][0] = colsum[nt][1] = colsum[nt][2] = colsum[nt][3] = 0.0f;
            for (int half = 0; half < 2; ++half) {
                int s;
                if (!acquire(s)) break;
                const uint8_t* sd = my_stages + s * G::kStageBytes;
                const uint8_t* ss = sd + G::kDataBytes;
#pragma unroll
                for (int ti = 0; ti < kHalf / 16; ++ti) {
                    float acc[NT][4];
                    nvfp4_tile_mma<DI, NT>(sd, ss, ti * 16 + g, c, qf, acc);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) colsum[nt][e] += fmaxf(acc[nt][e], 0.0f);
                }
                __syncwarp();  // every lane is done reading stage s before it is refilled
            }
            if (failed) break;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // rows g and g+8 of the same column, then the head weights
                float x0 = (colsum[nt][0] + colsum[nt][2]) * wq[nt][0];
                float x1 = (colsum[nt][1] + colsum[nt][3]) * wq[nt][1];
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
            continue;
        }

        float pool[NT][TPN];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < TPN; ++e) pool[nt][e] = p.pool_mode == 1 ? -INFINITY : 0.0f;
        for (int half = 0; half < 2; ++half) {
            const int hvalid = min(valid - half * kHalf, kHalf);
            if (hvalid <= 0) break;
            int s;
            if (!acquire(s)) break;
            const uint8_t* sd = my_stages + s * G::kStageBytes;
            const uint8_t* ss = sd + G::kDataBytes;
            const int64_t hbase = kbase + half * kHalf;
            const int ntiles = (hvalid + 15) >> 4;
            for (int ti = 0; ti < ntiles; ++ti) {
                const int r0 = ti * 16 + g, r1 = r0 + 8;
                float acc[NT][4];
                nvfp4_tile_mma<DI, NT>(sd, ss, r0, c, qf, acc);
                // epilogue: ReLU * w, sum over heads, mask, pool
                const int64_t j0 = hbase + r0, j1 = hbase + r1;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float v[2][2];  // [row][col]
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        v[0][e] = fmaxf(acc[nt][e], 0.0f) * wq[nt][e];
                        v[1][e] = fmaxf(acc[nt][2 + e], 0.0f) * wq[nt][e];
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
                        const int64_t pos = (int64_t)L - Tq + t;
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
            __syncwarp();  // every lane is done reading stage s before it is refilled
        }
        if (failed) break;

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
                    const int64_t pos = (int64_t)L - Tq + t;
                    const int64_t cnt = min64(kBlock, max64(0, pos + 1 - kbase));
                    float outv = -INFINITY;
                    if (cnt > 0) outv = p.pool_mode == 1 ? x * s_t : (x / (float)cnt) * s_t;
                    block_scores[((int64_t)b * Tq + t) * p.nbmax + n] = outv;
                }
            }
        }
    }
    // never leave with copies in flight into this warp's stages
    for (uint32_t j = slot; j < slot_issued; ++j)
        if (!mbar_wait(&my_bars[j % R], (j / R) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_DRAIN);
            break;
        }
}

template <int DI, int HI, int NT>
int launch_t(const Problem& p, float* bs, float* ts, bool pdl, cudaStream_t st) {
    auto kern = index_decode_kernel<DI, HI, NT>;
    const size_t smem = idx_smem_bytes<DI>(p.B);
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)idx_smem_bytes<DI>(kMaxB)) != cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * di.num_sms));
    cfg.blockDim = dim3(kIdxThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p, bs, ts) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

template <int DI, int HI>
int launch_nt(const Problem& p, float* bs, float* ts, bool pdl, cudaStream_t st) {
    const int nq = p.Tq * HI;
    if (nq <= 8) return launch_t<DI, HI, 1>(p, bs, ts, pdl, st);
    if (nq <= 16) return launch_t<DI, HI, 2>(p, bs, ts, pdl, st);
    if (nq <= 24) return launch_t<DI, HI, 3>(p, bs, ts, pdl, st);
    return launch_t<DI, HI, 4>(p, bs, ts, pdl, st);
}

template <int DI>
int launch_hi(const Problem& p, float* bs, float* ts, bool pdl, cudaStream_t st) {
    switch (p.HI) {
        case 1: return launch_nt<DI, 1>(p, bs, ts, pdl, st);
        case 2: return launch_nt<DI, 2>(p, bs, ts, pdl, st);
        case 4: return launch_nt<DI, 4>(p, bs, ts, pdl, st);
        case 8: return launch_nt<DI, 8>(p, bs, ts, pdl, st);
        default: return MSA_EUNSUPPORTED;
    }
}

}  // namespace

int index_decode_max_batch() { return kMaxB; }

int launch_index_decode(const Problem& p, float* block_scores, float* token_scores, bool pdl, cudaStream_t st) {
    if (p.B > kMaxB || p.Tq * p.HI > 32) return MSA_EUNSUPPORTED;
    if (p.DI == 128) return launch_hi<128>(p, block_scores, token_scores, pdl, st);
    if (p.DI == 64) return launch_hi<64>(p, block_scores, token_scores, pdl, st);
    return MSA_EUNSUPPORTED;
}

}  // namespace msa
