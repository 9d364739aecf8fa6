// attend.cu — exact softmax attention over the selected NVFP4 blocks (decode).
//
// "Main attention then runs exactly, but only over the top 16 blocks ... That
// caps each query at 2,048 keys" ("vLLM Adds Day-0 Support for
// MiniMax-M3.1-Flash", ainewsbites.com, "A model built for efficient
// inference").  Query head h reads KV head h / (Hq/Hkv); keys j > pos are
// masked; K and V are NVFP4 and dequantised in registers.
//
// Design (B200): one thread-block cluster of 4 CTAs x 4 warps per
// (sequence, query token, KV head): each of the 16 warps takes one selected
// block (split-K over the <= 16 blocks).  Each warp streams its block as four
// 32-key quarters (K and V nibbles + scales, 4.5 KB each) through a private
// 2-stage shared-memory ring with untiled bulk copies (cp.async.bulk, no
// multicast), so the next quarter lands while the current one is computed;
// 37 KB of shared memory and <= 128 registers per CTA let 4 CTAs (16 warps)
// share an SM and the whole 32 x 64K decode grid run in one wave.  Per quarter:
//   S^T = K Q^T    mma m16n8k16, A = dequantised K (exact f16, 16 keys),
//                  B = the G query heads of this KV head (8 columns) — the
//                  same tile routine as the indexer, no padded rows;
//   softmax        online over quarters (exp2 domain, fp32);
//   O^T += V^T P^T mma m16n8k16, A = dequantised V, B = P^T obtained from the
//                  S^T accumulators by one movmatrix (8x8 transpose) per 8 keys;
//                  output tile [128 dims x 8 heads], no padded rows.
// The partial (m, l, O) of the 4 warps are merged in shared memory, then the 4
// CTAs of the cluster merge through distributed shared memory (each CTA
// finalises 32 of the 128 dims).  No global scratch, no second launch, a
// fixed merge order (bitwise deterministic).
#include <cooperative_groups.h>

#include "internal.h"
#include "nvfp4_mma.cuh"
#include "select_row.cuh"

namespace msa {
namespace {

namespace cg = cooperative_groups;

constexpr int kAttWarps = 4;
constexpr int kAttCluster = 4;
constexpr int kAttThreads = 32 * kAttWarps;
constexpr int kD = 128;
constexpr int64_t kFusedSelectMaxBlocks = 1024;  // rows one warp selects from registers
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Per-warp ring of 2 shared-memory stages, each one 32-key quarter of the warp's
// block (K and V nibbles + scales of one KV head, 4.5 KB).
constexpr int kQuarter = 32;
constexpr int kKData = kQuarter * 64, kKScale = kQuarter * 8;
constexpr int kStage = 2 * (kKData + kKScale);  // 4.5 KB
constexpr int kWarpSmem = 2 * kStage;           // 9 KB: also holds the warp's partial O (4 KB) at the end
constexpr size_t kAttSmem = (size_t)kAttWarps * kWarpSmem + 2 * kAttWarps * sizeof(uint64_t) + 2 * 8 * sizeof(float);

// FUSED: the CTA first selects its row's blocks from the pooled scores (warp 0,
// rows of <= 1,024 blocks) instead of reading a selection written by select.cu.
template <int G, bool FUSED>
__global__ void __cluster_dims__(kAttCluster, 1, 1) __launch_bounds__(kAttThreads, 4)
    attend_kernel(const Problem p, const int32_t* __restrict__ sel, const float* __restrict__ block_scores,
                  int32_t* __restrict__ sel_out, float* __restrict__ out, float* __restrict__ lse) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAttWarps * kWarpSmem);  // [warp][2]
    float* cM = reinterpret_cast<float*>(bars + 2 * kAttWarps);
    float* cL = cM + 8;
    __shared__ float sM[kAttWarps][8], sL[kAttWarps][8];
    __shared__ int sh_sel[kTopK];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    uint8_t* wsm = smem + warp * kWarpSmem;
    uint64_t* wb = bars + 2 * warp;
    if (lane == 0) {
        mbar_init(&wb[0], 1);
        mbar_init(&wb[1], 1);
        fence_mbar_init();
    }
    __syncwarp();

    pdl_wait();
    pdl_launch_dependents();

    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int64_t unit = blockIdx.x / kAttCluster;  // ((b * Tq) + t) * Hkv + kvh
    const int kvh = (int)(unit % p.Hkv);
    const int64_t bt = unit / p.Hkv;
    const int b = (int)(bt / p.Tq), t = (int)(bt % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t pos = L - p.Tq + t;
    const int64_t nvis = pos / kBlock + 1;
    const int gw = crank * kAttWarps + warp;

    // query fragments: column g = query head kvh*G + g, dims permuted as the K rows
    uint32_t qf[1][8][2];
    if (g < G) {
        const __nv_bfloat16* qrow = p.q + ((bt * p.Hq) + (int64_t)kvh * G + g) * kD + c * 32;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(qrow + 8 * v);
            qf[0][2 * v][0] = bf16x2_to_f16x2(w4.x);
            qf[0][2 * v][1] = bf16x2_to_f16x2(w4.y);
            qf[0][2 * v + 1][0] = bf16x2_to_f16x2(w4.z);
            qf[0][2 * v + 1][1] = bf16x2_to_f16x2(w4.w);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qf[0][i][0] = qf[0][i][1] = 0u;
    }

    int blk;
    if constexpr (FUSED) {
        if (warp == 0) {
            const float* srow = block_scores + bt * p.nbmax;
            const int64_t r = nvis - 1;
            const int id = nvis <= 512 ? select_row_warp<16>(srow, nvis, r, lane) : select_row_warp<32>(srow, nvis, r, lane);
            if (lane < kTopK) {
                sh_sel[lane] = id;
                if (sel_out != nullptr && crank == 0 && kvh == 0) sel_out[bt * kTopK + lane] = id;
            }
        }
        __syncthreads();
        blk = gw < kTopK ? sh_sel[gw] : -1;
    } else {
        blk = gw < kTopK ? sel[bt * kTopK + gw] : -1;
    }
    if (blk >= nvis) {
        if (lane == 0) set_status(p.status, MSA_STATUS_SELECT);
        blk = -1;
    }
    int nk = 0, nq = 0;
    int64_t vec0 = 0;
    if (blk >= 0) {
        const int64_t kbase = (int64_t)blk * kBlock;
        nk = (int)min64(kBlock, pos + 1 - kbase);
        nq = (nk + kQuarter - 1) / kQuarter;
        vec0 = ((int64_t)b * p.Hkv + kvh) * p.lmax + kbase;
    }
    // quarter j of the block -> stage j & 1 (rows rounded up to 16; the cache holds whole blocks)
    auto issue = [&](int j) {
        const int rows = (min(kQuarter, nk - j * kQuarter) + 15) & ~15;
        uint8_t* st = wsm + (j & 1) * kStage;
        const int64_t v = vec0 + j * kQuarter;
        mbar_arrive_expect_tx(&wb[j & 1], (uint32_t)(2 * rows * (64 + 8)));
        bulk_g2s(st, p.k.data + v * 64, (uint32_t)(rows * 64), &wb[j & 1]);
        bulk_g2s(st + kKData, p.k.scale + v * 8, (uint32_t)(rows * 8), &wb[j & 1]);
        bulk_g2s(st + kKData + kKScale, p.v.data + v * 64, (uint32_t)(rows * 64), &wb[j & 1]);
        bulk_g2s(st + 2 * kKData + kKScale, p.v.scale + v * 8, (uint32_t)(rows * 8), &wb[j & 1]);
    };
    if (lane == 0) {
        if (nq > 0) issue(0);
        if (nq > 1) issue(1);
    }

    const float sc_log2 = p.softmax_scale * p.k.s_t * kLog2e;
    // per thread: query heads 2c and 2c+1
    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.0f, 0.0f};
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.0f;

    for (int j = 0; j < nq; ++j) {
        if (!mbar_wait(&wb[j & 1], (j >> 1) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_ATTEND);
            // one more bounded wait for the copies still in flight before the stages are reused
            for (int jj = j; jj < min(nq, j + 2); ++jj) mbar_wait(&wb[jj & 1], (jj >> 1) & 1u);
            nq = j;
            break;
        }
        const uint8_t* st = wsm + (j & 1) * kStage;
        const uint8_t* kd = st;
        const uint8_t* ksc = st + kKData;
        const uint8_t* vd = st + kKData + kKScale;
        const uint8_t* vsc = st + 2 * kKData + kKScale;
        const int qvalid = min(kQuarter, nk - j * kQuarter);
        const int ntiles = (qvalid + 15) >> 4;
        // ---- S^T = K Q^T for the quarter's keys: st4[kt] = rows (keys) g, g+8 x cols 2c, 2c+1
        float s4[2][4];
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            if (kt < ntiles) {
                float acc[1][4];
                nvfp4_tile_mma<128, 1>(kd, ksc, kt * 16 + g, c, qf, acc);
                const bool v0 = kt * 16 + g < qvalid, v1 = kt * 16 + g + 8 < qvalid;
                s4[kt][0] = v0 ? acc[0][0] * sc_log2 : -INFINITY;
                s4[kt][1] = v0 ? acc[0][1] * sc_log2 : -INFINITY;
                s4[kt][2] = v1 ? acc[0][2] * sc_log2 : -INFINITY;
                s4[kt][3] = v1 ? acc[0][3] * sc_log2 : -INFINITY;
            } else {
                s4[kt][0] = s4[kt][1] = s4[kt][2] = s4[kt][3] = -INFINITY;
            }
        }
        // ---- online softmax over the quarter (query heads 2c, 2c+1), exp2 domain
        float corr[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(fmaxf(s4[0][e], s4[0][2 + e]), fmaxf(s4[1][e], s4[1][2 + e]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m2[e], mx);
            corr[e] = exp2f(m2[e] - m_new);
            m2[e] = m_new;
            float l = 0.0f;
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                s4[kt][e] = exp2f(s4[kt][e] - m_new);
                s4[kt][2 + e] = exp2f(s4[kt][2 + e] - m_new);
                l += s4[kt][e] + s4[kt][2 + e];
            }
            l2[e] = l2[e] * corr[e] + l;
        }
        if (j > 0) {
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                o[mt][0] *= corr[0];
                o[mt][1] *= corr[1];
                o[mt][2] *= corr[0];
                o[mt][3] *= corr[1];
            }
        }
        // ---- O^T += V^T P^T, 16 keys at a time
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            if (kt < ntiles) {
                // P^T fragment (keys x heads) -> B operand (k = keys 2c.., n = head g)
                const uint32_t pb0 = movmatrix_trans(pack_f16x2(s4[kt][0], s4[kt][1]));
                const uint32_t pb1 = movmatrix_trans(pack_f16x2(s4[kt][2], s4[kt][3]));
                uint32_t vh[4][8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int key = kt * 16 + 2 * c + (i & 1) + 8 * (i >> 1);
                    uint2 vw = make_uint2(0u, 0u);
                    uint32_t vs = 0u;
                    if (key < qvalid) {  // masked keys read as 0 (their P is 0; V may hold anything)
                        vw = lds_v2(vd + key * 64 + g * 8);
                        vs = lds_u8(vsc + key * 8 + g);
                    }
                    e2m1x8_to_f16x8(vw.x, vh[i][0], vh[i][1], vh[i][2], vh[i][3]);
                    e2m1x8_to_f16x8(vw.y, vh[i][4], vh[i][5], vh[i][6], vh[i][7]);
                    const uint32_t sc = e4m3_bcast_f16x2(vs);
#pragma unroll
                    for (int m = 0; m < 8; ++m) vh[i][m] = hmul2(vh[i][m], sc);
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const uint32_t a0 = prmt(vh[0][mt], vh[1][mt], 0x5410u);
                    const uint32_t a1 = prmt(vh[0][mt], vh[1][mt], 0x7632u);
                    const uint32_t a2 = prmt(vh[2][mt], vh[3][mt], 0x5410u);
                    const uint32_t a3 = prmt(vh[2][mt], vh[3][mt], 0x7632u);
                    mma16816(o[mt], a0, a1, a2, a3, pb0, pb1);
                }
            }
        }
        __syncwarp();  // every lane is done with stage j & 1
        if (lane == 0 && j + 2 < nq) issue(j + 2);
    }
    uint8_t* stage = wsm;

    // ---- merge the 4 warps of this CTA (each warp's partial O goes into its own stage)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = l2[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (g == 0) {
            sM[warp][2 * c + e] = m2[e];
            sL[warp][2 * c + e] = l;
        }
    }
    __syncwarp();
    float* sOw = reinterpret_cast<float*>(stage);  // [8][kD]
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
        const int d = 16 * g + 2 * mt;
        sOw[(2 * c) * kD + d] = o[mt][0];
        sOw[(2 * c + 1) * kD + d] = o[mt][1];
        sOw[(2 * c) * kD + d + 1] = o[mt][2];
        sOw[(2 * c + 1) * kD + d + 1] = o[mt][3];
    }
    __syncthreads();
    float* sO0 = reinterpret_cast<float*>(smem);  // the CTA's merged partial, in warp 0's stage
    {
        const int q = threadIdx.x >> 4, d0 = (threadIdx.x & 15) * 8;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, sM[w][q]);
        float f[kAttWarps], Lc = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) {
            f[w] = sM[w][q] == -INFINITY ? 0.0f : exp2f(sM[w][q] - M);
            Lc += f[w] * sL[w][q];
        }
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) {
            const float* src = reinterpret_cast<const float*>(smem + w * kWarpSmem) + q * kD + d0;
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] += f[w] * src[j];
        }
        // every read of this (q, d0..d0+7) slice happened in this thread: safe to overwrite
#pragma unroll
        for (int j = 0; j < 8; ++j) sO0[q * kD + d0 + j] = acc[j];
        if ((threadIdx.x & 15) == 0) {
            cM[q] = M;
            cL[q] = Lc;
        }
    }
    cluster.sync();

    // ---- merge the 4 CTAs of the cluster: CTA r finalises dims [32r, 32r + 32)
    {
        const int q = threadIdx.x >> 4, d = 32 * crank + (threadIdx.x & 15) * 2;
        float Mr[kAttCluster], Lr[kAttCluster], O0[kAttCluster], O1[kAttCluster];
#pragma unroll
        for (int r = 0; r < kAttCluster; ++r) {
            const float* pm = cluster.map_shared_rank(cM, r);
            const float* pl = cluster.map_shared_rank(cL, r);
            const float* po = cluster.map_shared_rank(sO0, r);
            Mr[r] = pm[q];
            Lr[r] = pl[q];
            const float2 v2 = *reinterpret_cast<const float2*>(po + q * kD + d);
            O0[r] = v2.x;
            O1[r] = v2.y;
        }
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < kAttCluster; ++r) M = fmaxf(M, Mr[r]);
        float Lt = 0.0f, a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int r = 0; r < kAttCluster; ++r) {
            const float f = Mr[r] == -INFINITY ? 0.0f : exp2f(Mr[r] - M);
            Lt += f * Lr[r];
            a0 += f * O0[r];
            a1 += f * O1[r];
        }
        if (q < G) {
            const float inv = Lt > 0.0f ? p.v.s_t / Lt : 0.0f;
            float* orow = out + ((bt * p.Hq) + (int64_t)kvh * G + q) * kD;
            *reinterpret_cast<float2*>(orow + d) = make_float2(a0 * inv, a1 * inv);
            if (lse != nullptr && crank == 0 && (threadIdx.x & 15) == 0)
                lse[bt * p.Hq + (int64_t)kvh * G + q] = Lt > 0.0f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
        }
    }
    cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

template <int G, bool FUSED>
int launch_g(const Problem& p, const int32_t* sel, const float* bs, int32_t* sel_out, float* out, float* lse,
             bool pdl, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Tq * p.Hkv;
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(attend_kernel<G, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kAttSmem) != cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * kAttCluster));
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = kAttSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attend_kernel<G, FUSED>, p, sel, bs, sel_out, out, lse) != cudaSuccess)
        return MSA_ECUDA;
    return MSA_OK;
}

template <bool FUSED>
int launch_any(const Problem& p, const int32_t* sel, const float* bs, int32_t* sel_out, float* out, float* lse,
               bool pdl, cudaStream_t st) {
    if (p.D != kD) return MSA_EUNSUPPORTED;
    const int64_t units = (int64_t)p.B * p.Tq * p.Hkv;
    if (units * kAttCluster > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    switch (p.Hq / p.Hkv) {
        case 1: return launch_g<1, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 2: return launch_g<2, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 4: return launch_g<4, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 8: return launch_g<8, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        default: return MSA_EUNSUPPORTED;
    }
}

}  // namespace

int launch_attend(const Problem& p, const int32_t* sel, float* out, float* lse, bool pdl, cudaStream_t st) {
    return launch_any<false>(p, sel, nullptr, nullptr, out, lse, pdl, st);
}

int launch_select_attend(const Problem& p, const float* block_scores, int32_t* sel_out, float* out, float* lse,
                         bool pdl, cudaStream_t st) {
    if (p.nbmax > kFusedSelectMaxBlocks) return MSA_EUNSUPPORTED;
    return launch_any<true>(p, nullptr, block_scores, sel_out, out, lse, pdl, st);
}

}  // namespace msa
