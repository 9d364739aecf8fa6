// attend.cu — exact softmax attention over the selected NVFP4 blocks (decode).
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com,
// section "A model built for efficient inference"): softmax attention is computed
// exactly, but only over the 16 selected blocks of 128 tokens, so no query reads
// more than 2,048 keys.  Query head h reads KV head h / (Hq/Hkv); keys j > pos
// are masked; K and V are NVFP4 and dequantised in registers.
//
// Design (B200): one thread-block cluster of 4 CTAs x 4 warps per
// (sequence, query token, KV head): each of the 16 warps takes one selected
// block (split-K over the <= 16 blocks); grids of few such units use clusters
// of 8 CTAs (two warps per block) or 16 (four, one 32-key quarter each) to
// shorten each warp's serial chain.  Each warp streams its keys as 32-key quarters
// (K and V nibbles + scales, 4.5 KB each) through a private
// 2-stage shared-memory ring with untiled bulk copies (cp.async.bulk, no
// multicast), so the next quarter lands while the current one is computed;
// 37 KB of shared memory and <= 128 registers per CTA let 4 CTAs (16 warps)
// share an SM and the whole 32 x 64K decode grid run in one wave.  The
// per-quarter step (S^T = K Q^T, online softmax, O^T += V^T P^T on mma.sync
// m16n8k16 with K and V dequantised in registers) is att_quarter() of
// attend_quarter.cuh.
// The partial (m, l, O) of the 4 warps are merged in shared memory, then the
// CTAs of the cluster merge through distributed shared memory (each CTA
// finalises 128 / CL of the 128 dims).  With the selection fused in (rows of
// <= 1,024 blocks), every CTA first selects the row's blocks.  No global scratch,
// no second launch, a fixed merge order (bitwise deterministic).
#include <cooperative_groups.h>

#include "internal.h"
#include "attend_quarter.cuh"
#include "select_row.cuh"

namespace msa {
namespace {

namespace cg = cooperative_groups;

constexpr int kAttWarps = 4;
constexpr int kAttThreads = 32 * kAttWarps;
constexpr int kD = kAttD;
constexpr int64_t kFusedSelectMaxBlocks = 1024;  // rows one warp selects from registers

// Per-warp ring of 2 shared-memory stages, each one 32-key quarter of the warp's block.
constexpr int kWarpSmem = 2 * kAttStageBytes;  // 9 KB: also holds the warp's partial O (4 KB) at the end
constexpr size_t kAttSmem = (size_t)kAttWarps * kWarpSmem + 2 * kAttWarps * sizeof(uint64_t) + 2 * 8 * sizeof(float);

// FUSED: the CTA first selects its row's blocks from the pooled scores (rows of <= 1,024
// blocks: warp 0 alone up to 128, else all 4 warps in two levels) instead of reading a
// selection written by select.cu.
template <int G, bool FUSED, int CL>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(kAttThreads, 4)
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

    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    constexpr int kWPB = CL / 4;             // warps per selected block (1 or 2)
    constexpr int kQPW = 4 / kWPB;           // quarters per warp
    const int64_t unit = blockIdx.x / CL;  // ((b * Tq) + t) * Hkv + kvh
    const int kvh = (int)(unit % p.Hkv);
    const int64_t bt = unit / p.Hkv;
    const int b = (int)(bt / p.Tq), t = (int)(bt % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t pos = L - p.Tq + t;
    const int64_t nvis = pos / kBlock + 1;
    const int gw = crank * kAttWarps + warp;

    // The queries and lengths are not written by the kernel this one waits for (the
    // indexer or the selection, which waited for their own predecessors before letting
    // this grid start), so they load before the wait.
    uint32_t qf[1][8][2];
    att_load_q(p, bt, kvh, G, g, c, qf);

    pdl_wait();
    pdl_launch_dependents();

    int blk;
    if constexpr (FUSED) {
        const float* srow = block_scores + bt * p.nbmax;
        const int64_t r = nvis - 1;
        if (nvis <= 128) {
            if (warp == 0) select_row_warp<4>(srow, nvis, r, lane, sh_sel);
        } else {  // the CTA's 4 warps: 128 or 256 blocks each, then warp 0 over the 60 candidates
            __shared__ uint32_t ckey[kAttWarps * (kTopK - 1)];
            __shared__ int32_t cid[kAttWarps * (kTopK - 1)];
            if (nvis <= 512) select_row_cta<kAttWarps, 4>(srow, nvis, r, warp, lane, ckey, cid, sh_sel);
            else select_row_cta<kAttWarps, 8>(srow, nvis, r, warp, lane, ckey, cid, sh_sel);
        }
        __syncthreads();
        if (warp == 0 && lane < kTopK && sel_out != nullptr && crank == 0 && kvh == 0)
            sel_out[bt * kTopK + lane] = sh_sel[lane];
        blk = sh_sel[gw / kWPB];
    } else {
        blk = sel[bt * kTopK + gw / kWPB];
    }
    if (blk >= nvis) {
        if (lane == 0) set_status(p.status, MSA_STATUS_SELECT);
        blk = -1;
    }
    if (blk < p.blk_lo || blk >= p.blk_hi) blk = -1;  // another rank's block (context-parallel decode)
    int nk = 0, nq = 0;
    int64_t vec0 = 0;
    if (blk >= 0) {
        // this warp's part of the block: keys [part * 32 kQPW, (part + 1) * 32 kQPW)
        const int part0 = (gw % kWPB) * (kQPW * kAttQuarter);
        const int64_t kbase = (int64_t)blk * kBlock + part0;
        nk = (int)max64(0, min64(kQPW * kAttQuarter, pos + 1 - kbase));
        nq = (nk + kAttQuarter - 1) / kAttQuarter;
        vec0 = block_vec_any(p, b, blk, kvh, p.Hkv) + part0;
    }
    // quarter j of the block -> stage j & 1 (rows rounded up to 16; the cache holds whole blocks)
    auto issue = [&](int j) {
        const int rows = (min(kAttQuarter, nk - j * kAttQuarter) + 15) & ~15;
        att_issue_quarter(p, wsm + (j & 1) * kAttStageBytes, vec0 + j * kAttQuarter, rows, &wb[j & 1]);
    };
    if (lane == 0) {
        if (nq > 0) issue(0);
        if (nq > 1) issue(1);
    }

    const float sc_log2 = p.softmax_scale * p.k.s_t * kLog2e;
    AttAcc acc;
    att_init(acc);
    for (int j = 0; j < nq; ++j) {
        if (!mbar_wait(&wb[j & 1], (j >> 1) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_ATTEND);
            // one more bounded wait for the copies still in flight before the stages are reused
            for (int jj = j; jj < min(nq, j + 2); ++jj) mbar_wait(&wb[jj & 1], (jj >> 1) & 1u);
            nq = j;
            break;
        }
        att_quarter(wsm + (j & 1) * kAttStageBytes, min(kAttQuarter, nk - j * kAttQuarter), j == 0, qf, sc_log2, g,
                    c, acc);
        __syncwarp();  // every lane is done with stage j & 1
        if (lane == 0 && j + 2 < nq) issue(j + 2);
    }
    // ---- merge the 4 warps of this CTA (each warp's partial O goes into its own stage)
    att_reduce_l(acc);
    if (g == 0) {
        sM[warp][2 * c] = acc.m2[0];
        sM[warp][2 * c + 1] = acc.m2[1];
        sL[warp][2 * c] = acc.l2[0];
        sL[warp][2 * c + 1] = acc.l2[1];
    }
    __syncwarp();
    att_store_o(reinterpret_cast<float*>(wsm), g, c, acc);
    __syncthreads();
    float* sO0 = reinterpret_cast<float*>(smem);  // the CTA's merged partial, in warp 0's stage
    {
        // thread t merges float2 slots t, t + 128, t + 256, t + 384 of the [64][8] (pair, head)
        // array: all of head q = t % 8 (consecutive threads read consecutive 8-byte words)
        const int q = threadIdx.x & 7;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, sM[w][q]);
        float f[kAttWarps], Lc = 0.0f;
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) {
            f[w] = sM[w][q] == -INFINITY ? 0.0f : exp2f(sM[w][q] - M);
            Lc += f[w] * sL[w][q];
        }
        float2 acc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int w = 0; w < kAttWarps; ++w) {
            const float2* src = reinterpret_cast<const float2*>(smem + w * kWarpSmem);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 v = src[threadIdx.x + 128 * j];
                acc[j].x += f[w] * v.x;
                acc[j].y += f[w] * v.y;
            }
        }
        // every read of these slots happened in this thread: safe to overwrite
#pragma unroll
        for (int j = 0; j < 4; ++j) reinterpret_cast<float2*>(sO0)[threadIdx.x + 128 * j] = acc[j];
        if (threadIdx.x < 8) {
            cM[q] = M;
            cL[q] = Lc;
        }
    }
    cluster.sync();

    // ---- merge the CL CTAs of the cluster: CTA r finalises float2 slots [512 r / CL,
    // 512 (r + 1) / CL) of the (pair, head) array; slot e holds head e % 8 of dim pair e / 8
    if (threadIdx.x < 512 / CL) {
        const int e = (512 / CL) * crank + threadIdx.x;
        const int q = e & 7, pi = e >> 3;
        float Mr[CL], Lr[CL];
        float2 Or[CL];
#pragma unroll
        for (int r = 0; r < CL; ++r) {
            const float* pm = cluster.map_shared_rank(cM, r);
            const float* pl = cluster.map_shared_rank(cL, r);
            const float2* po = reinterpret_cast<const float2*>(cluster.map_shared_rank(sO0, r));
            Mr[r] = pm[q];
            Lr[r] = pl[q];
            Or[r] = po[e];
        }
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < CL; ++r) M = fmaxf(M, Mr[r]);
        float Lt = 0.0f, a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int r = 0; r < CL; ++r) {
            const float f = Mr[r] == -INFINITY ? 0.0f : exp2f(Mr[r] - M);
            Lt += f * Lr[r];
            a0 += f * Or[r].x;
            a1 += f * Or[r].y;
        }
        if (q < G) {
            const float inv = Lt > 0.0f ? p.v.s_t / Lt : 0.0f;
            store_out2(p, out, ((bt * p.Hq) + (int64_t)kvh * G + q) * kD + 2 * pi, a0 * inv, a1 * inv);
            if (lse != nullptr && crank == 0 && threadIdx.x < 8)
                lse[bt * p.Hq + (int64_t)kvh * G + q] = Lt > 0.0f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
        }
    }
    cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

template <int G, bool FUSED, int CL>
int launch_g(const Problem& p, const int32_t* sel, const float* bs, int32_t* sel_out, float* out, float* lse,
             bool pdl, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Tq * p.Hkv;
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(attend_kernel<G, FUSED, CL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kAttSmem) != cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * CL));
    cfg.blockDim = dim3(kAttThreads);
    cfg.dynamicSmemBytes = kAttSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attend_kernel<G, FUSED, CL>, p, sel, bs, sel_out, out, lse) != cudaSuccess)
        return MSA_ECUDA;
    return MSA_OK;
}

// Clusters of 16 CTAs (a non-portable size: used only where the device accepts it) with 4
// warps per selected block, one quarter each
template <int G, bool FUSED>
bool cluster16_ok() {
    static int ok_dev = -2, ok = 0;
    const DeviceInfo& di = device_info();
    if (ok_dev != di.device) {
        ok = 0;
        auto kern = attend_kernel<G, FUSED, 16>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttSmem) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(16);
            cfg.blockDim = dim3(kAttThreads);
            cfg.dynamicSmemBytes = kAttSmem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 16;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0) ok = 1;
        }
        cudaGetLastError();  // a refused query leaves no sticky error behind
        ok_dev = di.device;
    }
    return ok != 0;
}

// Few (row, KV head) units: clusters of 16 CTAs (one quarter-block per warp) when 16 CTAs per
// unit still fit in one wave of one CTA per SM, clusters of 8 (two warps per block) when the
// units are at most half the SM count, else clusters of 4 (one warp per block).  Smaller
// pieces per warp shorten each warp's serial chain where the grid leaves SMs idle.
template <int G, bool FUSED>
int launch_cl(const Problem& p, const int32_t* sel, const float* bs, int32_t* sel_out, float* out, float* lse,
              bool pdl, cudaStream_t st) {
    const int64_t units = (int64_t)p.B * p.Tq * p.Hkv;
    const int sms = device_info().num_sms;
    if (16 * units <= sms && cluster16_ok<G, FUSED>())
        return launch_g<G, FUSED, 16>(p, sel, bs, sel_out, out, lse, pdl, st);
    if (2 * units <= sms) return launch_g<G, FUSED, 8>(p, sel, bs, sel_out, out, lse, pdl, st);
    return launch_g<G, FUSED, 4>(p, sel, bs, sel_out, out, lse, pdl, st);
}

template <bool FUSED>
int launch_any(const Problem& p, const int32_t* sel, const float* bs, int32_t* sel_out, float* out, float* lse,
               bool pdl, cudaStream_t st) {
    if (p.D != kD) return MSA_EUNSUPPORTED;
    const int64_t units = (int64_t)p.B * p.Tq * p.Hkv;
    if (units * 8 > 0x7FFFFFFFll) return MSA_EUNSUPPORTED;
    switch (p.Hq / p.Hkv) {
        case 1: return launch_cl<1, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 2: return launch_cl<2, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 4: return launch_cl<4, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
        case 8: return launch_cl<8, FUSED>(p, sel, bs, sel_out, out, lse, pdl, st);
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
