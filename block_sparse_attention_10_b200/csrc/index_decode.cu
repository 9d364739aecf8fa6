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
//     untiled bulk copies (cp.async.bulk, no multicast) of 4.5 KB stages (64
//     keys at DI = 128, a whole block at DI = 64) into the warp's private ring
//     of 3 shared-memory stages, two ahead of the one being computed, each
//     stage with its own mbarrier.  A warp only ever waits on its own stages,
//     in order, so ~150 KB per SM are in flight while every warp computes.
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
//     (token, block) — the per-block routine of index_block.cuh.
#include "index_block.cuh"

namespace msa {
namespace {

constexpr int kIdxWarps = 8;
constexpr int kIdxThreads = 32 * kIdxWarps;
constexpr int kMaxB = 4096;
constexpr int kIdxRing = 3;  // stages per warp: 13.5 KB

constexpr size_t idx_smem_bytes(int B) {
    return (size_t)kIdxWarps * kIdxRing * (kIdxStageBytes + sizeof(uint64_t)) + (size_t)(2 * B + 2) * sizeof(int);
}

template <int DI, int HI, int NT, bool PAGED>
__global__ void __launch_bounds__(kIdxThreads, 2)
    index_decode_kernel(const Problem p, float* __restrict__ block_scores, float* __restrict__ token_scores) {
    constexpr int R = kIdxRing;
    constexpr int KPS = idx_stage_keys<DI>();

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kIdxWarps * R * kIdxStageBytes);
    int* prefix = reinterpret_cast<int*>(bars + kIdxWarps * R);  // [B + 1] units before sequence b
    int* lens = prefix + (p.B + 1);                               // [B] clamped lengths

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int B = p.B, Tq = p.Tq;
    uint8_t* my_stages = smem + warp * R * kIdxStageBytes;
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
                // the sequence's blocks inside [blk_lo, blk_hi)
                nb = (int)max64(0, min64((L + kBlock - 1) / kBlock, p.blk_hi) - p.blk_lo);
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

    // blocks past a sequence's length, or outside [blk_lo, blk_hi), score -inf (no unit covers them)
    {
        const int64_t total = (int64_t)B * Tq * p.nbmax;
        const int64_t stride = (int64_t)gridDim.x * kIdxThreads;
        for (int64_t i = (int64_t)blockIdx.x * kIdxThreads + threadIdx.x; i < total; i += stride) {
            const int64_t n = i % p.nbmax - p.blk_lo;
            const int b = (int)(i / (p.nbmax * Tq));
            if (n < 0 || n >= prefix[b + 1] - prefix[b]) block_scores[i] = -INFINITY;
        }
    }

    // this warp's contiguous range of units (sequence, block)
    const int64_t U = prefix[B];
    const int64_t Wt = (int64_t)gridDim.x * kIdxWarps;
    const int64_t gw = (int64_t)blockIdx.x * kIdxWarps + warp;
    const int64_t u_begin = U * gw / Wt, u_end = U * (gw + 1) / Wt;

    // issue side: walks the same (unit, stage) sequence as the compute side, R stages ahead
    int64_t iu = u_begin;
    int is = 0, ib = 0;
    uint32_t slot_issued = 0;
    auto issue_upto = [&](uint32_t limit) {
        while (slot_issued < limit && iu < u_end) {
            while (prefix[ib + 1] <= iu) ++ib;
            const int64_t n = p.blk_lo + (iu - prefix[ib]);
            const int valid = (int)min64(kBlock, lens[ib] - n * kBlock) - is * KPS;
            if (valid > 0) {
                if (lane == 0) {
                    const int rows = (min(valid, KPS) + 15) & ~15;
                    const int s = (int)(slot_issued % R);
                    const int64_t row0 = block_vec<PAGED>(p, ib, n, 0, 1) + is * KPS;
                    uint8_t* st = my_stages + s * kIdxStageBytes;
                    const uint32_t db = (uint32_t)(rows * (DI / 2)), sb = (uint32_t)(rows * (DI / 16));
                    mbar_arrive_expect_tx(&my_bars[s], db + sb);
                    bulk_g2s(st, p.ik.data + row0 * (DI / 2), db, &my_bars[s]);
                    bulk_g2s(st + kIdxStageData, p.ik.scale + row0 * (DI / 16), sb, &my_bars[s]);
                }
                ++slot_issued;
            }
            if (++is == kBlock / KPS) {
                is = 0;
                ++iu;
            }
        }
    };
    uint32_t slot = 0;
    // the next stage of this warp's stream (in order), or nullptr after a timeout
    auto acquire = [&]() -> const uint8_t* {
        issue_upto(slot + R);
        const int s = (int)(slot % R);
        if (!mbar_wait(&my_bars[s], (slot / R) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_CONSUMER);
            return nullptr;
        }
        ++slot;
        return my_stages + s * kIdxStageBytes;
    };

    IdxQuery<DI, NT> q;
    int cur_b = -1;
    int b = 0;
    for (int64_t u = u_begin; u < u_end; ++u) {
        while (prefix[b + 1] <= u) ++b;
        if (b != cur_b) {
            cur_b = b;
            idx_load_query<DI, HI, NT>(p, b, g, c, q);
        }
        if (!idx_block<DI, HI, NT>(p, b, p.blk_lo + (u - prefix[b]), lens[b], q, acquire, block_scores, token_scores,
                                   g, c))
            break;
    }
    // never leave with copies in flight into this warp's stages
    for (uint32_t j = slot; j < slot_issued; ++j)
        if (!mbar_wait(&my_bars[j % R], (j / R) & 1u)) {
            if (lane == 0) set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_DRAIN);
            break;
        }
}

template <int DI, int HI, int NT, bool PAGED>
int launch_t(const Problem& p, float* bs, float* ts, bool pdl, cudaStream_t st) {
    auto kern = index_decode_kernel<DI, HI, NT, PAGED>;
    const size_t smem = idx_smem_bytes(p.B);
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)idx_smem_bytes(kMaxB)) != cudaSuccess)
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
    const bool paged = p.block_table != nullptr;
    if (nq <= 8) return paged ? launch_t<DI, HI, 1, true>(p, bs, ts, pdl, st) : launch_t<DI, HI, 1, false>(p, bs, ts, pdl, st);
    if (nq <= 16) return paged ? launch_t<DI, HI, 2, true>(p, bs, ts, pdl, st) : launch_t<DI, HI, 2, false>(p, bs, ts, pdl, st);
    if (nq <= 24) return paged ? launch_t<DI, HI, 3, true>(p, bs, ts, pdl, st) : launch_t<DI, HI, 3, false>(p, bs, ts, pdl, st);
    return paged ? launch_t<DI, HI, 4, true>(p, bs, ts, pdl, st) : launch_t<DI, HI, 4, false>(p, bs, ts, pdl, st);
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
