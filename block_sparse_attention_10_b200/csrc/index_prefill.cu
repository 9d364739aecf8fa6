// index_prefill.cu — MSA indexer + block pooling for a chunk of many query tokens
// (chunked prefill), on the fifth-generation tensor cores.
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com,
// "A model built for efficient inference"): every query scores every visible
// key with the lightweight indexer, and the scores are pooled per 128-token
// block.  With Tq query tokens and HI heads this is a dense contraction
// [Tq*HI rows x DI] x [DI x L keys] per sequence with a causal mask at the end
// of the context — the pages' prefill optimisation is a fused prefill path.
// Reading: s = sum_h w_h ReLU(q_h . k); mean over the block's visible keys.
// Because the mean is linear, the block score of token t is
//     S[t, n] = (1/cnt) * sum_h w_h * sum_{j in n, j <= pos_t} ReLU(q_{t,h} . k_j),
// so each accumulator row (one (token, head)) only needs its own ReLU-sum over
// the block's columns; the head sum happens once per (token, block).
//
// Design (B200, one persistent CTA per SM, 10 warps):
//   * work unit = (sequence, 256 keys = 2 MSA blocks, up to 64 query tiles);
//   * warps 0-7 dequantise each unit's 256 NVFP4 keys into one of two bf16
//     shared tiles in the canonical K-major 128-byte-swizzle layout (e2m1*e4m3
//     is exact in bf16; the fp32 tensor scale is applied to the pooled score)
//     and run the epilogue.  The next unit's keys are written into the other
//     tile at the start of the current unit, while the MMAs of its first two
//     query tiles run, so the tensor pipe does not drain at unit boundaries;
//   * warp 9 (one lane) streams 128-row query tiles [128 x DI] bf16 with TMA
//     (128-byte swizzle, no multicast) into a 3-stage ring;
//   * warp 8 (one lane) issues tcgen05.mma 128 x 256 x 16 (bf16 -> fp32 in
//     tensor memory), double-buffered over 2 x 256 TMEM columns, and commits
//     to mbarriers;
//   * epilogue: each warp reads its 32 TMEM lanes x 128 columns (one block)
//     with tcgen05.ld, sums ReLU over the visible columns, applies head
//     weights, sums heads with shuffles and writes one pooled score.
// Query tiles whose tokens see none of the unit's keys are skipped entirely.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "tcgen05.cuh"

namespace msa {
namespace {

constexpr int kPfEpiWarps = 8;
constexpr int kPfMmaWarp = 8;
constexpr int kPfTmaWarp = 9;
constexpr int kPfThreads = 32 * 10;
constexpr int kPfQStages = 3;
constexpr int kPfRows = 128;    // M: query rows (token, head) per tile
constexpr int kPfKeys = 256;    // N: keys per unit (2 MSA blocks)
constexpr int kPfQChunk = 64;   // query tiles per unit
constexpr int kPfTmemCols = 512;

template <int DI>
struct PfGeom {
    static constexpr int kKB = DI / 64;                   // 128-byte K-blocks per row
    static constexpr int kQStage = kPfRows * DI * 2;      // bytes per query stage
    static constexpr int kQBlock = kPfRows * 128;         // one K-block of a query stage
    static constexpr int kKTile = kPfKeys * DI * 2;       // bf16 key tile
    static constexpr int kKBlock = kPfKeys * 128;         // one K-block of the key tile
    static constexpr size_t kSmem = 1024 + 2 * kKTile + kPfQStages * kQStage + 256;
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

struct PfShape {
    int nqt;      // query tiles per sequence
    int nqc;      // query chunks per sequence
    int nkt;      // key tiles (2 blocks) per sequence capacity
    int64_t units;
};

__device__ __forceinline__ PfShape pf_shape(const Problem& p, int HI) {
    PfShape s;
    s.nqt = (p.Tq * HI + kPfRows - 1) / kPfRows;
    s.nqc = (s.nqt + kPfQChunk - 1) / kPfQChunk;
    s.nkt = (int)((p.nbmax + 1) / 2);
    s.units = (int64_t)p.B * s.nkt * s.nqc;
    return s;
}

// Does any token of query tile qt see any of the keys [k0, k0 + 256)?
template <int HI>
__device__ __forceinline__ bool pf_tile_live(int qt, int64_t k0, int64_t L, int Tq) {
    const int tb = min(Tq, (qt + 1) * (kPfRows / HI));  // one past the tile's last token
    return k0 < L && k0 <= L - Tq + tb - 1;
}

template <int DI, int HI, bool PAGED>
__global__ void __launch_bounds__(kPfThreads, 1)
    index_prefill_kernel(const Problem p, float* __restrict__ block_scores, const __grid_constant__ CUtensorMap tmap) {
    using G = PfGeom<DI>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* kbuf = smem;  // two key tiles
    uint8_t* qbuf = smem + 2 * G::kKTile;
    uint64_t* q_full = reinterpret_cast<uint64_t*>(qbuf + kPfQStages * G::kQStage);
    uint64_t* q_empty = q_full + kPfQStages;
    uint64_t* t_full = q_empty + kPfQStages;
    uint64_t* t_empty = t_full + 2;
    uint64_t* k_full = t_empty + 2;  // [2]: key tile complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(k_full + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPfQStages; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&t_full[s], 1);
            mbar_init(&t_empty[s], kPfEpiWarps);
        }
        mbar_init(&k_full[0], kPfEpiWarps);
        mbar_init(&k_full[1], kPfEpiWarps);
        fence_mbar_init();
    }
    if (warp == kPfMmaWarp) {
        tmem_alloc(tmem_slot, kPfTmemCols);
        tmem_relinquish();
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    const PfShape sh = pf_shape(p, HI);
    const int Tq = p.Tq;
    const float s_t = p.ik.s_t;

    if (warp == kPfTmaWarp) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t qi = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < sh.units && ok; u += gridDim.x) {
                const int b = (int)(u / ((int64_t)sh.nkt * sh.nqc));
                const int64_t rem = u % ((int64_t)sh.nkt * sh.nqc);
                const int64_t k0 = (rem / sh.nqc) * kPfKeys;
                const int qc = (int)(rem % sh.nqc);
                const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, nullptr);
                for (int qt = qc * kPfQChunk; qt < min(sh.nqt, (qc + 1) * kPfQChunk); ++qt) {
                    if (!pf_tile_live<HI>(qt, k0, L, Tq)) continue;
                    const int s = (int)(qi % kPfQStages);
                    if (qi >= (uint32_t)kPfQStages && !mbar_wait(&q_empty[s], ((qi / kPfQStages) - 1) & 1u)) {
                        set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_PRODUCER);
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&q_full[s], (uint32_t)G::kQStage);
#pragma unroll
                    for (int kb = 0; kb < G::kKB; ++kb)
                        tma_load_3d(qbuf + s * G::kQStage + kb * G::kQBlock, &tmap, kb * 64, qt * kPfRows, b,
                                    &q_full[s]);
                    ++qi;
                }
            }
            // never leave with copies in flight into this CTA's shared memory
            for (uint32_t j = qi > (uint32_t)kPfQStages ? qi - kPfQStages : 0u; j < qi; ++j)
                if (!mbar_wait(&q_full[j % kPfQStages], (j / kPfQStages) & 1u)) {
                    set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_DRAIN);
                    break;
                }
        }
    } else if (warp == kPfMmaWarp) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfRows, kPfKeys);
            uint32_t qi = 0, ui = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < sh.units && ok; u += gridDim.x) {
                const int b = (int)(u / ((int64_t)sh.nkt * sh.nqc));
                const int64_t rem = u % ((int64_t)sh.nkt * sh.nqc);
                const int64_t k0 = (rem / sh.nqc) * kPfKeys;
                const int qc = (int)(rem % sh.nqc);
                const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, nullptr);
                const int qt_end = min(sh.nqt, (qc + 1) * kPfQChunk);
                bool any = false;
                for (int qt = qc * kPfQChunk; qt < qt_end; ++qt) any |= pf_tile_live<HI>(qt, k0, L, Tq);
                if (!any) continue;
                if (!mbar_wait(&k_full[ui & 1u], (ui >> 1) & 1u)) {
                    set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_CONSUMER);
                    break;
                }
                tcgen05_fence_after();
                for (int qt = qc * kPfQChunk; qt < qt_end; ++qt) {
                    if (!pf_tile_live<HI>(qt, k0, L, Tq)) continue;
                    const int s = (int)(qi % kPfQStages);
                    const int buf = (int)(qi & 1u);
                    if (!mbar_wait(&q_full[s], (qi / kPfQStages) & 1u) ||
                        (qi >= 2 && !mbar_wait(&t_empty[buf], ((qi >> 1) - 1) & 1u))) {
                        set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_CONSUMER);
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t qs = smem_u32(qbuf + s * G::kQStage),
                                   ks = smem_u32(kbuf + (ui & 1u) * G::kKTile);
#pragma unroll
                    for (int k = 0; k < DI / 16; ++k) {
                        const int kb = k >> 2, kk = k & 3;
                        umma_bf16_ss(tmem_base + (uint32_t)(buf * kPfKeys),
                                     umma_desc_k_sw128(qs + kb * G::kQBlock + kk * 32),
                                     umma_desc_k_sw128(ks + kb * G::kKBlock + kk * 32), idesc, k > 0 ? 1u : 0u);
                    }
                    umma_commit(&q_empty[s]);
                    umma_commit(&t_full[buf]);
                    ++qi;
                }
                ++ui;
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue warps
        const int et = threadIdx.x;  // 0..255
        // blocks past each sequence's length score -inf: one (sequence, token) row per thread
        // of the grid, each writing only its row's blocks past the sequence's length
        for (int64_t r = (int64_t)blockIdx.x * 256 + et; r < (int64_t)p.B * Tq; r += (int64_t)gridDim.x * 256) {
            const int b = (int)(r / Tq);
            const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, r % Tq == 0 ? p.status : nullptr);
            for (int64_t n = (L + kBlock - 1) / kBlock; n < p.nbmax; ++n) block_scores[r * p.nbmax + n] = -INFINITY;
        }
        const int quad = warp & 3, hb = warp >> 2;
        // Key dequantisation: each thread owns one 8-element chunk column of every kKeyStep-th
        // key of an MSA block (keys >= L read as 0); a block's loads are all issued before its
        // first conversion.
        constexpr int kChunksPerRow = DI / 8;
        constexpr int kKeyStep = 256 / kChunksPerRow;
        constexpr int kIt = kBlock / kKeyStep;  // chunks per thread per block
        static_assert(kBlock % kKeyStep == 0, "a thread's keys must not straddle a block inside one step");
        const int cr = et % kChunksPerRow, j0 = et / kChunksPerRow;
        const int ckb = cr >> 3, ccc = cr & 7;
        auto load_block = [&](int64_t uu, int h2, uint32_t(&wv)[kIt], uint32_t(&sv)[kIt]) {
            const int kb_b = (int)(uu / ((int64_t)sh.nkt * sh.nqc));
            const int64_t kb_k0 = ((uu % ((int64_t)sh.nkt * sh.nqc)) / sh.nqc) * kPfKeys;
            const int64_t kb_L = clamp_len(p.seq_lens[kb_b], Tq, p.lmax, nullptr);
            const int64_t vb = kb_k0 + h2 * kBlock < kb_L ? block_vec<PAGED>(p, kb_b, kb_k0 / kBlock + h2, 0, 1) : 0;
#pragma unroll
            for (int it = 0; it < kIt; ++it) {
                const int64_t vec = vb + j0 + it * kKeyStep;
                wv[it] = 0u;
                sv[it] = 0u;
                if (kb_k0 + h2 * kBlock + j0 + it * kKeyStep < kb_L) {
                    wv[it] = *reinterpret_cast<const uint32_t*>(p.ik.data + vec * (DI / 2) + cr * 4);
                    sv[it] = p.ik.scale[vec * (DI / 16) + (cr >> 1)];
                }
            }
        };
        auto store_block = [&](uint8_t* kdst, int h2, const uint32_t(&wv)[kIt], const uint32_t(&sv)[kIt]) {
#pragma unroll
            for (int it = 0; it < kIt; ++it) {
                const int j = h2 * kBlock + j0 + it * kKeyStep;
                uint32_t hh[4];
                e2m1x8_to_f16x8(wv[it], hh[0], hh[1], hh[2], hh[3]);
                const uint32_t s2 = e4m3_bcast_f16x2(sv[it]);
                uint4 o;
                uint32_t* op = &o.x;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t m = hmul2(hh[i], s2);  // e2m1 * e4m3, exact in f16 and in bf16
                    const __half2 vm = *reinterpret_cast<const __half2*>(&m);
                    const __nv_bfloat162 bb = __floats2bfloat162_rn(__low2float(vm), __high2float(vm));
                    op[i] = *reinterpret_cast<const uint32_t*>(&bb);
                }
                *reinterpret_cast<uint4*>(kdst + ckb * G::kKBlock + j * 128 + ((ccc ^ (j & 7)) << 4)) = o;
            }
        };
        auto publish = [&](uint32_t kbi) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&k_full[kbi]);
        };
        auto unit_live = [&](int64_t uu) {
            const int ub = (int)(uu / ((int64_t)sh.nkt * sh.nqc));
            const int64_t urem = uu % ((int64_t)sh.nkt * sh.nqc);
            const int64_t uk0 = (urem / sh.nqc) * kPfKeys;
            const int uqc = (int)(urem % sh.nqc);
            const int64_t uL = clamp_len(p.seq_lens[ub], Tq, p.lmax, nullptr);
            bool a2 = false;
            for (int qt = uqc * kPfQChunk; qt < min(sh.nqt, (uqc + 1) * kPfQChunk); ++qt)
                a2 |= pf_tile_live<HI>(qt, uk0, uL, Tq);
            return a2;
        };
        auto next_live = [&](int64_t uu) {
            for (uu += gridDim.x; uu < sh.units; uu += gridDim.x)
                if (unit_live(uu)) return uu;
            return sh.units;
        };
        // this CTA's first live unit: its keys go to tile 0 before any query tile
        int64_t u_live = (int64_t)blockIdx.x >= sh.units ? sh.units
                         : unit_live(blockIdx.x)            ? (int64_t)blockIdx.x
                                                            : next_live(blockIdx.x);
        if (u_live < sh.units) {
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t wv[kIt], sv[kIt];
                load_block(u_live, h2, wv, sv);
                store_block(kbuf, h2, wv, sv);
            }
            publish(0);
        }
        uint32_t qi = 0, ui = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < sh.units && ok; u += gridDim.x) {
            const int b = (int)(u / ((int64_t)sh.nkt * sh.nqc));
            const int64_t rem = u % ((int64_t)sh.nkt * sh.nqc);
            const int64_t k0 = (rem / sh.nqc) * kPfKeys;
            const int qc = (int)(rem % sh.nqc);
            const int64_t L = clamp_len(p.seq_lens[b], Tq, p.lmax, nullptr);
            const int64_t nb_b = (L + kBlock - 1) / kBlock;
            const int64_t n = k0 / kBlock + hb;  // this warp's block
            const int qt_end = min(sh.nqt, (qc + 1) * kPfQChunk);
            const bool any = u == u_live;
            // A live unit first writes the next live unit's keys into the other tile (free: its MMAs
            // ended before this unit's first tile); the MMAs of this unit's first two query tiles
            // need nothing from these warps and run meanwhile.
            if (any) {
                u_live = next_live(u);
                if (u_live < sh.units) {
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t wv[kIt], sv[kIt];
                        load_block(u_live, h2, wv, sv);
                        store_block(kbuf + ((ui + 1) & 1u) * G::kKTile, h2, wv, sv);
                    }
                    publish((ui + 1) & 1u);
                }
            }
            // Per tile, the row's token moves on by kPfRows / HI and its head stays the same, so the
            // token, its count of visible keys in this warp's block and its score address step by
            // constants (32-bit where the values are bounded by a block); the tail between tiles
            // is then the head sum and one store.
            const int row = quad * 32 + lane;
            const int h = row % HI;  // kPfRows is a multiple of HI
            const int q0 = qc * kPfQChunk;
            int t = (q0 * kPfRows + row) / HI;
            // visible keys of block n for token t: L - Tq + t + 1 - n * 128, clamped to [0, 128]
            const int64_t vis0 = L - Tq + 1 - n * kBlock;
            const bool n_ok = n < nb_b;
            const float wrow = p.w_idx != nullptr;  // weights are read per token below
            float* dst = block_scores + ((int64_t)b * Tq + t) * p.nbmax + n;
            const int64_t dst_step = (int64_t)(kPfRows / HI) * p.nbmax;
            // the tile's visibility and key count, computed one tile ahead (they fill the latency of
            // the previous tile's head sum)
            bool live = q0 < qt_end && pf_tile_live<HI>(q0, k0, L, Tq);
            bool t_ok = t < Tq && n_ok;
            int cnt = t_ok ? (int)min64(kBlock, max64(0, vis0 + t)) : 0;
            for (int qt = q0; qt < qt_end; ++qt, t += kPfRows / HI, dst += dst_step) {
                float sum = 0.0f;
                if (live) {
                    const int buf = (int)(qi & 1u);
                    if (!mbar_wait(&t_full[buf], (qi >> 1) & 1u)) {
                        set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_INDEX_CONSUMER);
                        ok = false;
                        break;
                    }
                    tcgen05_fence_after();
                    const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * kPfKeys + hb * kBlock);
                    // ReLU-sum over the visible columns: the block's 128 columns in one round trip
                    // to tensor memory (four loads, one wait), 4 independent packed accumulators
                    float2 acc2[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
                    float v[kBlock / 32][32];
#pragma unroll
                    for (int c4 = 0; c4 < kBlock / 32; ++c4) tmem_ld32(taddr + c4 * 32, v[c4]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < kBlock / 32; ++c4) {
                        if (cnt >= (c4 + 1) * 32) {
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                acc2[i & 3] = add_f32x2(acc2[i & 3], make_float2(fmaxf(v[c4][2 * i], 0.0f),
                                                                                fmaxf(v[c4][2 * i + 1], 0.0f)));
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int col = c4 * 32 + 2 * i;
                                acc2[i & 3] = add_f32x2(acc2[i & 3],
                                                        make_float2(col < cnt ? fmaxf(v[c4][2 * i], 0.0f) : 0.0f,
                                                                    col + 1 < cnt ? fmaxf(v[c4][2 * i + 1], 0.0f) : 0.0f));
                            }
                        }
                    }
                    sum = ((acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y)) + ((acc2[2].x + acc2[2].y) + (acc2[3].x + acc2[3].y));
                    tcgen05_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&t_empty[buf]);
                    ++qi;
                }
                const float x = t < Tq ? sum * (wrow != 0.0f ? p.w_idx[((int64_t)b * Tq + t) * HI + h] : 1.0f) : 0.0f;
                const bool st_ok = h == 0 && t_ok;
                const int st_cnt = cnt;
                {
                    const int tn = t + kPfRows / HI;
                    live = qt + 1 < qt_end && pf_tile_live<HI>(qt + 1, k0, L, Tq);
                    t_ok = tn < Tq && n_ok;
                    cnt = t_ok ? (int)min64(kBlock, max64(0, vis0 + tn)) : 0;
                }
                // head sum: the token's HI rows are HI consecutive lanes; every lane reads them at
                // once (independent shuffles) and adds pairwise
                float xs[HI];
#pragma unroll
                for (int o = 0; o < HI; ++o) xs[o] = __shfl_sync(0xffffffffu, x, (lane & ~(HI - 1)) + o);
#pragma unroll
                for (int w2 = HI / 2; w2 >= 1; w2 >>= 1)
#pragma unroll
                    for (int o = 0; o < w2; ++o) xs[o] += xs[o + w2];
                // mean over the visible keys; a full block divides by 128, a power of two (exact as a product)
                if (st_ok)
                    *dst = st_cnt == kBlock ? (xs[0] * (1.0f / kBlock)) * s_t
                                            : st_cnt > 0 ? (xs[0] / (float)st_cnt) * s_t : -INFINITY;
            }
            if (any) ++ui;
        }
    }

    tcgen05_fence_before();
    __syncthreads();
    if (warp == kPfMmaWarp) {
        tcgen05_fence_after();
        tmem_dealloc(tmem_base, kPfTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
}

template <int DI, int HI, bool PAGED>
int launch_pf(const Problem& p, float* bs, bool pdl, cudaStream_t st) {
    using G = PfGeom<DI>;
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return MSA_ECUDA;
    // query rows of one sequence: [B][Tq*HI][DI] bf16, 128 x 64 boxes, 128-byte swizzle
    CUtensorMap tmap;
    const cuuint64_t dims[3] = {(cuuint64_t)DI, (cuuint64_t)p.Tq * HI, (cuuint64_t)p.B};
    const cuuint64_t strides[2] = {(cuuint64_t)DI * 2, (cuuint64_t)p.Tq * HI * DI * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kPfRows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(p.q_idx), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MSA_ECUDA;
    auto kern = index_prefill_kernel<DI, HI, PAGED>;
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::kSmem) != cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)di.num_sms);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = G::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p, bs, tmap) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

template <int DI>
int launch_pf_hi(const Problem& p, float* bs, bool pdl, cudaStream_t st) {
    switch (p.HI) {
        case 1: return p.block_table ? launch_pf<DI, 1, true>(p, bs, pdl, st) : launch_pf<DI, 1, false>(p, bs, pdl, st);
        case 2: return p.block_table ? launch_pf<DI, 2, true>(p, bs, pdl, st) : launch_pf<DI, 2, false>(p, bs, pdl, st);
        case 4: return p.block_table ? launch_pf<DI, 4, true>(p, bs, pdl, st) : launch_pf<DI, 4, false>(p, bs, pdl, st);
        case 8: return p.block_table ? launch_pf<DI, 8, true>(p, bs, pdl, st) : launch_pf<DI, 8, false>(p, bs, pdl, st);
        default: return MSA_EUNSUPPORTED;
    }
}

}  // namespace

void* tensor_map_encode_entry() {
    static void* fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = ptr;
    }
    return fn;
}

int launch_index_prefill(const Problem& p, float* block_scores, bool pdl, cudaStream_t st) {
    if (p.pool_mode != 0) return MSA_EUNSUPPORTED;
    if (p.DI == 128) return launch_pf_hi<128>(p, block_scores, pdl, st);
    if (p.DI == 64) return launch_pf_hi<64>(p, block_scores, pdl, st);
    return MSA_EUNSUPPORTED;
}

}  // namespace msa
