// attend_prefill.cu — exact sparse attention for a chunk of many query tokens (chunked
// prefill) on the fifth-generation tensor cores.
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com, section "A
// model built for efficient inference"): every query token attends, with exact softmax,
// to the keys of its own 16 selected 128-token blocks that it can see; query head h reads
// KV head h / (Hq/Hkv).  The pages' prefill path fuses its steps ("Kernel and serving
// optimizations", same page); the design below is this library's.
//
// Decode attention gathers, per (token, KV head), its 16 blocks and dequantises them for
// that token alone.  With thousands of tokens in a chunk, each block is selected by tens
// of them, so this file turns the work around and goes block by block:
//   1. ap_count / ap_scan / ap_fill invert the selection: for every (sequence, block) the
//      list of (token, slot) pairs that selected it (slot = its place in the token's 16);
//      ap_tiles writes one 96-byte record per tile (item, coordinates, tokens, sequence
//      length, the next item's first tile, the 16 list entries);
//   2. ap_attend_kernel: one persistent CTA per SM walks items (sequence, KV head, block)
//      cut into tiles of 16 listed tokens x 8 query heads = 128 rows, the tiles spread
//      evenly over the CTAs.  Warp roles (16 warps, at most 128 registers each):
//        producer   bulk-copies tile records 6 tiles ahead into an 8-slot shared ring and
//                   gathers each tile's query rows (TMA from 16 lanes, 128-byte swizzle, one
//                   8-row atom per token, L2 evict-last, no multicast) into 2 stages;
//        dequant    a warpgroup that, item by item, loads the NVFP4 block straight from the
//                   caches into registers and writes K as bf16 [128 keys x 128 dims] and V
//                   transposed as f16 [128 dims x 128 keys] (divided by 128), both K-major
//                   with the 128-byte swizzle (e2m1 x e4m3 is exact in both types), into one
//                   of 2 item buffers, so the next item is ready before the current one ends;
//        MMA        one thread issues, in order of readiness,
//                     S = Q K^T  tcgen05.mma kind::f16, bf16, 128 x 128 x 128, fp32 in TMEM,
//                     O = P V    tcgen05.mma kind::f16, f16, A (= P) read from TMEM;
//        softmax    two warpgroups take alternate tiles (one TMEM lane = one row per thread),
//                   so one's exponentials overlap the other's TMEM traffic and output: read S
//                   (two passes of 32-column chunks: row max, then exponentials), mask keys
//                   past the token's position, write P = 2^(S c - m c) as f16 over S's first
//                   64 columns, then read O and write the row's unnormalised O / 128 (f16)
//                   with (m c, l) to the token's slot.
//      TMEM holds S / P of the two warpgroups at columns 0 / 128 and their O at 256 / 384;
//      S(i) reuses the columns of P(i - 2), so it is issued after P V(i - 2);
//   3. ap_merge_kernel combines each token's (up to) 16 slot partials in slot order:
//      out = s_V * 128 * sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// Every output row's arithmetic is independent of the tile row it occupies and the merge
// order is fixed, so results are bitwise reproducible although the lists are filled with
// atomics.  Every wait is bounded (MSA_STATUS_TIMEOUT | MSA_STATUS_AT_ATTEND).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "tcgen05.cuh"

namespace msa {
namespace {

constexpr int kApG = 8;                // query heads per KV head on this path
constexpr int kApTok = 128 / kApG;     // listed tokens per 128-row tile
constexpr int kApDqWarp = 8;           // warps 8..11: the dequantising warpgroup
constexpr int kApMmaWarp = 12;
constexpr int kApTmaWarp = 13;
constexpr int kApThreads = 32 * 16;    // warps 0..7: two softmax warpgroups (one per tile parity); 14, 15 idle
constexpr int kApTile = 32768;         // 128 rows x 128 16-bit elements: two 16 KB K-blocks
constexpr int kApKB = 16384;           // one K-block (64 elements of 128 rows)
// Two query stages: a third one (room exists once the raw block is read straight from the
// caches) made a few rows per step come out wrong, which the back-to-back bitwise test catches.
constexpr int kApQStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffKV = kApQStages * kApTile;   // 2 item buffers: K bf16 [key][dim], then V^T f16 [dim][key]
constexpr int kOffBar = kOffKV + 4 * kApTile;  // 37 mbarriers + the TMEM address
static_assert(kApQStages <= 3, "barrier layout holds 3 query stages");
constexpr int kOffInfo = kOffBar + 384;       // ring of 8 tile records
constexpr int kApInfoSlots = 8;
constexpr int kApRecAhead = 6;                // records in flight ahead of the tile being issued
constexpr size_t kApSmem = 1024 + kOffInfo + kApInfoSlots * 96;
constexpr uint32_t kApTmemCols = 512;  // S (then P) at columns 0 / 128, O at 256 / 384
constexpr float kApLog2e = 1.4426950408889634f;
constexpr float kApLn2 = 0.6931471805599453f;

// One tile, as ap_tiles_kernel writes it and the producer warp copies it (one 96-byte bulk
// copy) into the shared-memory ring read by the MMA thread and the tile's softmax warpgroup.
struct ApTileInfo {
    int32_t item, b, kvh, n, ntok, L;
    int32_t next;  // first tile of the next item (the loader and the dequantising warps jump there)
    int32_t pad;
    int32_t entry[kApTok];  // t * 16 + slot of the tile's tokens (0 past ntok)
};
static_assert(sizeof(ApTileInfo) == 96, "tile record layout");

struct ApWork {
    const int32_t* sel;         // [B][Tq][16]
    int32_t* cnt;               // [B * nbmax] tokens that selected block n of sequence b
    int32_t* cursor;            // [B * nbmax] fill positions
    int32_t* list_off;          // [B * nbmax] start of each list
    int32_t* tile_start;        // [items + 1] first tile of item (b, kvh, n); last entry = total
    int32_t* list;              // [B * Tq * 16] entries t * 16 + slot, grouped by (b, n)
    ApTileInfo* recs;    // [tile bound] one 96-byte record per tile (see ApTileInfo)
    float2* part_ml;            // [B][Tq][16][Hq]: (row max m * c, row sum l) of each slot's partial
    __half* part_o;             // [B][Tq][16][Hkv] blocks of 2 KB: [half][8-dim chunk][8 heads][8 dims]
};

// ------------------------------------------------------------------ selection inversion

__device__ __forceinline__ bool ap_valid_entry(const Problem& p, const int32_t* sel, int64_t e, int& b, int& t,
                                               int& n) {
    const int64_t bt = e / kTopK;
    b = (int)(bt / p.Tq);
    t = (int)(bt % p.Tq);
    n = sel[e];
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t nvis = (L - p.Tq + t) / kBlock + 1;
    if (n >= nvis) set_status(p.status, MSA_STATUS_SELECT);
    return n >= 0 && n < nvis;
}

__global__ void ap_count_kernel(const Problem p, const ApWork w) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)p.B * p.Tq * kTopK) return;
    int b, t, n;
    if (ap_valid_entry(p, w.sel, e, b, t, n)) atomicAdd(&w.cnt[(int64_t)b * p.nbmax + n], 1);
}

// Exclusive scan of `count(i)` for i < N into out[0..N] (out[N] = total) by one CTA of 1024 threads.
template <class Count>
__device__ __forceinline__ void ap_block_scan(int64_t N, Count&& count, int32_t* out, int32_t* warp_sums) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t carry = 0;
    for (int64_t base = 0; base < N; base += 1024) {
        const int64_t i = base + tid;
        const int32_t x = i < N ? count(i) : 0;
        int32_t v = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (lane == 31) warp_sums[warp] = v;
        __syncthreads();
        if (warp == 0) {
            int32_t s = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sums[lane] = s;  // inclusive sums of the warps
        }
        __syncthreads();
        const int32_t before = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + v - x;
        if (i < N) out[i] = before;
        const int32_t total = warp_sums[31];
        __syncthreads();  // warp_sums is rewritten by the next chunk
        carry += total;
    }
    if (tid == 0) out[N] = carry;
}

__global__ void __launch_bounds__(1024) ap_scan_kernel(const Problem p, const ApWork w) {
    __shared__ int32_t warp_sums[32];
    pdl_wait();
    pdl_launch_dependents();
    const int64_t lists = (int64_t)p.B * p.nbmax;
    ap_block_scan(lists, [&](int64_t i) { return w.cnt[i]; }, w.list_off, warp_sums);
    for (int64_t i = threadIdx.x; i < lists; i += 1024) w.cursor[i] = 0;
    // tiles of item (b, kvh, n): ceil(cnt[b][n] / 16)
    const int64_t items = lists * p.Hkv;
    ap_block_scan(
        items,
        [&](int64_t i) {
            const int64_t n = i % p.nbmax, b = i / (p.nbmax * p.Hkv);
            return (w.cnt[b * p.nbmax + n] + kApTok - 1) / kApTok;
        },
        w.tile_start, warp_sums);
}

__global__ void ap_fill_kernel(const Problem p, const ApWork w) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (int64_t)p.B * p.Tq * kTopK) return;
    int b, t, n;
    if (ap_valid_entry(p, w.sel, e, b, t, n)) {
        const int64_t ln = (int64_t)b * p.nbmax + n;
        const int at = atomicAdd(&w.cursor[ln], 1);
        w.list[w.list_off[ln] + at] = t * kTopK + (int)(e % kTopK);
    }
}

// One warp per item (b, kvh, n), one lane per tile: the tile's record (item, coordinates,
// tokens, clamped L, the next item's first tile and its 16 list entries), so that the attention
// kernel fetches one 96-byte record per tile with one bulk copy.
__global__ void ap_tiles_kernel(const Problem p, const ApWork w) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (item >= (int64_t)p.B * p.Hkv * p.nbmax) return;
    const int64_t n = item % p.nbmax, b = item / (p.nbmax * p.Hkv);
    const int64_t ln = b * p.nbmax + n;
    const int cnt = w.cnt[ln], off = w.list_off[ln], t0 = w.tile_start[item];
    const int L = (int)clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int next = w.tile_start[item + 1];
    const int kvh = (int)((item / p.nbmax) % p.Hkv);
    for (int j = lane; j * kApTok < cnt; j += 32) {
        const int ntok = min(kApTok, cnt - j * kApTok);
        int e[kApTok];
#pragma unroll
        for (int k = 0; k < kApTok; ++k) e[k] = k < ntok ? w.list[off + j * kApTok + k] : 0;
        int4* r = reinterpret_cast<int4*>(w.recs + t0 + j);
        r[0] = make_int4((int)item, (int)b, kvh, (int)n);
        r[1] = make_int4(ntok, L, next, 0);
#pragma unroll
        for (int k = 0; k < kApTok; k += 4) r[2 + k / 4] = make_int4(e[k], e[k + 1], e[k + 2], e[k + 3]);
    }
}

// ------------------------------------------------------------------ block-major attention

// TMA load of a 4-D box with an L2 eviction-priority hint (no multicast).
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const void* tmap, int c0, int c1, int c2, int c3,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h) {
    const __half2 v = *reinterpret_cast<const __half2*>(&h);
    const __nv_bfloat162 b = __floats2bfloat162_rn(__low2float(v), __high2float(v));
    return *reinterpret_cast<const uint32_t*>(&b);
}

// One thread's share (of 128) of an NVFP4 block (128 keys of one KV head), loaded straight
// from the caches into registers (read-only path; the caches hold whole 128-key blocks):
// K words i = 0..15 cover keys (tid + 128 i) / 16, dims 8 ((tid + 128 i) % 16) .. + 7 (the
// 128 threads read 512 contiguous bytes per i); V keys 8 (tid / 8) + a, dims 16 (tid % 8) .. + 15.
struct ApRawShare {
    uint32_t kw[16], ks[16];
    uint2 vx[8];
    uint32_t vs[8];
};

__device__ __forceinline__ void ap_raw_load(ApRawShare& r, const Problem& p, int64_t vec, int tid) {
    const uint8_t* kd = p.k.data + vec * 64;
    const uint8_t* kscale = p.k.scale + vec * 8;
    const uint8_t* vd = p.v.data + vec * 64;
    const uint8_t* vscale = p.v.scale + vec * 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int q = tid + 128 * i;
        r.kw[i] = __ldg(reinterpret_cast<const uint32_t*>(kd) + q);
        r.ks[i] = __ldg(kscale + (q >> 4) * 8 + ((q & 15) >> 1));
    }
    const int w16 = tid & 7, kg = tid >> 3;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int key = kg * 8 + a;
        r.vx[a] = __ldg(reinterpret_cast<const uint2*>(vd + key * 64 + w16 * 8));
        r.vs[a] = __ldg(vscale + key * 8 + w16);
    }
}

// K, bf16 [key][dim], 128-byte swizzle, K-major (e2m1 x e4m3 is exact in bf16); keys at or
// past nvalid become zeros.
__device__ __forceinline__ void ap_dequant_k(uint8_t* kt, const ApRawShare& r, int nvalid, int tid) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int q = tid + 128 * i;
        const int j = q >> 4, cr = q & 15;  // key j, dims 8 cr .. 8 cr + 7
        const bool live = j < nvalid;
        uint32_t h[4];
        e2m1x8_to_f16x8(live ? r.kw[i] : 0u, h[0], h[1], h[2], h[3]);
        const uint32_t s2 = e4m3_bcast_f16x2(live ? r.ks[i] : 0u);
        uint4 o;
        o.x = f16x2_to_bf16x2(hmul2(h[0], s2));
        o.y = f16x2_to_bf16x2(hmul2(h[1], s2));
        o.z = f16x2_to_bf16x2(hmul2(h[2], s2));
        o.w = f16x2_to_bf16x2(hmul2(h[3], s2));
        *reinterpret_cast<uint4*>(kt + (cr >> 3) * kApKB + j * 128 + (((cr & 7) ^ (j & 7)) << 4)) = o;
    }
}

// V^T, f16 [dim][key] divided by 128, 128-byte swizzle, K-major: thread = (dims 16 w16 ..
// 16 w16 + 15, keys 8 kg .. 8 kg + 7), written as 16 rows x one 16-byte chunk.
__device__ __forceinline__ void ap_dequant_vt(uint8_t* vt, const ApRawShare& r, int nvalid, int tid) {
    const int w16 = tid & 7, kg = tid >> 3;
    uint32_t rows[16][4];  // [dim 16 w16 + r][key pair i]
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // (key 2i, key 2i+1) scales times 2^-7: V^T is stored divided by 128 (exact in f16: every
        // product stays a multiple of 2^-24 below 2^11), so P V is O / 128 and fits f16 unnormalised
        const bool l0 = kg * 8 + 2 * i < nvalid, l1 = kg * 8 + 2 * i + 1 < nvalid;
        const uint32_t sc =
            hmul2(e4m3x2_to_f16x2((l0 ? r.vs[2 * i] : 0u) | ((l1 ? r.vs[2 * i + 1] : 0u) << 8)), 0x20002000u);
#pragma unroll
        for (int hw = 0; hw < 2; ++hw) {
            const uint32_t A = l0 ? (hw ? r.vx[2 * i].y : r.vx[2 * i].x) : 0u;
            const uint32_t Bw = l1 ? (hw ? r.vx[2 * i + 1].y : r.vx[2 * i + 1].x) : 0u;
            const uint32_t ev = (A & 0x0F0F0F0Fu) | ((Bw << 4) & 0xF0F0F0F0u);  // byte k: dim 8 hw + 2k
            const uint32_t od = ((A >> 4) & 0x0F0F0F0Fu) | (Bw & 0xF0F0F0F0u);  // byte k: dim 8 hw + 2k + 1
            uint32_t e[4], o[4];
            e2m1x8_to_f16x8(ev, e[0], e[1], e[2], e[3]);
            e2m1x8_to_f16x8(od, o[0], o[1], o[2], o[3]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                rows[8 * hw + 2 * k][i] = hmul2(e[k], sc);
                rows[8 * hw + 2 * k + 1][i] = hmul2(o[k], sc);
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 16; ++rr) {
        const int d = 16 * w16 + rr;
        *reinterpret_cast<uint4*>(vt + (kg >> 3) * kApKB + d * 128 + (((kg & 7) ^ (d & 7)) << 4)) =
            make_uint4(rows[rr][0], rows[rr][1], rows[rr][2], rows[rr][3]);
    }
}

// One row's softmax numerators: m = max of the row's first kvis scores of the S tile at
// taddr (128 fp32 TMEM columns of this thread's lane), P_k = 2^(S_k c - m c) (0 for k >= kvis),
// written as f16 pairs over the first 64 of those columns; returns the row sum of the fp32 P
// and sets mc = m c (0 for an empty row).  S is read twice (max, then exponentials) in chunks
// of 32 columns, in loops that are not unrolled: the code stays small enough for the
// instruction cache while the other warp roles run beside it.  MASKED = false: every key
// visible (kvis >= 128), no selects.
template <bool MASKED>
__device__ __forceinline__ float ap_softmax_row(uint32_t taddr, float c, int kvis, float& mc) {
    float mx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mx[j] = -INFINITY;
#pragma unroll 1
    for (int k0 = 0; k0 < 128; k0 += 32) {
        float v[32];
        tmem_ld32(taddr + k0, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k)
            if (!MASKED || k0 + k < kvis) mx[k & 7] = fmaxf(mx[k & 7], v[k]);
    }
    const float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
    mc = kvis > 0 ? m * c : 0.0f;
    float ls[4] = {0.f, 0.f, 0.f, 0.f};  // 4 independent partial sums
    // keys k0 .. k0 + 31 -> P columns k0 / 2 .. k0 / 2 + 15, which lie in S columns already read
#pragma unroll 1
    for (int k0 = 0; k0 < 128; k0 += 32) {
        float v[32];
        tmem_ld32(taddr + k0, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            float x0 = ex2_approx(fmaf(v[2 * u], c, -mc));
            float x1 = ex2_approx(fmaf(v[2 * u + 1], c, -mc));
            if (MASKED) {
                x0 = k0 + 2 * u < kvis ? x0 : 0.0f;
                x1 = k0 + 2 * u + 1 < kvis ? x1 : 0.0f;
            }
            ls[(2 * u) & 3] += x0;
            ls[(2 * u + 1) & 3] += x1;
            pk[u] = pack_f16x2(x0, x1);
        }
        tmem_st16(taddr + (k0 >> 1), pk);
    }
    return (ls[0] + ls[1]) + (ls[2] + ls[3]);
}

template <bool PAGED>
__global__ void __launch_bounds__(kApThreads, 1)
    ap_attend_kernel(const Problem p, const ApWork w, const __grid_constant__ CUtensorMap tmap) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bar + 0;       // [query stages]
    uint64_t* q_empty = bar + 3;      // [query stages]
    uint64_t* k_full = bar + 6;       // [2 item buffers]
    uint64_t* v_full = bar + 8;       // [2]
    uint64_t* kv_empty = bar + 10;    // [2]
    uint64_t* s_full = bar + 12;      // [2 warpgroups = tile parities]
    uint64_t* p_full = bar + 14;      // [2]
    uint64_t* o_full = bar + 16;      // [2]
    uint64_t* o_empty = bar + 18;     // [2]
    uint64_t* info_full = bar + 20;   // [8]
    uint64_t* info_empty = bar + 28;  // [8]
    uint64_t* done = bar + 36;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 37);
    ApTileInfo* info = reinterpret_cast<ApTileInfo*>(smem + kOffInfo);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kApQStages; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 4);
            mbar_init(&v_full[s], 4);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&o_full[s], 1);
            mbar_init(&o_empty[s], 4);
        }
        for (int s = 0; s < kApInfoSlots; ++s) {
            mbar_init(&info_full[s], 1);
            mbar_init(&info_empty[s], 4 + 2);  // the tile's warpgroup, the MMA thread, the producer
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == kApMmaWarp) {
        tmem_alloc(tmem_slot, kApTmemCols);
        tmem_relinquish();
    }
    tcgen05_fence_before();
    __syncthreads();
    tcgen05_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    // Data written by the kernels just before this one (launched as programmatic dependents) is read
    // on the L2 path (ld.global.cg): a plain load could hit a line left in this SM's L1 by an earlier
    // step that used the same workspace.
    const int64_t items = (int64_t)p.B * p.Hkv * p.nbmax;
    const int total = __ldcg(w.tile_start + items);
    const int t0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int t1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
    const int ntiles = t1 - t0;
    const int Tq = p.Tq;
    auto fail = [&]() { set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_ATTEND); };

    if (warp == kApTmaWarp) {
        // ------------------------------------------------------------ producer warp: tile records (bulk copies
        // kApRecAhead tiles ahead into the 8-slot ring) and each tile's query rows (TMA, one 8-row atom per
        // token, from 16 lanes).  No global load sits on this warp's path.
        if (ntiles > 0) {
            const uint64_t pol = l2_policy_evict_last();  // the queries are re-read by many tiles
            int recs = 0, seen = 0, issued = 0;  // records copied, records read here, query tiles issued
            bool ok = true;
            auto copy_rec = [&](int j) -> bool {  // lane 0: record of tile j into slot j & 7
                const int s8 = j & (kApInfoSlots - 1);
                if (j >= kApInfoSlots && !mbar_wait(&info_empty[s8], ((j >> 3) - 1) & 1)) return false;
                mbar_arrive_expect_tx(&info_full[s8], (uint32_t)sizeof(ApTileInfo));
                bulk_g2s(info + s8, w.recs + t0 + j, (uint32_t)sizeof(ApTileInfo), &info_full[s8]);
                return true;
            };
            if (lane == 0)
                for (; recs < min(kApRecAhead, ntiles) && ok; ++recs) ok = copy_rec(recs);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int i = 0; i < ntiles && ok; ++i) {
                const int sb = i % kApQStages, s8 = i & (kApInfoSlots - 1);
                if (lane == 0 && i >= kApQStages && !mbar_wait(&q_empty[sb], ((i / kApQStages) - 1) & 1)) ok = false;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok || !__all_sync(0xffffffffu, mbar_wait(&info_full[s8], (i >> 3) & 1))) {
                    ok = false;
                    break;
                }
                seen = i + 1;
                const int ntok = info[s8].ntok, b = info[s8].b, kvh = info[s8].kvh;
                const int e = lane < kApTok ? info[s8].entry[lane] : 0;
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&info_empty[s8]);
                    mbar_arrive_expect_tx(&q_full[sb], (uint32_t)(ntok * 2 * 1024));
                }
                __syncwarp();
                if (lane < ntok) {  // each lane gathers one token's 8 query heads
                    const int t = e / kTopK;
                    uint8_t* qs = smem + kOffQ + sb * kApTile + lane * 1024;
                    tma_load_4d_hint(qs, &tmap, 0, kvh * kApG, t, b, &q_full[sb], pol);
                    tma_load_4d_hint(qs + kApKB, &tmap, 64, kvh * kApG, t, b, &q_full[sb], pol);
                }
                issued = i + 1;
                if (lane == 0 && recs < ntiles) ok = copy_rec(recs++);
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            if (!ok && lane == 0) fail();
            // never leave with copies in flight into this CTA's shared memory
            if (lane == 0) {
                for (int i = max(0, issued - kApQStages); i < issued; ++i)
                    if (!mbar_wait(&q_full[i % kApQStages], (i / kApQStages) & 1)) {
                        fail();
                        break;
                    }
                for (int j = seen; j < recs; ++j)
                    if (!mbar_wait(&info_full[j & (kApInfoSlots - 1)], (j >> 3) & 1)) {
                        fail();
                        break;
                    }
            }
        }
    } else if (warp >= kApDqWarp && warp < kApDqWarp + 4) {
        // ------------------------------------------------------------ dequantising warpgroup: every item of
        // this CTA in order, into item buffer seq & 1 (free once the P V MMAs of item seq - 2 are done).  The
        // block's NVFP4 bytes are loaded into registers before that wait, so their latency overlaps it; K is
        // written first (the S MMAs wait for K only), then V^T.
        if (ntiles > 0) {
            const int tid = threadIdx.x - 32 * kApDqWarp;
            auto wait_all = [&](uint64_t* b_, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(b_, parity)) != 0;
            };
            int seq = -1;
            bool ok = true;
            for (int tau = t0; tau < t1;) {
                const int item = __ldcg(&w.recs[tau].item), Lr = __ldcg(&w.recs[tau].L), next = __ldcg(&w.recs[tau].next);
                tau = max(next, tau + 1);
                ++seq;
                const int kb = seq & 1;
                const int n = item % (int)p.nbmax, bk = item / (int)p.nbmax;
                const int kvh = bk % p.Hkv, b = bk / p.Hkv;
                const int nvalid = (int)min64(kBlock, max64(0, (int64_t)Lr - (int64_t)n * kBlock));
                ApRawShare r;
                ap_raw_load(r, p, block_vec<PAGED>(p, b, n, kvh, p.Hkv), tid);
                if (seq >= 2 && !wait_all(&kv_empty[kb], ((seq >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                uint8_t* kvb = smem + kOffKV + kb * 2 * kApTile;
                ap_dequant_k(kvb, r, nvalid, tid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&k_full[kb]);
                ap_dequant_vt(kvb + kApTile, r, nvalid, tid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&v_full[kb]);
            }
            if (!ok && lane == 0) fail();
        }
    } else if (warp == kApMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (one thread), scheduled by
        // readiness: P V(j) as soon as P(j), V and O(j & 1) are ready, S(i) as soon as its record, K and Q(i)
        // are, so that neither waits behind the other.  S(i) reuses the TMEM columns that held P(i - 2), so it
        // is issued only after P V(i - 2) (tcgen05.mma runs in issue order).  Polls are non-blocking; no
        // progress for the wait limit ends the loop with a timeout status.
        if (lane == 0 && ntiles > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(128, 128);
            constexpr uint32_t idesc_o = umma_idesc_f16_f32(128, 128);
            int ns = 0, npv = 0;             // next S tile, next P V tile
            int cur = -1, seq = -1;          // item of the last record read, its number in this CTA
            int kseq = -1, vseq = -1;        // last item whose K / V readiness was seen
            int sseq = -1;                   // item number of tile ns once its record is read (-1: not yet)
            int pend = -1;                   // item whose last P V went out before the next record was read
            int seq_of[4] = {0, 0, 0, 0};    // item number of S-issued tiles (at most 2 ahead of P V)
            bool ok = true;
            uint64_t last = globaltimer_ns();
            while (npv < ntiles) {
                bool progress = false;
                // ---- P V(npv)
                if (npv < ns) {
                    const int j = npv, g = j & 1, sj = seq_of[j & 3];
                    if (mbar_test(&p_full[g], (j >> 1) & 1) && (sj == vseq || mbar_test(&v_full[sj & 1], (sj >> 1) & 1)) &&
                        (j < 2 || mbar_test(&o_empty[g], ((j >> 1) - 1) & 1))) {
                        vseq = sj;
                        tcgen05_fence_after();
                        const uint32_t vt = smem_u32(smem + kOffKV + (sj & 1) * 2 * kApTile + kApTile);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            umma_f16_ts(tmem + 256 + g * 128, tmem + g * 128 + k * 8,
                                        umma_desc_k_sw128(vt + (k >> 2) * kApKB + (k & 3) * 32), idesc_o,
                                        k > 0 ? 1u : 0u);
                        umma_commit(&o_full[g]);
                        // the item's K and V buffer is free once its last P V is done
                        if (j + 1 < ns) {
                            if (seq_of[(j + 1) & 3] != sj) umma_commit(&kv_empty[sj & 1]);
                        } else if (sseq >= 0) {  // tile j + 1 = ns: its record is read already
                            if (sseq != sj) umma_commit(&kv_empty[sj & 1]);
                        } else if (j + 1 < ntiles) {
                            pend = sj;  // decided when tile j + 1's record is read
                        }
                        ++npv;
                        progress = true;
                    }
                }
                // ---- S(ns)
                if (ns < ntiles && npv >= ns - 1) {
                    const int i = ns, g = i & 1, s8 = i & (kApInfoSlots - 1);
                    if (sseq < 0 && mbar_test(&info_full[s8], (i >> 3) & 1)) {
                        const int item = info[s8].item;
                        mbar_arrive(&info_empty[s8]);
                        if (item != cur) {
                            cur = item;
                            ++seq;
                        }
                        sseq = seq;
                        if (pend >= 0) {
                            if (pend != sseq) umma_commit(&kv_empty[pend & 1]);
                            pend = -1;
                        }
                        progress = true;
                    }
                    if (sseq >= 0 && (sseq == kseq || mbar_test(&k_full[sseq & 1], (sseq >> 1) & 1)) &&
                        mbar_test(&q_full[i % kApQStages], (i / kApQStages) & 1)) {
                        kseq = sseq;
                        tcgen05_fence_after();
                        const uint32_t qa = smem_u32(smem + kOffQ + (i % kApQStages) * kApTile);
                        const uint32_t kt = smem_u32(smem + kOffKV + (sseq & 1) * 2 * kApTile);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            umma_bf16_ss(tmem + g * 128, umma_desc_k_sw128(qa + (k >> 2) * kApKB + (k & 3) * 32),
                                         umma_desc_k_sw128(kt + (k >> 2) * kApKB + (k & 3) * 32), idesc_s,
                                         k > 0 ? 1u : 0u);
                        umma_commit(&q_empty[i % kApQStages]);
                        umma_commit(&s_full[g]);
                        seq_of[i & 3] = sseq;
                        sseq = -1;
                        ++ns;
                        progress = true;
                    }
                }
                if (progress) {
                    last = globaltimer_ns();
                } else if (globaltimer_ns() - last > kWaitLimitNs) {
                    ok = false;
                    break;
                } else {
                    __nanosleep(32);  // leave the issue slots to the warps that compute
                }
            }
            if (!ok) fail();
            // every MMA issued has completed before the CTA releases its tensor memory
            umma_commit(done);
            if (!mbar_wait(done, 0)) fail();
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups: warpgroup g takes
        // the tiles of parity g, so that one warpgroup's exponentials overlap the other's tensor-memory
        // traffic and output.  Thread = one row (TMEM lane) = (token slot row / 8, query head row % 8).
        const int g = warp >> 2, qw = warp & 3;
        const int row = qw * 32 + lane, tslot = row >> 3, hq = row & 7;
        const uint32_t lane_base = tmem + ((uint32_t)(qw * 32) << 16);
        const float c = p.softmax_scale * p.k.s_t * kApLog2e;
        auto wait_all = [&](uint64_t* b_, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(b_, parity)) != 0;
        };
        bool ok = true;
        for (int i = g; i < ntiles; i += 2) {
            const int s8 = i & (kApInfoSlots - 1);
            if (!wait_all(&info_full[s8], (i >> 3) & 1)) {
                ok = false;
                break;
            }
            const ApTileInfo& ti = info[s8];
            const int n = ti.n, b = ti.b, kvh = ti.kvh, ntok = ti.ntok;
            const int64_t L = ti.L;
            const int e = tslot < ntok ? ti.entry[tslot] : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&info_empty[s8]);
            int kvis = 0;  // visible keys of the row's block (0: no token in this tile row)
            int64_t orow = -1;
            if (tslot < ntok) {
                const int t = e / kTopK, slot = e % kTopK;
                kvis = (int)min64(kBlock, L - Tq + t - (int64_t)n * kBlock + 1);
                orow = (((int64_t)b * Tq + t) * kTopK + slot) * p.Hq + kvh * kApG + hq;
            }
            if (!wait_all(&s_full[g], (i >> 1) & 1)) {
                ok = false;
                break;
            }
            tcgen05_fence_after();
            // no key masked in this warp: the unpredicated form
            float mc;
            const float l = __all_sync(0xffffffffu, kvis >= kBlock) ? ap_softmax_row<false>(lane_base + g * 128, c, kvis, mc)
                                                                    : ap_softmax_row<true>(lane_base + g * 128, c, kvis, mc);
            tmem_wait_st();
            tcgen05_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[g]);
            // ---- output: the row's O / 128 (f16) and (m c, l)
            if (!wait_all(&o_full[g], (i >> 1) & 1)) {
                ok = false;
                break;
            }
            tcgen05_fence_after();
            // the 8 heads of a token are interleaved at 8-dim (16-byte) granularity, so each store
            // below writes whole 128-byte lines: 8 lanes (heads) x 16 bytes per token
            uint4* dst = reinterpret_cast<uint4*>(w.part_o + (orow >> 3) * 1024) + hq;
#pragma unroll 1
            for (int c4 = 0; c4 < 4; ++c4) {
                float o[32];
                tmem_ld32(lane_base + 256 + g * 128 + c4 * 32, o);
                tmem_wait_ld();
                if (c4 == 3) {
                    tcgen05_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&o_empty[g]);
                }
                if (orow >= 0) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        __stcs(dst + (4 * c4 + q) * 8,
                               make_uint4(pack_f16x2(o[8 * q], o[8 * q + 1]), pack_f16x2(o[8 * q + 2], o[8 * q + 3]),
                                          pack_f16x2(o[8 * q + 4], o[8 * q + 5]),
                                          pack_f16x2(o[8 * q + 6], o[8 * q + 7])));
                }
            }
            if (orow >= 0) __stcs(w.part_ml + orow, make_float2(mc, l));
        }
        if (!ok && lane == 0) fail();
    }

    tcgen05_fence_before();
    __syncthreads();
    if (warp == kApMmaWarp) {
        tcgen05_fence_after();
        tmem_dealloc(tmem, kApTmemCols);
    }
}

// ------------------------------------------------------------------ merge of the slot partials

// One CTA of 128 threads per (sequence, token, KV head): one thread copies the group's valid
// slot partials (2 KB blocks of 8 heads x 128 dims, O / 128 in f16) and their (m, l) pairs into
// shared memory with bulk copies (one mbarrier), so the whole group is in flight at once without
// holding it in registers; then thread (head, 8 dims) combines the slots in slot order:
//   out = s_V * 128 * sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  lse = ln 2 * (M + log2 sum ...),
// stages the group's [8 heads][128 dims] output over the slot buffer and writes it in order.
constexpr int kMergeThreads = 128;
constexpr int kMergeSlot = kApG * 128 * 2;  // bytes of one slot partial of a group
constexpr size_t kMergeSmem = (size_t)kTopK * kMergeSlot + (size_t)kTopK * kApG * 8 + 16;
__global__ void __launch_bounds__(kMergeThreads) ap_merge_kernel(const Problem p, const ApWork w,
                                                                 float* __restrict__ out, float* __restrict__ lse) {
    extern __shared__ __align__(128) uint8_t msm[];
    const uint4* slots = reinterpret_cast<const uint4*>(msm);                            // [slot][128 x 16 B]
    const float2* mls = reinterpret_cast<const float2*>(msm + kTopK * kMergeSlot);       // [slot][8 heads]
    uint64_t* full = reinterpret_cast<uint64_t*>(msm + kTopK * kMergeSlot + kTopK * kApG * 8);
    pdl_wait();
    pdl_launch_dependents();
    const int64_t bk = blockIdx.x;  // (b * Tq + t) * Hkv + kvh
    const int j = threadIdx.x;      // position in the 2 KB block: (half * 8 + chunk) * 8 + head
    const int hh = j & 7, g8 = j >> 3;
    const int kvh = (int)(bk % p.Hkv);
    const int64_t bt = bk / p.Hkv;
    const int hq = kvh * kApG + hh;
    const int b = (int)(bt / p.Tq), t = (int)(bt % p.Tq);
    const int64_t L = clamp_len(p.seq_lens[b], p.Tq, p.lmax, nullptr);
    const int64_t nvis = (L - p.Tq + t) / kBlock + 1;
    const int4* selv = reinterpret_cast<const int4*>(w.sel + bt * kTopK);
    uint32_t valid = 0;  // bit s: slot s holds a visible selected block
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int4 x = __ldg(selv + q);
        const int id[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) valid |= (uint32_t)(id[r] >= 0 && id[r] < nvis) << (4 * q + r);
    }
    if (j == 0) {
        mbar_init(full, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (j == 0) {
        mbar_arrive_expect_tx(full, (uint32_t)__popc(valid) * (kMergeSlot + kApG * 8));
        for (int s2 = 0; s2 < kTopK; ++s2) {
            if (!((valid >> s2) & 1u)) continue;
            const int64_t pr = bt * kTopK + s2;  // (token, slot)
            bulk_g2s(msm + s2 * kMergeSlot, w.part_o + (pr * p.Hkv + kvh) * (kApG * 128), kMergeSlot, full);
            bulk_g2s(msm + kTopK * kMergeSlot + s2 * kApG * 8, w.part_ml + pr * p.Hq + kvh * kApG, kApG * 8, full);
        }
    }
    if (!mbar_wait(full, 0)) {
        set_status(p.status, MSA_STATUS_TIMEOUT | MSA_STATUS_AT_ATTEND);
        if (!mbar_wait(full, 0)) return;  // never leave with copies in flight, within the limit
        valid = 0;
    }
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < kTopK; ++s2)
        if ((valid >> s2) & 1u) M = fmaxf(M, mls[s2 * kApG + hh].x);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float W = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
        for (int s2 = 0; s2 < kTopK; ++s2) {
            if (!((valid >> s2) & 1u)) continue;
            const float2 ml = mls[s2 * kApG + hh];
            const float wt = ml.x == -INFINITY ? 0.0f : exp2f(ml.x - M);
            W += wt * ml.y;
            const uint4 ov = slots[s2 * (kMergeSlot / 16) + j];
            const uint32_t vv[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&vv[q]));
                acc[2 * q] += wt * f.x;
                acc[2 * q + 1] += wt * f.y;
            }
        }
    }
    const float inv = W > 0.0f ? 128.0f * p.v.s_t / W : 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] *= inv;
    if (g8 == 0 && lse != nullptr) lse[bt * p.Hq + hq] = W > 0.0f ? (M + log2f(W)) * kApLn2 : -INFINITY;
    // the group's output is [8 heads][128 dims], contiguous in out: stage it over the slot buffer
    // (every read of it is done at the barrier), then write it in order
    __syncthreads();
    float* st = reinterpret_cast<float*>(msm);
#pragma unroll
    for (int q = 0; q < 8; ++q) st[hh * 128 + g8 * 8 + q] = acc[q];
    __syncthreads();
    const int64_t o0 = (bt * p.Hq + kvh * kApG) * 128;  // first element of the group's 8 heads
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int e = 2 * (j + 128 * q);  // this thread's pairs are e, e + 256, e + 512, e + 768
        store_out2(p, out, o0 + e, st[e], st[e + 1]);
    }
}

// ------------------------------------------------------------------ host side

constexpr size_t kApAlign = 256;
size_t ap_round(size_t x) { return (x + kApAlign - 1) / kApAlign * kApAlign; }

struct ApLayout {
    size_t cnt, cursor, off, tstart, list, recs, lse, po, total;
};

ApLayout ap_layout(const Problem& p) {
    ApLayout a;
    const size_t lists = (size_t)p.B * p.nbmax, items = lists * p.Hkv, entries = (size_t)p.B * p.Tq * kTopK;
    size_t at = 0;
    a.cnt = at;
    at += ap_round(lists * 4);
    a.cursor = at;
    at += ap_round(lists * 4);
    a.off = at;
    at += ap_round(lists * 4);
    a.tstart = at;
    at += ap_round((items + 1) * 4);
    a.list = at;
    at += ap_round(entries * 4);
    a.recs = at;  // tiles <= sum over items of (listed tokens / 16 + 1)
    at += ap_round((entries * p.Hkv / kApTok + items + 1) * sizeof(ApTileInfo));
    a.lse = at;
    at += ap_round(entries * p.Hq * sizeof(float2));
    a.po = at;
    at += ap_round(entries * p.Hq * 128 * 2);
    a.total = at;
    return a;
}

cudaLaunchConfig_t ap_config(dim3 grid, dim3 block, size_t smem, bool pdl, cudaStream_t st,
                             cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <bool PAGED>
int launch_ap_attend(const Problem& p, const ApWork& w, bool pdl, cudaStream_t st) {
    auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (enc == nullptr) return MSA_ECUDA;
    // queries [B][Tq][Hq][128] bf16: boxes of 64 dims x 8 heads of one token, 128-byte swizzle
    CUtensorMap tmap;
    const cuuint64_t dims[4] = {128, (cuuint64_t)p.Hq, (cuuint64_t)p.Tq, (cuuint64_t)p.B};
    const cuuint64_t strides[3] = {(cuuint64_t)128 * 2, (cuuint64_t)p.Hq * 128 * 2, (cuuint64_t)p.Tq * p.Hq * 128 * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)kApG, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(p.q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return MSA_ECUDA;
    auto kern = ap_attend_kernel<PAGED>;
    static int configured_dev = -1;
    const DeviceInfo& di = device_info();
    if (configured_dev != di.device) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kApSmem) != cudaSuccess)
            return MSA_ECUDA;
        configured_dev = di.device;
    }
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = ap_config(dim3((unsigned)di.num_sms), dim3(kApThreads), kApSmem, pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, kern, p, w, tmap) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace

bool attend_prefill_supported(const Problem& p) {
    return (int64_t)p.Tq * p.HI > 32 && p.Hkv > 0 && p.Hq == kApG * p.Hkv && p.D == 128 &&
           (int64_t)p.B * p.Tq * kTopK * p.Hkv < 0x7FFFFFFFll && (int64_t)p.B * p.Hkv * p.nbmax < 0x7FFFFFFFll;
}

size_t attend_prefill_ws_bytes(const Problem& p) { return attend_prefill_supported(p) ? ap_layout(p).total : 0; }

int launch_attend_prefill(const Problem& p, const int32_t* sel, void* ws, float* out, float* lse, bool pdl,
                          cudaStream_t st) {
    if (!attend_prefill_supported(p)) return MSA_EUNSUPPORTED;
    const ApLayout a = ap_layout(p);
    uint8_t* base = static_cast<uint8_t*>(ws);
    ApWork w;
    w.sel = sel;
    w.cnt = reinterpret_cast<int32_t*>(base + a.cnt);
    w.cursor = reinterpret_cast<int32_t*>(base + a.cursor);
    w.list_off = reinterpret_cast<int32_t*>(base + a.off);
    w.tile_start = reinterpret_cast<int32_t*>(base + a.tstart);
    w.list = reinterpret_cast<int32_t*>(base + a.list);
    w.recs = reinterpret_cast<ApTileInfo*>(base + a.recs);
    w.part_ml = reinterpret_cast<float2*>(base + a.lse);
    w.part_o = reinterpret_cast<__half*>(base + a.po);
    const int64_t entries = (int64_t)p.B * p.Tq * kTopK;
    if (cudaMemsetAsync(w.cnt, 0, (size_t)p.B * p.nbmax * 4, st) != cudaSuccess) return MSA_ECUDA;
    cudaLaunchAttribute attr[1];
    const dim3 eg((unsigned)((entries + 255) / 256));
    cudaLaunchConfig_t cfg = ap_config(eg, dim3(256), 0, false, st, attr);
    if (cudaLaunchKernelEx(&cfg, ap_count_kernel, p, w) != cudaSuccess) return MSA_ECUDA;
    cfg = ap_config(dim3(1), dim3(1024), 0, pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, ap_scan_kernel, p, w) != cudaSuccess) return MSA_ECUDA;
    cfg = ap_config(eg, dim3(256), 0, pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, ap_fill_kernel, p, w) != cudaSuccess) return MSA_ECUDA;
    const int64_t items = (int64_t)p.B * p.Hkv * p.nbmax;
    cfg = ap_config(dim3((unsigned)((items * 32 + 255) / 256)), dim3(256), 0, pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, ap_tiles_kernel, p, w) != cudaSuccess) return MSA_ECUDA;
    const int r = p.block_table != nullptr ? launch_ap_attend<true>(p, w, pdl, st) : launch_ap_attend<false>(p, w, pdl, st);
    if (r != MSA_OK) return r;
    static int merge_dev = -1;
    if (merge_dev != device_info().device) {
        if (cudaFuncSetAttribute(ap_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMergeSmem) !=
            cudaSuccess)
            return MSA_ECUDA;
        merge_dev = device_info().device;
    }
    cfg = ap_config(dim3((unsigned)((int64_t)p.B * p.Tq * p.Hkv)), dim3(kMergeThreads), kMergeSmem, pdl, st, attr);
    if (cudaLaunchKernelEx(&cfg, ap_merge_kernel, p, w, out, lse) != cudaSuccess) return MSA_ECUDA;
    return MSA_OK;
}

}  // namespace msa
