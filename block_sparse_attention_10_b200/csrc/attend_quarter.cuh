// attend_quarter.cuh — one warp's exact-attention step over 32 keys of one KV head.
//
// Method ("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", ainewsbites.com, section "A
// model built for efficient inference"): attention over the selected blocks is exact
// softmax attention, not an approximation.  A warp computes the G query heads of one KV head against the
// keys of a 32-key quarter of a selected block and folds them into its running
// (max, sum, output) with the online softmax:
//   S^T = K Q^T    mma m16n8k16, A = dequantised K (exact f16, 16 keys), B = the G
//                  query heads (8 columns) — the same tile routine as the indexer;
//   softmax        online over quarters, exp2 domain, fp32; the running output is only
//                  rescaled when a quarter raises the running max;
//   O^T += V^T P^T mma m16n8k16, A = dequantised V, B = P^T taken from the S^T
//                  accumulators by one movmatrix (8x8 transpose) per 8 keys.  The A
//                  fragment pairs two keys per dim: the two keys' nibbles are interleaved
//                  bytewise first, so each converted f16x2 already holds that pair.
// Shared by the attention kernel (attend.cu) and the single-launch decode kernel
// (decode_fused.cu).  A quarter stage is K nibbles (32 x 64 B), K scales (32 x 8 B),
// V nibbles, V scales: 4.5 KB, the same size as an indexer stage.
#pragma once

#include "internal.h"
#include "nvfp4_mma.cuh"

namespace msa {

constexpr int kAttD = 128;
constexpr int kAttQuarter = 32;
constexpr int kAttKData = kAttQuarter * 64, kAttKScale = kAttQuarter * 8;
constexpr int kAttStageBytes = 2 * (kAttKData + kAttKScale);  // 4.5 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Per-thread running state: query heads 2c, 2c+1 (m, l) and the output tile, where
// thread (g, c) holds dims 16g + 2mt (+1 in elements 2, 3) of heads 2c, 2c+1.
struct AttAcc {
    float m2[2], l2[2];
    float o[8][4];
};

__device__ __forceinline__ void att_init(AttAcc& a) {
    a.m2[0] = a.m2[1] = -INFINITY;
    a.l2[0] = a.l2[1] = 0.0f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) a.o[mt][0] = a.o[mt][1] = a.o[mt][2] = a.o[mt][3] = 0.0f;
}

// Query fragments of row bt (= b * Tq + t), KV head kvh: column g = query head kvh*G + g,
// dims permuted as the K rows of nvfp4_tile_mma; columns g >= G are zero.
__device__ __forceinline__ void att_load_q(const Problem& p, int64_t bt, int kvh, int G, int g, int c,
                                           uint32_t (&qf)[1][8][2]) {
    if (g < G) {
        const __nv_bfloat16* qrow = p.q + ((bt * p.Hq) + (int64_t)kvh * G + g) * kAttD + c * 32;
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
}

// Bulk copies of one quarter (rows keys from cache vector vec, i.e. (b*Hkv + kvh)*lmax +
// key) into stage st; completes on bar.  One lane calls it.
__device__ __forceinline__ void att_issue_quarter(const Problem& p, uint8_t* st, int64_t vec, int rows,
                                                  uint64_t* bar) {
    mbar_arrive_expect_tx(bar, (uint32_t)(2 * rows * (64 + 8)));
    bulk_g2s(st, p.k.data + vec * 64, (uint32_t)(rows * 64), bar);
    bulk_g2s(st + kAttKData, p.k.scale + vec * 8, (uint32_t)(rows * 8), bar);
    bulk_g2s(st + kAttKData + kAttKScale, p.v.data + vec * 64, (uint32_t)(rows * 64), bar);
    bulk_g2s(st + 2 * kAttKData + kAttKScale, p.v.scale + vec * 8, (uint32_t)(rows * 8), bar);
}

// Folds the qvalid (1..32) leading keys of the quarter in stage st into a.
// sc_log2 = softmax scale * K tensor scale * log2(e).  first: a holds no key yet.
__device__ __forceinline__ void att_quarter(const uint8_t* st, int qvalid, bool first, const uint32_t (&qf)[1][8][2],
                                            float sc_log2, int g, int c, AttAcc& a) {
    const uint8_t* kd = st;
    const uint8_t* ksc = st + kAttKData;
    const uint8_t* vd = st + kAttKData + kAttKScale;
    const uint8_t* vsc = st + 2 * kAttKData + kAttKScale;
    const int ntiles = (qvalid + 15) >> 4;
    // ---- S^T = K Q^T for the quarter's keys: s4[kt] = rows (keys) g, g+8 x cols 2c, 2c+1
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
    // ---- online softmax over the quarter (query heads 2c, 2c+1)
    float corr[2] = {1.0f, 1.0f};
    bool grew = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(fmaxf(s4[0][e], s4[0][2 + e]), fmaxf(s4[1][e], s4[1][2 + e]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (mx > a.m2[e]) {
            corr[e] = ex2_approx(a.m2[e] - mx);  // 0 while nothing is accumulated (m = -inf)
            a.m2[e] = mx;
            grew = true;
        }
        float l = 0.0f;
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
            s4[kt][e] = ex2_approx(s4[kt][e] - a.m2[e]);
            s4[kt][2 + e] = ex2_approx(s4[kt][2 + e] - a.m2[e]);
            l += s4[kt][e] + s4[kt][2 + e];
        }
        a.l2[e] = a.l2[e] * corr[e] + l;
    }
    if (__any_sync(0xffffffffu, grew) && !first) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            a.o[mt][0] *= corr[0];
            a.o[mt][1] *= corr[1];
            a.o[mt][2] *= corr[0];
            a.o[mt][3] *= corr[1];
        }
    }
    // ---- O^T += V^T P^T, 16 keys at a time
#pragma unroll
    for (int kt = 0; kt < 2; ++kt) {
        if (kt < ntiles) {
            // P^T fragment (keys x heads) -> B operand (k = keys 2c.., n = head g)
            const uint32_t pb0 = movmatrix_trans(pack_f16x2(s4[kt][0], s4[kt][1]));
            const uint32_t pb1 = movmatrix_trans(pack_f16x2(s4[kt][2], s4[kt][3]));
            // V^T A fragments: for each key pair (2c, 2c+1) and (2c+8, 2c+9), interleave the two
            // keys' nibbles so that each byte holds one dim of both keys; the converter then
            // yields (key a, key b) f16x2 pairs of one dim directly
            // va[pr][m] / vb[pr][m]: f16x2 (key a, key b) of dim 16g + 2m / 16g + 2m + 1
            uint32_t va[2][8], vb[2][8];
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const int ka = kt * 16 + 2 * c + 8 * pr, kb = ka + 1;
                uint2 wa = make_uint2(0u, 0u), wb = make_uint2(0u, 0u);
                uint32_t sa = 0u, sb = 0u;
                if (qvalid == kAttQuarter || ka < qvalid) {
                    wa = lds_v2(vd + ka * 64 + g * 8);
                    sa = lds_u8(vsc + ka * 8 + g);
                }
                if (qvalid == kAttQuarter || kb < qvalid) {
                    wb = lds_v2(vd + kb * 64 + g * 8);
                    sb = lds_u8(vsc + kb * 8 + g);
                }
                const uint32_t sc = e4m3x2_to_f16x2(sa | (sb << 8));  // (scale a, scale b)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t A = h ? wa.y : wa.x, Bw = h ? wb.y : wb.x;
                    const uint32_t ev = (A & 0x0F0F0F0Fu) | ((Bw << 4) & 0xF0F0F0F0u);  // dims 8h + 0, 2, 4, 6
                    const uint32_t od = ((A >> 4) & 0x0F0F0F0Fu) | (Bw & 0xF0F0F0F0u);  // dims 8h + 1, 3, 5, 7
                    uint32_t e0, e1, e2, e3, o0, o1, o2, o3;
                    e2m1x8_to_f16x8(ev, e0, e1, e2, e3);
                    e2m1x8_to_f16x8(od, o0, o1, o2, o3);
                    // e2m1x8_to_f16x8 pairs nibbles (2k, 2k+1) of its word, i.e. byte k = (key a, key b) of one dim
                    va[pr][4 * h + 0] = hmul2(e0, sc);  // dim 8h + 0
                    va[pr][4 * h + 1] = hmul2(e1, sc);  // dim 8h + 2
                    va[pr][4 * h + 2] = hmul2(e2, sc);  // dim 8h + 4
                    va[pr][4 * h + 3] = hmul2(e3, sc);  // dim 8h + 6
                    vb[pr][4 * h + 0] = hmul2(o0, sc);  // dim 8h + 1
                    vb[pr][4 * h + 1] = hmul2(o1, sc);  // dim 8h + 3
                    vb[pr][4 * h + 2] = hmul2(o2, sc);  // dim 8h + 5
                    vb[pr][4 * h + 3] = hmul2(o3, sc);  // dim 8h + 7
                }
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                // rows g / g+8 of m-tile mt are dims 16g + 2mt / 16g + 2mt + 1
                mma16816(a.o[mt], va[0][mt], vb[0][mt], va[1][mt], vb[1][mt], pb0, pb1);
            }
        }
    }
}

// Sum of l over the 8 row groups: every lane then holds l of heads 2c, 2c+1.
__device__ __forceinline__ void att_reduce_l(AttAcc& a) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float l = a.l2[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        a.l2[e] = l;
    }
}

// The output tile as [dim pair (64)][head (8)][2] floats: one 16-byte store per m-tile.
__device__ __forceinline__ void att_store_o(float* dst, int g, int c, const AttAcc& a) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
        *reinterpret_cast<float4*>(dst + (8 * g + mt) * 16 + 4 * c) =
            make_float4(a.o[mt][0], a.o[mt][2], a.o[mt][1], a.o[mt][3]);
}

}  // namespace msa
