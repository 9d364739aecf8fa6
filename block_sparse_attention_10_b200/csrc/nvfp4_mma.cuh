// nvfp4_mma.cuh — one tensor-core tile of "NVFP4 rows x fp16 query columns".
#pragma once

#include "common.cuh"

namespace msa {

// Rows are NVFP4 vectors of dimension DI in shared memory (nibble rows of DI/2 bytes at
// sd, E4M3 scale rows of DI/16 bytes at ss).  The head dim is permuted identically on
// both operands so that thread (g = lane/4, c = lane%4) reads one contiguous 16-byte
// (DI = 128) or 8-byte (DI = 64) piece of its row: in k-step i its A-fragment columns
// {2c, 2c+1} / {2c+8, 2c+9} are dims DI/4*c + 4i + {0, 1} / {2, 3}, and the query
// fragments qf[nt][i][0..1] hold the same dims of query 8*nt + g.
// One 16-key tile: rows r0 and r0 + 8 of the stage, dequantised (E2M1 * E4M3, exact in
// f16) into A fragments, times the resident query fragments; acc = [NT n-tiles][c0..c3].
template <int DI, int NT>
__device__ __forceinline__ void nvfp4_tile_mma(const uint8_t* sd, const uint8_t* ss, int r0, int c,
                                         const uint32_t (&qf)[NT][DI / 16][2], float (&acc)[NT][4]) {
    constexpr int KS = DI / 16;
    const int r1 = r0 + 8;
    uint32_t h0[2 * KS], h1[2 * KS];
    uint32_t s0[KS], s1[KS];
    if constexpr (DI == 128) {
        const uint4 w0 = lds_v4(sd + r0 * 64 + c * 16);
        const uint4 w1 = lds_v4(sd + r1 * 64 + c * 16);
        const uint32_t sc0 = e4m3x2_to_f16x2(lds_u16(ss + r0 * 8 + c * 2));
        const uint32_t sc1 = e4m3x2_to_f16x2(lds_u16(ss + r1 * 8 + c * 2));
        e2m1x8_to_f16x8(w0.x, h0[0], h0[1], h0[2], h0[3]);
        e2m1x8_to_f16x8(w0.y, h0[4], h0[5], h0[6], h0[7]);
        e2m1x8_to_f16x8(w0.z, h0[8], h0[9], h0[10], h0[11]);
        e2m1x8_to_f16x8(w0.w, h0[12], h0[13], h0[14], h0[15]);
        e2m1x8_to_f16x8(w1.x, h1[0], h1[1], h1[2], h1[3]);
        e2m1x8_to_f16x8(w1.y, h1[4], h1[5], h1[6], h1[7]);
        e2m1x8_to_f16x8(w1.z, h1[8], h1[9], h1[10], h1[11]);
        e2m1x8_to_f16x8(w1.w, h1[12], h1[13], h1[14], h1[15]);
        const uint32_t a0 = prmt(sc0, sc0, 0x1010u), a1 = prmt(sc0, sc0, 0x3232u);
        const uint32_t b0 = prmt(sc1, sc1, 0x1010u), b1 = prmt(sc1, sc1, 0x3232u);
#pragma unroll
        for (int i = 0; i < KS; ++i) {
            s0[i] = i < 4 ? a0 : a1;
            s1[i] = i < 4 ? b0 : b1;
        }
    } else {
        const uint2 w0 = lds_v2(sd + r0 * 32 + c * 8);
        const uint2 w1 = lds_v2(sd + r1 * 32 + c * 8);
        const uint32_t a0 = e4m3_bcast_f16x2(lds_u8(ss + r0 * 4 + c));
        const uint32_t b0 = e4m3_bcast_f16x2(lds_u8(ss + r1 * 4 + c));
        e2m1x8_to_f16x8(w0.x, h0[0], h0[1], h0[2], h0[3]);
        e2m1x8_to_f16x8(w0.y, h0[4], h0[5], h0[6], h0[7]);
        e2m1x8_to_f16x8(w1.x, h1[0], h1[1], h1[2], h1[3]);
        e2m1x8_to_f16x8(w1.y, h1[4], h1[5], h1[6], h1[7]);
#pragma unroll
        for (int i = 0; i < KS; ++i) {
            s0[i] = a0;
            s1[i] = b0;
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
    for (int i = 0; i < KS; ++i) {
        const uint32_t ra0 = hmul2(h0[2 * i], s0[i]), ra2 = hmul2(h0[2 * i + 1], s0[i]);
        const uint32_t ra1 = hmul2(h1[2 * i], s1[i]), ra3 = hmul2(h1[2 * i + 1], s1[i]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(acc[nt], ra0, ra1, ra2, ra3, qf[nt][i][0], qf[nt][i][1]);
    }
}

}  // namespace msa
