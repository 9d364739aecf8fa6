// codec.cu — NVFP4 encode / decode / amax kernels.
//
// Format (readmex.ai "vLLM delivers day-0 support for MiniMax-M3.1-Flash",
// TL;DR: an NVFP4 KV cache for the indexer and the attention path; per-token
// size 34,560 vs 61,440 bytes in FP8 on ainewsbites.com "A model built for
// efficient inference", i.e. 9/16 byte per element): E2M1 codes, one E4M3
// scale per 16 elements, one fp32 scale per tensor.
//
// Encode is the cache write that precedes the MSA path.  Each thread owns one
// 16-element group: 64 B of fp32 in (4 x 128-bit loads), 8 B of codes + 1 B of
// scale out.  HBM-bound; the divisions are IEEE round-to-nearest (__fdiv_rn)
// and the rounding to E4M3 / E2M1 is the hardware's RNE + saturation, which
// is the definition the CPU oracle implements in plain C.
#include "internal.h"

namespace msa {

namespace {

__global__ void __launch_bounds__(256) nvfp4_encode_kernel(const float* __restrict__ x, int64_t ngroups,
                                                           float s_t, uint8_t* __restrict__ data,
                                                           uint8_t* __restrict__ scale) {
    const float six_st = __fmul_rn(6.0f, s_t);
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < ngroups;
         g += (int64_t)gridDim.x * blockDim.x) {
        const float4* src = reinterpret_cast<const float4*>(x + g * 16);
        float v[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 f = __ldcs(src + i);
            v[4 * i + 0] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const uint32_t sc = f32_to_e4m3_satfinite(__fdiv_rn(amax, six_st));
        const float denom = __fmul_rn(e4m3_to_f32(sc), s_t);
        uint32_t w[2] = {0u, 0u};
        if (denom != 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t byte = f32x2_to_e2m1x2_satfinite(__fdiv_rn(v[2 * i], denom), __fdiv_rn(v[2 * i + 1], denom));
                w[i / 4] |= byte << (8 * (i % 4));
            }
        }
        *reinterpret_cast<uint2*>(data + g * 8) = make_uint2(w[0], w[1]);
        scale[g] = (uint8_t)sc;
    }
}

__global__ void __launch_bounds__(256) nvfp4_decode_kernel(const uint8_t* __restrict__ data,
                                                           const uint8_t* __restrict__ scale, int64_t ngroups,
                                                           float s_t, float* __restrict__ out) {
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < ngroups;
         g += (int64_t)gridDim.x * blockDim.x) {
        uint2 w = *reinterpret_cast<const uint2*>(data + g * 8);
        const uint32_t s2 = e4m3_bcast_f16x2(scale[g]);
        uint32_t h[8];
        e2m1x8_to_f16x8(w.x, h[0], h[1], h[2], h[3]);
        e2m1x8_to_f16x8(w.y, h[4], h[5], h[6], h[7]);
        float4* dst = reinterpret_cast<float4*>(out + g * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // e2m1 * e4m3 is exact in f16 (<= 6 significant bits, 2^-10 .. 2688)
            const uint32_t p0 = hmul2(h[2 * i], s2), p1 = hmul2(h[2 * i + 1], s2);
            const __half2 a = *reinterpret_cast<const __half2*>(&p0);
            const __half2 b = *reinterpret_cast<const __half2*>(&p1);
            float4 f;
            f.x = __fmul_rn(__low2float(a), s_t);
            f.y = __fmul_rn(__high2float(a), s_t);
            f.z = __fmul_rn(__low2float(b), s_t);
            f.w = __fmul_rn(__high2float(b), s_t);
            __stcs(dst + i, f);
        }
    }
}

__global__ void __launch_bounds__(256) amax_kernel(const float* __restrict__ x, int64_t n,
                                                   unsigned int* __restrict__ out_bits) {
    float m = 0.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(__ldcs(x + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // non-negative floats order like their bit patterns
    if ((threadIdx.x & 31) == 0) atomicMax(out_bits, __float_as_uint(m));
}

}  // namespace

int launch_nvfp4_encode(const float* x, int64_t nvec, int dim, float s_t, uint8_t* data, uint8_t* scale,
                        cudaStream_t st) {
    const int64_t ngroups = nvec * (dim / 16);
    if (ngroups == 0) return MSA_OK;
    const int threads = 256;
    int64_t blocks = (ngroups + threads - 1) / threads;
    const int64_t cap = (int64_t)device_info().num_sms * 16;
    if (blocks > cap) blocks = cap;
    nvfp4_encode_kernel<<<(unsigned)blocks, threads, 0, st>>>(x, ngroups, s_t, data, scale);
    return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ECUDA;
}

int launch_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim, float s_t, float* out,
                        cudaStream_t st) {
    const int64_t ngroups = nvec * (dim / 16);
    if (ngroups == 0) return MSA_OK;
    const int threads = 256;
    int64_t blocks = (ngroups + threads - 1) / threads;
    const int64_t cap = (int64_t)device_info().num_sms * 16;
    if (blocks > cap) blocks = cap;
    nvfp4_decode_kernel<<<(unsigned)blocks, threads, 0, st>>>(data, scale, ngroups, s_t, out);
    return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ECUDA;
}

int launch_nvfp4_amax(const float* x, int64_t n, float* amax_out, cudaStream_t st) {
    if (cudaMemsetAsync(amax_out, 0, sizeof(float), st) != cudaSuccess) return MSA_ECUDA;
    if (n == 0) return MSA_OK;
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    const int64_t cap = (int64_t)device_info().num_sms * 8;
    if (blocks > cap) blocks = cap;
    amax_kernel<<<(unsigned)blocks, threads, 0, st>>>(x, n, reinterpret_cast<unsigned int*>(amax_out));
    return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ECUDA;
}

}  // namespace msa
