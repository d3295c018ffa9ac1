// quant.cu -- bf16 -> e4m3 block quantization for the FP8 attention variant
// ("Accelerating HunyuanVideo inference with ParaAttention" (WaveSpeed), § "FP8
// dynamic quantization": activations quantized to FP8 at run time; the format and
// the per-block power-of-two scaling below are the reading taken).
//
// Per (batch*head, block of `bs` tokens): the block's largest magnitude fixes a
// power-of-two scale 2^e, the smallest e with max * 2^-e <= 448; every value is
// scaled by 2^-e (exact) and rounded to the nearest e4m3 value (OCP E4M3FN: bias
// 7, 3 mantissa bits, largest finite 448), ties to the even code, magnitudes
// above 448 saturated (a block holding inf keeps the scale 2^0; NaN stays NaN and
// does not count toward the maximum).  A block's rows are contiguous in [B,H,N,d], so one CTA
// reads its bs*d values as 16-byte vectors, reduces the maximum, then converts.
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"

namespace fvattn {

namespace {

constexpr int kQuantThreads = 256;

// Two fp32 values -> two e4m3 codes (low byte from `lo`): nearest, ties to even,
// saturating to +-448 (the cvt .satfinite form).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kQuantThreads)
    quant_e4m3_kernel(const __nv_bfloat16 *__restrict__ X, int N, int d, int bs, int nb, uint8_t *__restrict__ out,
                      int32_t *__restrict__ scale_exp) {
    __shared__ float warp_max[kQuantThreads / 32];
    __shared__ int block_e;
    const int64_t bh = blockIdx.x / nb;
    const int b = static_cast<int>(blockIdx.x % nb);
    const int t0 = b * bs;
    const int rows = min(bs, N - t0);
    const int64_t first = (bh * N + t0) * static_cast<int64_t>(d);  // element index of the block's first value
    const int nvec = rows * d / 8;                                   // 8 bf16 per 16-byte vector (d % 8 == 0)
    const uint4 *src = reinterpret_cast<const uint4 *>(X + first);

    float m = 0.0f;
    for (int i = threadIdx.x; i < nvec; i += kQuantThreads) {
        const uint4 v = __ldg(src + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[k])), fabsf(bf16_hi(w[k]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float amax = 0.0f;
        for (int w = 0; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);
        int e = 0;
        if (amax > 0.0f && isfinite(amax)) {  // a block holding inf keeps the scale 2^0
            // ldexpf by a power of two is exact here (no overflow: amax * 2^-e stays near 448);
            // the start is within one step of the answer, the loops are bounded regardless
            e = ilogbf(amax) - 8;
            for (int k = 0; k < 4 && ldexpf(amax, -e) > 448.0f; ++k) ++e;
            for (int k = 0; k < 4 && ldexpf(amax, -(e - 1)) <= 448.0f; ++k) --e;
        }
        block_e = e;
        scale_exp[blockIdx.x] = e;
    }
    __syncthreads();
    const int e = block_e;
    uint2 *dst = reinterpret_cast<uint2 *>(out + first);  // 8 codes per input vector
    for (int i = threadIdx.x; i < nvec; i += kQuantThreads) {
        const uint4 v = __ldg(src + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) c[k] = e4m3x2(ldexpf(bf16_lo(w[k]), -e), ldexpf(bf16_hi(w[k]), -e));
        dst[i] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    }
}

}  // namespace

cudaError_t launch_quant_e4m3(const void *X, int64_t BH, int N, int d, int bs, uint8_t *out, int32_t *scale_exp,
                              cudaStream_t stream) {
    const int nb = (N + bs - 1) / bs;
    const int64_t blocks = BH * nb;
    if (blocks <= 0) return cudaSuccess;
    quant_e4m3_kernel<<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(X), N, d, bs, nb, out, scale_exp);
    return cudaGetLastError();
}

}  // namespace fvattn
