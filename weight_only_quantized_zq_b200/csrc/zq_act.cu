// zq_act.cu — activations given as bfloat16, for the tile kernel.
//
// The tensor cores multiply fp16 by fp16 here (the dequantized weights are
// fp16: bf16 weights would lose three bits), so bf16 activations are brought
// into fp16 first.  bf16 has fp32's exponent range and an 8-bit significand:
// scaled by a power of two that puts the row's largest |x| in [2^14, 2^15),
// every value at or above 2^-14 of the scaled range is exact in fp16 and only
// values below 2^-38 of the row's maximum round, far beneath the accuracy of
// the product.  The factor 2^-E is applied to the fp32 accumulators before
// the output is rounded.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zq_internal.h"

namespace zq {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// One block per token row.
__global__ void __launch_bounds__(256) bf16_rows_to_f16_kernel(const uint16_t *__restrict__ x, int K,
                                                              uint16_t *__restrict__ x16, float *__restrict__ f) {
    __shared__ float red[8];
    const size_t row = static_cast<size_t>(blockIdx.x) * K;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row);  // 8 values per 16 bytes (K % 128 == 0)
    const int n8 = K / 8;
    float amax = 0.0f;
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
        const uint4 v = src[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[j] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[j] >> 16))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) amax = fmaxf(amax, red[i]);
    // 2^E * amax in [2^14, 2^15); E = 0 for an all-zero row (amax is a normal
    // float or 0: bf16 subnormals are below 2^-126 and 2^E stays finite).
    int E = 0;
    if (amax > 0.0f) E = 14 - (static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127);
    // Rows whose largest |x| is below 2^-86 (scaled by at most 2^100) or above
    // 2^55 (fp16 would overflow) are outside the supported range.
    E = max(-40, min(E, 100));
    const float up = __uint_as_float(static_cast<uint32_t>(127 + E) << 23);
    uint4 *dst = reinterpret_cast<uint4 *>(x16 + row);
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
        const uint4 v = src[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2 h = __floats2half2_rn(bf16_bits_to_float(w[j] & 0xFFFFu) * up,
                                                bf16_bits_to_float(w[j] >> 16) * up);
            o[j] = *reinterpret_cast<const uint32_t *>(&h);
        }
        dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (threadIdx.x == 0) f[blockIdx.x] = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
}

cudaError_t launch_bf16_rows_to_f16(const uint16_t *x, int M, int K, uint16_t *x16, float *f, cudaStream_t stream) {
    bf16_rows_to_f16_kernel<<<static_cast<unsigned>(M), 256, 0, stream>>>(x, K, x16, f);
    return cudaGetLastError();
}

}  // namespace zq
