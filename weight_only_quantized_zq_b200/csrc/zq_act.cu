// zq_act.cu — activation copies for the tile kernel: bfloat16 activations
// brought into fp16, and the pair-permuted K order of its one-token-half
// plan.
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

#include "zq_device.cuh"
#include "zq_internal.h"

namespace zq {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Pair-permuted order of a 32-value chunk (the tile kernel's one-token-half
// plan): position 2w holds value pair_lo<B>(w), position 2w + 1 value
// pair_hi<B>(w), the order in which the dequant routine yields its fp16
// weight pairs, so that it stores them without restoring K order.
template <int B>
__device__ __forceinline__ void pair_permute(const uint16_t (&h)[32], uint32_t (&o)[16]) {
#pragma unroll
    for (int w = 0; w < 16; ++w)
        o[w] = static_cast<uint32_t>(h[pair_lo<B>(w)]) | (static_cast<uint32_t>(h[pair_hi<B>(w)]) << 16);
}
__device__ __forceinline__ void chunk_out(const uint16_t (&h)[32], int perm_bits, uint4 *dst) {
    uint32_t o[16];
    switch (perm_bits) {
        case 2: pair_permute<2>(h, o); break;
        case 3: pair_permute<3>(h, o); break;
        case 4: pair_permute<4>(h, o); break;
        case 8: pair_permute<8>(h, o); break;
        default:
#pragma unroll
            for (int w = 0; w < 16; ++w) o[w] = static_cast<uint32_t>(h[2 * w]) | (static_cast<uint32_t>(h[2 * w + 1]) << 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

// One block per token row: the row scaled to fp16 by 2^E, each 32-value
// chunk in natural order (perm_bits 0) or pair-permuted for b = perm_bits.
__global__ void __launch_bounds__(256) bf16_rows_to_f16_kernel(const uint16_t *__restrict__ x, int K, int perm_bits,
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
    for (int c = threadIdx.x; c < K / 32; c += blockDim.x) {  // one 32-value chunk per thread
        uint16_t h[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = src[4 * c + q];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                h[8 * q + 2 * j] = __half_as_ushort(__float2half_rn(bf16_bits_to_float(w[j] & 0xFFFFu) * up));
                h[8 * q + 2 * j + 1] = __half_as_ushort(__float2half_rn(bf16_bits_to_float(w[j] >> 16) * up));
            }
        }
        chunk_out(h, perm_bits, dst + 4 * c);
    }
    if (threadIdx.x == 0) f[blockIdx.x] = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
}

// fp16 rows, each 32-value chunk pair-permuted for b = bits: one chunk (64
// bytes) per thread.
__global__ void __launch_bounds__(256) x_pairperm_kernel(const uint16_t *__restrict__ x, long long chunks, int bits,
                                                        uint16_t *__restrict__ out) {
    const long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= chunks) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x) + 4 * c;
    uint16_t h[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 v = src[q];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            h[8 * q + 2 * j] = static_cast<uint16_t>(w[j] & 0xFFFFu);
            h[8 * q + 2 * j + 1] = static_cast<uint16_t>(w[j] >> 16);
        }
    }
    chunk_out(h, bits, reinterpret_cast<uint4 *>(out) + 4 * c);
}

cudaError_t launch_bf16_rows_to_f16(const uint16_t *x, int M, int K, int perm_bits, uint16_t *x16, float *f,
                                    cudaStream_t stream) {
    bf16_rows_to_f16_kernel<<<static_cast<unsigned>(M), 256, 0, stream>>>(x, K, perm_bits, x16, f);
    return cudaGetLastError();
}

cudaError_t launch_x_pairperm(const uint16_t *x, int M, int K, int bits, uint16_t *out, cudaStream_t stream) {
    const long long chunks = static_cast<long long>(M) * (K / 32);
    x_pairperm_kernel<<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, stream>>>(x, chunks, bits, out);
    return cudaGetLastError();
}

}  // namespace zq
