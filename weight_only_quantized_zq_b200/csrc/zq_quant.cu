// zq_quant.cu — quantize-and-pack and the unpack test hook (sm_100a).
//
// Quantizer: [wiki] "ZSE - open-source движок для запуска LLM локально на GPU -
// 2026", section "Формат модели .zse" (scale = (max - min)/15, zero = min,
// q = clamp(round((w - zero)/scale), 0, 15), fp16 scale/zero, two INT4 codes per
// byte, low nibble first), generalised to L = 2^b - 1 for the per-tensor INT2-8
// widths of "ZSE: A Memory-Efficient LLM Inference Engine with Smart Resource
// Orchestration", section "Technical Architecture".
//
// Symmetric variant: the same section lists symmetric INT8 quantization
// (reserved) without a formula.  Q = 2^(b-1) - 1, scale = fp16(max|w| / Q),
// q = clamp(round(w / scale), -Q, Q), stored in the asymmetric format as
// code = q + 2^(b-1) with zero = -2^(b-1) * scale (exact: a power-of-two
// multiple), so every linear kernel computes code*scale + zero = q*scale.
//
// Arithmetic: fp64 with explicit round-to-nearest intrinsics (no contraction),
// one rounding to fp16 for the stored scale and zero, q from the STORED fp16
// values, round half to even.  This makes the result bit-identical to any
// IEEE-754 implementation of the same steps.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zq_device.cuh"
#include "zq_internal.h"
#include "zq_quant.h"
#include "zq_quant_warp.cuh"

namespace zq {

// Per-call status words for the non-finite check.  A call owns one slot, keyed
// by a unique call id, so no clearing is needed between calls.
__device__ unsigned long long g_quant_status[kQuantStatusSlots];

// One warp per (row, block of 128 weights: 1, 2 or 4 groups).  Each lane owns
// 4 consecutive weights.
template <bool SYMMETRIC>
__global__ void __launch_bounds__(256) quantize_pack_kernel(
    const float *__restrict__ w, int N, int K, int bits, int group, uint32_t *__restrict__ packed,
    uint16_t *__restrict__ scales, uint16_t *__restrict__ zeros, int slot,
    unsigned long long call_id) {
    __shared__ uint32_t words[8][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = K / 128;  // blocks per row
    const long long item = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (item >= static_cast<long long>(N) * G) return;
    const int n = static_cast<int>(item / G), g = static_cast<int>(item % G);

    const float4 v4 = *reinterpret_cast<const float4 *>(w + static_cast<size_t>(n) * K +
                                                        static_cast<size_t>(g) * 128 + lane * 4);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    uint16_t s16, z16;
    if (!quantize_group_warp<SYMMETRIC>(v, bits, lane, words[warp], s16, z16, group)) {
        if (lane == 0) atomicExch(&g_quant_status[slot], call_id);
        return;
    }
    const int nw = 4 * bits;
    const size_t wpr = static_cast<size_t>(K) * bits / 32;
    if (lane < nw) packed[static_cast<size_t>(n) * wpr + static_cast<size_t>(g) * nw + lane] = words[warp][lane];
    const int lpg = group >> 2;  // lanes per group; the first lane of each writes its scale and zero
    if ((lane & (lpg - 1)) == 0) {
        const int per = 128 / group;
        const size_t at = static_cast<size_t>(n) * (K / group) + static_cast<size_t>(g) * per + lane / lpg;
        scales[at] = s16;
        zeros[at] = z16;
    }
}

// Unpack test hook: one thread per 32-code chunk, through unpack_pair<B>, the
// routine the linear kernels use.
template <int B>
__global__ void unpack_kernel(const uint32_t *__restrict__ packed, int N, int K,
                              uint8_t *__restrict__ codes) {
    const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int chunks_per_row = K / 32;
    if (t >= static_cast<long long>(N) * chunks_per_row) return;
    const int n = static_cast<int>(t / chunks_per_row), c = static_cast<int>(t % chunks_per_row);
    const uint32_t *src = packed + static_cast<size_t>(n) * (static_cast<size_t>(K) * B / 32) +
                          static_cast<size_t>(c) * B;
    uint32_t w[B];
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = src[i];
    uint8_t *dst = codes + static_cast<size_t>(n) * K + static_cast<size_t>(c) * 32;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const uint32_t h2 = unpack_pair<B>(w, p);
        const float lo = h2f_bits(h2 & 0xFFFFu), hi = h2f_bits(h2 >> 16);
        dst[pair_lo<B>(p)] = static_cast<uint8_t>(lo);
        dst[pair_hi<B>(p)] = static_cast<uint8_t>(hi);
    }
}

cudaError_t launch_quantize_pack(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                                 uint16_t *scales, uint16_t *zeros, int slot,
                                 unsigned long long call_id, cudaStream_t stream) {
    const long long items = static_cast<long long>(N) * (K / 128);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    quantize_pack_kernel<false><<<blocks, 256, 0, stream>>>(w, N, K, bits, group, packed, scales, zeros, slot,
                                                            call_id);
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack_symmetric(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                                           uint16_t *scales, uint16_t *zeros, int slot,
                                           unsigned long long call_id, cudaStream_t stream) {
    const long long items = static_cast<long long>(N) * (K / 128);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    quantize_pack_kernel<true><<<blocks, 256, 0, stream>>>(w, N, K, bits, group, packed, scales, zeros, slot,
                                                           call_id);
    return cudaGetLastError();
}

cudaError_t read_quant_status(int slot, unsigned long long *value, cudaStream_t stream) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(value, g_quant_status, sizeof(unsigned long long),
                                              sizeof(unsigned long long) * slot,
                                              cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

cudaError_t launch_unpack(const uint32_t *packed, int N, int K, int bits, uint8_t *codes,
                          cudaStream_t stream) {
    const long long threads = static_cast<long long>(N) * (K / 32);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    switch (bits) {
        case 2: unpack_kernel<2><<<blocks, 256, 0, stream>>>(packed, N, K, codes); break;
        case 3: unpack_kernel<3><<<blocks, 256, 0, stream>>>(packed, N, K, codes); break;
        case 4: unpack_kernel<4><<<blocks, 256, 0, stream>>>(packed, N, K, codes); break;
        default: unpack_kernel<8><<<blocks, 256, 0, stream>>>(packed, N, K, codes); break;
    }
    return cudaGetLastError();
}

}  // namespace zq
