// zq_kv.cu — zKV, the quantized KV cache with sliding precision (sm_100a).
//
// "ZSE: Motor de inferência de LLM de código aberto com inicializações a frio
// de 3,9 segundos", section "Componentes da arquitetura", and "ZSE: A
// Memory-Efficient LLM Inference Engine with Smart Resource Orchestration",
// section "Technical Architecture", name zKV: a KV cache quantized with
// "sliding precision" for about 4x less memory.  Here the newest `window`
// tokens of a plane stay in an fp16 ring and every older token sits in the
// store, quantized with the weights' group codec (zq_quant_warp.cuh).
//
// Append: one warp per (item, head, group of 128).  Ring items are the new
// tokens that end in the ring; each takes over slot t % window, first moving
// the slot's previous token to the store (read before the overwrite, by the
// same lanes), so the slots are disjoint between warps.  Direct items (only
// when more than `window` tokens arrive at once) are new tokens that leave the
// window within the same call; they go straight from the input to the store.
// The result equals appending the tokens one at a time.
//
// Gather: one thread per (token, head, 32-value chunk): a ring row is copied,
// a store row is unpacked with the linear kernels' exact unpack and
// dequantized by one HFMA2, fp16(q * scale + zero) with one rounding.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zq_device.cuh"
#include "zq_quant.h"
#include "zq_quant_warp.cuh"

namespace zq {

__device__ int g_kv_error;  // ZQ_ERR_NONFINITE once a row held NaN or Inf

__global__ void __launch_bounds__(256) kv_append_kernel(const KvArgs a, const uint16_t *__restrict__ rows, int t0,
                                                        int n, int r0, long long total_warps) {
    __shared__ uint32_t words[8][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * 8 + warp;
    if (gw >= total_warps) return;
    const int G = a.dim / 128;
    const int g = static_cast<int>(gw % G);
    const long long rest = gw / G;
    const int h = static_cast<int>(rest % a.heads);
    const int item = static_cast<int>(rest / a.heads);
    const int m = t0 + n - r0;  // ring items: tokens r0 .. t0+n-1
    const size_t row_vals = static_cast<size_t>(a.heads) * a.dim;
    const size_t off = static_cast<size_t>(h) * a.dim + static_cast<size_t>(g) * 128 + lane * 4;

    int t_store = -1;  // token quantized into the store by this warp
    uint2 raw = make_uint2(0u, 0u);
    if (item < m) {
        const int t = r0 + item;
        // Previous occupant of slot t % window: the newest earlier token of
        // the same slot, t - window * (floor((t - t0) / window) + 1).
        const int u = t - a.window * ((t - t0) / a.window + 1);
        uint16_t *slot = a.ring + static_cast<size_t>(t % a.window) * row_vals + off;
        const uint2 in = *reinterpret_cast<const uint2 *>(rows + static_cast<size_t>(t - t0) * row_vals + off);
        if (u >= 0) {
            raw = *reinterpret_cast<const uint2 *>(slot);
            t_store = u;
        }
        *reinterpret_cast<uint2 *>(slot) = in;
    } else {
        const int t = t0 + (item - m);
        raw = *reinterpret_cast<const uint2 *>(rows + static_cast<size_t>(t - t0) * row_vals + off);
        t_store = t;
    }
    if (t_store < 0) return;  // the same for the whole warp
    const float v[4] = {h2f_bits(raw.x & 0xFFFFu), h2f_bits(raw.x >> 16), h2f_bits(raw.y & 0xFFFFu),
                        h2f_bits(raw.y >> 16)};
    uint16_t s16, z16;
    if (!quantize_group_warp<false>(v, a.bits, lane, words[warp], s16, z16)) {
        if (lane == 0) atomicExch(&g_kv_error, 3);  // ZQ_ERR_NONFINITE
        return;
    }
    const int nw = 4 * a.bits;
    const size_t hrow = static_cast<size_t>(t_store) * a.heads + h;  // (token, head) row of the store
    if (lane < nw) a.packed[hrow * (static_cast<size_t>(a.dim) * a.bits / 32) + static_cast<size_t>(g) * nw + lane] =
        words[warp][lane];
    if (lane == 0) {
        a.scales[hrow * G + g] = s16;
        a.zeros[hrow * G + g] = z16;
    }
}

template <int B>
__global__ void __launch_bounds__(256) kv_gather_kernel(const KvArgs a, int t_total, int t_a,
                                                        uint16_t *__restrict__ out, long long total_threads) {
    const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
    if (i >= total_threads) return;
    const int C = a.dim / 32;  // chunks per head row
    const int c = static_cast<int>(i % C);
    const long long rest = i / C;
    const int h = static_cast<int>(rest % a.heads);
    const int j = static_cast<int>(rest / a.heads);
    const int t = t_a + j;
    uint4 *dst = reinterpret_cast<uint4 *>(out + (static_cast<size_t>(j) * a.heads + h) * a.dim + c * 32);
    if (t >= t_total - a.window) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            a.ring + (static_cast<size_t>(t % a.window) * a.heads + h) * a.dim + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = src[q];
        return;
    }
    const size_t hrow = static_cast<size_t>(t) * a.heads + h;
    const uint32_t *src = a.packed + hrow * (static_cast<size_t>(a.dim) * B / 32) + static_cast<size_t>(c) * B;
    uint32_t w[B];
#pragma unroll
    for (int q = 0; q < B; ++q) w[q] = src[q];
    const int G = a.dim / 128;
    const uint32_t s2 = static_cast<uint32_t>(a.scales[hrow * G + c / 4]) * 0x10001u;
    const uint32_t z2 = static_cast<uint32_t>(a.zeros[hrow * G + c / 4]) * 0x10001u;
    uint32_t o[16];  // natural order, two values per word
#pragma unroll
    for (int q = 0; q < 16; ++q) o[q] = 0u;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const uint32_t v = hfma2_bits(unpack_pair<B>(w, p), s2, z2);
        const int lo = pair_lo<B>(p), hi = pair_hi<B>(p);
        o[lo / 2] |= (v & 0xFFFFu) << (16 * (lo & 1));
        o[hi / 2] |= (v >> 16) << (16 * (hi & 1));
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
}

cudaError_t launch_kv_append(const KvArgs &a, const uint16_t *rows, int t0, int n, cudaStream_t stream) {
    const int r0 = (t0 + n - a.window > t0) ? t0 + n - a.window : t0;  // first new token kept in the ring
    const long long warps = static_cast<long long>(n) * a.heads * (a.dim / 128);  // n items: ring, then direct
    const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
    kv_append_kernel<<<blocks, 256, 0, stream>>>(a, rows, t0, n, r0, warps);
    return cudaGetLastError();
}

cudaError_t launch_kv_gather(const KvArgs &a, int t_total, int t_a, int t_b, uint16_t *out, cudaStream_t stream) {
    const long long threads = static_cast<long long>(t_b - t_a) * a.heads * (a.dim / 32);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    switch (a.bits) {
        case 2: kv_gather_kernel<2><<<blocks, 256, 0, stream>>>(a, t_total, t_a, out, threads); break;
        case 3: kv_gather_kernel<3><<<blocks, 256, 0, stream>>>(a, t_total, t_a, out, threads); break;
        case 4: kv_gather_kernel<4><<<blocks, 256, 0, stream>>>(a, t_total, t_a, out, threads); break;
        default: kv_gather_kernel<8><<<blocks, 256, 0, stream>>>(a, t_total, t_a, out, threads); break;
    }
    return cudaGetLastError();
}

cudaError_t read_kv_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_kv_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_kv_error, &zero, sizeof(int));
}

}  // namespace zq
