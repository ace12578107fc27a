// zq_tp.cu — the reduction step of a tensor-parallel (K-split) linear layer.
//
// [wiki] "ZSE - open-source движок для запуска LLM локально на GPU - 2026",
// section "Тензорный параллелизм": weights are sharded across processes,
// column-parallel for QKV/Gate/Up and row-parallel for O/Down, with NCCL
// collectives (AllReduce, ReduceScatter, ...).  A row-parallel shard holds a
// slice of K (whole groups of 128) and yields fp32 partial sums of the full
// output (zq_linear_partial); this kernel adds the shards' partial sums in a
// fixed order and rounds once to fp16.  The partial buffers may live on this
// GPU or be peers' memory reached over NVLink (plain loads).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zq_internal.h"

namespace zq {

struct ReduceArgs {
    const float *parts[kMaxReduceParts];
    int n_parts;
    int vec;  // every pointer 16-byte aligned and count % 4 == 0: float4 loads
    size_t count;
    uint16_t *out;
};

__global__ void __launch_bounds__(256) reduce_partials_kernel(const __grid_constant__ ReduceArgs a) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (a.vec) {
        const size_t n4 = a.count / 4;
        for (; i < n4; i += stride) {
            float4 s = __ldcg(reinterpret_cast<const float4 *>(a.parts[0]) + i);
            for (int p = 1; p < a.n_parts; ++p) {  // fixed order: part 0, 1, 2, ...
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.parts[p]) + i);
                s.x += v.x;
                s.y += v.y;
                s.z += v.z;
                s.w += v.w;
            }
            const __half2 lo = __floats2half2_rn(s.x, s.y), hi = __floats2half2_rn(s.z, s.w);
            uint2 o;
            o.x = *reinterpret_cast<const uint32_t *>(&lo);
            o.y = *reinterpret_cast<const uint32_t *>(&hi);
            reinterpret_cast<uint2 *>(a.out)[i] = o;
        }
    } else {
        for (; i < a.count; i += stride) {
            float s = __ldcg(a.parts[0] + i);
            for (int p = 1; p < a.n_parts; ++p) s += __ldcg(a.parts[p] + i);
            a.out[i] = __half_as_ushort(__float2half_rn(s));
        }
    }
}

cudaError_t launch_reduce_partials(const float *const *parts, int n_parts, size_t count, uint16_t *out,
                                   cudaStream_t stream) {
    ReduceArgs a = {};
    bool vec = (count % 4) == 0;
    for (int p = 0; p < n_parts; ++p) {
        a.parts[p] = parts[p];
        vec = vec && (reinterpret_cast<uintptr_t>(parts[p]) % 16) == 0;
    }
    a.n_parts = n_parts;
    a.vec = vec ? 1 : 0;
    a.count = count;
    a.out = out;
    const size_t items = vec ? count / 4 : count;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t blocks_needed = (items + 255) / 256;
    const unsigned blocks = static_cast<unsigned>(blocks_needed < static_cast<size_t>(sms) * 8 ? blocks_needed
                                                                                           : static_cast<size_t>(sms) * 8);
    reduce_partials_kernel<<<blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace zq
