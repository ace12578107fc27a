// zq_internal.h — declarations shared between the host entry points and the
// kernel translation units of libzq.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace zq {

constexpr int kGroup = 128;
constexpr int kQuantStatusSlots = 64;

// ---------------------------------------------------------------- decode --
// A decode launch processes up to kMaxDecodeOps independent linear layers of
// one bit width with M <= 64.  The work is a sequence of steps, one step =
// (op, row block, 128-wide group); op o owns steps [step0, step0 + row_blocks*G)
// in row-block-major order.  Warp w of W takes steps [T*w/W, T*(w+1)/W)
// (stream-K): a row block cut by a warp boundary is summed from per-warp
// partial slots by the last warp to finish it.

constexpr int kMaxDecodeOps = 128;
constexpr int kMaxPrepEntries = 64;
constexpr int kDecodeWarpsPerCta = 4;

struct DecodeOp {
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *zeros;
    const uint16_t *xperm;  // workspace: M_pad x K fp16, pair-permuted, 2^-s-scaled activations
    const float *sx;        // workspace: G x M_pad x 2 fp32 (sum x, bias) per group and token
    uint16_t *out;          // M x N fp16
    long long step0;        // first step of this op
    int M, N, K, G;
    int row_blocks;
    int su;                 // steps per row block: ceil(G / GPS)
};

struct DecodeParams {
    long long total_steps;
    float *part;             // workspace: 2 partial slots per warp, slot_floats each
    unsigned int *cnt;       // workspace: one arrival counter per warp (zero between calls)
    int slot_floats;         // rows * max M
    int n_ops;
    DecodeOp ops[kMaxDecodeOps];
};

struct PrepEntry {
    const uint16_t *x;  // M x K fp16
    uint16_t *xperm;    // M_pad x K
    float *sx;          // G x M_pad x 2: (sum of x, 1024 * sum of scaled x)
    int M, M_pad, K, bits;
};

struct PrepParams {
    int n_entries;
    int pad_;
    long long warp_prefix[kMaxPrepEntries + 1];  // warps before entry i
    PrepEntry e[kMaxPrepEntries];
};

// Decode tiling.  A warp step covers 16 weight rows x GPS groups (a 256-byte
// row segment at 4 and 8 bits: longer DRAM bursts than one group per row).
__host__ __device__ constexpr int decode_rows(int) { return 16; }
__host__ __device__ constexpr int decode_gps(int bits) { return bits == 8 ? 2 : 4; }
__host__ __device__ constexpr int decode_seg(int bits) { return decode_gps(bits) * 16 * bits; }
// Shared-memory row stride.  2, 4 and 8 bits use an XOR swizzle of the 16-byte
// chunks (decode_swizzle) to keep fragment reads bank-conflict free; 3 bits
// pads each row by 16 bytes instead.
__host__ __device__ constexpr int decode_row_stride(int bits) { return decode_seg(bits) + (bits == 3 ? 16 : 0); }
__host__ __device__ constexpr int decode_swizzle(int bits, int row, int chunk) {
    return bits == 2 ? chunk ^ ((row & 3) << 1) : bits == 4 ? chunk ^ ((row & 1) << 2) : bits == 8 ? chunk ^ (row & 1) : chunk;
}
__host__ __device__ constexpr int decode_stage(int bits) { return 16 * decode_row_stride(bits); }
// cp.async ring depth: about 12 KB of codes per warp.
__host__ __device__ constexpr int decode_depth(int bits) {
    return 12288 / decode_stage(bits) < 2 ? 2 : 12288 / decode_stage(bits) > 8 ? 8 : 12288 / decode_stage(bits);
}
inline size_t decode_smem_bytes(int bits, int) {
    return static_cast<size_t>(kDecodeWarpsPerCta) * decode_depth(bits) * decode_stage(bits);
}
inline int mt_for_m(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

cudaError_t launch_quantize_pack(const float *w, int N, int K, int bits, uint32_t *packed,
                                 uint16_t *scales, uint16_t *zeros, int slot,
                                 unsigned long long call_id, cudaStream_t stream);
cudaError_t read_quant_status(int slot, unsigned long long *value, cudaStream_t stream);
cudaError_t launch_unpack(const uint32_t *packed, int N, int K, int bits, uint8_t *codes,
                          cudaStream_t stream);

cudaError_t launch_prefill(const uint16_t *x, const uint32_t *packed, const uint16_t *scales,
                           const uint16_t *zeros, int bits, int M, int N, int K, uint16_t *out, int num_sms,
                           cudaStream_t stream);
cudaError_t read_prefill_error(int *err);

// Largest M handled by the decode family; larger M goes to the prefill family.
constexpr int kDecodeMaxM = 64;

cudaError_t launch_prep(const PrepParams &p, long long total_warps, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, int bits, int mt, int n_ctas, cudaStream_t stream);
cudaError_t decode_ctas_per_sm(int bits, int mt, int *ctas);

}  // namespace zq
