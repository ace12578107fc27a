// zq_internal.h — declarations shared between the host entry points and the
// kernel translation units of libzq.  Not part of the public ABI.
#pragma once

#include <cuda.h>
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

constexpr int kMaxDecodeOps = 112;
constexpr int kMaxPrepEntries = 64;
constexpr int kDecodeWarpsPerCta = 4;

struct alignas(64) DecodeOp {
    CUtensorMap tmap;       // packed codes as a 2-D uint8 tensor: box = 16 rows x one step's bytes
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
    int sz_vec;             // G % GPS == 0: scales/zeros of a step are one aligned vector per row
    int pad_;
};

struct DecodeParams {
    long long total_steps;
    float *part;             // workspace: 2 partial slots per chunk, slot_floats each
    unsigned int *cnt;       // workspace: [0] work counter (reset by prep), [1 + k] arrival counter of chunk k
    int slot_floats;         // rows * max M
    int n_ops;
    int log2c;               // chunk = 2^log2c consecutive steps
    int n_chunks;
    int dynamic;             // 1: chunks beyond the first per warp are taken from cnt[0]
    int pad_;
    DecodeOp ops[kMaxDecodeOps];
};
static_assert(sizeof(DecodeParams) <= 32000, "kernel parameter space");

struct PrepEntry {
    const uint16_t *x;  // M x K fp16
    uint16_t *xperm;    // M_pad x K
    float *sx;          // G x M_pad x 2: (sum of x, 1024 * sum of scaled x)
    int M, M_pad, K, bits;
};

struct PrepParams {
    unsigned int *work;  // decode work counter, reset to 0 (may be null)
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
// Per-warp ring stage: the step's codes (dense, written by TMA) followed by
// the step's scales and zeros, 16 rows x {scales, zeros} x GPS halves.
__host__ __device__ constexpr int decode_sz_bytes(int bits) { return 16 * 2 * decode_gps(bits) * 2; }
__host__ __device__ constexpr int decode_stage(int bits) { return 16 * decode_seg(bits) + decode_sz_bytes(bits); }
// Ring depth: about 13 KB per warp, at least 3 stages.
__host__ __device__ constexpr int decode_depth(int bits) {
    return 13312 / decode_stage(bits) < 3 ? 3 : 13312 / decode_stage(bits) > 6 ? 6 : 13312 / decode_stage(bits);
}
inline size_t decode_smem_bytes(int bits, int) {
    return static_cast<size_t>(kDecodeWarpsPerCta) * (decode_depth(bits) * decode_stage(bits) + 8 * decode_depth(bits)) +
           128;
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
cudaError_t read_decode_error(int *err);
cudaError_t encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t dim0,
                                 uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                                 CUtensorMapSwizzle swizzle);

// Largest M handled by the decode family; larger M goes to the prefill family.
constexpr int kDecodeMaxM = 64;

cudaError_t launch_prep(const PrepParams &p, long long total_warps, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, int bits, int mt, int n_ctas, cudaStream_t stream);
cudaError_t decode_ctas_per_sm(int bits, int mt, int *ctas);

}  // namespace zq
