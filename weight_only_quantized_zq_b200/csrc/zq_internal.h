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
// one bit width with M <= 64.  Work is split into units (op, row block,
// K slice) and spread over all warps of a persistent grid by cost (bytes).

constexpr int kMaxDecodeOps = 128;
constexpr int kMaxPrepEntries = 64;
constexpr int kDecodeWarpsPerCta = 4;

struct DecodeOp {
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *zeros;
    const uint16_t *xperm;  // workspace: M_pad x K fp16, chunk-permuted activations
    const float *sx;        // workspace: G x M_pad x 2 fp32 (sum x, bias) per group and token
    uint16_t *out;          // M x N fp16
    float *part;            // workspace: split-K partials (S > 1) or null
    unsigned int *cnt;      // workspace: split-K arrival counters (S > 1) or null
    long long cost0;        // cost of all earlier ops (prefix)
    long long unit_cost;    // cost of one unit
    int M, N, K, G;
    int S;                  // K slices
    int gps;                // groups per slice (last slice may be shorter)
    int row_blocks;
    int pad_;
};

struct DecodeParams {
    long long total_cost;
    int n_ops;
    int pad_;
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

// Decode tiling for a token-tile count MT (tokens padded to 8*MT).
__host__ __device__ constexpr int decode_rt(int mt) { return mt == 1 ? 4 : mt == 2 ? 2 : 1; }
__host__ __device__ constexpr int decode_rows(int mt) { return 16 * decode_rt(mt); }
// cp.async ring depth: about 12 KB of codes per warp.
__host__ __device__ constexpr int decode_depth(int bits, int mt) {
    return (12288 / (decode_rows(mt) * 16 * bits)) < 2 ? 2
         : (12288 / (decode_rows(mt) * 16 * bits)) > 8 ? 8
                                                       : 12288 / (decode_rows(mt) * 16 * bits);
}
inline size_t decode_smem_bytes(int bits, int mt) {
    return static_cast<size_t>(kDecodeWarpsPerCta) * decode_depth(bits, mt) * decode_rows(mt) * 16 * bits;
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
