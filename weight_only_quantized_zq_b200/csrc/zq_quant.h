// zq_quant.h — internal declarations of the quantizer variants beyond the
// asymmetric one (whose launcher sits with the other kernel launchers), and
// of the KV-cache store built on the same codec.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace zq {

// Symmetric quantize-and-pack: Q = 2^(bits-1) - 1, scale = fp16(max|w| / Q),
// q = clamp(round_half_even(w / scale), -Q, Q), stored as code = q + 2^(bits-1)
// with zero = -2^(bits-1) * scale.  Same launch shape and status slot protocol
// as launch_quantize_pack; a group whose zero is not a finite fp16 also sets
// the status slot.
cudaError_t launch_quantize_pack_symmetric(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                                           uint16_t *scales, uint16_t *zeros, int slot,
                                           unsigned long long call_id, cudaStream_t stream);

// ------------------------------------------------------------- KV cache --
// One K or V plane of the quantized KV cache (zq_kv.h): fp16 ring of the
// newest `window` tokens, quantized store of the older ones.
struct KvArgs {
    uint16_t *ring;
    uint32_t *packed;
    uint16_t *scales;
    uint16_t *zeros;
    int window, heads, dim, bits;
};

// Appends rows (fp16 n x heads x dim) to a plane holding t0 tokens.
cudaError_t launch_kv_append(const KvArgs &a, const uint16_t *rows, int t0, int n, cudaStream_t stream);
// Tokens [t_a, t_b) of a plane holding t_total tokens, as fp16, into out.
cudaError_t launch_kv_gather(const KvArgs &a, int t_total, int t_a, int t_b, uint16_t *out, cudaStream_t stream);
// Reads and clears the device word that records a non-finite KV row.
cudaError_t read_kv_error(int *err);

}  // namespace zq
