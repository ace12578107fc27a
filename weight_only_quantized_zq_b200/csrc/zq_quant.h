// zq_quant.h — internal declarations of the quantizer variants beyond the
// asymmetric one (whose launcher sits with the other kernel launchers).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace zq {

// Symmetric quantize-and-pack: Q = 2^(bits-1) - 1, scale = fp16(max|w| / Q),
// q = clamp(round_half_even(w / scale), -Q, Q), stored as code = q + 2^(bits-1)
// with zero = -2^(bits-1) * scale.  Same launch shape and status slot protocol
// as launch_quantize_pack; a group whose zero is not a finite fp16 also sets
// the status slot.
cudaError_t launch_quantize_pack_symmetric(const float *w, int N, int K, int bits, uint32_t *packed,
                                           uint16_t *scales, uint16_t *zeros, int slot,
                                           unsigned long long call_id, cudaStream_t stream);

}  // namespace zq
