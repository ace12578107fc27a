// zq_prefill.h — internal declarations of the tile kernel's two shared-memory
// plans (zq_prefill.cu).  A launch whose ops all have M <= kPrefillHalfTokens
// runs the one-token-half plan, whose x tensor maps have boxes of
// kPrefillHalfTokens rows; any other launch runs the two-half plan with boxes
// of 256 rows.  The host builds every op's map with prefill_box_rows() of the
// launch, so maps and plan always agree.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "zq_internal.h"

namespace zq {

constexpr int kPrefillHalfTokens = 128;

// Tensor map of x (M x K fp16) with boxes of 64 k x box_rows tokens, 128-byte swizzle.
cudaError_t prefill_x_map_rows(CUtensorMap *map, const uint16_t *x, int M, int K, int box_rows);

// Tensor map of fp16 weights W (N x K) with boxes of 64 k x 256 rows, 128-byte
// swizzle: the W slab of the tile kernel for bits = 16.
cudaError_t prefill_w_map(CUtensorMap *map, const uint16_t *w, int N, int K);

// Token rows per x box of a launch: 128 if every op has M <= 128, else 256.
// Reads only the ops' M, so it may be called before their maps are built.
int prefill_box_rows(const PrefillGroup &pg);

}  // namespace zq
