// zq_prefill.h — internal declarations of the tile kernel's three plans
// (zq_prefill.cu).  A launch whose ops all have M <= kPrefillHalfTokens runs
// the one-token-half plan (256-token tiles, x boxes of kPrefillHalfTokens
// rows); a launch of b-bit codes with some M >= kPairMinM runs the CTA-pair
// plan (512-token tiles, x boxes of kPrefillHalfTokens rows); any other runs
// the two-half plan (256-token tiles, x boxes of 256 rows).  The host builds every
// op's map and tile count from prefill_plan() of the launch, so maps, tiles
// and plan always agree.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "zq_internal.h"

namespace zq {

constexpr int kPrefillHalfTokens = 128;
constexpr int kPrefillQuarterTokens = 64;  // x stage rows of the one-half plan when every M <= 64 (b <= 4)

// Tensor map of x (M x K fp16) with boxes of 64 k x box_rows tokens, 128-byte swizzle.
cudaError_t prefill_x_map_rows(CUtensorMap *map, const uint16_t *x, int M, int K, int box_rows);

// Tensor map of fp16 weights W (N x K) with boxes of 64 k x 256 rows, 128-byte
// swizzle: the W slab of the tile kernel for bits = 16.
cudaError_t prefill_w_map(CUtensorMap *map, const uint16_t *w, int N, int K);

constexpr int kPlanOneHalf = 0, kPlanTwoHalves = 1, kPlanPair = 2, kPlanOneHalf64 = 3;
constexpr int kPairMinM = 512;  // the CTA-pair plan runs launches with some M >= 512

// Plan of a launch from its ops' M (read only; may be called before the maps
// are built) and bit width.
int prefill_plan(const PrefillGroup &pg, int bits);
// Token rows per x box, tokens per tile, and tiles of an M x N op, per plan.
int prefill_box_rows(int plan);
int prefill_tok_tile(int plan);
int prefill_tiles(int M, int N, int plan);

}  // namespace zq
