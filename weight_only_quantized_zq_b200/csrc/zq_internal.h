// zq_internal.h — declarations shared between the host entry points and the
// kernel translation units of libzq.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace zq {

constexpr int kGroup = 128;

// Records the message returned by zq_last_error() for the calling thread.
void set_last_error(const char *msg);
constexpr int kQuantStatusSlots = 64;

// ---------------------------------------------------------------- decode --
// A decode launch processes up to kMaxDecodeOps independent linear layers of
// one bit width with M <= kDecodeMaxM.  The work is a sequence of CTA steps, one step =
// (op, row block of decode_cta_rows rows, GPS consecutive groups of 128); op o owns steps
// [step0, step0 + row_blocks * su) in row-block-major order.  The steps are
// cut into chunks (whole row blocks, or 2^log2c consecutive steps); a CTA
// starts with chunk blockIdx.x and, in dynamic mode, takes further chunks from
// a counter.  A row block cut by a chunk boundary is summed from per-chunk
// partial slots by the last warp to finish a piece of it.

constexpr int kMaxDecodeOps = 112;
constexpr int kMaxPrepEntries = 64;
constexpr int kDecodeWarpsPerCta = 4;

struct alignas(64) DecodeOp {
    CUtensorMap tmap;       // packed codes as a 2-D uint8 tensor: box = decode_cta_rows rows x box_w bytes
    const uint16_t *scales;
    const uint16_t *zeros;
    const uint16_t *xg;     // workspace: pair-permuted, 2^(E-s)-scaled, chunk-swizzled fp16 activations
                            // by decode step, [K / (128 GPS)][x_rows][GPS x 128] (x_rows = M with one
                            // token tile, else M_pad)
    const float *sx;        // workspace: records (sum x, -f * 1024 * sum x', f, 0) fp32 per token and
                            // group by step, [K / (128 GPS)][x_rows][RS] (RS = decode_rec_stride >= GPS
                            // slots, group g at slot g % GPS); f = 2^-E undoes the power-of-two x' scale
    uint16_t *out;          // M x N fp16, or null when out32 is set
    float *out32;           // M x N fp32 (partial sums, not rounded), or null
    int step0;              // first CTA step of this op
    int unit0;              // first row block of this op (counted over the launch)
    int M, N, K, G;
    int row_blocks;         // ceil(N / decode_cta_rows)
    int su;                 // steps per row block: ceil(G / GPS)
    int sz_vec;             // G % GPS == 0: a step's scales/zeros of one row are one aligned vector
    int out_bf16;           // 1: out holds bfloat16 (bf16 activations), else fp16
};

// Kernel parameters of a decode launch of at most CAP ops.  They travel with
// every launch, so launches of few ops use a small block (a 28 KB block cost
// 2-3 us of latency per single-op call).
template <int CAP>
struct DecodeParamsT {
    float *part;             // workspace: 2 partial slots per chunk, slot_floats each
    unsigned int *cnt;       // workspace: [0] chunk counter (reset by prep), [1 + k] pieces of chunk k's row block
    int total_steps;
    int n_ops;
    int slot_floats;         // decode_cta_rows x M_pad
    int log2c;               // fixed chunks: 2^log2c consecutive steps
    int n_chunks;
    int units;               // 1: a chunk is one whole row block
    int dynamic;             // 1: chunks beyond the first per CTA are taken from cnt[0]
    int depth;               // ring stages
    int codes_bytes;         // codes of one stage (decode_cta_rows x one step's bytes), multiple of 1024
    int meta_bytes;          // rest of one stage, multiple of 16
    int off_sz, off_sx, off_x, off_desc;  // offsets inside a stage's meta part
    unsigned long long wait_ns;           // limit of a bounded wait (see wait_limit_ns)
    DecodeOp ops[CAP];
};
constexpr int kSmallLaunchOps = 8;  // ops (and distinct activations) of a small decode launch
using DecodeParams = DecodeParamsT<kMaxDecodeOps>;
using DecodeParamsSmall = DecodeParamsT<kSmallLaunchOps>;
static_assert(sizeof(DecodeParams) <= 32000, "kernel parameter space");

struct PrepEntry {
    const uint16_t *x;  // M x K fp16
    uint16_t *xg;       // [step][x_rows][GPS x 128], chunk-swizzled per group and token; rows >= M are zeros
    float *sx;          // [step][x_rows][RS] x 4: (sum of x, -f * 1024 * sum of scaled x, f, 0); zeros for rows >= M
    int M, x_rows, K, bits;  // x_rows: M with one token tile, else the padded M_pad
    int gps, rs;             // groups per decode step, record slots per token (decode_gps, decode_rec_stride)
    int x_bf16;              // 1: x holds bfloat16, else fp16
};

template <int CAP>
struct PrepParamsT {
    unsigned int *work;  // decode chunk counter, reset to 0 (may be null)
    int n_entries;
    int pad_;
    long long warp_prefix[CAP + 1];  // warps before entry i
    PrepEntry e[CAP];
};
using PrepParams = PrepParamsT<kMaxPrepEntries>;
using PrepParamsSmall = PrepParamsT<kSmallLaunchOps>;

// Decode tiling.  A CTA step covers 64 x RT weight rows x GPS groups; each of
// the 4 warps computes RT row tiles of 16.  With one or two token tiles RT = 1
// and GPS = 4 (2 at b = 8); with four token tiles GPS = 2 and, for b <= 4,
// RT = 2, so that each activation fragment a warp loads serves 32 weight rows
// while a stage (128 rows of codes, 2 x 32 x 256 bytes of activations) leaves
// room for a 3-stage ring at 2 CTAs per SM (b = 8 and fp16 weights, twice the
// code bytes per row, keep 64-row steps).  M = 17-32 ran 27 % faster with
// RT = 2; M = 9-16 about 1 % slower, so two token tiles keep RT = 1.
__host__ __device__ constexpr int decode_row_tiles(int bits, int mt) { return (mt >= 4 && bits <= 4) ? 2 : 1; }
__host__ __device__ constexpr int decode_cta_rows(int bits, int mt) {
    return 16 * kDecodeWarpsPerCta * decode_row_tiles(bits, mt);
}
// CTAs per SM the decode kernel's registers are budgeted for (its launch
// bounds) and the host's ring sizing aims at: 4 with one token tile (128
// registers), 3 with two, 2 with four.
__host__ __device__ constexpr int decode_reg_ctas(int, int mt) { return mt == 1 ? 4 : mt == 2 ? 3 : 2; }
__host__ __device__ constexpr int decode_gps(int bits, int mt) {
    return bits == 16 ? 1 : (bits == 8 || mt >= 4) ? 2 : 4;
}
__host__ __device__ constexpr int decode_seg(int bits, int mt) { return decode_gps(bits, mt) * 16 * bits; }
// Record slots (16 bytes) per token in a decode step's block of records: one
// spare slot when GPS > 1, so that the records of tokens 2c (c = 0..3),
// which a quad of lanes reads at once, start in four different bank quads (a
// token stride of 4 * 16 = 64 bytes would put all four in the same banks).
__host__ __device__ constexpr int decode_rec_stride(int bits, int mt) {
    return decode_gps(bits, mt) + (decode_gps(bits, mt) > 1 ? 1 : 0);
}
// Codes of a step land as 128-byte-wide TMA boxes with the 128-byte swizzle
// when a row segment is a whole number of 128-byte spans.  Otherwise (b = 3:
// 192 bytes) as one unswizzled box 16 bytes wider than the segment: a shared
// memory row pitch of 208 bytes (52 words) puts the 8 rows of a fragment load
// in 8 different bank quads, where 192 (48 words) would give only two.  The
// extra 16 bytes are the start of the next step's codes (or zero fill).
__host__ __device__ constexpr bool decode_swizzled(int bits, int mt) { return decode_seg(bits, mt) % 128 == 0; }
__host__ __device__ constexpr int decode_box_w(int bits, int mt) {
    return decode_swizzled(bits, mt) ? 128 : decode_seg(bits, mt) + 16;
}
__host__ __device__ constexpr int decode_boxes(int bits, int mt) {
    return decode_swizzled(bits, mt) ? decode_seg(bits, mt) / 128 : 1;
}
// Shared-memory bytes of one stage of codes.
__host__ __device__ constexpr int decode_codes_bytes(int bits, int mt) {
    return decode_cta_rows(bits, mt) * decode_boxes(bits, mt) * decode_box_w(bits, mt);
}
// Token tiles of 8 for the decode kernel (M <= kDecodeMaxM): 1, 2 or 4.
inline int mt_for_m(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : 4; }

cudaError_t launch_quantize_pack(const float *w, int N, int K, int bits, int group, uint32_t *packed,
                                 uint16_t *scales, uint16_t *zeros, int slot,
                                 unsigned long long call_id, cudaStream_t stream);
cudaError_t read_quant_status(int slot, unsigned long long *value, cudaStream_t stream);
cudaError_t launch_unpack(const uint32_t *packed, int N, int K, int bits, uint8_t *codes,
                          cudaStream_t stream);
// The tile kernel's dequant routine over a whole tensor (test hook): w_hat fp16 N x K.
cudaError_t launch_dequant_test(const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros, int bits,
                                int group, int N, int K, uint16_t *w_hat, cudaStream_t stream);

// ---------------------------------------------------------------- prefill --
// A prefill launch runs up to kMaxPrefillOps independent ops of one bit width
// as one persistent grid over all their 256-token x 256-row output tiles,
// handed out dynamically from a counter (the last two words of the
// workspace's counter region).
constexpr int kMaxPrefillOps = 64;

struct alignas(64) PrefillOp {
    CUtensorMap xmap;  // x (M x K fp16): 64 k x 256 (one-half plan: 128) tokens per box, 128-byte swizzle
    CUtensorMap wmap;  // fp16 weights only (bits 16): W (N x K fp16), 64 k x 256 rows per box, 128-byte swizzle
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *zeros;
    uint16_t *out;   // M x N fp16 (bf16 with out_bf16), or null when out32 is set
    float *out32;    // M x N fp32 (partial sums, not rounded), or null
    const float *xscale;  // bf16 activations: per-token factor 2^-E of the fp16 copy xmap reads, else null
    int M, N, K;
    int gshift;     // log2(group) - 5: groups of 32, 64 or 128 codes
    int out_bf16;   // 1: round the output to bfloat16
    int tok_tiles;  // ceil(M / tokens per tile): 256, or 512 in the CTA-pair plan
    int tile0;      // first tile of this op in the launch
};

struct PrefillGroup {
    int n_ops;
    int n_tiles;
    unsigned long long wait_ns;  // limit of a bounded wait (see wait_limit_ns)
    unsigned int *tile_ctr;      // workspace: [0] next tile ticket, [1] CTAs finished; both 0 between launches
    PrefillOp ops[kMaxPrefillOps];
};
static_assert(sizeof(PrefillGroup) <= 32000, "kernel parameter space");

cudaError_t prefill_x_map(CUtensorMap *map, const uint16_t *x, int M, int K);
cudaError_t launch_prefill_group(const PrefillGroup &pg, int bits, int num_sms, cudaStream_t stream);
cudaError_t read_prefill_error(int *err);
cudaError_t read_decode_error(int *err);
// Limit of the kernels' bounded waits, passed to every launch as a kernel
// parameter (2 s unless the test hook zq_set_wait_limit_ns changed it).
unsigned long long wait_limit_ns();
cudaError_t encode_tensor_map_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t dim0,
                                 uint64_t dim1, uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                                 CUtensorMapSwizzle swizzle);

// Largest M handled by the mma.sync decode kernel; larger M goes to the
// tcgen05 tile kernel (which, with one token tile, also streams the weights
// once, and from 17 tokens on is the faster of the two).
constexpr int kDecodeMaxM = 32;

// bf16 activations for the tile kernel: each token row of x (M x K bfloat16)
// scaled by a power of two 2^E (E per row, from the row's largest |x|) and
// rounded to fp16 into x16, each 32-value chunk in natural order (perm_bits 0)
// or pair-permuted for b = perm_bits (2, 3, 4, 8); f[m] = 2^-E undoes the
// scaling in the epilogue.
cudaError_t launch_bf16_rows_to_f16(const uint16_t *x, int M, int K, int perm_bits, uint16_t *x16, float *f,
                                    cudaStream_t stream);
// fp16 x (M x K) -> out with every 32-value chunk pair-permuted for b = bits
// (the x the tile kernel's one-token-half plan reads).
cudaError_t launch_x_pairperm(const uint16_t *x, int M, int K, int bits, uint16_t *out, cudaStream_t stream);

// Partial-sum reduction: out[i] = fp16(sum of parts[p][i], p in order).
constexpr int kMaxReduceParts = 16;
cudaError_t launch_reduce_partials(const float *const *parts, int n_parts, size_t count, uint16_t *out,
                                   cudaStream_t stream);

cudaError_t launch_prep(const PrepParams &p, long long total_warps, cudaStream_t stream);
cudaError_t launch_prep(const PrepParamsSmall &p, long long total_warps, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, int bits, int mt, int n_ctas, size_t smem, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParamsSmall &p, int bits, int mt, int n_ctas, size_t smem, cudaStream_t stream);
// CTAs per SM that the registers of decode_kernel<bits, mt> allow with `smem`
// bytes of dynamic shared memory each.
cudaError_t decode_ctas_per_sm(int bits, int mt, size_t smem, int *ctas);

}  // namespace zq
