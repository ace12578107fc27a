// zq_prefill.cu — tile kernel (M > 32): dequantize-to-shared-memory GEMM on
// the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA).
//
// What it computes: out = x · dequant(W)^T with dequant(W) = q * scale + zero per
// group of 128 along K ([wiki] "ZSE - open-source движок для запуска LLM
// локально на GPU - 2026", section "Формат модели .zse").  The pages' tiled
// shared-memory matmul (section "Оркестратор и GPU-ядра", TILE = 32) is prior
// art only.
//
// CTA tile: 256 tokens x 256 weight rows, K in slabs of 64 (one 128-byte
// swizzle atom of fp16).  Warp roles:
//   warps 0-3  epilogue: TMEM -> registers (tcgen05.ld) -> fp16 -> global;
//   warp 4     TMA producer for x (2-D tensor map, SWIZZLE_128B) and TMEM owner;
//   warp 5     MMA issuer: one thread issues tcgen05.mma (M=128, N=256, K=16)
//              for the two 128-token halves into 2 x 256 fp32 TMEM columns;
//   warps 6-13 dequant producers (6-21 in the one-half plan): packed codes ->
//              exact fp16 codes (zq_device.cuh) -> fp16(q*s + z) with one
//              fused HFMA2 rounding -> K-order restored with PRMT -> UMMA
//              K-major SWIZZLE_128B layout.
// A launch is one persistent grid (a CTA per SM) over all tiles of up to 64
// independent ops of one bit width, handed out round-robin in op order (the
// host puts the longest K first).
// A ring of (x, W) slabs is handed over with mbarriers; stage release is
// tcgen05.commit.  Every wait is bounded: after ~2 s it raises an abort flag,
// records ZQ_ERR_TIMEOUT in a device word and all roles drain and exit (TMEM
// is always freed).
//
// Two shared-memory plans:
//   * two token halves (a launch with some M > 128): 3 stages of
//     (x 256 x 64, W 256 x 64); the dequant threads keep the codes, scales and
//     zeros of the next group in registers;
//   * one token half (every M <= 128, i.e. 17..128 tokens): the x stages hold
//     128 tokens, and the space this frees becomes a ring of per-thread code
//     slots that cp.async fills several groups ahead, so that enough weight
//     bytes are in flight per SM; with the codes out of the registers, 16
//     dequant warps fit, each owning one row chunk per slab.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "zq_device.cuh"
#include "zq_internal.h"
#include "zq_prefill.h"

namespace zq {

__device__ int g_prefill_error;  // 0 = ok, else a ZQ_ERR_* code from a kernel

namespace pf {

constexpr int kTokTile = 256;   // tokens per CTA tile (two MMA halves of 128)
constexpr int kRowTile = 256;   // weight rows per CTA tile (MMA N)
constexpr int kBK = 64;         // K per slab
constexpr int kMaxStages = 4;
constexpr int kSlabB = kRowTile * kBK * 2;  // 32 KB
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kDqWarp0 = 6;
constexpr int kTmemCols = 512;
// Drains after an abort wait for copies and MMAs already issued; they ignore
// the abort flag and the adjustable limit and give up only after this bound.
constexpr unsigned long long kDrainNs = 2000000000ull;  // 2 s

// Tiles are handed out dynamically: the scheduler warp takes tickets from a
// counter in the workspace and writes the tile numbers, in order, into a ring
// of kTileRing entries; every role reads the ring in the same order and
// releases an entry as soon as it has read it.  The ring is deeper than the
// furthest any reader runs ahead of another (the dequant issue cursor, a few
// blocks ahead of its consume cursor, which leads the epilogue by a few
// slabs), so no reader waits on the scheduler for long.
constexpr int kTileRing = 16;

struct Ctl {
    int tq[kTileRing];                     // tile numbers, -1 = no more tiles
    unsigned long long tq_full[kTileRing];
    unsigned long long tq_empty[kTileRing];
    unsigned long long full[kMaxStages];   // W slab dequantized (one arrival per dequant warp)
    unsigned long long xfull[kMaxStages];  // x slab landed (the TMA warp's expect_tx + the copy's bytes)
    unsigned long long empty[kMaxStages];
    // accumulator buffer b complete / drained: the one-token-half plan uses
    // TMEM columns [256b, 256b + 256) for tile i with b = i % 2, so a tile's
    // MMAs run while the previous tile is drained; the two-half plan holds
    // both token halves in its 512 columns and uses buffer 0 alone
    unsigned long long acc_full[2];
    unsigned long long acc_empty[2];
    unsigned long long mma_done;           // every tcgen05.mma this CTA issued has completed
    uint32_t tmem_base;
    int abort;
};

// Shared-memory plan (byte offsets from a 1024-byte aligned base):
//   [0, kOffB)          x slabs, kStages x kSlabA (TMA, SWIZZLE_128B)
//   [kOffB, kOffCodes)  dequantized W slabs, kStages x kSlabB (SWIZZLE_128B)
//   [kOffCodes, kOffCtl) code slots (one token half only): slot = one group
//                       of the tile's 256 rows, laid out per thread (below),
//                       then one (scale | zero << 16) word per (row, chunk)
//   [kOffCtl, ...)      barriers and flags
template <int B, bool ONE, int XR = ONE ? 128 : 256>
struct Plan {
    // Dequant warps: 16 in the one-half plan (its code ring keeps their
    // registers low), 8 in the two-half plan (register prefetch); none for
    // fp16 weights (B = 16), which TMA copies into the W stages as they are.
    static constexpr int kDqWarps = B == 16 ? 0 : ONE ? 16 : 8;
    static constexpr int kSchedWarp = kDqWarp0 + kDqWarps;  // the tile scheduler (lane 0)
    static constexpr int kThreads = 32 * (kSchedWarp + 1);
    // readers of every tile-ring entry: TMA and MMA lanes, epilogue and dequant warps
    static constexpr int kTileReaders = 2 + kEpiWarps + kDqWarps;
    // XR: token rows of an x stage.  With every M <= 64 (XR = 64, b <= 4) the
    // x stage is half as large and the space becomes a fourth W stage (one
    // code slot fewer); the MMA still reads 128 A rows, rows 64..127 from the
    // bytes after the slab, whose accumulator rows are never stored.
    static constexpr int kStages = B == 16 ? 3 : (ONE && B == 8) ? 2 : XR == 64 ? 4 : 3;
    static constexpr int kSlabA = XR * kBK * 2;
    static constexpr int kSlots = (!ONE || B == 16) ? 0
                                  : XR == 64 ? (B == 2 ? 5 : B == 3 ? 4 : 3)
                                             : (B == 2 ? 6 : B == 3 ? 5 : B == 4 ? 4 : 3);
    static constexpr int kSlotCodes = 1024 * (4 * B);  // 256 rows x 2 slabs x 2 chunks of 32 codes
    // + a (scale | zero << 16) word per (row, chunk, slab): the two slabs of a
    // block of 128 codes fall in different groups when groups are 32 or 64
    static constexpr int kSlotBytes = kSlotCodes + 1024 * 4;
    static constexpr int kOffB = kStages * kSlabA;
    static constexpr int kOffCodes = kOffB + kStages * kSlabB;
    static constexpr int kOffCtl = kOffCodes + kSlots * kSlotBytes;
    static constexpr size_t kBytes = kOffCtl + sizeof(Ctl) + 1024;  // + alignment slack
    static_assert(kStages <= kMaxStages, "barrier arrays");
    static_assert(kOffB % 1024 == 0 && kOffCodes % 1024 == 0, "SWIZZLE_128B stages need 1024-byte alignment");
    static_assert(kBytes <= 232448, "227 KB of shared memory per CTA");
    static_assert(!ONE || B == 16 || kSlots >= 3, "the scale/zero hand-off needs a prefetch distance of 2 groups");
    static_assert(XR == (ONE ? XR : 256) && (XR != 64 || (ONE && B <= 4)), "x rows per plan");
};

// Bounded wait: false if the CTA is aborting or the limit was reached.  The
// first test of the phase is inline and the polling loop a call, so a wait
// whose phase has completed costs one try_wait (the call alone cost 6-7 % of
// the tile kernel's time at 40-256 tokens).
__device__ __noinline__ bool mbar_wait_poll(unsigned long long *bar, uint32_t parity, volatile int *abort,
                                            unsigned long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit) {
                *abort = 1;
                atomicExch(&g_prefill_error, 5);  // ZQ_ERR_TIMEOUT
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(unsigned long long *bar, uint32_t parity, volatile int *abort,
                                          unsigned long long limit) {
    return mbar_try_wait(bar, parity) || mbar_wait_poll(bar, parity, abort, limit);
}

// Wait of a drain: for a phase that work already issued will complete; no
// abort check, bounded by kDrainNs.
__device__ __noinline__ void mbar_drain(unsigned long long *bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > kDrainNs) break;
}

// Tile number of ring entry j (whole warp or one lane): -1 when the tiles are
// exhausted, -2 when the wait gave up (the CTA is aborting).
__device__ __forceinline__ int tile_at(Ctl &c, uint32_t j, volatile int *abort, unsigned long long limit) {
    if (!mbar_wait(&c.tq_full[j % kTileRing], (j / kTileRing) & 1u, abort, limit)) return -2;
    return *reinterpret_cast<volatile int *>(&c.tq[j % kTileRing]);
}

__device__ __forceinline__ void tile_release(Ctl &c, uint32_t j) { mbar_arrive(&c.tq_empty[j % kTileRing]); }

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory descriptor: K-major, SWIZZLE_128B, 8-row groups 1024 B
// apart (rows of 128 bytes), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address
    d |= static_cast<uint64_t>(1) << 16;                   // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                   // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                   // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D.
constexpr uint32_t kIdesc = (1u << 4)                       // D format f32
                            | (0u << 7) | (0u << 10)        // A, B format f16
                            | (static_cast<uint32_t>(kRowTile >> 3) << 17)  // N
                            | (static_cast<uint32_t>(128 >> 4) << 24);     // M

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(unsigned long long *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Split form of tmem_ld32: the load is issued, and its registers are valid
// only after tmem_wait32 on the same array (which waits for every earlier
// tcgen05.ld of the thread and ties the registers to the wait, so no use of
// them moves above it).
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Two outputs rounded (nearest even) to fp16, or to bfloat16 for bf16 activations.
__device__ __forceinline__ uint32_t pack_out2(float lo, float hi, int bf16) {
    if (bf16) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t *>(&b);
    }
    return pack_half2(lo, hi);
}

// Epilogue store of 32 accumulator columns (weight rows col0 .. col0 + 31) of
// token row `tok`: scaled by the token's factor fs (bf16 activations), then
// fp32 partials (out32), or fp16 / bf16 rounded to nearest even; rows and
// tokens past the op's N and M are not stored.
__device__ __forceinline__ void store_cols32(const PrefillOp &op, int tok, int col0, uint32_t (&r)[32], float fs) {
    if (op.xscale != nullptr) {
#pragma unroll
        for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * fs);
    }
    if (tok >= op.M || col0 >= op.N) return;
    if (op.out32) {
        // fp32 partial sums (a K-split shard), not rounded
        float *dst = op.out32 + static_cast<size_t>(tok) * op.N + col0;
        if ((op.N % 4) == 0 && col0 + 32 <= op.N) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                reinterpret_cast<uint4 *>(dst)[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q)
                if (col0 + q < op.N) dst[q] = __uint_as_float(r[q]);
        }
        return;
    }
    uint16_t *dst = op.out + static_cast<size_t>(tok) * op.N + col0;
    if ((op.N % 8) == 0 && col0 + 32 <= op.N) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            reinterpret_cast<uint4 *>(dst)[q] = make_uint4(
                pack_out2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]), op.out_bf16),
                pack_out2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]), op.out_bf16),
                pack_out2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]), op.out_bf16),
                pack_out2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]), op.out_bf16));
    } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
            if (col0 + q < op.N) dst[q] = static_cast<uint16_t>(pack_out2(__uint_as_float(r[q]), 0.0f, op.out_bf16));
    }
}

// Tile t of a launch -> (op, weight-row tile, token tile).  The tiles of op o
// are [tile0, tile0 + tok_tiles * row_tiles); within an op token tiles vary
// fastest, so the CTAs working at the same time share one weight tile (L2
// reuse).
struct TileRef {
    int o, n0, t0;
};
__device__ __forceinline__ TileRef locate(const PrefillGroup &p, int t, int tok_tile = kTokTile) {
    int lo = 0, hi = p.n_ops - 1;  // last op with tile0 <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.ops[mid].tile0 <= t) lo = mid;
        else hi = mid - 1;
    }
    const int local = t - p.ops[lo].tile0;
    const int tt = p.ops[lo].tok_tiles;
    return TileRef{lo, (local / tt) * kRowTile, (local % tt) * tok_tile};
}

// True when some code of the group dequantizes past the fp16 range: the top
// of the group, L*s + z (s >= 0, so every q*s + z is at most that), rounds to
// +inf.  Only groups whose range reaches the fp16 limit (|w| near 65504) do.
template <int B>
__device__ __forceinline__ bool dequant_overflows(uint32_t sz) {
    constexpr uint32_t kL2 = (B == 2 ? 0x4200u : B == 3 ? 0x4700u : B == 4 ? 0x4B80u : 0x5BF8u) * 0x10001u;  // (L, L)
    const uint32_t top = hfma2_bits(kL2, (sz & 0xFFFFu) * 0x10001u, (sz >> 16) * 0x10001u);
    return (top & 0x7FFFu) == 0x7C00u;
}

__device__ __forceinline__ uint32_t hmin2_bits(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Dequantize this thread's 32-code chunk of one W row into 4 x 16 bytes of
// fp16 (q*s + z, one rounding), via the shared unpack: in natural K order, or
// (NATURAL = false) in the pair order of the unpack, word p holding codes
// pair_lo(p) and pair_hi(p), for an x copy permuted the same way.  In a group
// that reaches past the fp16 range (`ovf`), values that round to +inf are held
// at 65504, the largest finite fp16 (a relative change below 2^-11).
template <int B, bool NATURAL = true>
__device__ __forceinline__ void dequant_chunk(const uint32_t (&w)[B], uint32_t sz, uint32_t (&o)[16], bool ovf) {
    const uint32_t s2 = (sz & 0xFFFFu) * 0x10001u;  // (s, s)
    const uint32_t z2 = (sz >> 16) * 0x10001u;      // (z, z)
    uint32_t v[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) v[p] = hfma2_bits(unpack_pair<B>(w, p), s2, z2);
    if (ovf) {
#pragma unroll
        for (int p = 0; p < 16; ++p) v[p] = hmin2_bits(v[p], 0x7BFF7BFFu);
    }
    if constexpr (!NATURAL) {
#pragma unroll
        for (int p = 0; p < 16; ++p) o[p] = v[p];
    } else {
        // Pairs p (even) and p+1 hold codes (lo, hi) and (lo+1, hi+1): two
        // PRMTs give the natural pairs (lo, lo+1) and (hi, hi+1).
#pragma unroll
        for (int p = 0; p < 16; p += 2) {
            const int lo = pair_lo<B>(p), hi = pair_hi<B>(p);
            o[lo / 2] = prmt(v[p], v[p + 1], 0x5410u);
            o[hi / 2] = prmt(v[p], v[p + 1], 0x7632u);
        }
    }
}

template <int B>
__device__ __forceinline__ void load_chunk(uint32_t (&w)[B], const uint32_t *src) {
    if constexpr (B == 2) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src);
        w[0] = v.x;
        w[1] = v.y;
    } else if constexpr (B == 3) {
        w[0] = src[0];
        w[1] = src[1];
        w[2] = src[2];
    } else if constexpr (B == 4) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
        const uint4 v0 = reinterpret_cast<const uint4 *>(src)[0];
        const uint4 v1 = reinterpret_cast<const uint4 *>(src)[1];
        w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    }
}


// Two consecutive 16-bit values from a 4-byte aligned address (read-only path).
__device__ __forceinline__ uint32_t ldg_u32_nc(const uint16_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// cp.async of U bytes (16, 8 or 4) global -> shared.
template <int U>
__device__ __forceinline__ void cp_async_u(void *dst, const void *src) {
    if constexpr (U == 16) cp_async16(dst, src);
    else if constexpr (U == 8) cp_async8(dst, src);
    else cp_async4(dst, src);
}

// Scales and zeros of one block of 128 codes as loaded (not yet packed into
// the slot's (scale | zero << 16) words), and how they were loaded.
constexpr int kSzNone = 0;        // nothing loaded (past the last block)
constexpr int kSzOne = 1;         // one group: s[r][0], z[r][0]
constexpr int kSzSplit = 2;       // groups of 32 or 64: [r][0] for slab 0, [r][1] for slab 1
constexpr int kSzPair = 3;        // this group and the next: the low and high halves of s[r][0], z[r][0]
constexpr int kSzPairSecond = 4;  // the second group of a pair: nothing of its own
template <int RPT>
struct ScaleSet {
    uint32_t s[RPT][2], z[RPT][2];
    int mode;
};

// Dequant producer of the one-token-half plan.  Its NT threads own the 512
// (row, chunk) pairs of each slab, pair q = d + NT * r (r < 512 / NT) of
// thread d being row (q % 256) / 2 + 128 * (q / 256), 32-code chunk q % 2 --
// the two-half plan's assignment when NT = 256.  Codes travel through a ring
// of kSlots shared-memory slots filled by cp.async kSlots - 1 groups ahead.
// Within a slot each thread's data is spread in U-byte units, unit u of thread
// d at (u * NT + d) * U, so the copies and the loads of a warp are contiguous.
// Scales and zeros (2-byte aligned, too small for cp.async) are loaded into a
// register set when their group's codes are issued and written to the slot
// two groups later, packed only then; the two register sets alternate, hence
// the loop below is unrolled twice.  With groups of 128 and an even number of
// groups per row, the scales (and zeros) of two consecutive groups are one
// 4-byte load, made with the first group's codes, and both groups' words are
// written two groups later.
template <int B, int XR>
__device__ __forceinline__ void dequant_ring(const PrefillGroup &p, uint8_t *sb, uint8_t *scode, Ctl &c,
                                             int d, int lane) {
    using P = Plan<B, true, XR>;
    constexpr int NT = 32 * P::kDqWarps;
    constexpr int RPT = 512 / NT;                     // rows per thread
    constexpr int kS = P::kSlots;
    constexpr int PD = kS - 1;                        // groups in flight
    constexpr int U = B == 3 ? 4 : B == 2 ? 8 : 16;   // bytes per copy
    constexpr int UPC = 4 * B / U;                    // copies per 32-code chunk
    static_assert(RPT * NT == 512, "thread count");
    volatile int *abort = &c.abort;
    const int ch = d & 1;
    int rows[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int q = d + NT * r;
        rows[r] = (q % 256) / 2 + 128 * (q / 256);
    }

    // Issue cursor: the block of 128 codes whose codes are copied next, in the
    // tile of ring entry jp (the issue cursor reads each entry first; the
    // consume cursor, later, releases it).
    uint32_t jp = 0;
    int tp = tile_at(c, jp, abort, p.wait_ns), gp = 0, Gp = 0, gsh = 2;
    // groups of 128 and an even count per row: with the arrays 16-byte aligned
    // (checked by the host), the scales of groups 2i and 2i + 1 are 4-byte aligned
    bool pair2 = false;
    const uint32_t *prow[RPT];
    const uint16_t *psr[RPT], *pzr[RPT];
    auto start_issue = [&]() {
        if (tp >= 0) {
            const TileRef tr = locate(p, tp);
            const PrefillOp &op = p.ops[tr.o];
            Gp = op.K / kGroup;
            gsh = op.gshift;
            const size_t gs = static_cast<size_t>(op.K) >> (op.gshift + 5);  // scales per row
            pair2 = gsh == 2 && (gs & 1) == 0;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int n = min(tr.n0 + rows[r], op.N - 1);
                prow[r] = op.packed + static_cast<size_t>(n) * (static_cast<size_t>(op.K) * B / 32);
                psr[r] = op.scales + static_cast<size_t>(n) * gs;
                pzr[r] = op.zeros + static_cast<size_t>(n) * gs;
            }
        }
    };
    start_issue();
    ScaleSet<RPT> szA, szB;
    szA.mode = szB.mode = kSzNone;
    // Block j of this CTA's sequence: first store the scale/zero words of
    // block j - 2 (held in `set`) into its slot (and those of block j - 1
    // into its slot, after a pair load), then copy block j's codes into slot
    // j % kS and load its scales and zeros into `set`: slab h of the block
    // uses group (4 * gp + 2h + ch) >> gshift.  Block j - 1's slot is free for
    // its words by then: the slot's previous block was consumed before block
    // j - 1 was issued.  Past the last block only the store and an empty
    // commit remain, so that every block index commits exactly one cp.async
    // group.
    auto issue = [&](int j, ScaleSet<RPT> &set) {
        if (j >= 2 && set.mode != kSzNone && set.mode != kSzPairSecond) {
            // the words of block j - 2 (and, after a pair load, of block j - 1)
            uint32_t *zs = reinterpret_cast<uint32_t *>(scode + ((j - 2) % kS) * P::kSlotBytes + P::kSlotCodes);
            uint32_t *zn = reinterpret_cast<uint32_t *>(scode + ((j - 1) % kS) * P::kSlotBytes + P::kSlotCodes);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const uint32_t w0 = prmt(set.s[r][0], set.z[r][0], 0x5410u);
                zs[(2 * r) * NT + d] = w0;
                zs[(2 * r + 1) * NT + d] = set.mode == kSzSplit ? prmt(set.s[r][1], set.z[r][1], 0x5410u) : w0;
                if (set.mode == kSzPair) {
                    const uint32_t w1 = prmt(set.s[r][0], set.z[r][0], 0x7632u);
                    zn[(2 * r) * NT + d] = w1;
                    zn[(2 * r + 1) * NT + d] = w1;
                }
            }
        }
        set.mode = kSzNone;
        if (tp >= 0) {
            uint8_t *cs = scode + (j % kS) * P::kSlotBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    const uint8_t *src = reinterpret_cast<const uint8_t *>(prow[r] + (4 * gp + 2 * h + ch) * B);
#pragma unroll
                    for (int u = 0; u < UPC; ++u)
                        cp_async_u<U>(cs + (((h * RPT + r) * UPC + u) * NT + d) * U, src + u * U);
                }
            // The loaded values stay as they are until their words are stored
            // two blocks later: packing them here would wait for the loads.
            if (gsh != 2) {
                // groups of 32 or 64: the block's two slabs of this chunk lie in
                // groups g0 and g1 > g0
                const int g0 = (4 * gp + ch) >> gsh, g1 = (4 * gp + 2 + ch) >> gsh;
                set.mode = kSzSplit;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    set.s[r][0] = ldg_u16_nc(psr[r] + g0);
                    set.z[r][0] = ldg_u16_nc(pzr[r] + g0);
                    set.s[r][1] = ldg_u16_nc(psr[r] + g1);
                    set.z[r][1] = ldg_u16_nc(pzr[r] + g1);
                }
            } else if (pair2 && (gp & 1) == 0) {
                // groups gp and gp + 1 with one 4-byte load each of scales and zeros
                set.mode = kSzPair;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    set.s[r][0] = ldg_u32_nc(psr[r] + gp);
                    set.z[r][0] = ldg_u32_nc(pzr[r] + gp);
                }
            } else if (pair2) {
                set.mode = kSzPairSecond;  // loaded, and stored, with block gp - 1
            } else {
                set.mode = kSzOne;
#pragma unroll
                for (int r = 0; r < RPT; ++r) {
                    set.s[r][0] = ldg_u16_nc(psr[r] + gp);
                    set.z[r][0] = ldg_u16_nc(pzr[r] + gp);
                }
            }
            if (++gp == Gp) {
                gp = 0;
                tp = tile_at(c, ++jp, abort, p.wait_ns);
                start_issue();
            }
        }
        cp_async_commit();
    };
#pragma unroll
    for (int j = 0; j + 1 < PD; j += 2) {  // group j uses register set j & 1
        issue(j, szA);
        issue(j + 1, szB);
    }
    if constexpr (PD & 1) issue(PD - 1, szA);

    // Consume cursor: group i of tile t, ring entry jc (released by the warp
    // once read: the issue cursor has read it already).
    uint32_t jc = 0;
    int t = tile_at(c, jc, abort, p.wait_ns), g = 0, G = t >= 0 ? p.ops[locate(p, t).o].K / kGroup : 0;
    __syncwarp();
    if (lane == 0) tile_release(c, jc);
    uint32_t it = 0;  // W stages filled so far
    auto consume = [&](int i) -> bool {
        cp_async_wait<PD>();               // this thread's copies of group i have landed
        const uint32_t z = opaque_zero();  // orders the slot loads after the wait
        const uint32_t cs = smem_u32(scode + (i % kS) * P::kSlotBytes) + z;
        uint32_t sz[RPT][2];
        bool ovf[RPT][2];
#pragma unroll
        for (int r = 0; r < RPT; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sz[r][h] = lds_u32(cs + P::kSlotCodes + 4 * ((2 * r + h) * NT + d));
                ovf[r][h] = dequant_overflows<B>(sz[r][h]);
            }
        // both slabs' codes, loaded before the waits for their W stages
        uint32_t wall[2][RPT][B];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int u = 0; u < UPC; ++u) {
                    const uint32_t a = cs + (((h * RPT + r) * UPC + u) * NT + d) * U;
                    uint32_t(&w)[B] = wall[h][r];
                    if constexpr (U == 16) {
                        const uint4 v = lds_v4(a);
                        w[4 * u] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
                    } else if constexpr (U == 8) {
                        const uint2 v = lds_v2(a);
                        w[2 * u] = v.x; w[2 * u + 1] = v.y;
                    } else {
                        w[u] = lds_u32(a);
                    }
                }
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // the two slabs of this group
            const int st = it % P::kStages;
            const uint32_t round = it / P::kStages;
            if (!mbar_wait(&c.empty[st], (round & 1u) ^ 1u, abort, p.wait_ns)) return false;
            uint8_t *bs = sb + st * kSlabB;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int row = rows[r];
                uint32_t o[16];
                dequant_chunk<B, false>(wall[h][r], sz[r][h], o, ovf[r][h]);  // x is pair-permuted
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c16 = (4 * ch + j) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(bs + row * 128 + c16 * 16) =
                        make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&c.full[st]);
            ++it;
        }
        if (++g == G) {
            g = 0;
            t = tile_at(c, ++jc, abort, p.wait_ns);
            __syncwarp();
            if (lane == 0 && t != -2) tile_release(c, jc);
            if (t >= 0) G = p.ops[locate(p, t).o].K / kGroup;
        }
        return true;
    };
    ScaleSet<RPT> &set_even = (PD & 1) ? szB : szA;  // register set of block i + PD, i even
    ScaleSet<RPT> &set_odd = (PD & 1) ? szA : szB;
#pragma unroll 1
    for (int i = 0;; i += 2) {
        if (t < 0 || *abort) break;
        issue(i + PD, set_even);
        if (!consume(i)) break;
        if (t < 0 || *abort) break;
        issue(i + 1 + PD, set_odd);
        if (!consume(i + 1)) break;
    }
    cp_async_wait<0>();  // no copy may land after the CTA has exited
}

template <int B, bool ONE, int XR>
__global__ void __launch_bounds__(Plan<B, ONE, XR>::kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillGroup p) {
    using P = Plan<B, ONE, XR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sa = base;                  // x slabs
    uint8_t *sb = base + P::kOffB;       // W slabs
    uint8_t *scode = base + P::kOffCodes;
    Ctl &sm = *reinterpret_cast<Ctl *>(base + P::kOffCtl);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = p.n_tiles;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kTileRing; ++i) {
            mbar_init(&sm.tq_full[i], 1);
            mbar_init(&sm.tq_empty[i], P::kTileReaders);
        }
        for (int s = 0; s < P::kStages; ++s) {
            if constexpr (B != 16) mbar_init(&sm.full[s], P::kDqWarps);
            mbar_init(&sm.xfull[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], kEpiWarps);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kTmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    pdl_wait();  // x may be produced by the previous kernel in the stream
    pdl_launch_dependents();

    if (warp == P::kSchedWarp) {
        // Tile scheduler: tickets from the launch's counter, in order, into the
        // ring; an entry is refilled once every reader has released it.  The
        // ring is 16 tiles deep, so the scheduler sleeps between polls and
        // leaves the issue slots of its SM sub-partition to the dequant warps.
        if (lane == 0) {
            for (uint32_t i = 0;; ++i) {
                if (i >= kTileRing) {
                    unsigned long long *bar = &sm.tq_empty[i % kTileRing];
                    const uint32_t par = ((i / kTileRing) - 1u) & 1u;
                    const unsigned long long t0 = globaltimer();
                    bool ok = true;
                    while (!mbar_try_wait(bar, par)) {
                        if (*abort || globaltimer() - t0 > p.wait_ns) {
                            ok = false;
                            break;
                        }
                        __nanosleep(1000);
                    }
                    if (!ok) {
                        if (!*abort) {
                            *abort = 1;
                            atomicExch(&g_prefill_error, 5);  // ZQ_ERR_TIMEOUT
                        }
                        break;
                    }
                }
                const unsigned int v = atomicAdd(p.tile_ctr, 1u);
                const int t = v < static_cast<unsigned int>(n_tiles) ? static_cast<int>(v) : -1;
                *reinterpret_cast<volatile int *>(&sm.tq[i % kTileRing]) = t;
                mbar_arrive(&sm.tq_full[i % kTileRing]);  // release: publishes the entry
                if (t < 0) break;
            }
        }
    } else if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t it = 0;
            for (uint32_t j = 0;; ++j) {
                const int t = tile_at(sm, j, abort, p.wait_ns);
                if (t != -2) tile_release(sm, j);
                if (t < 0 || *abort) break;
                const TileRef tr = locate(p, t);
                const PrefillOp &op = p.ops[tr.o];
                const int slabs = op.K / kBK;
                for (int s = 0; s < slabs; ++s, ++it) {
                    const int st = it % P::kStages;
                    const uint32_t round = it / P::kStages;
                    if (!mbar_wait(&sm.empty[st], (round & 1u) ^ 1u, abort, p.wait_ns)) break;
                    if constexpr (B == 16) {
                        // fp16 weights: the W slab is copied as it is, in the same
                        // 128-byte swizzled K-major layout the dequant warps write
                        mbar_arrive_expect_tx(&sm.xfull[st], P::kSlabA + kSlabB);
                        tma_load_2d(sb + st * kSlabB, &op.wmap, s * kBK, tr.n0, &sm.xfull[st]);
                    } else {
                        mbar_arrive_expect_tx(&sm.xfull[st], P::kSlabA);
                    }
                    tma_load_2d(sa + st * P::kSlabA, &op.xmap, s * kBK, tr.t0, &sm.xfull[st]);
                }
            }
            // Copies still in flight (only after an abort) must land before
            // the CTA can exit.  `it` copies were issued; a slot is refilled only
            // after the MMA consumed its previous copy, so only the last
            // kStages can be pending, one per slot.  The x-only barriers
            // complete on the copies' bytes alone, whatever the other roles did.
            for (uint32_t k = 0; k < P::kStages && k < it; ++k) {
                const uint32_t j = it - 1 - k;
                mbar_drain(&sm.xfull[j % P::kStages], (j / P::kStages) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            uint32_t it = 0, tile_i = 0;
            bool issued = false;
            for (uint32_t j = 0;; ++j, ++tile_i) {
                const int t = tile_at(sm, j, abort, p.wait_ns);
                if (t != -2) tile_release(sm, j);
                if (t < 0 || *abort) break;
                const TileRef tr = locate(p, t);
                const int slabs = p.ops[tr.o].K / kBK;
                // the second 128-token half only when it holds tokens
                const bool half1 = !ONE && tr.t0 + 128 < p.ops[tr.o].M;
                // accumulator buffer of this tile and the number of earlier uses of it
                const uint32_t ab = ONE ? (tile_i & 1u) : 0u, au = ONE ? (tile_i >> 1) : tile_i;
                if (!mbar_wait(&sm.acc_empty[ab], (au & 1u) ^ 1u, abort, p.wait_ns)) break;
                tc_fence_after();
                const uint32_t tacc = tmem + ab * kRowTile;
                bool ok = true;
                for (int s = 0; s < slabs; ++s, ++it) {
                    const int st = it % P::kStages;
                    if (!mbar_wait(&sm.xfull[st], (it / P::kStages) & 1u, abort, p.wait_ns) ||
                        (B != 16 && !mbar_wait(&sm.full[st], (it / P::kStages) & 1u, abort, p.wait_ns))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issued = true;
                    const uint32_t a0 = smem_u32(sa + st * P::kSlabA);
                    const uint32_t b0 = smem_u32(sb + st * kSlabB);
                    if (half1) {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint64_t bd = sdesc_sw128(b0 + kk * 32);
                            const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                            umma_f16(tmem, sdesc_sw128(a0 + kk * 32), bd, acc);
                            umma_f16(tmem + kRowTile, sdesc_sw128(a0 + P::kSlabA / 2 + kk * 32), bd, acc);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                            umma_f16(tacc, sdesc_sw128(a0 + kk * 32), sdesc_sw128(b0 + kk * 32), acc);
                        }
                    }
                    umma_commit(&sm.empty[st]);
                }
                if (!ok) break;
                umma_commit(&sm.acc_full[ab]);
            }
            // Every MMA issued must have completed before TMEM is freed and the
            // CTA exits (after an abort no epilogue waited for them).
            if (issued) {
                umma_commit(&sm.mma_done);
                mbar_drain(&sm.mma_done, 0u);
            }
        }
    } else if (warp >= kDqWarp0) {
        if constexpr (B == 16) {
            // no dequant warps for fp16 weights
        } else if constexpr (ONE) {
            dequant_ring<B, XR>(p, sb, scode, sm, threadIdx.x - 32 * kDqWarp0, lane);
        } else {
        // 256 threads: thread d owns rows d/2 and d/2 + 128 of the tile and the
        // 32-code chunk d%2 of every slab.  Codes, scales and zeros of the next
        // group (two slabs) are prefetched into registers.
        const int d = threadIdx.x - 32 * kDqWarp0;
        const int ch = d & 1;
        uint32_t it = 0;
        uint32_t wn[2][2][B], szn[2][2];  // [slab of block][row][word], [slab][row]
        // Row pointers of the tile being fetched (set when it starts).
        const uint32_t *rowp[2];
        const uint16_t *srow[2], *zrow[2];
        int gsh = 2;                      // log2(group) - 5 of the tile being fetched
        auto start_tile = [&](int t) -> int {  // returns the tile's count of 128-code blocks
            const TileRef tr = locate(p, t);
            const PrefillOp &op = p.ops[tr.o];
            const int G = op.K / kGroup;
            gsh = op.gshift;
            const size_t gs = static_cast<size_t>(op.K) >> (op.gshift + 5);  // scales per row
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = min(tr.n0 + d / 2 + 128 * i, op.N - 1);
                rowp[i] = op.packed + static_cast<size_t>(r) * (static_cast<size_t>(op.K) * B / 32);
                srow[i] = op.scales + static_cast<size_t>(r) * gs;
                zrow[i] = op.zeros + static_cast<size_t>(r) * gs;
            }
            return G;
        };
        auto fetch = [&](int g) {
            // slab h of block g: codes 128g + 64h + 32ch .. +31, group (4g + 2h + ch) >> gsh
            const int g0 = (4 * g + ch) >> gsh, g1 = (4 * g + 2 + ch) >> gsh;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    load_chunk<B>(wn[h][i], rowp[i] + static_cast<size_t>(4 * g + 2 * h + ch) * B);
                if (gsh == 2) {
                    // groups of 128: the scale and the zero as loaded, packed
                    // when the block is used (packing here would wait for them)
                    szn[0][i] = ldg_u16_nc(srow[i] + g0);
                    szn[1][i] = ldg_u16_nc(zrow[i] + g0);
                } else {
                    szn[0][i] = ldg_u16_nc(srow[i] + g0) | (ldg_u16_nc(zrow[i] + g0) << 16);
                    szn[1][i] = ldg_u16_nc(srow[i] + g1) | (ldg_u16_nc(zrow[i] + g1) << 16);
                }
            }
        };
        // Tiles from the ring: entry jn is read (and released) by the fetch
        // cursor, one block ahead of the dequant.
        uint32_t jn = 0;
        int t = tile_at(sm, jn, abort, p.wait_ns), g = 0, groups = 0, groups_n = 0;
        __syncwarp();
        if (lane == 0 && t != -2) tile_release(sm, jn);
        if (t >= 0) {
            groups = start_tile(t);
            fetch(0);
        }
        bool ok = true;
        while (t >= 0 && ok && !*abort) {
            uint32_t wc[2][2][B], szc[2][2];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int q = 0; q < B; ++q) wc[h][i][q] = wn[h][i][q];
            bool ovf[2][2];
            if (gsh == 2) {  // gsh is still the current tile's
#pragma unroll
                for (int i = 0; i < 2; ++i) szc[0][i] = szc[1][i] = prmt(szn[0][i], szn[1][i], 0x5410u);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int i = 0; i < 2; ++i) szc[h][i] = szn[h][i];
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 2; ++i) ovf[h][i] = dequant_overflows<B>(szc[h][i]);
            int t_n = t, g_n = g + 1;
            groups_n = groups;
            if (g_n == groups) {
                g_n = 0;
                t_n = tile_at(sm, ++jn, abort, p.wait_ns);
                __syncwarp();
                if (lane == 0 && t_n != -2) tile_release(sm, jn);
                if (t_n >= 0) groups_n = start_tile(t_n);
            }
            if (t_n >= 0) fetch(g_n);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // the two slabs of this group
                const int st = it % P::kStages;
                const uint32_t round = it / P::kStages;
                if (!mbar_wait(&sm.empty[st], (round & 1u) ^ 1u, abort, p.wait_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *bs = sb + st * kSlabB;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int row = d / 2 + 128 * i;
                    uint32_t o[16];
                    dequant_chunk<B>(wc[h][i], szc[h][i], o, ovf[h][i]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int c16 = (4 * ch + j) ^ (row & 7);
                        *reinterpret_cast<uint4 *>(bs + row * 128 + c16 * 16) =
                            make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                    }
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.full[st]);
                ++it;
            }
            t = t_n;
            g = g_n;
            groups = groups_n;
        }
        }
    } else {
        // Epilogue warps 0..3: TMEM lanes 32*warp .. +31 = tokens of each half.
        uint32_t tile_i = 0;
        for (uint32_t j = 0;; ++j, ++tile_i) {
            const int t = tile_at(sm, j, abort, p.wait_ns);
            __syncwarp();
            if (lane == 0 && t != -2) tile_release(sm, j);
            if (t < 0 || *abort) break;
            const uint32_t ab = ONE ? (tile_i & 1u) : 0u, au = ONE ? (tile_i >> 1) : tile_i;
            if (!mbar_wait(&sm.acc_full[ab], au & 1u, abort, p.wait_ns)) break;
            tc_fence_after();
            const TileRef tr = locate(p, t);
            const PrefillOp &op = p.ops[tr.o];
            const int n0 = tr.n0, t0 = tr.t0;
#pragma unroll 1
            for (int half = 0; half < (!ONE && t0 + 128 < op.M ? 2 : 1); ++half) {
                const int tok = t0 + 128 * half + 32 * warp + lane;
                // bf16 activations: the token's power-of-two factor undoes the
                // scaling of the fp16 copy the MMAs read
                const float fs = (op.xscale != nullptr && tok < op.M) ? op.xscale[tok] : 1.0f;
                const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + (half + ab) * kRowTile;
                if constexpr (ONE) {
                    // 22 warps: no registers for a second buffer
#pragma unroll 1
                    for (int cc = 0; cc < kRowTile / 32; ++cc) {
                        uint32_t r[32];
                        tmem_ld32(ta + cc * 32, r);
                        store_cols32(op, tok, n0 + cc * 32, r, fs);
                    }
                } else {
                    // 32 columns at a time, the next load in flight while the
                    // previous columns are converted and stored
                    uint32_t ra[32], rb[32];
                    tmem_ld32_issue(ta, ra);
#pragma unroll 1
                    for (int cc = 0; cc < kRowTile / 32; cc += 2) {
                        tmem_wait32(ra);
                        tmem_ld32_issue(ta + (cc + 1) * 32, rb);
                        store_cols32(op, tok, n0 + cc * 32, ra, fs);
                        tmem_wait32(rb);
                        if (cc + 2 < kRowTile / 32) tmem_ld32_issue(ta + (cc + 2) * 32, ra);
                        store_cols32(op, tok, n0 + (cc + 1) * 32, rb, fs);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kTmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
    // The last CTA to finish sets the launch's tile counter back to zero for
    // the next launch on the stream (which reads it only after this grid has
    // completed: its schedulers start after griddepcontrol.wait).
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.tile_ctr + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.tile_ctr, 0u);
            atomicExch(p.tile_ctr + 1, 0u);
        }
    }
}

// ------------------------------------------------------------ CTA pairs --
// Pair plan (every launch with some M > 128 and b-bit codes): a cluster of
// two CTAs on two SMs computes a 512-token x 256-row tile with
// tcgen05.mma.cta_group::2 (M = 256 tokens, N = 256 weight rows, K = 16).  The
// pair's MMA takes its A operand (x) 128 token rows from each CTA and its B
// operand (the dequantized W) 128 weight rows from each CTA, and keeps each
// CTA's 128 token rows of the accumulator in that CTA's tensor memory.  So each
// SM dequantizes only its own 128 weight rows of a slab for 512 tokens (two
// MMA halves of 256): half the dequant work per multiply-add of a 256 x 256
// one-SM tile, and half its shared-memory operand traffic.
//
// Per CTA (rank r of the pair): x slab = tokens t0 + 256h + 128r + [0, 128)
// for halves h = 0, 1 (two TMA boxes of 128 rows, 32 KB), W slab = rows
// n0 + 128r + [0, 128) (16 KB).  The even CTA (the leader) issues every MMA.
// Hand-offs between the two CTAs:
//   * x and W: each CTA's TMA copies complete on its own xfull barrier and
//     its dequant warps arrive on its own full barrier; in the peer one
//     relay thread waits for both and arrives on the leader's pfull barrier
//     (one cluster-scope release per slab, by a thread with no loads in
//     flight: a cluster-scope release by the dequant threads themselves
//     would wait for their prefetch loads of the next block).  With every
//     copy completing in its own CTA, each CTA can drain its own copies
//     after an abort before it leaves;
//   * stage free, accumulator full, all MMAs done: the leader's
//     tcgen05.commit arrives on the barrier of both CTAs (multicast commit);
//   * accumulator half drained: the epilogue warps of both CTAs arrive on
//     the leader's acc_empty barrier of that token half (after
//     tcgen05.wait::ld and the tcgen05 fence, so the leader's next MMAs
//     cannot overwrite unread columns); the halves complete and drain one
//     after the other, so the epilogue overlaps the MMAs (see the issuer).
// No TMA copy here multicasts: each CTA loads its own operands.  Tiles are
// assigned statically (pair c takes tiles c, c + pairs, ...), ops with the
// longest K first.
constexpr int kPairTok = 512;      // tokens per pair tile
constexpr int kPairStages = 4;

struct PairCtl {
    unsigned long long full[kPairStages];   // both: this CTA's W slab written (kDqWarps arrivals)
    unsigned long long pfull[kPairStages];  // leader: the peer's x and W slabs ready (the peer's relay)
    unsigned long long xfull[kPairStages];  // both: this CTA's x slab landed (expect_tx + the copies)
    unsigned long long empty[kPairStages];  // both: the pair's MMAs on the stage completed
    unsigned long long acc_full[2];         // both: token half h of a tile's accumulator complete
    unsigned long long acc_empty[2];        // leader: half h drained by both CTAs' epilogues (2 x kEpiWarps)
    unsigned long long mma_done;            // both: every MMA the leader issued has completed
    uint32_t tmem_base;
    int abort;
};

struct PairPlan {
    static constexpr int kDqWarps = 8;  // thread d: row d / 2 of this CTA's 128, 32-code chunk d % 2
    static constexpr int kThreads = 32 * (kDqWarp0 + kDqWarps);
    static constexpr int kSlabX = 2 * kPrefillHalfTokens * kBK * 2;  // 32 KB
    static constexpr int kSlabW = 128 * kBK * 2;                     // 16 KB
    static constexpr int kOffW = kPairStages * kSlabX;
    static constexpr int kOffCtl = kOffW + kPairStages * kSlabW;
    static constexpr size_t kBytes = kOffCtl + sizeof(PairCtl) + 1024;
    static_assert(kOffW % 1024 == 0 && kOffCtl % 1024 == 0, "SWIZZLE_128B stages need 1024-byte alignment");
    static_assert(kBytes <= 232448, "227 KB of shared memory per CTA");
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrival on a barrier of either CTA of the pair: release at cluster scope
// (orders this thread's earlier memory operations, and what it acquired,
// before the arrival for a waiter in the other CTA), or at CTA scope (the
// ordering the tcgen05 fences already give: tensor-memory reads before the
// leader's next MMAs).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(unsigned long long *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bounded wait, with cluster-scope acquire (CL: the barrier's arrivals
// release data written by the other CTA's threads) or CTA-scope acquire (TMA
// bytes, tcgen05 commits, tensor-memory hand-offs).  On a timeout both CTAs
// of the pair are told to abort (their own flag and the peer's) and
// ZQ_ERR_TIMEOUT is recorded.  As in mbar_wait, the first test is inline.
template <bool CL = false>
__device__ __noinline__ bool pair_wait_poll(unsigned long long *bar, uint32_t parity, volatile int *abort,
                                            uint32_t peer_abort, unsigned long long limit) {
    auto ready = [&]() { return CL ? mbar_try_wait_cl(bar, parity) : mbar_try_wait(bar, parity); };
    if (ready()) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (ready()) return true;
        if ((it & 15u) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > limit) {
                *abort = 1;
                asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
                atomicExch(&g_prefill_error, 5);  // ZQ_ERR_TIMEOUT
                return false;
            }
        }
    }
}
template <bool CL = false>
__device__ __forceinline__ bool pair_wait(unsigned long long *bar, uint32_t parity, volatile int *abort,
                                          uint32_t peer_abort, unsigned long long limit) {
    const bool ok = CL ? mbar_try_wait_cl(bar, parity) : mbar_try_wait(bar, parity);
    return ok || pair_wait_poll<CL>(bar, parity, abort, peer_abort, limit);
}
__device__ __noinline__ void pair_drain(unsigned long long *bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait_cl(bar, parity))
        if (globaltimer() - t0 > kDrainNs) break;
}

// Instruction descriptor, kind::f16 for the pair: fp16 A and B (K-major), fp32
// D, M = 256 (tokens, 128 per CTA), N = 256 (weight rows, 128 per CTA).
constexpr uint32_t kIdescPair = (1u << 4) | (static_cast<uint32_t>(256 >> 3) << 17) |
                                (static_cast<uint32_t>(256 >> 4) << 24);

__device__ __forceinline__ void umma_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdescPair), "r"(accumulate)
        : "memory");
}
// Completion of the leader's MMAs issued so far, arriving on `bar` in both CTAs.
__device__ __forceinline__ void umma_commit_pair(unsigned long long *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

template <int B>
// 14 warps, one CTA per SM: 128 registers per thread (four warps share a
// sub-partition's 16K registers).
__global__ void __launch_bounds__(PairPlan::kThreads, 1) prefill_pair_kernel(const __grid_constant__ PrefillGroup p) {
    using P = PairPlan;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sx = base;            // x slabs
    uint8_t *sw = base + P::kOffW;  // W slabs (this CTA's 128 rows)
    PairCtl &c = *reinterpret_cast<PairCtl *>(base + P::kOffCtl);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);
    const int n_tiles = p.n_tiles;
    volatile int *abort = &c.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&c.full[s], P::kDqWarps);
            mbar_init(&c.pfull[s], 1);
            mbar_init(&c.xfull[s], 1);
            mbar_init(&c.empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&c.acc_full[h], 1);
            mbar_init(&c.acc_empty[h], 2 * kEpiWarps);
        }
        mbar_init(&c.mma_done, 1);
        c.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kTmaWarp) {
        // both CTAs' warp kTmaWarp allocate together: the same 512 columns in each
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&c.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any arrival from the peer
    tc_fence_after();
    const uint32_t tmem = c.tmem_base;
    const uint32_t peer_abort = peer_addr(&c.abort, rank ^ 1u);

    pdl_wait();  // x may be produced by the previous kernel in the stream
    pdl_launch_dependents();

    if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = pair; t < n_tiles && !*abort; t += pairs) {
                const TileRef tr = locate(p, t, kPairTok);
                const PrefillOp &op = p.ops[tr.o];
                const int slabs = op.K / kBK;
                const int nh = tr.t0 + 256 < op.M ? 2 : 1;  // token halves that hold tokens
                bool ok = true;
                for (int s = 0; s < slabs; ++s, ++it) {
                    const int st = it % kPairStages;
                    if (!pair_wait(&c.empty[st], ((it / kPairStages) & 1u) ^ 1u, abort, peer_abort, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&c.xfull[st], static_cast<uint32_t>(nh * (P::kSlabX / 2)));
                    for (int h = 0; h < nh; ++h)
                        tma_load_2d(sx + st * P::kSlabX + h * (P::kSlabX / 2), &op.xmap, s * kBK,
                                    tr.t0 + 256 * h + 128 * static_cast<int>(rank), &c.xfull[st]);
                }
                if (!ok) break;
            }
            // Copies still in flight (only after an abort) must land before
            // the CTA can exit: a stage is refilled only after the pair's MMAs
            // consumed its previous copy, so only the last kPairStages copies
            // can be pending, one per slot; their barriers complete on the
            // copies' bytes alone.
            for (uint32_t k = 0; k < kPairStages && k < it; ++k) {
                const uint32_t j = it - 1 - k;
                pair_drain(&c.xfull[j % kPairStages], (j / kPairStages) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0 && rank == 1) {
            // Relay: each stage of this CTA, once its x slab has landed and
            // its W slab is written, to the leader's pfull.
            const uint32_t pfull_leader0 = peer_addr(&c.pfull[0], 0);
            uint32_t it = 0;
            bool ok = true;
            for (int t = pair; t < n_tiles && ok && !*abort; t += pairs) {
                const int slabs = p.ops[locate(p, t, kPairTok).o].K / kBK;
                for (int s = 0; s < slabs; ++s, ++it) {
                    const int st = it % kPairStages;
                    const uint32_t par = (it / kPairStages) & 1u;
                    if (!pair_wait(&c.xfull[st], par, abort, peer_abort, p.wait_ns) ||
                        !pair_wait(&c.full[st], par, abort, peer_abort, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_cluster(pfull_leader0 + st * static_cast<uint32_t>(sizeof(unsigned long long)));
                }
            }
        }
        if (lane == 0 && rank == 0) {
            // Order of a tile's MMAs: the first H slabs (H = min(stages,
            // slabs)) for token half 0, then the same slabs for half 1; the
            // middle slabs both halves each; the last T slabs again half 0
            // first (then acc_full[0]), then half 1 (then acc_full[1]).  So
            // half 0 of the accumulator completes, and is drained, while half
            // 1's last MMAs run, and the next tile's half-0 MMAs run while
            // half 1 is drained: the tensor pipe waits for the epilogue only
            // where a drain outlasts H (or T) slabs of one half's MMAs.
            uint32_t it = 0, tile_i = 0;
            auto operands = [&](uint32_t j) -> bool {  // stage of slab j filled in both CTAs
                const int st = j % kPairStages;
                const uint32_t par = (j / kPairStages) & 1u;
                if (!pair_wait(&c.xfull[st], par, abort, peer_abort, p.wait_ns) ||
                    !pair_wait(&c.full[st], par, abort, peer_abort, p.wait_ns) ||
                    !pair_wait<true>(&c.pfull[st], par, abort, peer_abort, p.wait_ns))
                    return false;
                tc_fence_after();
                return true;
            };
            auto mma_half = [&](uint32_t j, int s, int h) {  // slab j (s-th of its tile), token half h
                const int st = j % kPairStages;
                const uint32_t a0 = smem_u32(sx + st * P::kSlabX + h * (P::kSlabX / 2));
                const uint32_t b0 = smem_u32(sw + st * P::kSlabW);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    umma_pair(tmem + h * kRowTile, sdesc_sw128(a0 + kk * 32), sdesc_sw128(b0 + kk * 32),
                              (s > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = true;
            for (int t = pair; t < n_tiles && ok; t += pairs, ++tile_i) {
                if (*abort) break;
                const TileRef tr = locate(p, t, kPairTok);
                const PrefillOp &op = p.ops[tr.o];
                const int S = op.K / kBK;
                const bool half1 = tr.t0 + 256 < op.M;
                const int H = min(kPairStages, S), T = min(kPairStages, S - H);
                const uint32_t pe = (tile_i & 1u) ^ 1u;  // parity of the previous tile's drains
                // head: half 0, then half 1 of slabs [0, H)
                if (!pair_wait(&c.acc_empty[0], pe, abort, peer_abort, p.wait_ns)) break;
                tc_fence_after();
                for (int s = 0; s < H && ok; ++s) {
                    ok = operands(it + s);
                    if (ok) mma_half(it + s, s, 0);
                }
                if (!ok) break;
                if (H == S) umma_commit_pair(&c.acc_full[0]);
                if (!pair_wait(&c.acc_empty[1], pe, abort, peer_abort, p.wait_ns)) break;
                tc_fence_after();
                for (int s = 0; s < H; ++s) {
                    if (half1) mma_half(it + s, s, 1);
                    umma_commit_pair(&c.empty[(it + s) % kPairStages]);
                }
                if (H == S) umma_commit_pair(&c.acc_full[1]);
                // middle: both halves per slab
                for (int s = H; s < S - T && ok; ++s) {
                    ok = operands(it + s);
                    if (!ok) break;
                    mma_half(it + s, s, 0);
                    if (half1) mma_half(it + s, s, 1);
                    umma_commit_pair(&c.empty[(it + s) % kPairStages]);
                }
                if (!ok) break;
                // tail: half 0, then half 1 of slabs [S - T, S)
                if (T > 0) {
                    for (int s = S - T; s < S && ok; ++s) {
                        ok = operands(it + s);
                        if (ok) mma_half(it + s, s, 0);
                    }
                    if (!ok) break;
                    umma_commit_pair(&c.acc_full[0]);
                    for (int s = S - T; s < S; ++s) {
                        if (half1) mma_half(it + s, s, 1);
                        umma_commit_pair(&c.empty[(it + s) % kPairStages]);
                    }
                    umma_commit_pair(&c.acc_full[1]);
                }
                it += S;
            }
            // Always signalled (even with no MMA issued): both CTAs wait for it
            // before TMEM is freed and before either CTA exits.
            umma_commit_pair(&c.mma_done);
        }
    } else if (warp >= kDqWarp0) {
        // Thread d: row d / 2 of this CTA's 128 weight rows, 32-code chunk
        // d % 2 of every slab.  The codes, scales and zeros of a block (128
        // codes: two slabs) are loaded into registers three blocks ahead of
        // their use (register sets A, B and C rotate; two at b = 8), so that
        // about six slabs of dequant time cover the loads' latency; with groups
        // of 128 the scale and the zero stay as loaded until the block is used,
        // where they become its (scale | zero << 16) word.
        const int d = threadIdx.x - 32 * kDqWarp0;
        const int row = d >> 1, ch = d & 1;
        const uint32_t *rowp = nullptr;
        const uint16_t *srow = nullptr, *zrow = nullptr;
        int gsh = 2;
        // fetch cursor: tile tf, block gf of blocks_f
        int tf = pair, gf = 0, blocks_f = 0;
        auto start_tile = [&](int t) {
            const TileRef tr = locate(p, t, kPairTok);
            const PrefillOp &op = p.ops[tr.o];
            gsh = op.gshift;
            const size_t gs = static_cast<size_t>(op.K) >> (op.gshift + 5);  // scales per row
            const int r = min(tr.n0 + 128 * static_cast<int>(rank) + row, op.N - 1);
            rowp = op.packed + static_cast<size_t>(r) * (static_cast<size_t>(op.K) * B / 32);
            srow = op.scales + static_cast<size_t>(r) * gs;
            zrow = op.zeros + static_cast<size_t>(r) * gs;
            blocks_f = op.K / kGroup;
        };
        if (tf < n_tiles) start_tile(tf);
        auto fetch_next = [&](uint32_t (&w)[2][B], uint32_t (&sz)[2]) {
            if (tf >= n_tiles) return;
            // slab h of block gf: codes 128gf + 64h + 32ch .. +31, group (4gf + 2h + ch) >> gsh
#pragma unroll
            for (int h = 0; h < 2; ++h) load_chunk<B>(w[h], rowp + static_cast<size_t>(4 * gf + 2 * h + ch) * B);
            const int g0 = (4 * gf + ch) >> gsh, g1 = (4 * gf + 2 + ch) >> gsh;  // one group with groups of 128
            if (gsh == 2) {
                // the scale and the zero as loaded: the consumer packs them
                // (packing here would wait for the loads)
                sz[0] = ldg_u16_nc(srow + g0);
                sz[1] = ldg_u16_nc(zrow + g0);
            } else {
                sz[0] = ldg_u16_nc(srow + g0) | (ldg_u16_nc(zrow + g0) << 16);
                sz[1] = ldg_u16_nc(srow + g1) | (ldg_u16_nc(zrow + g1) << 16);
            }
            if (++gf == blocks_f) {
                gf = 0;
                tf += pairs;
                if (tf < n_tiles) start_tile(tf);
            }
        };
        // consume cursor: tile tc, block gc of blocks_c; slab counter it
        int tc = pair, gc = 0, blocks_c = 0, gsh_c = 2;
        if (tc < n_tiles) {
            const PrefillOp &op = p.ops[locate(p, tc, kPairTok).o];
            blocks_c = op.K / kGroup;
            gsh_c = op.gshift;
        }
        uint32_t it = 0;
        auto consume = [&](uint32_t (&w)[2][B], uint32_t (&sz)[2]) -> bool {
            if (tc >= n_tiles || *abort) return false;
            uint32_t wc[2][B], szc[2];
            bool ovf[2];
            if (gsh_c == 2) {
                szc[0] = szc[1] = prmt(sz[0], sz[1], 0x5410u);
            } else {
                szc[0] = sz[0];
                szc[1] = sz[1];
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int q = 0; q < B; ++q) wc[h][q] = w[h][q];
                ovf[h] = dequant_overflows<B>(szc[h]);
            }
            fetch_next(w, sz);  // the set is free again: load the block two ahead
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // the two slabs of this block
                const int st = it % kPairStages;
                if (!pair_wait(&c.empty[st], ((it / kPairStages) & 1u) ^ 1u, abort, peer_abort, p.wait_ns))
                    return false;
                uint8_t *bs = sw + st * P::kSlabW;
                uint32_t o[16];
                dequant_chunk<B>(wc[h], szc[h], o, ovf[h]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c16 = (4 * ch + j) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(bs + row * 128 + c16 * 16) =
                        make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                }
                fence_proxy_async();  // the generic writes, visible to the MMA's (async-proxy) reads
                __syncwarp();
                if (lane == 0) mbar_arrive(&c.full[st]);
                ++it;
            }
            if (++gc == blocks_c) {
                gc = 0;
                tc += pairs;
                if (tc < n_tiles) {
                    const PrefillOp &op = p.ops[locate(p, tc, kPairTok).o];
                    blocks_c = op.K / kGroup;
                    gsh_c = op.gshift;
                }
            }
            return true;
        };
        uint32_t wA[2][B], szA[2], wB[2][B], szB[2], wC[2][B], szC[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            szA[h] = szB[h] = szC[h] = 0u;
#pragma unroll
            for (int q = 0; q < B; ++q) wA[h][q] = wB[h][q] = wC[h][q] = 0u;
        }
        fetch_next(wA, szA);
        fetch_next(wB, szB);
        if constexpr (B == 8) {
            // b = 8: twice the code words per block; two sets fit the registers
#pragma unroll 1
            while (consume(wA, szA) && consume(wB, szB)) {
            }
        } else {
            fetch_next(wC, szC);
#pragma unroll 1
            while (consume(wA, szA) && consume(wB, szB) && consume(wC, szC)) {
            }
        }
    } else if (warp < kEpiWarps) {
        // Epilogue warps 0..3: TMEM lanes 32*warp .. +31 = this CTA's token
        // rows of each half; columns = the tile's 256 weight rows.
        uint32_t tile_i = 0;
        for (int t = pair; t < n_tiles; t += pairs, ++tile_i) {
            if (*abort) break;
            const TileRef tr = locate(p, t, kPairTok);
            const PrefillOp &op = p.ops[tr.o];
            const int nh = tr.t0 + 256 < op.M ? 2 : 1;
            bool ok = true;
            for (int half = 0; half < 2; ++half) {  // drained in the order the MMAs complete them
                if (!pair_wait(&c.acc_full[half], tile_i & 1u, abort, peer_abort, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (half < nh) {
                    const int tok = tr.t0 + 256 * half + 128 * static_cast<int>(rank) + 32 * warp + lane;
                    const float fs = (op.xscale != nullptr && tok < op.M) ? op.xscale[tok] : 1.0f;
                    // 32 columns at a time, the next load in flight while the
                    // previous columns are converted and stored
                    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + half * kRowTile;
                    uint32_t ra[32], rb[32];
                    tmem_ld32_issue(ta, ra);
#pragma unroll 1
                    for (int cc = 0; cc < kRowTile / 32; cc += 2) {
                        tmem_wait32(ra);
                        tmem_ld32_issue(ta + (cc + 1) * 32, rb);
                        store_cols32(op, tok, tr.n0 + cc * 32, ra, fs);
                        tmem_wait32(rb);
                        if (cc + 2 < kRowTile / 32) tmem_ld32_issue(ta + (cc + 2) * 32, ra);
                        store_cols32(op, tok, tr.n0 + (cc + 1) * 32, rb, fs);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(peer_addr(&c.acc_empty[half], 0));
            }
            if (!ok) break;
        }
    }

    // Every MMA of the pair has completed before either CTA frees TMEM or
    // exits (the leader's MMAs read both CTAs' shared memory and write both
    // CTAs' TMEM).
    if (warp == kMmaWarp && lane == 0) pair_drain(&c.mma_done, 0u);
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == kTmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// Dequant test hook: one thread per (row, 32-code chunk) runs dequant_chunk,
// the tile kernel's own routine (unpack, one-HFMA2 rounding, K-order restore,
// overflow hold), and writes the 32 fp16 values to w_hat (N x K, natural order).
template <int B>
__global__ void dequant_test_kernel(const uint32_t *__restrict__ packed, const uint16_t *__restrict__ scales,
                                    const uint16_t *__restrict__ zeros, int N, int K, int gshift,
                                    uint16_t *__restrict__ w_hat) {
    const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int chunks = K / 32;
    if (t >= static_cast<long long>(N) * chunks) return;
    const int n = static_cast<int>(t / chunks), c = static_cast<int>(t % chunks);
    uint32_t w[B];
    load_chunk<B>(w, packed + static_cast<size_t>(n) * (static_cast<size_t>(K) * B / 32) + static_cast<size_t>(c) * B);
    const size_t gi = static_cast<size_t>(n) * (static_cast<size_t>(K) >> (gshift + 5)) + (c >> gshift);
    const uint32_t sz = scales[gi] | (static_cast<uint32_t>(zeros[gi]) << 16);
    uint32_t o[16];
    dequant_chunk<B>(w, sz, o, dequant_overflows<B>(sz));
    uint4 *dst = reinterpret_cast<uint4 *>(w_hat + static_cast<size_t>(n) * K + static_cast<size_t>(c) * 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

}  // namespace pf

cudaError_t launch_dequant_test(const uint32_t *packed, const uint16_t *scales, const uint16_t *zeros, int bits,
                                int group, int N, int K, uint16_t *w_hat, cudaStream_t stream) {
    const long long threads = static_cast<long long>(N) * (K / 32);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    const int gshift = group == 32 ? 0 : group == 64 ? 1 : 2;
    switch (bits) {
        case 2: pf::dequant_test_kernel<2><<<blocks, 256, 0, stream>>>(packed, scales, zeros, N, K, gshift, w_hat); break;
        case 3: pf::dequant_test_kernel<3><<<blocks, 256, 0, stream>>>(packed, scales, zeros, N, K, gshift, w_hat); break;
        case 4: pf::dequant_test_kernel<4><<<blocks, 256, 0, stream>>>(packed, scales, zeros, N, K, gshift, w_hat); break;
        default: pf::dequant_test_kernel<8><<<blocks, 256, 0, stream>>>(packed, scales, zeros, N, K, gshift, w_hat); break;
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ host --

template <int B, bool ONE, int XR = ONE ? 128 : 256>
static cudaError_t launch_prefill_t(const PrefillGroup &pg, int n_ctas, cudaStream_t stream) {
    constexpr size_t smem = pf::Plan<B, ONE, XR>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(pf::prefill_kernel<B, ONE, XR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_ctas));
    cfg.blockDim = dim3(pf::Plan<B, ONE, XR>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, pf::prefill_kernel<B, ONE, XR>, pg);
}

cudaError_t prefill_x_map(CUtensorMap *map, const uint16_t *x, int M, int K) {
    return prefill_x_map_rows(map, x, M, K, pf::kTokTile);
}

cudaError_t prefill_x_map_rows(CUtensorMap *map, const uint16_t *x, int M, int K, int box_rows) {
    return encode_tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, static_cast<uint64_t>(K),
                                static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, pf::kBK,
                                static_cast<uint32_t>(box_rows), CU_TENSOR_MAP_SWIZZLE_128B);
}

int prefill_plan(const PrefillGroup &pg, int bits) {
    int max_m = 0;
    for (int i = 0; i < pg.n_ops; ++i) max_m = pg.ops[i].M > max_m ? pg.ops[i].M : max_m;
    if (max_m <= kPrefillQuarterTokens && bits <= 4) return kPlanOneHalf64;
    if (max_m <= kPrefillHalfTokens) return kPlanOneHalf;
    // CTA pairs from 512 tokens: below, a pair tile's second token half is
    // empty and the one-CTA two-half plan was faster (M = 256: 3.4 against
    // 5.5 ms on the 28-layer stack)
    return (bits == 16 || max_m < kPairMinM) ? kPlanTwoHalves : kPlanPair;
}

int prefill_box_rows(int plan) {
    return plan == kPlanTwoHalves ? pf::kTokTile : plan == kPlanOneHalf64 ? kPrefillQuarterTokens : kPrefillHalfTokens;
}

int prefill_tok_tile(int plan) { return plan == kPlanPair ? pf::kPairTok : pf::kTokTile; }

int prefill_tiles(int M, int N, int plan) {
    const int tt = prefill_tok_tile(plan);
    return ((M + tt - 1) / tt) * ((N + pf::kRowTile - 1) / pf::kRowTile);
}

// Pair plan: clusters of two CTAs, as many pairs as fit at once (at most one
// per tile); the count that fits is queried once per bit width.
template <int B>
static cudaError_t launch_pair_t(const PrefillGroup &pg, int num_sms, cudaStream_t stream) {
    constexpr size_t smem = pf::PairPlan::kBytes;
    cudaError_t e = cudaFuncSetAttribute(pf::prefill_pair_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (num_sms / 2)));
    cfg.blockDim = dim3(pf::PairPlan::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    static std::atomic<int> fit{0};
    int pairs_fit = fit.load();
    if (pairs_fit == 0) {
        e = cudaOccupancyMaxActiveClusters(&pairs_fit, pf::prefill_pair_kernel<B>, &cfg);
        if (e != cudaSuccess) return e;
        if (pairs_fit < 1) return cudaErrorInvalidConfiguration;
        fit.store(pairs_fit);
    }
    const int pairs = pg.n_tiles < pairs_fit ? pg.n_tiles : pairs_fit;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    return cudaLaunchKernelEx(&cfg, pf::prefill_pair_kernel<B>, pg);
}

cudaError_t launch_prefill_group(const PrefillGroup &pg, int bits, int num_sms, cudaStream_t stream) {
    const int n_ctas = pg.n_tiles < num_sms ? pg.n_tiles : num_sms;
    const int plan = prefill_plan(pg, bits);
    if (plan == kPlanPair) {
        switch (bits) {
            case 2: return launch_pair_t<2>(pg, num_sms, stream);
            case 3: return launch_pair_t<3>(pg, num_sms, stream);
            case 4: return launch_pair_t<4>(pg, num_sms, stream);
            default: return launch_pair_t<8>(pg, num_sms, stream);
        }
    }
    if (plan == kPlanOneHalf64) {
        switch (bits) {
            case 2: return launch_prefill_t<2, true, kPrefillQuarterTokens>(pg, n_ctas, stream);
            case 3: return launch_prefill_t<3, true, kPrefillQuarterTokens>(pg, n_ctas, stream);
            default: return launch_prefill_t<4, true, kPrefillQuarterTokens>(pg, n_ctas, stream);
        }
    }
    if (plan == kPlanOneHalf) {
        switch (bits) {
            case 2: return launch_prefill_t<2, true>(pg, n_ctas, stream);
            case 3: return launch_prefill_t<3, true>(pg, n_ctas, stream);
            case 4: return launch_prefill_t<4, true>(pg, n_ctas, stream);
            case 8: return launch_prefill_t<8, true>(pg, n_ctas, stream);
            default: return launch_prefill_t<16, true>(pg, n_ctas, stream);
        }
    }
    switch (bits) {
        case 2: return launch_prefill_t<2, false>(pg, n_ctas, stream);
        case 3: return launch_prefill_t<3, false>(pg, n_ctas, stream);
        case 4: return launch_prefill_t<4, false>(pg, n_ctas, stream);
        case 8: return launch_prefill_t<8, false>(pg, n_ctas, stream);
        default: return launch_prefill_t<16, false>(pg, n_ctas, stream);
    }
}

cudaError_t prefill_w_map(CUtensorMap *map, const uint16_t *w, int N, int K) {
    return encode_tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w, static_cast<uint64_t>(K),
                                static_cast<uint64_t>(N), static_cast<uint64_t>(K) * 2, pf::kBK,
                                static_cast<uint32_t>(pf::kRowTile), CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t read_prefill_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_prefill_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_prefill_error, &zero, sizeof(int));
}

}  // namespace zq
