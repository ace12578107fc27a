// zq_decode.cu — decode kernel (M <= 32): skinny tensor-core GEMM that streams
// the packed weights exactly once.  (From 17 tokens on the tcgen05 tile kernel
// of zq_prefill.cu, with a single token tile, streams them faster.)
//
// What it computes: y = x · dequant(W)^T with dequant(W) = q * scale + zero per
// group of 128 along K ([wiki] "ZSE - open-source движок для запуска LLM
// локально на GPU - 2026", section "Формат модели .zse").  The pages' INT4 GEMV
// for small batches (section "Оркестратор и GPU-ядра": 128-bit weight loads,
// batched GEMV) is prior art only; this is a B200 design:
//
//  * Per group the dequant is factored:
//        sum_k x_k (q_k s + z) = s * sum_k q_k x_k + z * sum_k x_k,
//    so the hot loop multiplies EXACT integer codes (fp16) with fp16 x on the
//    tensor cores (mma.sync m16n8k16, fp32 accumulate), and the scale/zero are
//    applied once per group in fp32.  sum_k x_k per group is precomputed.
//  * Swap-AB: weight rows fill the 16-row side of the MMA, tokens the 8-column
//    side, so M = 1..8 costs one MMA column tile.
//  * Codes become biased fp16 pairs, 1024 + q * 2^s, with one LOP3 per two codes
//    (zq_device.cuh) and go to the tensor cores as they are: the activations
//    are pre-permuted once per call into the same pair order and pre-scaled by
//    2^(E - s) (exact; E per token and group keeps x' in fp16's normal range),
//    so each product is 1024 * x' + 2^E * q * x, and the per-group bias
//    1024 * sum(x') is subtracted, and 2^E divided out, in fp32 once per group.
//    The canonical packed layout is consumed as stored.
//  * A CTA step is 64 weight rows (128 with four token tiles and b <= 4) x
//    GPS groups.  One ring of shared-memory
//    stages per CTA, filled in turn by the four warps (stage t by warp t % 4,
//    the scheduling state handed from one producing warp to the next through
//    shared memory): one TMA 2-D copy per 128-byte column of the codes, with
//    the 128-byte swizzle so the fragment loads are free of bank conflicts
//    (one unswizzled 208-byte box at b = 3); bulk copies of the step's
//    activations and group sums; cp.async for scales and zeros.  All four
//    warps consume, each 16 of the rows (32 with 128-row steps: two row tiles
//    share every activation fragment).  A step descriptor travels in the
//    stage, so the consumers keep no scheduling state.
//  * A persistent grid covers every SM.  The steps of all ops of a launch are
//    cut into chunks: whole row blocks (large launches, longest first) or
//    2^c consecutive steps (small launches, split along K).  A CTA starts with
//    chunk blockIdx.x and takes further chunks from a counter.  A row block
//    cut by a chunk boundary is reduced by the last warp to finish a piece of
//    it, in chunk order, so results are deterministic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "zq_device.cuh"
#include "zq_internal.h"

namespace zq {

template <int I, int N, typename F>
__device__ __forceinline__ void static_for_impl(F &f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for_impl<I + 1, N>(f);
    }
}
// Calls f(integral_constant<int, i>) for i = 0 .. N-1 (compile-time indices).
template <int N, typename F>
__device__ __forceinline__ void static_for(F &&f) {
    static_for_impl<0, N>(f);
}

// ------------------------------------------------------------------ prep --
// One warp per (entry, padded token, group).  Tokens < M: the group's 128
// activations, pair-permuted and scaled by 2^(E - s), into xg (M x K,
// row-major).  E is chosen per (token, group) from the group's largest |x| so
// that the scaled values sit near 2^14: whatever the magnitude of the
// activations (fp16 subnormals included), x' keeps fp16's full precision
// instead of sliding into the subnormal range, where x * 2^-s would lose bits
// or flush to zero.  Every scaling is by a power of two, so it is exact and the
// kernel undoes it with the factor f = 2^-E in fp32.
// Lane c of the MMA reads 16-byte chunks 4c .. 4c+3 of its token's row; they
// are stored at x_chunk(c, q, token & 7), so that the 8 lanes of a quarter
// warp (two tokens x four lanes) always hit 8 different bank groups.  Every
// padded token gets its group record (sum x, -f * 1024 * sum x', f, 0):
// zeros past M.

__host__ __device__ constexpr int x_chunk(int c, int q, int t7) { return (4 * c + (q ^ (2 * (c >> 1)))) ^ t7; }

// Exponent E of the (token, group) scaling: 2^E * max|x| lies in [2^14, 2^15);
// E = 0 for an all-zero group.  fp16 activations give E in [-1, 38]; bf16
// ones (fp32's exponent range) are held to [-40, 100], i.e. groups whose
// largest |x| is in [2^-86, 2^55).
__device__ __forceinline__ int prep_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127;  // floor(log2 amax)
    return max(-40, min(14 - ex, 100));
}

// One activation as float: fp16 bits, or bfloat16 bits (the top half of a binary32).
template <bool BF16>
__device__ __forceinline__ float act_bits(uint32_t h) {
    if constexpr (BF16) return __uint_as_float(h << 16);
    else return h2f_bits(h);
}

__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }

template <int B, bool BF16>
__device__ __forceinline__ float prep_group(const uint16_t *xrow, uint16_t *prow, int lane, int t7, int E) {
    float bias = 0.0f;  // sum of the scaled activations written by this lane
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int q = lane + 32 * h;  // 64 pairs per group
        const int c = q / 16, p = q % 16;
        // exact powers of two: the codes of the two halves may sit at different offsets
        const float sl = pow2f(E - pair_shift_lo<B>(p)), sh = pow2f(E - pair_shift_hi<B>(p));
        const __half lo = __float2half_rn(act_bits<BF16>(xrow[32 * c + pair_lo<B>(p)]) * sl);
        const __half hi = __float2half_rn(act_bits<BF16>(xrow[32 * c + pair_hi<B>(p)]) * sh);
        bias += __half2float(lo) + __half2float(hi);
        const int word = (x_chunk(c, p >> 2, t7) << 2) | (p & 3);
        reinterpret_cast<uint32_t *>(prow)[word] = __half_as_ushort(lo) | (__half_as_ushort(hi) << 16);
    }
    return bias;
}

template <class PP>
__global__ void __launch_bounds__(256) prep_kernel(const __grid_constant__ PP p,
                                                   long long total_warps) {
    pdl_wait();  // x may be the output of the previous kernel in the stream
    if (p.work != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.work = 0u;
    const long long gw = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw < total_warps) {
        int e = 0;
        while (e + 1 < p.n_entries && p.warp_prefix[e + 1] <= gw) ++e;
        const PrepEntry &en = p.e[e];
        const long long local = gw - p.warp_prefix[e];
        const int G = en.K / kGroup;
        const int t = static_cast<int>(local / G), g = static_cast<int>(local % G);
        // Both outputs by decode step (GPS groups): [step][token][GPS groups]
        // of x' and [step][token][RS records], so a step's x' and records for
        // all staged tokens are two contiguous blocks (two bulk copies).
        const int gps = en.gps;
        const size_t blk = static_cast<size_t>(g / gps) * en.x_rows + t;  // (step, token)
        float4 *dst = reinterpret_cast<float4 *>(en.sx) + blk * en.rs + g % gps;
        uint16_t *prow = en.xg + (blk * gps + g % gps) * kGroup;
        if (t >= en.M) {
            if (lane == 0) *dst = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            reinterpret_cast<uint2 *>(prow)[lane] = make_uint2(0u, 0u);
        } else {
            const uint16_t *xrow = en.x + static_cast<size_t>(t) * en.K + static_cast<size_t>(g) * kGroup;
            const uint2 v = reinterpret_cast<const uint2 *>(xrow)[lane];
            const bool bf = en.x_bf16 != 0;
            const float x0 = bf ? act_bits<true>(v.x & 0xFFFFu) : act_bits<false>(v.x & 0xFFFFu);
            const float x1 = bf ? act_bits<true>(v.x >> 16) : act_bits<false>(v.x >> 16);
            const float x2 = bf ? act_bits<true>(v.y & 0xFFFFu) : act_bits<false>(v.y & 0xFFFFu);
            const float x3 = bf ? act_bits<true>(v.y >> 16) : act_bits<false>(v.y >> 16);
            float s = x0 + x1 + x2 + x3;
            float amax = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const int E = prep_exponent(amax);
            float b;
            if (bf) {
                switch (en.bits) {
                    case 2: b = prep_group<2, true>(xrow, prow, lane, t & 7, E); break;
                    case 3: b = prep_group<3, true>(xrow, prow, lane, t & 7, E); break;
                    case 4: b = prep_group<4, true>(xrow, prow, lane, t & 7, E); break;
                    case 8: b = prep_group<8, true>(xrow, prow, lane, t & 7, E); break;
                    default: b = prep_group<16, true>(xrow, prow, lane, t & 7, E); break;
                }
            } else {
                switch (en.bits) {
                    case 2: b = prep_group<2, false>(xrow, prow, lane, t & 7, E); break;
                    case 3: b = prep_group<3, false>(xrow, prow, lane, t & 7, E); break;
                    case 4: b = prep_group<4, false>(xrow, prow, lane, t & 7, E); break;
                    case 8: b = prep_group<8, false>(xrow, prow, lane, t & 7, E); break;
                    default: b = prep_group<16, false>(xrow, prow, lane, t & 7, E); break;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                b += __shfl_xor_sync(0xffffffffu, b, o);
            }
            // f * (acc - 1024 * b) = fma(acc, f, -f * 1024 * b): the products
            // by the power of two f are exact.
            const float f = pow2f(-E);
            // fp16 weights (bits 16) carry no 1024 bias
            const float bias = en.bits == 16 ? 0.0f : 1024.0f * b;
            if (lane == 0) *dst = make_float4(s, -(f * bias), f, 0.0f);
        }
    }
    // Dependents may be scheduled only now, i.e. after everything enqueued
    // before this kernel has completed (they read weights before their wait).
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- decode --

struct Cursor {
    int s;         // step index
    int o, rb, j;  // op, row block, step within the row block
    bool valid;
};

template <class DP>
__device__ __forceinline__ void cursor_init(Cursor &cu, const DP &p, int s, int s_end) {
    cu.s = s;
    cu.valid = s < s_end;
    int lo = 0, hi = p.n_ops - 1;  // last op with step0 <= s
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.ops[mid].step0 <= s) lo = mid;
        else hi = mid - 1;
    }
    const int o = lo;
    const int local = s - p.ops[o].step0;
    cu.o = o;
    cu.rb = local / p.ops[o].su;
    cu.j = local - cu.rb * p.ops[o].su;
}

template <class DP>
__device__ __forceinline__ void cursor_next(Cursor &cu, const DP &p, int s_end) {
    ++cu.s;
    cu.valid = cu.s < s_end;
    if (++cu.j == p.ops[cu.o].su) {
        cu.j = 0;
        if (++cu.rb == p.ops[cu.o].row_blocks) {
            cu.rb = 0;
            if (cu.o + 1 < p.n_ops) ++cu.o;
        }
    }
}

// Steps [begin, end) of chunk k: one whole row block, or 2^log2c steps.
template <class DP>
__device__ __forceinline__ void chunk_range(const DP &p, int k, int &begin, int &end) {
    if (p.units) {
        int lo = 0, hi = p.n_ops - 1;  // last op with unit0 <= k
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.ops[mid].unit0 <= k) lo = mid;
            else hi = mid - 1;
        }
        begin = p.ops[lo].step0 + (k - p.ops[lo].unit0) * p.ops[lo].su;
        end = begin + p.ops[lo].su;
    } else {
        begin = k << p.log2c;
        end = min(begin + (1 << p.log2c), p.total_steps);
    }
}

// Step descriptor, written by the producer into the stage (32 bytes).
//   x: op, y: row block, z: step within the row block,
//   w: number of groups | flags << 8;
//   second int4: chunk, first step of the row block, M, unused.
constexpr int kFlagLast = 1;   // last step of this chunk's piece of the row block: emit
constexpr int kFlagHead = 2;   // the row block started in an earlier chunk
constexpr int kFlagTail = 4;   // the row block continues in a later chunk
constexpr int kFlagEnd = 8;    // no more work for this CTA
constexpr int kFlagSzVec = 16; // scales and zeros are in the stage

// One k16 step of a group: biased codes of pairs 2J, 2J+1 (rows gq, gq + 8)
// times the activation pairs; J is a compile-time index so the unpack masks
// are instruction immediates.
template <int BITS, int J, bool INIT>
__device__ __forceinline__ void mma_j(float (&acc)[4], const uint32_t (&w)[2][BITS], const uint32_t (&xf)[16],
                                      uint32_t magic) {
    const uint32_t a0 = unpack_biased_c<BITS, 2 * J>(w[0], magic);
    const uint32_t a1 = unpack_biased_c<BITS, 2 * J>(w[1], magic);
    const uint32_t a2 = unpack_biased_c<BITS, 2 * J + 1>(w[0], magic);
    const uint32_t a3 = unpack_biased_c<BITS, 2 * J + 1>(w[1], magic);
    if constexpr (INIT) {
        const float zero4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma_16816(acc, a0, a1, a2, a3, xf[2 * J], xf[2 * J + 1], zero4);
    } else {
        mma_16816(acc, a0, a1, a2, a3, xf[2 * J], xf[2 * J + 1], acc);
    }
}

// One group (16 rows x 128 k) into acc: eight dependent k16 steps.  (Two
// interleaved accumulator chains measured no faster at one token and 5 %
// slower at four: their four registers cost more than the shorter chain.)
template <int BITS>
__device__ __forceinline__ void mma_group(float (&acc)[4], const uint32_t (&w)[2][BITS], const uint32_t (&xf)[16],
                                          uint32_t magic) {
    mma_j<BITS, 0, true>(acc, w, xf, magic);
    mma_j<BITS, 1, false>(acc, w, xf, magic);
    mma_j<BITS, 2, false>(acc, w, xf, magic);
    mma_j<BITS, 3, false>(acc, w, xf, magic);
    mma_j<BITS, 4, false>(acc, w, xf, magic);
    mma_j<BITS, 5, false>(acc, w, xf, magic);
    mma_j<BITS, 6, false>(acc, w, xf, magic);
    mma_j<BITS, 7, false>(acc, w, xf, magic);
}

// The output value rounded to fp16, or to bfloat16 for bf16 activations
// (nearest even, either way).
__device__ __forceinline__ uint16_t round_out(float v, int bf16) {
    return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

// Device record of a decode kernel that gave up a bounded wait (ZQ_ERR_TIMEOUT).
__device__ int g_decode_error;

// Bound of the drain after an abort, which waits for copies already issued
// and does not follow the adjustable limit of the other waits (p.wait_ns).
constexpr unsigned long long kDecodeDrainNs = 2000000000ull;  // 2 s

// Bounded wait of the whole warp for a phase of `bar`; the answer is the same
// in every lane (a lane that ran out makes the warp give up).
__device__ __forceinline__ bool wait_phase(unsigned long long *bar, uint32_t parity, unsigned long long limit) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const unsigned long long t0 = globaltimer();
        while (!(ok = mbar_try_wait(bar, parity)))
            if (globaltimer() - t0 > limit) break;
    }
    return __all_sync(0xffffffffu, ok);
}

// Scheduling state of a CTA's producer, handed from one producing warp to
// the next.
struct ProdState {
    int s, o, rb, j, valid;   // cursor of the next step to stage
    int chunk, begin, end;    // its chunk and that chunk's steps
    unsigned int ticket;      // counter value for the chunk after this one
    int done;                 // the end marker has been staged
    int slot, round;          // ring slot and round of the next stage: seq = round * depth + slot
    int seq;                  // stages filled so far
};

__device__ __forceinline__ void st_release_shared(int *a, int v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(a)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_shared(const int *a) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(a)) : "memory");
    return v;
}

// Bounded wait of the whole warp until *seq == target; it sleeps between
// polls so that a waiting warp leaves the issue slots to the others.
__device__ __forceinline__ bool wait_seq(const int *seq, int target, unsigned long long limit) {
    bool ok = ld_acquire_shared(seq) == target;
    if (!ok) {
        const unsigned long long t0 = globaltimer();
        while (!(ok = ld_acquire_shared(seq) == target)) {
            if (globaltimer() - t0 > limit) break;
            __nanosleep(64);
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// Box row (within its 8-row half) that MMA row g of a warp reads.  With the
// 128-byte swizzle a 16-byte chunk of box row r sits at chunk ^ (r & 7); a
// quarter warp covers MMA rows 2j and 2j+1, and this choice of box rows puts
// its 8 fragment loads in 8 different bank groups.
template <int BITS, int MT>
__device__ __forceinline__ int box_row(int g) {
    if constexpr (!decode_swizzled(BITS, MT) || BITS == 8 || BITS == 16) return g;  // b = 8: chunks 2c ^ g differ
    else if constexpr (BITS == 4) return (g >> 1) + 4 * (g & 1);       // rows 2j, 2j+1 -> j, j+4
    else return 2 * (g & 3) + (g >> 2);                                // b = 2 (half-warp phases)
}

template <int BITS, int MT, class DP>
__global__ void __launch_bounds__(kDecodeWarpsPerCta * 32, decode_reg_ctas(BITS, MT))
    decode_kernel(const __grid_constant__ DP p) {
    constexpr int GPS = decode_gps(BITS, MT);
    constexpr int SEG = decode_seg(BITS, MT);       // bytes of one row per step
    constexpr bool SWZ = decode_swizzled(BITS, MT);
    constexpr int BOXW = decode_box_w(BITS, MT);
    constexpr int NBOX = decode_boxes(BITS, MT);
    constexpr int RT = decode_row_tiles(BITS, MT);  // row tiles of 16 per warp
    constexpr int ROWS = decode_cta_rows(BITS, MT); // weight rows per CTA step
    constexpr int BOXB = BOXW * ROWS;               // bytes of one TMA box
    constexpr int GB = 16 * BITS;                   // bytes of one row of one group
    constexpr int MPAD = 8 * MT;
    constexpr int SZB = 2 * GPS;                    // bytes of scales (or zeros) of one row per step
    constexpr int RS = decode_rec_stride(BITS, MT); // record slots per staged token

    extern __shared__ uint8_t smem_raw[];
    // Swizzled TMA destinations need 1024-byte alignment (the host adds slack).
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int D = p.depth, CB = p.codes_bytes, MB = p.meta_bytes;
    uint8_t *meta = ring + D * CB;  // per stage: scales/zeros, group sums, activations, descriptor
    unsigned long long *full = reinterpret_cast<unsigned long long *>(meta + D * MB);
    unsigned long long *empty = full + D;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2;  // MMA group id: row (A, C) / token (B)
    const int c = lane & 3;    // quad position: 32-code chunk (A, B) / token pair (C)
    const int gr = box_row<BITS, MT>(gq);  // weight row (mod 8) of MMA row gq
    const int nch = p.n_chunks;

    if (threadIdx.x == 0) {
        for (int i = 0; i < D; ++i) {
            mbar_init(&full[i], 33);  // 32 cp.async arrivals + the producer's arrive(.expect_tx)
            mbar_init(&empty[i], kDecodeWarpsPerCta);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    pdl_wait();  // the prepared activations and the counter come from the prep kernel
    pdl_launch_dependents();

    // ---- producer ----------------------------------------------------------
    // Stage t is filled by warp t % 4, in order: the scheduling state (cursor
    // and chunk) lives in shared memory and is handed from one producing warp
    // to the next through `seq` (the number of stages filled so far).
    ProdState *ps = reinterpret_cast<ProdState *>(empty + D);
    if (threadIdx.x == 0) {
        int b = 0, e = 0;
        if (static_cast<int>(blockIdx.x) < nch) chunk_range(p, blockIdx.x, b, e);
        Cursor cu;
        cursor_init(cu, p, b, e);
        ps->s = cu.s;
        ps->o = cu.o;
        ps->rb = cu.rb;
        ps->j = cu.j;
        ps->valid = cu.valid ? 1 : 0;
        ps->chunk = blockIdx.x;
        ps->begin = b;
        ps->end = e;
        ps->ticket = p.dynamic ? atomicAdd(p.cnt, 1u) : 0u;  // fetched one chunk ahead of its use
        ps->done = 0;
        ps->slot = 0;
        ps->round = 0;
        ps->seq = 0;
    }
    __syncthreads();

    // Fills stage `target` (after its previous contents were released by all
    // warps); false if a wait ran out.  Whole warp, uniform control flow.
    auto produce = [&](int target) -> bool {
        if (!wait_seq(&ps->seq, target, p.wait_ns)) return false;
        Cursor ld;
        ld.s = ps->s;
        ld.o = ps->o;
        ld.rb = ps->rb;
        ld.j = ps->j;
        ld.valid = ps->valid != 0;
        int ld_chunk = ps->chunk, ld_begin = ps->begin, ld_end = ps->end;
        unsigned int ticket = ps->ticket;
        // slot and round of stage `target` (no division by the runtime depth)
        const int slot_ld = ps->slot, round_ld = ps->round;
        const bool wrap = slot_ld + 1 == D;
        if (ps->done) {
            __syncwarp();
            if (lane == 0) {
                ps->slot = wrap ? 0 : slot_ld + 1;
                ps->round = round_ld + (wrap ? 1 : 0);
                st_release_shared(&ps->seq, target + 1);
            }
            return true;
        }
        if (round_ld > 0 && !wait_phase(&empty[slot_ld], (round_ld - 1) & 1, p.wait_ns)) return false;
        if (!ld.valid && p.dynamic) {
            // Chunks only grow, so a CTA stops at its first ticket past the end
            // and never holds an unused valid one.
            const int k = static_cast<int>(gridDim.x + ticket);
            if (k < nch) {
                if (lane == 0) ticket = atomicAdd(p.cnt, 1u);
                ld_chunk = k;
                chunk_range(p, k, ld_begin, ld_end);
                cursor_init(ld, p, ld_begin, ld_end);
            }
        }
        uint8_t *st = ring + slot_ld * CB;
        uint8_t *sm = meta + slot_ld * MB;
        int4 *dsc = reinterpret_cast<int4 *>(sm + p.off_desc);
        int done = 0;
        if (ld.valid) {
            const DecodeOp &op = p.ops[ld.o];
            const int g0 = ld.j * GPS;
            const int ng = min(GPS, op.G - g0);
            const int xrows = MT == 1 ? op.M : MPAD;  // staged token rows
            const int unit_start = ld.s - ld.j;
            int flags = 0;
            const int SU = op.su;
            if (ld.j + 1 == SU || ld.s + 1 == ld_end) flags |= kFlagLast;
            if (unit_start < ld_begin) flags |= kFlagHead;
            if (unit_start + SU > ld_end) flags |= kFlagTail;
            if (op.sz_vec) {
                flags |= kFlagSzVec;
#pragma unroll
                for (int h = 0; h < ROWS / 32; ++h) {
                    const int r = lane + 32 * h;
                    const int rg = min(ld.rb * ROWS + r, op.N - 1);
                    const size_t src = static_cast<size_t>(rg) * op.G + g0;
                    uint8_t *dst = sm + p.off_sz + r * 2 * SZB;
                    if constexpr (SZB == 8) {
                        cp_async8(dst, op.scales + src);
                        cp_async8(dst + 8, op.zeros + src);
                    } else {
                        cp_async4(dst, op.scales + src);
                        cp_async4(dst + 4, op.zeros + src);
                    }
                }
            }
            cp_async_arrive_noinc(&full[slot_ld]);
            fence_proxy_async();  // earlier reads of this slot precede the async-proxy overwrite
            if (lane == 0) {
                dsc[0] = make_int4(ld.o, ld.rb, ld.j, ng | (flags << 8));
                dsc[1] = make_int4(ld_chunk, unit_start, op.M, 0);
                // the step's x' and records for all staged tokens: two
                // contiguous blocks (a last step with ng < GPS groups copies
                // its unused group slots too)
                const uint32_t xbytes = static_cast<uint32_t>(xrows * GPS * 256);
                const uint32_t sbytes = static_cast<uint32_t>(xrows * RS * 16);
                mbar_arrive_expect_tx(&full[slot_ld], NBOX * BOXB + xbytes + sbytes);
#pragma unroll
                for (int b = 0; b < NBOX; ++b)
                    tma_load_2d(st + b * BOXB, &op.tmap, g0 * GB + b * BOXW, ld.rb * ROWS, &full[slot_ld]);
                const size_t blk = static_cast<size_t>(ld.j) * xrows;  // first (step, token) block
                bulk_load(sm + p.off_x, op.xg + blk * (GPS * kGroup), xbytes, &full[slot_ld]);
                bulk_load(sm + p.off_sx, op.sx + blk * (RS * 4), sbytes, &full[slot_ld]);
            }
            __syncwarp();
            cursor_next(ld, p, ld_end);
        } else {
            cp_async_arrive_noinc(&full[slot_ld]);
            if (lane == 0) {
                dsc[0] = make_int4(0, 0, 0, kFlagEnd << 8);
                mbar_arrive(&full[slot_ld]);
            }
            done = 1;
        }
        __syncwarp();
        if (lane == 0) {
            ps->s = ld.s;
            ps->o = ld.o;
            ps->rb = ld.rb;
            ps->j = ld.j;
            ps->valid = ld.valid ? 1 : 0;
            ps->chunk = ld_chunk;
            ps->begin = ld_begin;
            ps->end = ld_end;
            ps->ticket = ticket;
            ps->done = done;
            ps->slot = wrap ? 0 : slot_ld + 1;
            ps->round = round_ld + (wrap ? 1 : 0);
            st_release_shared(&ps->seq, target + 1);
        }
        return true;
    };

    bool aborted = false;
    for (int t = warp; t < D - 1 && !aborted; t += kDecodeWarpsPerCta) aborted = !produce(t);

    // ---- consumers (all warps) ---------------------------------------------
    // Per-lane byte offsets into a stage, fixed for the whole kernel (shared
    // memory is addressed with 32-bit offsets from the stage bases).
    //   codes: the lane's chunk of group gi of row (warp*16*RT + rt*16 +
    //          h*8 + gr) at cofs[rt][h][k] + a compile-time part (RT row tiles
    //          of 16 per warp); with the 128-byte swizzle the
    //          chunk index is ((gi*GB % 128)/16) ^ lanex.
    //   x':    token gq's staged row is GPS*256 bytes, group gi at +gi*256,
    //          the lane's chunk q of it at x_chunk(c, q, gq).
    //   sums:  (sum x, -f * bias, f, 0) of token 8mt + 2c of group gi at
    //          off_sx + ((8mt + 2c) * RS + gi) * 16, token 8mt + 2c + 1
    //          RS * 16 bytes on; lanes of tokens >= M read other bytes of the
    //          stage (their columns are padding).
    int lanex;
    if constexpr (BITS == 4) lanex = c ^ gr;
    else if constexpr (BITS == 2) lanex = (c >> 1) ^ gr;
    else if constexpr (BITS == 16) lanex = 4 * (c & 1);  // fp16: box c >> 1, chunks (lanex + j) ^ gr
    else lanex = (2 * c) ^ gr;  // b = 8: chunks lanex and lanex ^ 1
    uint32_t cofs[RT][2][2];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t crow = (warp * 16 * RT + rt * 16 + h * 8 + gr) * (SWZ ? 128 : BOXW);
            uint32_t(&cf)[2] = cofs[rt][h];
            if constexpr (BITS == 16) {
                cf[0] = cf[1] = crow + (c >> 1) * BOXB;
            } else if constexpr (!SWZ) {
                cf[0] = cf[1] = crow + 4 * BITS * c;
            } else if constexpr (BITS == 4) {
                cf[0] = crow + (lanex << 4);
                cf[1] = crow + ((lanex ^ 4) << 4);
            } else if constexpr (BITS == 8) {
                cf[0] = crow + (lanex << 4);
                cf[1] = crow + ((lanex ^ 1) << 4);
            } else {  // b = 2: group gi at chunk (2gi ^ lanex), half c & 1
                cf[0] = cf[1] = crow + 8 * (c & 1);
            }
        }
    uint32_t xq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) xq[q] = p.off_x + gq * (GPS * 256) + (x_chunk(c, q, gq) << 4);
    const uint32_t sxo = p.off_sx + 2 * c * RS * 16;
    uint32_t szq[RT][2];  // scale/zero words of rows warp*16*RT + rt*16 + h*8 + gr
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) szq[rt][h] = p.off_sz + (warp * 16 * RT + rt * 16 + h * 8 + gr) * 2 * SZB;
    const uint32_t ring_s = smem_u32(ring), meta_s = smem_u32(meta);

    float tot[MT][RT][4];
#pragma unroll
    for (int b = 0; b < MT; ++b)
#pragma unroll
        for (int rt = 0; rt < RT; ++rt)
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[b][rt][i] = 0.0f;
    const uint32_t magic = kMagic;
    // B fragments (activations) of one token tile.  With one tile only the
    // lanes of tokens < M load them; the rest keep stale values (their C
    // columns are never stored), so the fragments live across steps.
    uint32_t xf1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) xf1[i] = 0u;
    int slot = 0, n_seen = 0;  // stages this warp has waited for
    int deferred = -1;         // stage this warp still has to fill
    uint32_t par = 0;

#pragma unroll 1
    while (!aborted) {
        {
            // Stage to fill now, by its warp.  If the previous producer has not
            // handed over yet, consume first and fill it afterwards.
            const int target = n_seen + D - 1;
            if (target % kDecodeWarpsPerCta == warp) {
                if (__all_sync(0xffffffffu, ld_acquire_shared(&ps->seq) == target)) {
                    if (!produce(target)) {
                        aborted = true;
                        break;
                    }
                } else {
                    deferred = target;
                }
            }
        }
        if (!wait_phase(&full[slot], par, p.wait_ns)) {
            aborted = true;
            break;
        }
        const uint32_t z = opaque_zero();  // orders the stage loads after the wait
        const uint32_t stb = ring_s + slot * CB + z, smb = meta_s + slot * MB + z;
        const uint4 d0 = lds_v4(smb + p.off_desc);
        const uint4 d1 = lds_v4(smb + p.off_desc + 16);
        const int flags = static_cast<int>(d0.w) >> 8;
        ++n_seen;
        if (flags & kFlagEnd) {
            if (deferred >= 0 && !produce(deferred)) aborted = true;  // later producers wait for it
            break;
        }
        const int ng = d0.w & 0xFF;
        const int M = static_cast<int>(d1.z);
        const int o = static_cast<int>(d0.x), rb = static_cast<int>(d0.y);

        // Scales and zeros of rows rt*16 + gr and rt*16 + gr + 8 for the GPS groups.
        uint32_t szs[RT][2][(GPS + 1) / 2], szz[RT][2][(GPS + 1) / 2];
        if constexpr (BITS == 16) {
            // fp16 weights: no scales or zeros
        } else if (flags & kFlagSzVec) {
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if constexpr (GPS == 4) {
                        const uint4 v = lds_v4(smb + szq[rt][h]);
                        szs[rt][h][0] = v.x; szs[rt][h][1] = v.y; szz[rt][h][0] = v.z; szz[rt][h][1] = v.w;
                    } else {
                        const uint2 v = lds_v2(smb + szq[rt][h]);
                        szs[rt][h][0] = v.x; szz[rt][h][0] = v.y;
                    }
                }
        } else {
            const DecodeOp &op = p.ops[o];
            const int g0 = static_cast<int>(d0.z) * GPS;
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = min(rb * ROWS + warp * 16 * RT + rt * 16 + h * 8 + gr, op.N - 1);
#pragma unroll
                    for (int i = 0; i < GPS / 2; ++i) {
                        const int ga = min(g0 + 2 * i, op.G - 1), gb = min(g0 + 2 * i + 1, op.G - 1);
                        const size_t ia = static_cast<size_t>(r) * op.G + ga, ib = static_cast<size_t>(r) * op.G + gb;
                        szs[rt][h][i] = ldg_u16_nc(op.scales + ia) | (ldg_u16_nc(op.scales + ib) << 16);
                        szz[rt][h][i] = ldg_u16_nc(op.zeros + ia) | (ldg_u16_nc(op.zeros + ib) << 16);
                    }
                }
        }

        auto group = [&](auto gi_c, auto one_c) {
            constexpr int gi = decltype(gi_c)::value;
            constexpr bool one_token = decltype(one_c)::value;
            // this thread's 32-code chunk of rows rt*16 + gr and rt*16 + gr + 8
            uint32_t wv[RT][2][BITS];
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (BITS == 16) {
                    // fp16 weights: the lane's 32 codes are 64 bytes, 4 chunks
                    // of box c >> 1 (2-way bank conflicts: lanes c and c + 2
                    // read the same chunks of the two boxes)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 v = lds_v4(stb + cofs[rt][h][0] + (((lanex + j) ^ gr) << 4));
                        wv[rt][h][4 * j] = v.x;
                        wv[rt][h][4 * j + 1] = v.y;
                        wv[rt][h][4 * j + 2] = v.z;
                        wv[rt][h][4 * j + 3] = v.w;
                    }
                } else if constexpr (SWZ && BITS == 4) {
                    const uint4 v = lds_v4(stb + cofs[rt][h][gi & 1] + (gi * GB / 128) * BOXB);
                    wv[rt][h][0] = v.x;
                    wv[rt][h][1] = v.y;
                    wv[rt][h][2] = v.z;
                    wv[rt][h][3] = v.w;
                } else if constexpr (SWZ && BITS == 8) {
                    const uint4 v0 = lds_v4(stb + cofs[rt][h][0] + gi * BOXB);
                    const uint4 v1 = lds_v4(stb + cofs[rt][h][1] + gi * BOXB);
                    wv[rt][h][0] = v0.x; wv[rt][h][1] = v0.y; wv[rt][h][2] = v0.z; wv[rt][h][3] = v0.w;
                    wv[rt][h][4] = v1.x; wv[rt][h][5] = v1.y; wv[rt][h][6] = v1.z; wv[rt][h][7] = v1.w;
                } else if constexpr (SWZ) {
                    static_assert(BITS == 2, "swizzled layouts: b = 2, 4, 8");
                    const uint2 v = lds_v2(stb + cofs[rt][h][0] + (((2 * gi) ^ lanex) << 4));
                    wv[rt][h][0] = v.x;
                    wv[rt][h][1] = v.y;
                } else if constexpr (BITS == 2) {
                    const uint2 v = lds_v2(stb + cofs[rt][h][0] + gi * GB);
                    wv[rt][h][0] = v.x;
                    wv[rt][h][1] = v.y;
                } else {
                    static_assert(BITS == 3, "unswizzled layouts: b = 2 (2 groups per step), 3");
                    wv[rt][h][0] = lds_u32(stb + cofs[rt][h][0] + gi * GB);
                    wv[rt][h][1] = lds_u32(stb + cofs[rt][h][0] + gi * GB + 4);
                    wv[rt][h][2] = lds_u32(stb + cofs[rt][h][0] + gi * GB + 8);
                }
            }
            float sc[RT][2], zr[RT][2];
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if constexpr (BITS != 16) {
                        constexpr bool hi = (gi & 1) != 0;
                        sc[rt][h] = half_of<hi>(szs[rt][h][gi / 2]);
                        zr[rt][h] = half_of<hi>(szz[rt][h][gi / 2]);
                    } else {  // fp16 weights: no scale, no zero
                        sc[rt][h] = 1.0f;
                        zr[rt][h] = 0.0f;
                    }
                }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t xfm[16];
                uint32_t (&xf)[16] = MT == 1 ? xf1 : xfm;
                // Several tiles: all MPAD token rows are staged (zeros past M).
                if (MT > 1 || gq < M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = lds_v4(smb + xq[q] + (mt * 8 * GPS + gi) * 256);
                        xf[4 * q + 0] = v.x;
                        xf[4 * q + 1] = v.y;
                        xf[4 * q + 2] = v.z;
                        xf[4 * q + 3] = v.w;
                    }
                }
                const uint4 sa = lds_v4(smb + sxo + (8 * mt * RS + gi) * 16);
                uint4 sb = make_uint4(0u, 0u, 0u, 0u);
                if constexpr (!one_token) sb = lds_v4(smb + sxo + ((8 * mt + 1) * RS + gi) * 16);
                // tot += s * f * (acc - bias) + z * sum(x): the z * sum(x) term
                // first (it needs no MMA result, and its operands die early),
                // then s * f * (acc - bias) with f * (acc - bias) as one FMA (f
                // is the token's power-of-two x' scale); with one token the odd
                // C columns are padding.  The B fragments serve every row tile.
#pragma unroll
                for (int rt = 0; rt < RT; ++rt) {
                    float(&tt)[4] = tot[mt][rt];
#pragma unroll
                    for (int h = 0; h < 2; ++h) tt[2 * h] = fmaf(zr[rt][h], __uint_as_float(sa.x), tt[2 * h]);
                    if constexpr (!one_token) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) tt[2 * h + 1] = fmaf(zr[rt][h], __uint_as_float(sb.x), tt[2 * h + 1]);
                    }
                    float acc[4];
                    mma_group<BITS>(acc, wv[rt], xf, magic);
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tt[2 * h] = fmaf(sc[rt][h], fmaf(acc[2 * h], __uint_as_float(sa.z), __uint_as_float(sa.y)),
                                         tt[2 * h]);
                    if constexpr (!one_token) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tt[2 * h + 1] = fmaf(
                                sc[rt][h], fmaf(acc[2 * h + 1], __uint_as_float(sb.z), __uint_as_float(sb.y)),
                                tt[2 * h + 1]);
                    }
                }
            }
        };
        auto groups = [&](auto one_c) {
            if (ng == GPS) {
                static_for<GPS>([&](auto gi_c) { group(gi_c, one_c); });
            } else {
                static_for<GPS>([&](auto gi_c) {
                    constexpr int gv = decltype(gi_c)::value;
                    if (gv < ng) group(gi_c, one_c);
                });
            }
        };
        if (MT == 1 && M == 1) groups(std::true_type{});
        else groups(std::false_type{});

        // Release the stage.
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == D) {
            slot = 0;
            par ^= 1u;
        }
        if (deferred >= 0) {
            const bool ok = produce(deferred);
            deferred = -1;
            if (!ok) {
                aborted = true;
                break;
            }
        }

        if (flags & kFlagLast) {
            // End of this chunk's piece of a row block: emit.
            const DecodeOp &op = p.ops[o];
            const int r0 = rb * ROWS;
            if (!(flags & (kFlagHead | kFlagTail))) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int row = r0 + warp * 16 * RT + rt * 16 + (i >> 1) * 8 + gr;
                            const int tok = 8 * mt + 2 * c + (i & 1);
                            if (row < op.N && tok < M) {
                                const size_t at = static_cast<size_t>(tok) * op.N + row;
                                if (op.out32) op.out32[at] = tot[mt][rt][i];
                                else op.out[at] = round_out(tot[mt][rt][i], op.out_bf16);
                            }
                        }
            } else {
                // Partial piece: slot (k, 0) holds chunk k's head piece, (k, 1) its tail piece.
                const int chunk = d1.x, unit_start = d1.y;
                float *slot_p = p.part + (static_cast<size_t>(chunk) * 2 + ((flags & kFlagHead) ? 0 : 1)) * p.slot_floats;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rl = warp * 16 * RT + rt * 16 + (i >> 1) * 8 + gr;
                            const int tok = 8 * mt + 2 * c + (i & 1);
                            if (tok < M) slot_p[rl * M + tok] = tot[mt][rt][i];
                        }
                const int w_first = unit_start >> p.log2c;               // chunks holding the
                const int w_last = (unit_start + op.su - 1) >> p.log2c;   // pieces of this row block
                __threadfence();
                __syncwarp();
                unsigned int prev = 0;
                if (lane == 0) prev = atomicAdd(p.cnt + 1 + w_first, 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == static_cast<unsigned int>(kDecodeWarpsPerCta * (w_last - w_first + 1) - 1)) {
                    // Last piece in: sum the pieces in chunk order (deterministic).
                    __threadfence();
                    for (int idx = lane; idx < ROWS * M; idx += 32) {
                        float sum = __ldcg(p.part + (static_cast<size_t>(w_first) * 2 + 1) * p.slot_floats + idx);
                        for (int ww = w_first + 1; ww <= w_last; ++ww)
                            sum += __ldcg(p.part + static_cast<size_t>(ww) * 2 * p.slot_floats + idx);
                        const int row = idx / M, tok = idx - row * M;
                        if (r0 + row < op.N) {
                            const size_t at = static_cast<size_t>(tok) * op.N + r0 + row;
                            if (op.out32) op.out32[at] = sum;
                            else op.out[at] = round_out(sum, op.out_bf16);
                        }
                    }
                    if (lane == 0) p.cnt[1 + w_first] = 0u;  // ready for the next call
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) tot[mt][rt][i] = 0.0f;
        }
    }

    if (aborted && lane == 0) atomicExch(&g_decode_error, 5);  // ZQ_ERR_TIMEOUT
    // Copies still in flight (only after an abort) must land before the CTA
    // can exit: every warp waits, bounded, for each stage filled so far that
    // it did not wait for itself.
    if (aborted) {
        const int filled = ld_acquire_shared(&ps->seq);
        for (int k = n_seen; k < filled; ++k) {
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(&full[k % D], (k / D) & 1u) && globaltimer() - t0 < kDecodeDrainNs) {
            }
        }
    }
}

// ------------------------------------------------------------------ host --

cudaError_t read_decode_error(int *err) {
    cudaError_t e = cudaMemcpyFromSymbol(err, g_decode_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(int));
}

template <class PP>
static cudaError_t launch_prep_t(const PP &p, long long total_warps, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((total_warps + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prep_kernel<PP>, p, total_warps);
}
cudaError_t launch_prep(const PrepParams &p, long long total_warps, cudaStream_t stream) {
    return launch_prep_t(p, total_warps, stream);
}
cudaError_t launch_prep(const PrepParamsSmall &p, long long total_warps, cudaStream_t stream) {
    return launch_prep_t(p, total_warps, stream);
}

constexpr int kDecodeMaxSmem = 227 * 1024;

template <int BITS, int MT, class DP>
static cudaError_t set_smem_t() {
    static bool configured = false;  // benign race: the attribute call is idempotent
    if (configured) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS, MT, DP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDecodeMaxSmem);
    if (e == cudaSuccess) configured = true;
    return e;
}

template <int BITS, int MT, class DP>
static cudaError_t launch_decode_t(const DP &p, int n_ctas, size_t smem, cudaStream_t stream) {
    cudaError_t e = set_smem_t<BITS, MT, DP>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_ctas));
    cfg.blockDim = dim3(kDecodeWarpsPerCta * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, MT, DP>, p);
}

template <int BITS, int MT>
static cudaError_t occupancy_t(size_t smem, int *ctas) {
    cudaError_t e = set_smem_t<BITS, MT, DecodeParams>();
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, decode_kernel<BITS, MT, DecodeParams>,
                                                         kDecodeWarpsPerCta * 32, smem);
}

#define ZQ_DISPATCH_BITS_MT(FN, ...)                                   \
    switch (bits * 16 + mt) {                                          \
        case 2 * 16 + 1: return FN<2, 1>(__VA_ARGS__);                 \
        case 2 * 16 + 2: return FN<2, 2>(__VA_ARGS__);                 \
        case 2 * 16 + 4: return FN<2, 4>(__VA_ARGS__);                 \
        case 3 * 16 + 1: return FN<3, 1>(__VA_ARGS__);                 \
        case 3 * 16 + 2: return FN<3, 2>(__VA_ARGS__);                 \
        case 3 * 16 + 4: return FN<3, 4>(__VA_ARGS__);                 \
        case 4 * 16 + 1: return FN<4, 1>(__VA_ARGS__);                 \
        case 4 * 16 + 2: return FN<4, 2>(__VA_ARGS__);                 \
        case 4 * 16 + 4: return FN<4, 4>(__VA_ARGS__);                 \
        case 8 * 16 + 1: return FN<8, 1>(__VA_ARGS__);                 \
        case 8 * 16 + 2: return FN<8, 2>(__VA_ARGS__);                 \
        case 8 * 16 + 4: return FN<8, 4>(__VA_ARGS__);                 \
        case 16 * 16 + 1: return FN<16, 1>(__VA_ARGS__);               \
        case 16 * 16 + 2: return FN<16, 2>(__VA_ARGS__);               \
        case 16 * 16 + 4: return FN<16, 4>(__VA_ARGS__);               \
        default: return cudaErrorInvalidValue;                         \
    }

cudaError_t launch_decode(const DecodeParams &p, int bits, int mt, int n_ctas, size_t smem, cudaStream_t stream) {
    ZQ_DISPATCH_BITS_MT(launch_decode_t, p, n_ctas, smem, stream)
}
cudaError_t launch_decode(const DecodeParamsSmall &p, int bits, int mt, int n_ctas, size_t smem,
                          cudaStream_t stream) {
    ZQ_DISPATCH_BITS_MT(launch_decode_t, p, n_ctas, smem, stream)
}

cudaError_t decode_ctas_per_sm(int bits, int mt, size_t smem, int *ctas) {
    ZQ_DISPATCH_BITS_MT(occupancy_t, smem, ctas)
}

}  // namespace zq
