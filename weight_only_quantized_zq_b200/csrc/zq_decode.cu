// zq_decode.cu — decode family (M <= 64): skinny tensor-core GEMM that streams
// the packed weights exactly once.
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
//    2^-s (exact), so each product is 1024 * x' + q * x, and the per-group bias
//    1024 * sum(x') is subtracted in fp32 once per group.  The canonical packed
//    layout is consumed as stored.
//  * Packed codes stream through a per-warp shared-memory ring with cp.async
//    (16-byte chunks, several steps in flight, no register cost); the ring is
//    per warp, so no block-level barrier is needed.
//  * A persistent grid covers every SM.  The steps (op, row block, group) of
//    all ops of a launch are cut into one contiguous range per warp (stream-K),
//    so a whole stack of layers runs as one balanced launch and a small layer
//    is split along K; a row block cut by a warp boundary is reduced by the
//    last warp to finish it, in warp order, so results are deterministic.
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
// One warp per (entry, padded token, group): writes the pair-permuted copy of
// x and the fp32 group sum.  Tokens >= M are written as zeros.

template <int B>
__device__ __forceinline__ float prep_group(const uint16_t *xrow, uint16_t *prow, int lane) {
    float bias = 0.0f;  // sum of the scaled activations written by this lane
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int q = lane + 32 * h;  // 64 pairs per group
        const int c = q / 16, p = q % 16;
        const float sc = 1.0f / static_cast<float>(1 << pair_shift<B>(p));  // exact power of two
        const __half lo = __float2half_rn(h2f_bits(xrow[32 * c + pair_lo<B>(p)]) * sc);
        const __half hi = __float2half_rn(h2f_bits(xrow[32 * c + pair_hi<B>(p)]) * sc);
        bias += __half2float(lo) + __half2float(hi);
        reinterpret_cast<uint32_t *>(prow)[16 * c + p] = __half_as_ushort(lo) | (__half_as_ushort(hi) << 16);
    }
    return bias;
}

__global__ void __launch_bounds__(256) prep_kernel(const __grid_constant__ PrepParams p,
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
        uint16_t *prow = en.xperm + static_cast<size_t>(t) * en.K + static_cast<size_t>(g) * kGroup;
        float2 *dst = reinterpret_cast<float2 *>(en.sx) + static_cast<size_t>(g) * en.M_pad + t;
        if (t >= en.M) {
            reinterpret_cast<uint2 *>(prow)[lane] = make_uint2(0u, 0u);
            if (lane == 0) *dst = make_float2(0.0f, 0.0f);
        } else {
            const uint16_t *xrow = en.x + static_cast<size_t>(t) * en.K + static_cast<size_t>(g) * kGroup;
            const uint2 v = reinterpret_cast<const uint2 *>(xrow)[lane];
            float s = h2f_bits(v.x & 0xFFFFu) + h2f_bits(v.x >> 16) + h2f_bits(v.y & 0xFFFFu) +
                      h2f_bits(v.y >> 16);
            float b;
            switch (en.bits) {
                case 2: b = prep_group<2>(xrow, prow, lane); break;
                case 3: b = prep_group<3>(xrow, prow, lane); break;
                case 4: b = prep_group<4>(xrow, prow, lane); break;
                default: b = prep_group<8>(xrow, prow, lane); break;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                b += __shfl_xor_sync(0xffffffffu, b, o);
            }
            if (lane == 0) *dst = make_float2(s, 1024.0f * b);
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
    int SU, RB;    // steps per row block and row blocks of op o
    bool valid;
};

__device__ __forceinline__ void cursor_init(Cursor &cu, const DecodeParams &p, int s, int s_end) {
    cu.s = s;
    cu.valid = s < s_end;
    int lo = 0, hi = p.n_ops - 1;  // last op with step0 <= s
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.ops[mid].step0 <= s) lo = mid;
        else hi = mid - 1;
    }
    const int o = lo;
    const int local = s - static_cast<int>(p.ops[o].step0);
    cu.o = o;
    cu.SU = p.ops[o].su;
    cu.RB = p.ops[o].row_blocks;
    cu.rb = local / cu.SU;
    cu.j = local - cu.rb * cu.SU;
}

__device__ __forceinline__ void cursor_next(Cursor &cu, const DecodeParams &p, int s_end) {
    ++cu.s;
    cu.valid = cu.s < s_end;
    if (++cu.j == cu.SU) {
        cu.j = 0;
        if (++cu.rb == cu.RB) {
            cu.rb = 0;
            if (cu.o + 1 < p.n_ops) {
                ++cu.o;
                cu.SU = p.ops[cu.o].su;
                cu.RB = p.ops[cu.o].row_blocks;
            }
        }
    }
}

// Warp whose step range contains step s (ranges are [T*w/W, T*(w+1)/W)).
__device__ __forceinline__ int warp_of(long long s, long long W, long long T) {
    return static_cast<int>(((s + 1) * W - 1) / T);
}

// Scales and zeros of rows (gq, gq + 8) for the GPS groups of a step, packed as
// fp16 pairs: sz[h][i] holds groups (2i, 2i+1) of row half h; [2 + ...] zeros.
template <int GPS>
__device__ __forceinline__ void load_scale_zero(uint32_t (&sz)[2][GPS], const DecodeOp &op, int r0, int g0,
                                                int gq) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = min(r0 + h * 8 + gq, op.N - 1);
        const size_t idx = static_cast<size_t>(r) * op.G + g0;
        if (((r * op.G + g0) % GPS) == 0 && g0 + GPS <= op.G) {
            if constexpr (GPS == 4) {
                const uint2 s2 = *reinterpret_cast<const uint2 *>(op.scales + idx);
                const uint2 z2 = *reinterpret_cast<const uint2 *>(op.zeros + idx);
                sz[h][0] = s2.x;
                sz[h][1] = s2.y;
                sz[h][2] = z2.x;
                sz[h][3] = z2.y;
            } else {
                sz[h][0] = *reinterpret_cast<const uint32_t *>(op.scales + idx);
                sz[h][1] = *reinterpret_cast<const uint32_t *>(op.zeros + idx);
            }
        } else {
#pragma unroll
            for (int i = 0; i < GPS / 2; ++i) {
                const int ga = min(g0 + 2 * i, op.G - 1), gb = min(g0 + 2 * i + 1, op.G - 1);
                const size_t ia = static_cast<size_t>(r) * op.G + ga, ib = static_cast<size_t>(r) * op.G + gb;
                sz[h][i] = ldg_u16_nc(op.scales + ia) | (ldg_u16_nc(op.scales + ib) << 16);
                sz[h][GPS / 2 + i] = ldg_u16_nc(op.zeros + ia) | (ldg_u16_nc(op.zeros + ib) << 16);
            }
        }
    }
}

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

// One group (16 rows x 128 k) into acc.  With SPLIT the even and odd k-steps
// run as two independent accumulator chains, halving the dependent MMA
// latency; worth its four registers only when few token tiles are live.
template <int BITS, bool SPLIT>
__device__ __forceinline__ void mma_group(float (&acc)[4], const uint32_t (&w)[2][BITS], const uint32_t (&xf)[16],
                                          uint32_t magic) {
    if constexpr (SPLIT) {
        float acc2[4];
        mma_j<BITS, 0, true>(acc, w, xf, magic);
        mma_j<BITS, 1, true>(acc2, w, xf, magic);
        mma_j<BITS, 2, false>(acc, w, xf, magic);
        mma_j<BITS, 3, false>(acc2, w, xf, magic);
        mma_j<BITS, 4, false>(acc, w, xf, magic);
        mma_j<BITS, 5, false>(acc2, w, xf, magic);
        mma_j<BITS, 6, false>(acc, w, xf, magic);
        mma_j<BITS, 7, false>(acc2, w, xf, magic);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += acc2[i];
    } else {
        mma_j<BITS, 0, true>(acc, w, xf, magic);
        mma_j<BITS, 1, false>(acc, w, xf, magic);
        mma_j<BITS, 2, false>(acc, w, xf, magic);
        mma_j<BITS, 3, false>(acc, w, xf, magic);
        mma_j<BITS, 4, false>(acc, w, xf, magic);
        mma_j<BITS, 5, false>(acc, w, xf, magic);
        mma_j<BITS, 6, false>(acc, w, xf, magic);
        mma_j<BITS, 7, false>(acc, w, xf, magic);
    }
}

// Device record of a decode kernel that gave up a bounded wait (ZQ_ERR_TIMEOUT).
__device__ int g_decode_error;

constexpr unsigned long long kDecodeWaitNs = 2000000000ull;  // 2 s

template <int BITS, int MT>
__global__ void __launch_bounds__(kDecodeWarpsPerCta * 32, MT == 1 ? 4 : 2)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int ROWS = 16;
    constexpr int GPS = decode_gps(BITS);
    constexpr int GB = 16 * BITS;                 // bytes of one row of one group
    constexpr int SEG = decode_seg(BITS);         // bytes of one row per step
    constexpr int CODES = ROWS * SEG;             // TMA box bytes
    constexpr int STAGE = decode_stage(BITS);
    constexpr int D = decode_depth(BITS);
    constexpr int MPAD = 8 * MT;
    constexpr int SZB = 2 * GPS;                  // bytes of scales (or zeros) of one row per step

    extern __shared__ __align__(128) uint8_t smem_raw[];
    // TMA destinations: 128-byte aligned (the host adds 128 bytes of slack).
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2;  // MMA group id: row (A, C) / token (B)
    const int c = lane & 3;    // quad position: 32-code chunk (A, B) / token pair (C)
    uint8_t *ring = smem + warp * D * STAGE;
    unsigned long long *bars =
        reinterpret_cast<unsigned long long *>(smem + kDecodeWarpsPerCta * D * STAGE) + warp * D;

    // Work is cut into chunks of C = 2^log2c consecutive steps.  Warp w starts
    // with chunk w; in dynamic mode it then takes chunks W, W+1, ... from a
    // counter (reset by the prep kernel), so faster SMs take more of them.  A
    // row block cut by chunk boundaries is summed from per-chunk partial slots
    // by the last piece to finish.
    const int T = static_cast<int>(p.total_steps);
    const int log2c = p.log2c;
    const int nch = p.n_chunks;
    const int W = gridDim.x * kDecodeWarpsPerCta;
    const int gw = blockIdx.x * kDecodeWarpsPerCta + warp;

    if (lane == 0)
        for (int i = 0; i < D; ++i) mbar_init(&bars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();

    int cs_chunk = gw;  // chunk being computed
    int cs_end = min((cs_chunk + 1) << log2c, T);
    Cursor cs;
    cursor_init(cs, p, gw < nch ? gw << log2c : T, gw < nch ? cs_end : 0);
    Cursor ld = cs;
    int ld_end = cs_end;
    int pend = -1;          // chunk taken by the loader, not yet reached by the consumer
    bool need_take = false; // the loader ran out of its chunk
    bool may_take = false;  // the counter may be read (after the PDL wait)
    // Loader: codes of 16 rows x GPS groups by one TMA (out-of-range rows and
    // groups read as zeros), then scales and zeros by one cp.async per lane.
    auto issue = [&](const Cursor &cu, int slot) {
        const DecodeOp &op = p.ops[cu.o];
        const int g0 = cu.j * GPS;
        const int r0 = cu.rb * ROWS;
        uint8_t *st = ring + slot * STAGE;
        if (lane == 0) {
            fence_proxy_async();  // the warp's reads of this slot precede the overwrite
            mbar_arrive_expect_tx(&bars[slot], CODES);
            tma_load_2d(st, &op.tmap, g0 * GB, r0, &bars[slot]);
        }
        if (op.sz_vec) {
            const int row = lane >> 1;
            const int r = min(r0 + row, op.N - 1);
            const uint16_t *src = ((lane & 1) ? op.zeros : op.scales) + static_cast<size_t>(r) * op.G + g0;
            if constexpr (SZB == 8)
                cp_async8(st + CODES + lane * 8, src);
            else
                cp_async4(st + CODES + lane * SZB, src);
        }
    };

    // Loader cursor: advance; at the end of its chunk take the next one
    // (dynamic mode, once the counter may be read).
    auto ld_advance = [&]() {
        cursor_next(ld, p, ld_end);
        if (!ld.valid && p.dynamic) need_take = true;
    };
    auto ld_take = [&]() {
        if (!need_take || !may_take) return;
        need_take = false;
        int k = 0;
        if (lane == 0) k = W + static_cast<int>(atomicAdd(p.cnt, 1u));
        k = __shfl_sync(0xffffffffu, k, 0);
        if (k < nch) {
            pend = k;
            ld_end = min((k + 1) << log2c, T);
            cursor_init(ld, p, k << log2c, ld_end);
        }
    };

    // Prologue: weights do not depend on the previous kernel; start them now.
    int slot_ld = 0, slot_cs = 0;
    uint32_t par_cs = 0;          // parity of the next phase of slot_cs
    int n_issued = 0, n_consumed = 0;
#pragma unroll 1
    for (int i = 0; i < D - 1; ++i) {
        if (ld.valid) {
            issue(ld, slot_ld);
            ld_advance();
            ++n_issued;
        }
        cp_async_commit();
        slot_ld = slot_ld + 1 == D ? 0 : slot_ld + 1;
    }
    pdl_wait();  // the prepared activations come from the previous kernel
    pdl_launch_dependents();
    may_take = true;

    float tot[MT][4];
#pragma unroll
    for (int b = 0; b < MT; ++b)
#pragma unroll
        for (int i = 0; i < 4; ++i) tot[b][i] = 0.0f;
    const uint32_t magic = kMagic;
    bool aborted = false;

#pragma unroll 1
    while (cs.valid && !aborted) {
        __syncwarp();
        ld_take();
        if (ld.valid) {
            issue(ld, slot_ld);
            ld_advance();
            ++n_issued;
        }
        cp_async_commit();
        slot_ld = slot_ld + 1 == D ? 0 : slot_ld + 1;

        const DecodeOp &op = p.ops[cs.o];
        const int r0 = cs.rb * ROWS;
        const int g0 = cs.j * GPS;
        const int ng = min(GPS, op.G - g0);

        // Per-step bases of the activation fragments and group sums; the
        // groups of the step are at immediate offsets from them.
        const uint16_t *xb[MT];
        const float *sbb[MT];
        bool xon[MT], sbon[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int tok = 8 * mt + gq;
            xon[mt] = tok < op.M;
            sbon[mt] = 8 * mt + 2 * c < op.M;
            xb[mt] = op.xperm + static_cast<size_t>(xon[mt] ? tok : 0) * op.K + static_cast<size_t>(g0) * kGroup + 32 * c;
            sbb[mt] = op.sx + 2 * (static_cast<size_t>(g0) * MPAD + 8 * mt + 2 * c);
        }
        const bool one_token = op.M == 1;
        // Activation fragments, ping-pong by group parity; group 0 is loaded
        // before the waits, group gi + 1 while group gi computes.
        uint32_t xf[2][MT][16];
        auto load_x = [&](uint32_t (&dst)[MT][16], int gi) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                if (xon[mt]) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 w = ldg_u4(xb[mt] + gi * kGroup + 8 * q);
                        dst[mt][4 * q + 0] = w.x;
                        dst[mt][4 * q + 1] = w.y;
                        dst[mt][4 * q + 2] = w.z;
                        dst[mt][4 * q + 3] = w.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) dst[mt][q] = 0u;
                }
            }
        };
        load_x(xf[0], 0);

        // Wait for this step's codes (TMA, bounded) and scales/zeros (cp.async).
        {
            bool ok = mbar_try_wait(&bars[slot_cs], par_cs);
            if (!ok) {
                const unsigned long long t0 = globaltimer();
                while (!(ok = mbar_try_wait(&bars[slot_cs], par_cs)))
                    if (globaltimer() - t0 > kDecodeWaitNs) break;
            }
            if (!ok) {
                if (lane == 0) atomicExch(&g_decode_error, 5);  // ZQ_ERR_TIMEOUT
                aborted = true;
                break;
            }
        }
        cp_async_wait<D - 1>();
        __syncwarp();
        const uint8_t *st = ring + slot_cs * STAGE;
        ++n_consumed;
        if (++slot_cs == D) {
            slot_cs = 0;
            par_cs ^= 1u;
        }

        // Scales and zeros of rows gq and gq + 8 for the GPS groups.
        uint32_t szs[2][GPS / 2], szz[2][GPS / 2];
        if (op.sz_vec) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = h * 8 + gq;
                if constexpr (GPS == 4) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(st + CODES + row * 16);
                    szs[h][0] = v.x;
                    szs[h][1] = v.y;
                    szz[h][0] = v.z;
                    szz[h][1] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2 *>(st + CODES + row * 8);
                    szs[h][0] = v.x;
                    szz[h][0] = v.y;
                }
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = min(r0 + h * 8 + gq, op.N - 1);
#pragma unroll
                for (int i = 0; i < GPS / 2; ++i) {
                    const int ga = min(g0 + 2 * i, op.G - 1), gb = min(g0 + 2 * i + 1, op.G - 1);
                    const size_t ia = static_cast<size_t>(r) * op.G + ga, ib = static_cast<size_t>(r) * op.G + gb;
                    szs[h][i] = ldg_u16_nc(op.scales + ia) | (ldg_u16_nc(op.scales + ib) << 16);
                    szz[h][i] = ldg_u16_nc(op.zeros + ia) | (ldg_u16_nc(op.zeros + ib) << 16);
                }
            }
        }

        auto group = [&](auto gi_c) {
            constexpr int gi = decltype(gi_c)::value;
            // next group's activation fragments, one group ahead
            if (gi + 1 < GPS) load_x(xf[(gi + 1) & 1], gi + 1);
            // this thread's 32-code chunk of rows gq and gq + 8 (dense rows of SEG bytes)
            uint32_t wv[2][BITS];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint8_t *rp = st + (h * 8 + gq) * SEG + gi * GB;
                if constexpr (BITS == 2) {
                    const uint2 v = *reinterpret_cast<const uint2 *>(rp + 8 * c);
                    wv[h][0] = v.x;
                    wv[h][1] = v.y;
                } else if constexpr (BITS == 3) {
                    const uint32_t *q = reinterpret_cast<const uint32_t *>(rp + 12 * c);
                    wv[h][0] = q[0];
                    wv[h][1] = q[1];
                    wv[h][2] = q[2];
                } else if constexpr (BITS == 4) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(rp + 16 * c);
                    wv[h][0] = v.x;
                    wv[h][1] = v.y;
                    wv[h][2] = v.z;
                    wv[h][3] = v.w;
                } else {
                    const uint4 v0 = *reinterpret_cast<const uint4 *>(rp + 32 * c);
                    const uint4 v1 = *reinterpret_cast<const uint4 *>(rp + 32 * c + 16);
                    wv[h][0] = v0.x; wv[h][1] = v0.y; wv[h][2] = v0.z; wv[h][3] = v0.w;
                    wv[h][4] = v1.x; wv[h][5] = v1.y; wv[h][6] = v1.z; wv[h][7] = v1.w;
                }
            }
            constexpr int hi = gi & 1;
            const float sc[2] = {h2f_bits(hi ? (szs[0][gi / 2] >> 16) : (szs[0][gi / 2] & 0xFFFFu)),
                                 h2f_bits(hi ? (szs[1][gi / 2] >> 16) : (szs[1][gi / 2] & 0xFFFFu))};
            const float zr[2] = {h2f_bits(hi ? (szz[0][gi / 2] >> 16) : (szz[0][gi / 2] & 0xFFFFu)),
                                 h2f_bits(hi ? (szz[1][gi / 2] >> 16) : (szz[1][gi / 2] & 0xFFFFu))};
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const float4 sb = sbon[mt] ? *reinterpret_cast<const float4 *>(sbb[mt] + gi * 2 * MPAD)
                                           : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                float acc[4];
                mma_group<BITS, MT == 1>(acc, wv, xf[gi & 1][mt], magic);
                // tot += s * (acc - bias) + z * sum(x); with one token the odd
                // C columns are padding.
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    tot[mt][2 * h] = fmaf(sc[h], acc[2 * h] - sb.y, fmaf(zr[h], sb.x, tot[mt][2 * h]));
                if (MT > 1 || !one_token) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tot[mt][2 * h + 1] = fmaf(sc[h], acc[2 * h + 1] - sb.w, fmaf(zr[h], sb.z, tot[mt][2 * h + 1]));
                }
            }
        };
        if (ng == GPS) {
            static_for<GPS>(group);
        } else {
            static_for<GPS>([&](auto gi_c) {
                constexpr int gv = decltype(gi_c)::value;
                if (gv < ng) group(gi_c);
            });
        }

        if (cs.j + 1 == cs.SU || cs.s + 1 == cs_end) {
            // End of this chunk's piece of a row block: emit.
            const int unit_start = cs.s - cs.j;
            const bool head = unit_start < (cs_chunk << log2c);  // started in an earlier chunk
            const bool tail = unit_start + cs.SU > cs_end;      // continues in a later chunk
            if (!head && !tail) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = r0 + (i >> 1) * 8 + gq;
                        const int tok = 8 * mt + 2 * c + (i & 1);
                        if (row < op.N && tok < op.M)
                            op.out[static_cast<size_t>(tok) * op.N + row] =
                                __half_as_ushort(__float2half_rn(tot[mt][i]));
                    }
            } else {
                // Partial piece: slot (k, 0) holds chunk k's head piece, (k, 1) its tail piece.
                float *slot = p.part + (static_cast<size_t>(cs_chunk) * 2 + (head ? 0 : 1)) * p.slot_floats;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int row = (i >> 1) * 8 + gq;
                        const int tok = 8 * mt + 2 * c + (i & 1);
                        if (tok < op.M) slot[row * op.M + tok] = tot[mt][i];
                    }
                const int w_first = unit_start >> log2c;                 // chunks holding the
                const int w_last = (unit_start + cs.SU - 1) >> log2c;    // pieces of this row block
                __threadfence();
                __syncwarp();
                unsigned int prev = 0;
                if (lane == 0) prev = atomicAdd(p.cnt + 1 + w_first, 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == static_cast<unsigned int>(w_last - w_first)) {
                    // Last piece in: sum the pieces in warp order (deterministic).
                    __threadfence();
                    for (int idx = lane; idx < ROWS * op.M; idx += 32) {
                        float sum = __ldcg(p.part + (static_cast<size_t>(w_first) * 2 + 1) * p.slot_floats + idx);
                        for (int ww = w_first + 1; ww <= w_last; ++ww)
                            sum += __ldcg(p.part + static_cast<size_t>(ww) * 2 * p.slot_floats + idx);
                        const int row = idx / op.M, tok = idx - row * op.M;
                        if (r0 + row < op.N)
                            op.out[static_cast<size_t>(tok) * op.N + r0 + row] =
                                __half_as_ushort(__float2half_rn(sum));
                    }
                    if (lane == 0) p.cnt[1 + w_first] = 0u;  // ready for the next call
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) tot[mt][i] = 0.0f;
        }
        if (cs.s + 1 == cs_end) {
            // chunk done: continue with the chunk the loader took, if any
            if (pend >= 0) {
                cs_chunk = pend;
                pend = -1;
                cs_end = min((cs_chunk + 1) << log2c, T);
                cursor_init(cs, p, cs_chunk << log2c, cs_end);
            } else {
                cs.valid = false;
            }
        } else {
            cursor_next(cs, p, cs_end);
        }
    }
    // Copies still in flight (only after an abort) must land before the CTA
    // can exit: wait for every issued, unconsumed stage, bounded.
    cp_async_wait<0>();
    for (int k = n_consumed; k < n_issued; ++k) {
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(&bars[k % D], (k / D) & 1u) && globaltimer() - t0 < kDecodeWaitNs) {
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

cudaError_t launch_prep(const PrepParams &p, long long total_warps, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((total_warps + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prep_kernel, p, total_warps);
}

template <int BITS, int MT>
static cudaError_t launch_decode_t(const DecodeParams &p, int n_ctas, cudaStream_t stream) {
    const size_t smem = decode_smem_bytes(BITS, MT);
    static bool configured = false;  // benign race: the attribute call is idempotent
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS, MT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured = true;
    }
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
    return cudaLaunchKernelEx(&cfg, decode_kernel<BITS, MT>, p);
}

template <int BITS, int MT>
static cudaError_t occupancy_t(int *ctas) {
    const size_t smem = decode_smem_bytes(BITS, MT);
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<BITS, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, decode_kernel<BITS, MT>,
                                                         kDecodeWarpsPerCta * 32, smem);
}

#define ZQ_DISPATCH_BITS_MT(FN, ...)                                   \
    switch (bits * 16 + mt) {                                          \
        case 2 * 16 + 1: return FN<2, 1>(__VA_ARGS__);                 \
        case 2 * 16 + 2: return FN<2, 2>(__VA_ARGS__);                 \
        case 2 * 16 + 4: return FN<2, 4>(__VA_ARGS__);                 \
        case 2 * 16 + 8: return FN<2, 8>(__VA_ARGS__);                 \
        case 3 * 16 + 1: return FN<3, 1>(__VA_ARGS__);                 \
        case 3 * 16 + 2: return FN<3, 2>(__VA_ARGS__);                 \
        case 3 * 16 + 4: return FN<3, 4>(__VA_ARGS__);                 \
        case 3 * 16 + 8: return FN<3, 8>(__VA_ARGS__);                 \
        case 4 * 16 + 1: return FN<4, 1>(__VA_ARGS__);                 \
        case 4 * 16 + 2: return FN<4, 2>(__VA_ARGS__);                 \
        case 4 * 16 + 4: return FN<4, 4>(__VA_ARGS__);                 \
        case 4 * 16 + 8: return FN<4, 8>(__VA_ARGS__);                 \
        case 8 * 16 + 1: return FN<8, 1>(__VA_ARGS__);                 \
        case 8 * 16 + 2: return FN<8, 2>(__VA_ARGS__);                 \
        case 8 * 16 + 4: return FN<8, 4>(__VA_ARGS__);                 \
        case 8 * 16 + 8: return FN<8, 8>(__VA_ARGS__);                 \
        default: return cudaErrorInvalidValue;                         \
    }

cudaError_t launch_decode(const DecodeParams &p, int bits, int mt, int n_ctas, cudaStream_t stream) {
    ZQ_DISPATCH_BITS_MT(launch_decode_t, p, n_ctas, stream)
}

cudaError_t decode_ctas_per_sm(int bits, int mt, int *ctas) { ZQ_DISPATCH_BITS_MT(occupancy_t, ctas) }

}  // namespace zq
