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
//  * A persistent grid covers every SM; work units (op, row block, K slice) are
//    spread over warps by byte cost, so a whole stack of layers runs as one
//    launch and a single small layer is split along K (partials reduced by the
//    last-arriving warp in a fixed order, so results are deterministic).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zq_device.cuh"
#include "zq_internal.h"

namespace zq {

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
    int o, u, g, g_end, r0, rb, slice;
    bool valid;
};

template <int ROWS>
__device__ __forceinline__ void cursor_unit(Cursor &cu, const DecodeParams &p, long long c_end) {
    while (cu.o < p.n_ops && cu.u >= p.ops[cu.o].row_blocks * p.ops[cu.o].S) {
        ++cu.o;
        cu.u = 0;
    }
    cu.valid = false;
    if (cu.o >= p.n_ops) return;
    const DecodeOp &op = p.ops[cu.o];
    if (op.cost0 + static_cast<long long>(cu.u) * op.unit_cost >= c_end) return;
    cu.rb = cu.u / op.S;
    cu.slice = cu.u - cu.rb * op.S;
    cu.r0 = cu.rb * ROWS;
    cu.g = cu.slice * op.gps;
    cu.g_end = min(op.G, cu.g + op.gps);
    cu.valid = true;
}

template <int ROWS>
__device__ __forceinline__ void cursor_next(Cursor &cu, const DecodeParams &p, long long c_end) {
    if (++cu.g == cu.g_end) {
        ++cu.u;
        cursor_unit<ROWS>(cu, p, c_end);
    }
}

// Per-step operands other than the codes (activations, group sums, scales,
// zeros), loaded one step ahead into registers so their L1/L2 latency overlaps
// the previous step's math.
template <int MT, int RT>
struct StepOperands {
    uint32_t xf[MT][16];  // B fragments: 16 half2 pairs per token tile
    float4 sb[MT];        // (sum x, bias) for this thread's two C-fragment tokens
    uint32_t sz[RT][2];   // (scale | zero << 16) of this thread's C-fragment rows
};

template <int MT, int RT>
__device__ __forceinline__ void load_operands(StepOperands<MT, RT> &v, const DecodeOp &op, const Cursor &cu,
                                              int gq, int c) {
    constexpr int MPAD = 8 * MT;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int tok = 8 * mt + gq;
        if (tok < op.M) {
            const uint16_t *xp = op.xperm + static_cast<size_t>(tok) * op.K + static_cast<size_t>(cu.g) * kGroup + 32 * c;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = ldg_u4(xp + 8 * q);
                v.xf[mt][4 * q + 0] = w.x;
                v.xf[mt][4 * q + 1] = w.y;
                v.xf[mt][4 * q + 2] = w.z;
                v.xf[mt][4 * q + 3] = w.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) v.xf[mt][q] = 0u;
        }
        if (8 * mt + 2 * c < op.M)
            v.sb[mt] = *reinterpret_cast<const float4 *>(op.sx + 2 * (static_cast<size_t>(cu.g) * MPAD + 8 * mt + 2 * c));
        else
            v.sb[mt] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = min(cu.r0 + rt * 16 + h * 8 + gq, op.N - 1);
            const size_t idx = static_cast<size_t>(r) * op.G + cu.g;
            v.sz[rt][h] = ldg_u16_nc(op.scales + idx) | (ldg_u16_nc(op.zeros + idx) << 16);
        }
}

template <int BITS, int MT>
__global__ void __launch_bounds__(kDecodeWarpsPerCta * 32, MT == 1 ? 4 : 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int RT = decode_rt(MT);
    constexpr int ROWS = 16 * RT;
    constexpr int D = decode_depth(BITS, MT);
    constexpr int ROW_BYTES = 16 * BITS;  // one row of one group
    constexpr int STAGE = ROWS * ROW_BYTES;
    constexpr int CHUNKS = ROWS * BITS;   // 16-byte chunks per stage
    constexpr int CPL = (CHUNKS + 31) / 32;
    constexpr int MPAD = 8 * MT;

    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2;  // MMA group id: row (A, C) / token (B)
    const int c = lane & 3;    // quad position: 32-code chunk (A, B) / token pair (C)
    uint8_t *ring = smem + warp * D * STAGE;

    const long long W = static_cast<long long>(gridDim.x) * kDecodeWarpsPerCta;
    const long long gw = static_cast<long long>(blockIdx.x) * kDecodeWarpsPerCta + warp;
    const long long c_begin = p.total_cost * gw / W;
    const long long c_end = p.total_cost * (gw + 1) / W;

    Cursor nx;  // next step to compute (operands prefetched for it)
    {
        int o = 0;
        while (o + 1 < p.n_ops && p.ops[o + 1].cost0 <= c_begin) ++o;
        const DecodeOp &op = p.ops[o];
        const long long rel = c_begin - op.cost0;
        nx.o = o;
        nx.u = static_cast<int>((rel + op.unit_cost - 1) / op.unit_cost);
        cursor_unit<ROWS>(nx, p, c_end);
    }
    Cursor ld = nx;

    auto issue = [&](const Cursor &cu, int slot) {
        const DecodeOp &op = p.ops[cu.o];
        const size_t row_stride = static_cast<size_t>(op.K) * BITS / 8;  // bytes
        const uint8_t *base = reinterpret_cast<const uint8_t *>(op.packed) +
                              static_cast<size_t>(cu.g) * ROW_BYTES;
        uint8_t *st = ring + slot * STAGE;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int ch = lane + 32 * i;
            if (CHUNKS % 32 == 0 || ch < CHUNKS) {
                const int row = ch / BITS, part = ch % BITS;
                const int r = min(cu.r0 + row, op.N - 1);
                const int pp = BITS == 8 ? (part ^ (row & 7)) : part;
                cp_async16(st + row * ROW_BYTES + pp * 16, base + static_cast<size_t>(r) * row_stride + part * 16);
            }
        }
    };

    // Prologue: weights do not depend on the previous kernel; start them now.
    int slot_ld = 0, slot_cs = 0;
#pragma unroll 1
    for (int i = 0; i < D - 1; ++i) {
        if (ld.valid) {
            issue(ld, slot_ld);
            cursor_next<ROWS>(ld, p, c_end);
        }
        cp_async_commit();
        slot_ld = slot_ld + 1 == D ? 0 : slot_ld + 1;
    }
    pdl_wait();  // the prepared activations come from the previous kernel
    pdl_launch_dependents();

    StepOperands<MT, RT> opA, opB;
    if (nx.valid) load_operands<MT, RT>(opA, p.ops[nx.o], nx, gq, c);

    float tot[RT][MT][4];
#pragma unroll
    for (int a = 0; a < RT; ++a)
#pragma unroll
        for (int b = 0; b < MT; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i) tot[a][b][i] = 0.0f;
    const float zero4[4] = {0.0f, 0.0f, 0.0f, 0.0f};

    // One step: consume `cv` (operands of the step at `nx`), prefetch the next
    // step's operands into `nv`.
    auto step = [&](const StepOperands<MT, RT> &cv, StepOperands<MT, RT> &nv) {
        const Cursor cs = nx;
        cursor_next<ROWS>(nx, p, c_end);
        if (nx.valid) load_operands<MT, RT>(nv, p.ops[nx.o], nx, gq, c);

        __syncwarp();
        if (ld.valid) {
            issue(ld, slot_ld);
            cursor_next<ROWS>(ld, p, c_end);
        }
        cp_async_commit();
        slot_ld = slot_ld + 1 == D ? 0 : slot_ld + 1;

        cp_async_wait<D - 1>();
        __syncwarp();
        const uint8_t *st = ring + slot_cs * STAGE;
        slot_cs = slot_cs + 1 == D ? 0 : slot_cs + 1;

#pragma unroll
        for (int rt = 0; rt < RT; ++rt) {
            uint32_t wv[2][BITS];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = rt * 16 + h * 8 + gq;
                const uint8_t *rp = st + row * ROW_BYTES;
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
                    const uint4 v0 = *reinterpret_cast<const uint4 *>(rp + 16 * ((2 * c) ^ (row & 7)));
                    const uint4 v1 = *reinterpret_cast<const uint4 *>(rp + 16 * ((2 * c + 1) ^ (row & 7)));
                    wv[h][0] = v0.x; wv[h][1] = v0.y; wv[h][2] = v0.z; wv[h][3] = v0.w;
                    wv[h][4] = v1.x; wv[h][5] = v1.y; wv[h][6] = v1.z; wv[h][7] = v1.w;
                }
            }
            float acc[MT][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t a0 = unpack_biased<BITS>(wv[0], 2 * j);
                const uint32_t a1 = unpack_biased<BITS>(wv[1], 2 * j);
                const uint32_t a2 = unpack_biased<BITS>(wv[0], 2 * j + 1);
                const uint32_t a3 = unpack_biased<BITS>(wv[1], 2 * j + 1);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    if (j == 0)
                        mma_16816(acc[mt], a0, a1, a2, a3, cv.xf[mt][2 * j], cv.xf[mt][2 * j + 1], zero4);
                    else
                        mma_16816(acc[mt], a0, a1, a2, a3, cv.xf[mt][2 * j], cv.xf[mt][2 * j + 1], acc[mt]);
                }
            }
            // Per-group epilogue: tot += s * (acc - bias) + z * sum(x).
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float sc = h2f_bits(cv.sz[rt][h] & 0xFFFFu);
                const float zr = h2f_bits(cv.sz[rt][h] >> 16);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    float &t0 = tot[rt][mt][2 * h], &t1 = tot[rt][mt][2 * h + 1];
                    t0 = fmaf(sc, acc[mt][2 * h] - cv.sb[mt].y, fmaf(zr, cv.sb[mt].x, t0));
                    t1 = fmaf(sc, acc[mt][2 * h + 1] - cv.sb[mt].w, fmaf(zr, cv.sb[mt].z, t1));
                }
            }
        }

        if (cs.g + 1 == cs.g_end) {
            // End of a unit: emit.
            const DecodeOp &op = p.ops[cs.o];
            if (op.S == 1) {
#pragma unroll
                for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int row = cs.r0 + rt * 16 + (i >> 1) * 8 + gq;
                            const int tok = 8 * mt + 2 * c + (i & 1);
                            if (row < op.N && tok < op.M)
                                op.out[static_cast<size_t>(tok) * op.N + row] =
                                    __half_as_ushort(__float2half_rn(tot[rt][mt][i]));
                        }
            } else {
                float *pb = op.part + (static_cast<size_t>(cs.rb) * op.S + cs.slice) * ROWS * MPAD;
#pragma unroll
                for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int row = rt * 16 + hh * 8 + gq;
                            *reinterpret_cast<float2 *>(pb + row * MPAD + 8 * mt + 2 * c) =
                                make_float2(tot[rt][mt][2 * hh], tot[rt][mt][2 * hh + 1]);
                        }
                __threadfence();
                __syncwarp();
                unsigned int prev = 0;
                if (lane == 0) prev = atomicAdd(op.cnt + cs.rb, 1u);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == static_cast<unsigned int>(op.S - 1)) {
                    __threadfence();
                    const float *p0 = op.part + static_cast<size_t>(cs.rb) * op.S * ROWS * MPAD;
                    for (int idx = lane; idx < ROWS * op.M; idx += 32) {
                        const int row = idx / op.M, tok = idx - row * op.M;
                        float s = 0.0f;
                        for (int sl = 0; sl < op.S; ++sl)
                            s += __ldcg(p0 + (static_cast<size_t>(sl) * ROWS + row) * MPAD + tok);
                        if (cs.r0 + row < op.N)
                            op.out[static_cast<size_t>(tok) * op.N + cs.r0 + row] =
                                __half_as_ushort(__float2half_rn(s));
                    }
                    if (lane == 0) op.cnt[cs.rb] = 0u;  // ready for the next call
                }
            }
#pragma unroll
            for (int rt = 0; rt < RT; ++rt)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) tot[rt][mt][i] = 0.0f;
        }
    };

#pragma unroll 1
    while (nx.valid) {
        step(opA, opB);
        if (!nx.valid) break;
        step(opB, opA);
    }
    cp_async_wait<0>();
}

// ------------------------------------------------------------------ host --

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
