// zq_quant_warp.cuh — one warp quantizes one block of 128 weights: one group
// of 128, or 2 groups of 64, or 4 of 32 (shared by quantize-and-pack and the
// KV-cache store).
//
// Asymmetric ([wiki] "ZSE - open-source движок для запуска LLM локально на GPU -
// 2026", section "Формат модели .zse", with L = 2^b - 1): zero = fp16(min),
// scale = fp16((max - min) / L) in fp64 with one rounding, q = clamp(round((w -
// zero) / scale), 0, L) from the stored fp16 values, round half to even; a
// group whose scale is 0 gets all q = 0.  Symmetric (the same section's
// INT8-symmetric, at every width): Q = 2^(b-1) - 1, scale = fp16(max|w| / Q),
// q = clamp(round(w / scale), -Q, Q), stored as q + 2^(b-1) with zero =
// -2^(b-1) * scale.  Explicit round-to-nearest fp64 intrinsics, no
// contraction: bit-identical to any IEEE-754 implementation of these steps.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace zq {

__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
    return __half_as_ushort(__double2half(v));
}

// Lane l holds weights 4l .. 4l+3 of the block in v; a group is `group`
// consecutive weights (32, 64 or 128), i.e. the group/4 lanes starting at a
// multiple of group/4.  On success the block's 4*bits packed words
// (little-endian bitstream, code k at bits [k*b, k*b+b); groups never straddle
// words) are in words[0 .. 4*bits) (this warp's shared-memory scratch) and every
// lane holds the fp16 bits of its group's scale and zero.  Returns false, in
// every lane, if a weight is NaN, infinite or above 65504 in magnitude, or
// (symmetric) a zero would not be a finite fp16; then nothing is written.
template <bool SYMMETRIC>
__device__ __forceinline__ bool quantize_group_warp(const float (&v)[4], int bits, int lane, uint32_t *words,
                                                    uint16_t &s16, uint16_t &z16, int group = 128) {
    const int L = (1 << bits) - 1;
    bool bad = false;
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        bad |= !(fabsf(v[i]) <= 65504.0f);  // NaN compares false
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
    if (__any_sync(0xffffffffu, bad)) return false;
    const int lanes_per_group = group >> 2;  // 8, 16 or 32: the xor steps below stay inside a group
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float omn = __shfl_xor_sync(0xffffffffu, mn, o), omx = __shfl_xor_sync(0xffffffffu, mx, o);
        if (o < lanes_per_group) {
            mn = fminf(mn, omn);
            mx = fmaxf(mx, omx);
        }
    }
    uint32_t chunk = 0;  // this lane's 4 codes, 4*bits bits
    if constexpr (SYMMETRIC) {
        const double half = static_cast<double>(1 << (bits - 1)), Q = half - 1.0;
        s16 = f64_to_f16_bits(__ddiv_rn(static_cast<double>(fmaxf(-mn, mx)), Q));
        const double s = static_cast<double>(__half2float(__ushort_as_half(s16)));
        const double z = __dmul_rn(-half, s);
        if (__any_sync(0xffffffffu, z < -65504.0)) return false;  // a zero would not be a finite fp16
        z16 = f64_to_f16_bits(z);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            double t = 0.0;
            if (s != 0.0) t = fmin(fmax(rint(__ddiv_rn(static_cast<double>(v[i]), s)), -Q), Q);
            chunk |= static_cast<uint32_t>(t + half) << (bits * i);
        }
    } else {
        z16 = f64_to_f16_bits(static_cast<double>(mn));
        s16 = f64_to_f16_bits(
            __ddiv_rn(__dsub_rn(static_cast<double>(mx), static_cast<double>(mn)), static_cast<double>(L)));
        const double s = static_cast<double>(__half2float(__ushort_as_half(s16)));
        const double z = static_cast<double>(__half2float(__ushort_as_half(z16)));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t q = 0;
            if (s != 0.0) {
                double t = rint(__ddiv_rn(__dsub_rn(static_cast<double>(v[i]), z), s));
                t = fmin(fmax(t, 0.0), static_cast<double>(L));
                q = static_cast<uint32_t>(t);
            }
            chunk |= q << (bits * i);
        }
    }
    // Assemble the group's 4*bits words: lane's chunk starts at stream bit 4*bits*lane.
    const int nw = 4 * bits;
    if (lane < nw) words[lane] = 0;
    __syncwarp();
    const int bit0 = 4 * bits * lane;
    const int wi = bit0 >> 5, off = bit0 & 31;
    atomicOr(&words[wi], chunk << off);
    if (off + 4 * bits > 32) atomicOr(&words[wi + 1], chunk >> (32 - off));
    __syncwarp();
    return true;
}

}  // namespace zq
