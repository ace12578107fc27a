// zq_device.cuh — device building blocks shared by the zq kernels (sm_100a).
//
// Code unpack ([wiki] = "ZSE - open-source движок для запуска LLM локально на
// GPU - 2026", section "Формат модели .zse": b-bit codes, asymmetric scale and
// zero per 128 weights; the pages' DSL names INT4 unpack intrinsics in section
// "Компилятор").  The codes are turned into exact fp16 integers with the
// magic-exponent construction: a code q placed in the mantissa bits [s, s+b) of
// a binary16 whose exponent field encodes 1024 reads as 1024 + q * 2^s (the
// "biased" value); one fused multiply-add by (2^-s, -1024 * 2^-s) gives q
// exactly.  One LOP3 builds two such halves at once (one per 16-bit half of a
// 32-bit register), so the unpack yields half2 PAIRS of codes.  Which two codes share a pair depends on
// b; it is fixed by pair_lo()/pair_hi() below, and the activation side is
// permuted to the same order, so no repack of the canonical layout is needed.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace zq {

// ---------------------------------------------------------------- PTX bits --

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t r;  // (a & mask) | magic
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
    return r;
}

// Same with the mask as an instruction immediate (no register for it).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t lop_and_or_imm(uint32_t a, uint32_t magic) {
    uint32_t r;  // (a & MASK) | magic
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "n"(MASK), "r"(magic));
    return r;
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

__device__ __forceinline__ uint32_t shf_r(uint32_t lo, uint32_t hi, uint32_t s) {
    uint32_t r;  // low 32 bits of (hi:lo) >> s, s < 32
    asm("shf.r.clamp.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(lo), "r"(hi), "r"(s));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// D = A * B + C, m16n8k16, A row-major fp16, B col-major fp16, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1,
                                          const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// Programmatic dependent launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Ampere-style asynchronous global->shared copies, 16 bytes, L2 only.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t ldg_u16_nc(const uint16_t *p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_u4(const void *p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// mbarrier primitives (shared::cta).
__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 2-D TMA tile load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *map, int x, int y, unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory loads by 32-bit shared-window address.  They carry no memory
// clobber, so the compiler schedules them freely; a caller that must order
// them after a barrier wait adds opaque_zero() (taken after the wait) to the
// address.
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
// A zero the compiler cannot see through, produced at this point of the
// program order (volatile asm statements keep their relative order).
__device__ __forceinline__ uint32_t opaque_zero() {
    uint32_t z;
    asm volatile("mov.u32 %0, 0;" : "=r"(z));
    return z;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, unsigned long long *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed;
// the arrival counts toward the barrier's expected count.
__device__ __forceinline__ void cp_async_arrive_noinc(unsigned long long *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Ampere-style asynchronous copy of 8 bytes (L1-allocating form; sizes 4/8).
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

__device__ __forceinline__ float h2f_bits(uint32_t h) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// fp16 in the low (HI = false) or high half of a 32-bit word, as float.
template <bool HI>
__device__ __forceinline__ float half_of(uint32_t w) {
    const __half2 h = *reinterpret_cast<const __half2 *>(&w);
    return HI ? __high2float(h) : __low2float(h);
}

// ------------------------------------------------------------ code unpack --
//
// A thread owns one 32-code chunk of a group: b consecutive uint32 words that
// hold codes 0..31 of the chunk (the chunk starts on a word boundary for every
// b because 32*b bits is a whole number of words).  pair p (0..15) is a half2
// whose low half is code pair_lo(p) and whose high half is code pair_hi(p).

// b = 3: the 96-bit chunk (code j at stream bits 3j..3j+2) is read through
// eight 32-bit windows (stream bits n..n+31); pairs 2q and 2q+1 come from
// window q, their low codes at offsets 4..9 or so of the low half and their
// high codes in the high half.  The windows at n = 0, 32, 64 are the words
// themselves, the other five cost one shift each: 21 instructions per 32
// codes.  Codes (a, b) and (a+1, b+1) of each window keep a and b even, so
// two PRMTs still restore natural K order from pairs 2q and 2q+1.
__host__ __device__ constexpr int i3_win(int q) {
    return q == 0 ? 0 : q == 1 ? 4 : q == 2 ? 10 : q == 3 ? 32 : q == 4 ? 38 : q == 5 ? 56 : q == 6 ? 64 : 74;
}
__host__ __device__ constexpr int i3_lo(int q) {
    return q == 0 ? 0 : q == 1 ? 2 : q == 2 ? 4 : q == 3 ? 12 : q == 4 ? 14 : q == 5 ? 20 : q == 6 ? 22 : 26;
}
__host__ __device__ constexpr int i3_hi(int q) {
    return q == 0 ? 6 : q == 1 ? 8 : q == 2 ? 10 : q == 3 ? 16 : q == 4 ? 18 : q == 5 ? 24 : q == 6 ? 28 : 30;
}

template <int B>
__host__ __device__ constexpr int pair_lo(int p) {
    return B == 2 ? 16 * (p / 8) + p % 8
         : B == 3 ? i3_lo(p / 2) + p % 2
         : B == 4 ? 8 * (p / 4) + p % 4
         : B == 8 ? 4 * (p / 2) + p % 2
                  : 2 * p;  // B = 16 (fp16 weights): word p holds codes 2p, 2p + 1
}
template <int B>
__host__ __device__ constexpr int pair_hi(int p) {
    return B == 3 ? i3_hi(p / 2) + p % 2 : pair_lo<B>(p) + (B == 2 ? 8 : B == 4 ? 4 : B == 8 ? 2 : 1);
}

// fp16x2 constants: magic 1024 in both halves; (2^-s_lo, 2^-s_hi);
// (-1024 * 2^-s_lo, -1024 * 2^-s_hi).
constexpr uint32_t kMagic = 0x64006400u;
__host__ __device__ constexpr uint32_t mul_s2(int slo, int shi) {
    return ((15u - slo) << 10) | (((15u - shi) << 10) << 16);
}
__host__ __device__ constexpr uint32_t add_s2(int slo, int shi) {
    return (0x8000u | ((25u - slo) << 10)) | ((0x8000u | ((25u - shi) << 10)) << 16);
}

// Mantissa offsets of the codes of pair p (low and high half): the biased
// pair reads (1024 + q_lo * 2^s_lo, 1024 + q_hi * 2^s_hi).  Equal in both
// halves except at b = 3.
template <int B>
__host__ __device__ constexpr int pair_shift_lo(int p) {
    return B == 2 ? ((p % 8) < 5 ? 2 * (p % 8) : 2 * (p % 8 - 5))
         : B == 3 ? 3 * pair_lo<3>(p) - i3_win(p / 2)
         : B == 4 ? 4 * (p % 2)
                  : 0;  // b = 8, and fp16 weights (no offset, no bias)
}
template <int B>
__host__ __device__ constexpr int pair_shift_hi(int p) {
    return B == 3 ? 3 * pair_hi<3>(p) - i3_win(p / 2) - 16 : pair_shift_lo<B>(p);
}

// Every b = 3 pair: codes inside their window half, offsets 0..7 (so that
// 1024 + q * 2^s, q <= 7, is exact), and the quads the PRMT restore needs.
__host__ __device__ constexpr bool i3_table_ok() {
    unsigned seen = 0;
    for (int p = 0; p < 16; ++p) {
        const int lo = pair_lo<3>(p), hi = pair_hi<3>(p);
        const int slo = pair_shift_lo<3>(p), shi = pair_shift_hi<3>(p);
        if (slo < 0 || slo > 7 || shi < 0 || shi > 7) return false;
        if ((seen >> lo) & 1u || (seen >> hi) & 1u) return false;
        seen |= (1u << lo) | (1u << hi);
        if (p % 2 == 0 && (lo % 2 != 0 || hi % 2 != 0 || pair_lo<3>(p + 1) != lo + 1 || pair_hi<3>(p + 1) != hi + 1))
            return false;
    }
    return seen == 0xFFFFFFFFu;
}
static_assert(i3_table_ok(), "b = 3 pair table");

// Biased pair: one LOP3 (plus a shift shared by several pairs).
template <int B>
__device__ __forceinline__ uint32_t unpack_biased(const uint32_t (&w)[B], int p);

// b = 2: word i holds codes 16i..16i+15 at bits 2j.  Codes j and j+8 sit 16
// bits apart; j = 0..4 are at mantissa offsets 0..8 of their halves, j = 5..7
// are read from the word shifted right by 10.
template <>
__device__ __forceinline__ uint32_t unpack_biased<2>(const uint32_t (&w)[2], int p) {
    const uint32_t u = w[p / 8];
    const int j = p % 8;
    if (j < 5) return lop_and_or(u, 0x00030003u << (2 * j), kMagic);
    return lop_and_or(u >> 10, 0x00030003u << (2 * (j - 5)), kMagic);
}

// b = 3: window q = p / 2 of the 96-bit chunk (stream bits n..n+31, n =
// i3_win(q)), then one LOP3 keeps the pair's two codes.
__device__ __forceinline__ uint32_t i3_window(const uint32_t (&w)[3], int n) {
    return n == 0 ? w[0] : n < 32 ? shf_r(w[0], w[1], n) : n == 32 ? w[1] : n < 64 ? shf_r(w[1], w[2], n - 32)
                         : n == 64 ? w[2] : (w[2] >> (n - 64));
}
template <>
__device__ __forceinline__ uint32_t unpack_biased<3>(const uint32_t (&w)[3], int p) {
    return lop_and_or(i3_window(w, i3_win(p / 2)),
                      (0x7u << pair_shift_lo<3>(p)) | (0x7u << (16 + pair_shift_hi<3>(p))), kMagic);
}

// b = 4: word i holds codes 8i..8i+7 (nibbles); pairs (j, j+4) at mantissa
// offsets 0 and 4, from the word and from the word shifted right by 8.
template <>
__device__ __forceinline__ uint32_t unpack_biased<4>(const uint32_t (&w)[4], int p) {
    const uint32_t u = (p % 4) < 2 ? w[p / 4] : (w[p / 4] >> 8);
    return (p % 2) == 0 ? lop_and_or(u, 0x000F000Fu, kMagic) : lop_and_or(u, 0x00F000F0u, kMagic);
}

// b = 8: word i holds codes 4i..4i+3 (bytes); pairs (0,2) and (1,3).
template <>
__device__ __forceinline__ uint32_t unpack_biased<8>(const uint32_t (&w)[8], int p) {
    const uint32_t u = (p % 2) == 0 ? w[p / 2] : (w[p / 2] >> 8);
    return lop_and_or(u, 0x00FF00FFu, kMagic);
}

// Biased pair with the pair index known at compile time: the LOP3 mask is an
// immediate.  Same pairs as unpack_biased<B>(w, P).
template <int B, int P>
__device__ __forceinline__ uint32_t unpack_biased_c(const uint32_t (&w)[B], uint32_t magic) {
    if constexpr (B == 2) {
        constexpr int j = P % 8;
        if constexpr (j < 5) return lop_and_or_imm<(0x00030003u << (2 * j))>(w[P / 8], magic);
        else return lop_and_or_imm<(0x00030003u << (2 * (j - 5)))>(w[P / 8] >> 10, magic);
    } else if constexpr (B == 3) {
        constexpr uint32_t mask = (0x7u << pair_shift_lo<3>(P)) | (0x7u << (16 + pair_shift_hi<3>(P)));
        return lop_and_or_imm<mask>(i3_window(w, i3_win(P / 2)), magic);
    } else if constexpr (B == 4) {
        const uint32_t u = (P % 4) < 2 ? w[P / 4] : (w[P / 4] >> 8);
        return lop_and_or_imm<((P % 2) == 0 ? 0x000F000Fu : 0x00F000F0u)>(u, magic);
    } else if constexpr (B == 8) {
        const uint32_t u = (P % 2) == 0 ? w[P / 2] : (w[P / 2] >> 8);
        return lop_and_or_imm<0x00FF00FFu>(u, magic);
    } else {
        static_assert(B == 16, "b = 2, 3, 4, 8 or fp16 weights");
        return w[P];  // fp16 weights: the pair as stored, no bias
    }
}

// Exact codes: one HFMA2 by (2^-s, -1024 * 2^-s), per half, removes bias and
// offset.
template <int B>
__device__ __forceinline__ uint32_t unpack_pair(const uint32_t (&w)[B], int p) {
    const int slo = pair_shift_lo<B>(p), shi = pair_shift_hi<B>(p);
    return hfma2_bits(unpack_biased<B>(w, p), mul_s2(slo, shi), add_s2(slo, shi));
}

}  // namespace zq
