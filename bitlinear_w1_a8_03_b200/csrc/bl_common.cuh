// Device helpers shared by the BitLinear kernels (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bitlinear.h"

namespace bl {

constexpr int kMaxGroup = BITLINEAR_MAX_GROUP;

// bfloat16 is the upper half of a binary32, so widening is exact.
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

template <typename T>
__device__ __forceinline__ float load_as_f32(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_as_f32<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float load_as_f32<uint16_t>(const uint16_t* p, int64_t i) {
    return bf16_bits_to_f32(p[i]);
}

// d = c + Σ_i a.u8[i] · b.s8[i]  (unsigned codes times signed activations)
__device__ __forceinline__ int dp4a_u8s8(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// d = c + Σ_i a.s8[i] · b.s8[i]
__device__ __forceinline__ int dp4a_s8s8(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 16-byte read of data used once: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte read of data shared by many warps (activations): read-only, L1-cached.
__device__ __forceinline__ uint4 ld_shared_ro16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// Dequantisation scale of one token: RN32(RN64(α·β / 127)).  α and β are
// binary32, so their product is exact in binary64.
__device__ __forceinline__ float dequant_scale(float alpha, float beta) {
    double s = __dmul_rn((double)alpha, (double)beta);
    s = __ddiv_rn(s, 127.0);
    return __double2float_rn(s);
}

// Per-row factor of the fast path of quantize_one: c = RN(127·RN(1/β)), or
// NaN (every element takes the exact path) when β >= 2^120 or is not finite,
// where RN(1/β) could lose relative precision.
__device__ __forceinline__ float quant_factor(float beta, float scale) {
    return beta < 0x1p120f ? __fmul_rn(scale, __frcp_rn(beta)) : __int_as_float(0x7fffffff);
}

// clip(rint(RN(RN(127·v) / β)), -127, 127), exactly (the per-token int8
// quantisation of "1.58-bit 大模型极限量化实战" §2.4), with c = quant_factor(β, 127).
// Fast path: q = RN(v·c) is within 4·2^-24 relative of t = RN(127·v)/β
// (three binary32 roundings against one), so for |v| <= β it is within
// 127·4·2^-24 + 127·2^-24 < 4e-5 of RN(t).  When q is farther than 1e-4 from
// every half-integer, q and RN(t) lie on the same side of it and round to the
// same integer, which is at most 127 in magnitude (|q| < 127.5), so no clip
// is needed.  Otherwise (rare; always for non-finite q) the exact quotient
// is taken and clipped.
__device__ __forceinline__ int8_t quantize_one(float v, float beta, float c) {
    const float q = __fmul_rn(v, c);
    float r = rintf(q);  // round half to even
    if (!(fabsf(__fsub_rn(q, r)) < 0.4999f)) {
        r = rintf(__fdiv_rn(__fmul_rn(v, 127.0f), beta));
        r = fminf(fmaxf(r, -127.0f), 127.0f);
    }
    return (int8_t)__float2int_rn(r);
}

// quantize_one of N consecutive elements (N a multiple of 4), packed four
// codes to a word (element e in byte e % 4 of word e / 4); with qmax = 7 (and
// c = quant_factor(β, 7)) the codes of quantize_one_a4, as int8 bytes.  The rounding uses
// t = RN(q + 1.5·2^23): for |q| < 2^22 the sum lies where binary32 steps are
// 1, so t - 1.5·2^23 is rint(q) (ties to even, as RN breaks them) and the low
// byte of t's bits is that integer in two's complement; this avoids the
// float-to-integer conversions.  The fast values of all N are formed first;
// the exact path runs only for the elements that need it, behind one branch.
template <int N>
__device__ __forceinline__ void quantize_codes(const float (&f)[N], float beta, float c, uint32_t (&w)[N / 4],
                                               float qmax = 127.0f) {
    constexpr float kRound = 12582912.0f;  // 1.5·2^23
    float t[N];
    uint32_t bad = 0;
#pragma unroll
    for (int e = 0; e < N; ++e) {
        const float q = __fmul_rn(f[e], c);
        t[e] = __fadd_rn(q, kRound);
        const float r = __fsub_rn(t[e], kRound);
        bad |= (fabsf(__fsub_rn(q, r)) < 0.4999f ? 0u : 1u) << e;
    }
    if (bad) {
#pragma unroll
        for (int e = 0; e < N; ++e)
            if ((bad >> e) & 1u) {
                float r = rintf(__fdiv_rn(__fmul_rn(f[e], qmax), beta));
                r = fminf(fmaxf(r, -qmax), qmax);  // also maps NaN to -qmax
                t[e] = __fadd_rn(r, kRound);
            }
    }
#pragma unroll
    for (int g = 0; g < N / 4; ++g) {
        const uint32_t lo = __byte_perm(__float_as_uint(t[4 * g]), __float_as_uint(t[4 * g + 1]), 0x0040);
        const uint32_t hi = __byte_perm(__float_as_uint(t[4 * g + 2]), __float_as_uint(t[4 * g + 3]), 0x0040);
        w[g] = __byte_perm(lo, hi, 0x5410);
    }
}

// clip(rint(RN(RN(7·v) / β)), -7, 7): the 4-bit variant of quantize_one, with
// c = quant_factor(β, 7) and the same argument (q within 7·5·2^-24 of RN(t)).
__device__ __forceinline__ int quantize_one_a4(float v, float beta, float c) {
    const float q = __fmul_rn(v, c);
    float r = rintf(q);
    if (!(fabsf(__fsub_rn(q, r)) < 0.4999f)) {
        r = rintf(__fdiv_rn(__fmul_rn(v, 7.0f), beta));
        r = fminf(fmaxf(r, -7.0f), 7.0f);
    }
    return __float2int_rn(r);
}

// Dequantisation scale of one token for 4-bit activations: RN32(RN64(α·β / 7)).
__device__ __forceinline__ float dequant_scale_a4(float alpha, float beta) {
    double s = __dmul_rn((double)alpha, (double)beta);
    s = __ddiv_rn(s, 7.0);
    return __double2float_rn(s);
}

// Eight 4-bit activations (two's complement nibbles, element 2i in the low
// nibble of byte i) as two words of four int8: the nibbles are spread to bytes
// and sign-extended without borrows between bytes: ((u ^ 8) | 0x80) - 8, then ^ 0x80.
__device__ __forceinline__ void unpack_a4(uint32_t w, uint32_t& lo4, uint32_t& hi4) {
    const uint32_t even = w & 0x0F0F0F0Fu;         // elements 0, 2, 4, 6
    const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
    uint32_t a = __byte_perm(even, odd, 0x5140);   // 0, 1, 2, 3
    uint32_t b = __byte_perm(even, odd, 0x7362);   // 4, 5, 6, 7
    a = (((a ^ 0x08080808u) | 0x80808080u) - 0x08080808u) ^ 0x80808080u;
    b = (((b ^ 0x08080808u) | 0x80808080u) - 0x08080808u) ^ 0x80808080u;
    lo4 = a;
    hi4 = b;
}

}  // namespace bl
