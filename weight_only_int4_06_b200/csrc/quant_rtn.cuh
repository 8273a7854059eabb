// The round-to-nearest group quantiser, shared by w4_quantize_pack and the AWQ fake-quantiser so
// that both produce bit-identical codes.
//
// "GPTQ, AWQ and the rules of post-training quantization", section "The problem both methods
// solve": weights are rounded to the nearest level of a small integer format; "AutoGPTQ vs The
// Stack v2": one scale and one zero point per group of 128 consecutive k.
//
// Every step below is a single correctly rounded fp32 operation written with an explicit _rn
// intrinsic, so no contraction or fast-math rewriting can change a code:
//   lo = min(0, min v), hi = max(0, max v); s32 = (hi - lo) / 15;
//   s16 = s32 rounded toward +inf to fp16 (1.0 for an all-zero group);
//   z = clamp(rint(-lo / s16), 0, 15); q = clamp(rint(v / s16) + z, 0, 15), rint = half to even.
// Rounding s16 up makes the 16 levels span [lo, hi], so |v - (q - z) s16| <= s16 / 2.
#pragma once

#include "common.cuh"

namespace w4 {

struct GroupQuant {
    float sf;      // s16 as fp32
    float rcp;     // 1 / sf rounded to nearest (correctly rounded reciprocal)
    int z;         // zero point 0..15
    __half s16;    // fp16 scale
    bool overflow; // s16 is +inf
};

// Correctly rounded a / b from the correctly rounded reciprocal y = RN(1/b), by Markstein's
// correction step (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990): with q0 = RN(a*y) within one ulp of
// a/b, the remainder r = a - b*q0 is exact in one fma and RN(q0 + r*y) is the correctly rounded
// quotient.  Valid here because b is a positive normal fp32 value (an fp16 scale), a is finite
// and |a / b| < 2^24, so nothing over- or underflows.  An exact binary quotient is never a
// rounding midpoint, so the result is unique and equals IEEE division.
__device__ __forceinline__ float div_rn_from_rcp(float a, float b, float y) {
    const float q0 = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(r, y, q0);
}

// rint (round half to even) of an fp32 value with |x| < 2^22: adding 1.5 * 2^23 moves x into the
// binade [2^23, 2^24) whose spacing is 1, so the IEEE round-to-nearest-even of the addition is
// the rounding of x; the integer is the difference of the bit patterns (both in that binade).
__device__ __forceinline__ int rint_small(float x) {
    const float t = __fadd_rn(x, 12582912.0f);  // 1.5 * 2^23 (even, so ties keep x's parity rule)
    return __float_as_int(t) - 0x4B400000;      // bit pattern of 1.5 * 2^23
}

__device__ __forceinline__ GroupQuant group_params(float lo, float hi) {
    GroupQuant p;
    const float d = __fsub_rn(hi, lo);
    __half s = __float2half_ru(div_rn_from_rcp(d, 15.0f, __frcp_rn(15.0f)));  // d / 15, IEEE-exact
    if (d == 0.0f) s = __float2half_rn(1.0f);
    p.s16 = s;
    p.sf = __half2float(s);
    p.rcp = __frcp_rn(p.sf);
    p.overflow = isinf(p.sf);
    if (p.overflow) {  // codes are unspecified then; keep every intermediate finite
        p.sf = 1.0f;
        p.rcp = 1.0f;
    }
    const int z = rint_small(div_rn_from_rcp(-lo, p.sf, p.rcp));  // -lo / s16 in [0, 15 + 2^-20]
    p.z = min(max(z, 0), 15);
    return p;
}

// q = clamp(rint(v / s16) + z, 0, 15) with v / s16 the correctly rounded fp32 quotient
// (|v / s16| <= 15 + 2^-20 because the 16 levels span the zero-inclusive range).
__device__ __forceinline__ uint32_t quant_code(float v, const GroupQuant& p) {
    const int q = rint_small(div_rn_from_rcp(v, p.sf, p.rcp)) + p.z;
    return (uint32_t)min(max(q, 0), 15);
}

// Eight codes of an unclipped group packed into one word (lowest k in the lowest nibble).
// Same codes as quant_code: on the zero-inclusive range rint(v / s16) + z is never below 0
// (RN and rint are odd-symmetric and monotone, and z = rint(-lo / s16) is never clamped since
// -lo / s16 <= 15 (1 + 2^-23)), so only the upper clamp remains.  It is taken on the biased sum
// t = RN(v / s16) + 1.5 * 2^23 (see rint_small) against the float whose bit pattern is that of
// 1.5 * 2^23 + 15 - z: both are positive floats of one binade, so the float minimum is the integer
// minimum of the patterns.  The word is then sum_i (bits(t_i) - bits(1.5 * 2^23) + z) 16^i, formed
// modulo 2^32 as (z - bits(1.5 * 2^23)) * 0x11111111 + sum_i bits(t_i) 16^i: every field lies in
// [0, 15], so the modular sum has the fields of the exact one.  A group whose scale overflowed
// has unspecified codes (its status is reported); the arithmetic keeps them inside the word.
__device__ __forceinline__ uint32_t quant_pack8_rtn(const float (&v)[8], const GroupQuant& p) {
    const float top = __int_as_float(0x4B400000 + 15 - p.z);
    uint32_t word = (uint32_t)(p.z - 0x4B400000) * 0x11111111u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float t = fminf(__fadd_rn(div_rn_from_rcp(v[i], p.sf, p.rcp), 12582912.0f), top);
        word += __float_as_uint(t) * (1u << (4 * i));
    }
    return word;
}

// Eight consecutive fp16 weights (one 16-byte load) -> fp32, optionally times act_scale.
__device__ __forceinline__ void load8_scaled(const uint4 raw, const float* a, float (&v)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
    if (a) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], a[i]);
    }
}

}  // namespace w4
