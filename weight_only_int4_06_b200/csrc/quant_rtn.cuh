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
    int z;         // zero point 0..15
    __half s16;    // fp16 scale
    bool overflow; // s16 is +inf
};

__device__ __forceinline__ GroupQuant group_params(float lo, float hi) {
    GroupQuant p;
    const float d = __fsub_rn(hi, lo);
    __half s = __float2half_ru(__fdiv_rn(d, 15.0f));
    if (d == 0.0f) s = __float2half_rn(1.0f);
    p.s16 = s;
    p.sf = __half2float(s);
    p.overflow = isinf(p.sf);
    const int z = __float2int_rn(__fdiv_rn(-lo, p.sf));
    p.z = min(max(z, 0), 15);
    return p;
}

__device__ __forceinline__ uint32_t quant_code(float v, const GroupQuant& p) {
    const int q = __float2int_rn(__fdiv_rn(v, p.sf)) + p.z;
    return (uint32_t)min(max(q, 0), 15);
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
