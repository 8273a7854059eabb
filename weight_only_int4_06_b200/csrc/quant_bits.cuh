// Group quantisation with L = 2^b - 1 steps and the little-endian bit-stream packing of b-bit
// codes, shared by the b-bit quantiser and GPTQ.  The arithmetic is the INT4 quantiser's
// (quant_rtn.cuh) with 15 replaced by L, so b = 4 gives the same scales, zero points and codes,
// and the bit stream of 4-bit codes is the nibble layout.
#pragma once

#include "quant_rtn.cuh"

namespace w4 {

// group_params with L steps instead of 15 (see quant_rtn.cuh for the arithmetic).
__device__ __forceinline__ GroupQuant group_params_steps(float lo, float hi, int L) {
    GroupQuant p;
    const float fl = (float)L;
    const float d = __fsub_rn(hi, lo);
    __half s = __float2half_ru(div_rn_from_rcp(d, fl, __frcp_rn(fl)));
    if (d == 0.0f) s = __float2half_rn(1.0f);
    p.s16 = s;
    p.sf = __half2float(s);
    p.rcp = __frcp_rn(p.sf);
    p.overflow = isinf(p.sf);
    if (p.overflow) {
        p.sf = 1.0f;
        p.rcp = 1.0f;
    }
    const int z = rint_small(div_rn_from_rcp(-lo, p.sf, p.rcp));
    p.z = min(max(z, 0), L);
    return p;
}

// clamp(rint(v / s16) + z, 0, L); the quotient is clamped to +-1024 first so that the rounding
// helper's range holds for any input (beyond that the code saturates either way).
__device__ __forceinline__ int quant_code_steps(float v, const GroupQuant& p, int L) {
    const float x = fminf(fmaxf(div_rn_from_rcp(v, p.sf, p.rcp), -1024.0f), 1024.0f);
    return min(max(rint_small(x) + p.z, 0), L);
}

// Word w of one group's bit stream from the group's codes (codes[k], k < group).
__device__ __forceinline__ uint32_t stream_word(const uint8_t* codes, int bits, int w) {
    const int b0 = 32 * w;
    const int k0 = b0 / bits, k1 = (b0 + 31) / bits;
    uint32_t word = 0;
    for (int k = k0; k <= k1; ++k) {
        const int pos = bits * k - b0;
        const uint32_t c = codes[k];
        word |= pos >= 0 ? (c << pos) : (c >> (-pos));
    }
    return word;
}

}  // namespace w4
