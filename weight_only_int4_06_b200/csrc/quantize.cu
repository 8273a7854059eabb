// w4_quantize_pack kernel: group-wise INT4 round-to-nearest quantisation and nibble packing.
//
// A group is 128 consecutive k of one row; in a row-major [N, K] matrix with K % 128 == 0 the
// groups are contiguous 256-byte runs, so the whole problem is a flat list of N*K/128 groups.
// QL lanes take one group (a warp takes 32 / QL groups per step): each lane loads 256 / QL bytes
// (16 / QL 16-byte chunks of 8 weights), the QL lanes reduce min/max with log2(QL) shuffles, and
// each lane quantises its weights into 16 / QL packed words, stored as one vector (lowest k in the
// lowest nibble).  Few lanes per group amortise the group's range, scale and zero point over many
// weights; without act_scale the range is found with packed fp16 min/max (exact: the conversion
// to fp32 is exact and monotone) and the minimum and the negated maximum share one shuffle.  HBM
// traffic per weight: 2 B read + 0.5 B written + 3/128 B of scale/zero.
#include "internal.h"
#include "quant_rtn.cuh"

namespace w4 {

constexpr int QL = 4;  // lanes per group

template <bool HAS_SCALE>
__global__ void __launch_bounds__(256, HAS_SCALE ? 2 : 4) quantize_pack_kernel(
    const uint4* __restrict__ W, const float* __restrict__ act, int64_t n_groups, int G,
    uint32_t* __restrict__ packed, __half* __restrict__ scales, uint8_t* __restrict__ zeros,
    int* status) {
    constexpr int CH = 16 / QL;   // 16-byte chunks per lane
    constexpr int GW = 32 / QL;   // groups per warp per step
    const int lane = threadIdx.x & 31;
    const int sub = lane / QL;    // which group of the warp's step
    const int lq = lane % QL;     // this lane's slice of the group
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_steps = (n_groups + GW - 1) / GW;

    int64_t st = warp;
    uint4 raw[CH];
    auto load = [&](int64_t step, uint4 (&r)[CH]) {
        const int64_t f = step * GW + sub;
#pragma unroll
        for (int j = 0; j < CH; ++j)
            r[j] = (step < n_steps && f < n_groups) ? ldg_stream(W + f * 16 + lq * CH + j) : make_uint4(0u, 0u, 0u, 0u);
    };
    load(st, raw);
    for (; st < n_steps; st += nwarps) {
        uint4 nxt[CH];
        load(st + nwarps, nxt);  // the next step's loads are in flight while this one is quantised
        const int64_t f = st * GW + sub;
        const bool valid = f < n_groups;
        const int64_t k0 = HAS_SCALE && valid ? (f % G) * 128 + 8 * CH * lq : 0;
        // chunk j's 8 weights in fp32, times act_scale when given (recomputed where needed: the
        // products are correctly rounded, so both passes see the same values)
        auto chunk = [&](int j, float (&v)[8]) {
            if (HAS_SCALE) {
                const float4 a0 = __ldg(reinterpret_cast<const float4*>(act + k0 + 8 * j));
                const float4 a1 = __ldg(reinterpret_cast<const float4*>(act + k0 + 8 * j) + 1);
                const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                load8_scaled(raw[j], a, v);
            } else {
                load8_scaled(raw[j], nullptr, v);
            }
        };
        float lo, hi;
        if (HAS_SCALE) {
            float mn = 0.0f, mx = 0.0f;  // the range includes 0 in any case
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                float v[8];
                chunk(j, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    mn = fminf(mn, v[i]);
                    mx = fmaxf(mx, v[i]);
                }
            }
#pragma unroll
            for (int o = QL / 2; o; o >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            lo = mn;
            hi = mx;
        } else {
            const __half2* h = reinterpret_cast<const __half2*>(raw);
            __half2 mn2 = h[0], mx2 = h[0];
#pragma unroll
            for (int i = 1; i < 4 * CH; ++i) {
                mn2 = __hmin2(mn2, h[i]);
                mx2 = __hmax2(mx2, h[i]);
            }
            // (min, -max) in one pair: one shuffle and one packed minimum per step
            const __half mn1 = __hmin(__low2half(mn2), __high2half(mn2));
            const __half mx1 = __hmax(__low2half(mx2), __high2half(mx2));
            __half2 pr = __halves2half2(mn1, __hneg(mx1));
#pragma unroll
            for (int o = QL / 2; o; o >>= 1) {
                uint32_t u = *reinterpret_cast<uint32_t*>(&pr);
                u = __shfl_xor_sync(0xffffffffu, u, o);
                pr = __hmin2(pr, *reinterpret_cast<__half2*>(&u));
            }
            lo = __low2float(pr);
            hi = -__high2float(pr);
        }
        const GroupQuant p = group_params(fminf(lo, 0.0f), fmaxf(hi, 0.0f));
        if (valid) {
            uint32_t w[CH];
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                float v[8];
                chunk(j, v);
                w[j] = quant_pack8_rtn(v, p);
            }
            uint32_t* dst = packed + f * 16 + lq * CH;
            if constexpr (CH == 4) {
                *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int j = 0; j < CH; ++j) dst[j] = w[j];
            }
            if (lq == 0) {
                scales[f] = p.s16;
                zeros[f] = (uint8_t)p.z;
                if (p.overflow) record_status(status, W4_ERR_RANGE);
            }
        }
#pragma unroll
        for (int j = 0; j < CH; ++j) raw[j] = nxt[j];
    }
}

cudaError_t launch_quantize_pack(const uint16_t* W, int64_t N, int64_t K, const float* act_scale,
                                 uint32_t* packed, uint16_t* scales, uint8_t* zeros, int* status,
                                 cudaStream_t stream) {
    const int64_t G = K / 128;
    const int64_t n_groups = N * G;
    const int threads = 256;
    const int64_t want = (n_groups + 8 * (32 / QL) - 1) / (8 * (32 / QL));  // one step per warp
    // one wave: 4 (2 with act_scale) resident blocks per SM, the kernels' register bounds
    const int64_t cap = (int64_t)device_sm_count() * (act_scale ? 2 : 4);
    const int blocks = (int)(want < cap ? want : cap);
    if (act_scale) {
        quantize_pack_kernel<true><<<blocks, threads, 0, stream>>>(
            reinterpret_cast<const uint4*>(W), act_scale, n_groups, (int)G, packed,
            reinterpret_cast<__half*>(scales), zeros, status);
    } else {
        quantize_pack_kernel<false><<<blocks, threads, 0, stream>>>(
            reinterpret_cast<const uint4*>(W), nullptr, n_groups, (int)G, packed,
            reinterpret_cast<__half*>(scales), zeros, status);
    }
    return cudaGetLastError();
}

}  // namespace w4
