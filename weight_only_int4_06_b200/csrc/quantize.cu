// w4_quantize_pack kernel: group-wise INT4 round-to-nearest quantisation and nibble packing.
//
// A group is 128 consecutive k of one row; in a row-major [N, K] matrix with K % 128 == 0 the
// groups are contiguous 256-byte runs, so the whole problem is a flat list of N*K/128 groups.
// One warp takes two groups per step: lanes 0-15 the first, lanes 16-31 the second.  Each lane
// loads 16 bytes (8 weights), the half-warp reduces min/max with four shuffles, every lane
// quantises its 8 weights into one uint32 word (lowest k in the lowest nibble) and the 16 lanes
// store the group's 64 packed bytes contiguously.  HBM traffic per weight: 2 B read +
// 0.5 B written + 3/128 B of scale/zero -- the kernel is bound by HBM bandwidth.
#include "internal.h"
#include "quant_rtn.cuh"

namespace w4 {

template <bool HAS_SCALE>
__device__ __forceinline__ void quantize_group_slice(const uint4 raw, int64_t f, bool valid, int l16, int G,
                                                     const float* __restrict__ act,
                                                     uint32_t* __restrict__ packed, __half* __restrict__ scales,
                                                     uint8_t* __restrict__ zeros, int* status) {
    float v[8];
    if (valid) {
        if (HAS_SCALE) {
            const int64_t k0 = (f % G) * 128 + 8 * l16;
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(act + k0));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(act + k0) + 1);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            load8_scaled(raw, a, v);
        } else {
            load8_scaled(raw, nullptr, v);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int o = 8; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const GroupQuant p = group_params(fminf(mn, 0.0f), fmaxf(mx, 0.0f));
    if (valid) {
        packed[f * 16 + l16] = quant_pack8_rtn(v, p);
        if (l16 == 0) {
            scales[f] = p.s16;
            zeros[f] = (uint8_t)p.z;
            if (p.overflow) record_status(status, W4_ERR_RANGE);
        }
    }
}

template <bool HAS_SCALE>
__global__ void __launch_bounds__(256) quantize_pack_kernel(
    const uint4* __restrict__ W, const float* __restrict__ act, int64_t n_groups, int G,
    uint32_t* __restrict__ packed, __half* __restrict__ scales, uint8_t* __restrict__ zeros,
    int* status) {
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 4;   // which group of the pair
    const int l16 = lane & 15;   // 8-weight slice within the group
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_pairs = (n_groups + 1) >> 1;

    // Two pairs per iteration, both loads in flight before either is processed.
    for (int64_t pair = warp; pair < n_pairs; pair += 2 * nwarps) {
        const int64_t f0 = 2 * pair + sub;
        const int64_t f1 = 2 * (pair + nwarps) + sub;
        const bool v0 = f0 < n_groups, v1 = f1 < n_groups;
        uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = make_uint4(0u, 0u, 0u, 0u);
        if (v0) r0 = ldg_stream(W + f0 * 16 + l16);
        if (v1) r1 = ldg_stream(W + f1 * 16 + l16);
        quantize_group_slice<HAS_SCALE>(r0, f0, v0, l16, G, act, packed, scales, zeros, status);
        if (pair + nwarps < n_pairs)  // warp-uniform
            quantize_group_slice<HAS_SCALE>(r1, f1, v1, l16, G, act, packed, scales, zeros, status);
    }
}

cudaError_t launch_quantize_pack(const uint16_t* W, int64_t N, int64_t K, const float* act_scale,
                                 uint32_t* packed, uint16_t* scales, uint8_t* zeros, int* status,
                                 cudaStream_t stream) {
    const int64_t G = K / 128;
    const int64_t n_groups = N * G;
    const int64_t n_pairs = (n_groups + 1) / 2;
    const int threads = 256;
    const int64_t want = (n_pairs + 7) / 8;  // one pair per warp
    const int64_t cap = (int64_t)device_sm_count() * 8;
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
