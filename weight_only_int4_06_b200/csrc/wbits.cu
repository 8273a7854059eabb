// Other weight widths and column orders.
//
// "AutoGPTQ vs The Stack v2": GPTQ to 2/3/4/8-bit codes, per-group scales and zero points, and an
// optional act-order (desc_act); "GPTQ, AWQ and the rules of post-training
// quantization", sections "AWQ: find the one percent that matters" (INT3, group 128) and "What
// activation-awareness buys and what it does not" (INT2, group 64).
//
//   * b-bit groups: the INT4 quantiser's rules with L = 2^b - 1 steps (zero-inclusive range, fp32
//     steps, fp16 scale rounded up, z and q clamped to [0, L]); codes form one little-endian bit
//     stream per row (code k in bits b k .. b k + b - 1; stream bit j in bit j % 32 of word j / 32),
//     so b = 4 is exactly the nibble layout.  Every group starts on a word boundary (group * b is a
//     multiple of 32 for the supported widths and group sizes).
//   * the matmul for b-bit weights: dequantise to fp16 (w = (q - z) s, exact in fp32, rounded once
//     to fp16, as the tcgen05 INT4 GEMM does) into a workspace, then the tcgen05 GEMM with an fp16
//     weight operand.  Two passes, not fused: the fused kernels serve INT4.
//   * activation preparation: X'[m, i] = X[m, perm[i]] (act-order: weights stored in processing
//     order), optionally divided by a per-channel scale, fp16(fp32(x) / s), so that an AWQ scale
//     can be applied to activations that were not produced already divided.
#include "common.cuh"
#include "internal.h"
#include "quant_bits.cuh"

namespace w4 {

// ------------------------------------------------------------------------------- quantise + pack
// One warp per group, lane l holding the group's elements [l V, l V + V), V = GROUP / 32.
template <int GROUP>
__global__ void __launch_bounds__(256) quantize_bits_kernel(const __half* __restrict__ W, const float* __restrict__ act,
                                                            int64_t N, int K, int bits,
                                                            uint32_t* __restrict__ packed,
                                                            __half* __restrict__ scales,
                                                            uint8_t* __restrict__ zeros, int* status) {
    constexpr int V = GROUP / 32;
    __shared__ uint8_t codes[8][GROUP];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = (1 << bits) - 1;
    const int G = K / GROUP;
    const int nwords = GROUP * bits / 32;
    const int64_t n_groups = N * G;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t f = gw; f < n_groups; f += nw) {  // warp-uniform loop
        const int64_t n = f / G;
        const int g = (int)(f - n * G);
        const int64_t e0 = n * K + (int64_t)g * GROUP + lane * V;
        float v[V];
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            v[i] = __half2float(W[e0 + i]);
            if (act) v[i] = __fmul_rn(v[i], act[g * GROUP + lane * V + i]);
            lo = fminf(lo, v[i]);
            hi = fmaxf(hi, v[i]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const GroupQuant p = group_params_steps(lo, hi, L);
#pragma unroll
        for (int i = 0; i < V; ++i) codes[warp][lane * V + i] = (uint8_t)quant_code_steps(v[i], p, L);
        __syncwarp();
        if (lane < nwords)
            packed[n * ((int64_t)K * bits / 32) + (int64_t)g * nwords + lane] = stream_word(codes[warp], bits, lane);
        if (lane == 0) {
            scales[f] = p.s16;
            zeros[f] = (uint8_t)p.z;
            if (p.overflow) record_status(status, W4_ERR_RANGE);
        }
        __syncwarp();  // codes[warp] is rewritten by the next group
    }
}

cudaError_t launch_quantize_bits(const uint16_t* W, int64_t N, int64_t K, int bits, int group, const float* act_scale,
                                 uint32_t* packed, uint16_t* scales, uint8_t* zeros, int* status,
                                 cudaStream_t stream) {
    const int64_t n_groups = N * (K / group);
    const int64_t want = (n_groups + 7) / 8;
    const int64_t cap = (int64_t)device_sm_count() * 16;
    const int blocks = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    const __half* w = reinterpret_cast<const __half*>(W);
    __half* s = reinterpret_cast<__half*>(scales);
    if (group == 64)
        quantize_bits_kernel<64><<<blocks, 256, 0, stream>>>(w, act_scale, N, (int)K, bits, packed, s, zeros, status);
    else
        quantize_bits_kernel<128><<<blocks, 256, 0, stream>>>(w, act_scale, N, (int)K, bits, packed, s, zeros, status);
    return cudaGetLastError();
}

// --------------------------------------------------------------------------- dequantise (matmul)
// Wd[n, k] = fp16((q - z) * s), one thread per element.
__global__ void dequant_bits_kernel(const uint32_t* __restrict__ packed, const __half* __restrict__ scales,
                                    const uint8_t* __restrict__ zeros, int64_t N, int K, int bits, int group,
                                    __half* __restrict__ Wd) {
    const int64_t total = N * K;
    const int64_t wpr = (int64_t)K * bits / 32;  // words per row
    const uint32_t mask = (1u << bits) - 1u;
    const int G = K / group;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = e / K;
        const int k = (int)(e - n * K);
        const int pos = bits * k;
        const int w = pos >> 5, off = pos & 31;
        const uint32_t* row = packed + n * wpr;
        uint32_t c = row[w] >> off;
        if (off + bits > 32) c |= row[w + 1] << (32 - off);
        c &= mask;
        const int gi = k / group;
        const float s = __half2float(scales[n * G + gi]);
        const int z = zeros[n * G + gi];
        Wd[e] = __float2half_rn((float)((int)c - z) * s);
    }
}

cudaError_t launch_wb_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, int bits, int group, uint16_t* Y,
                           void* ws, int* status, cudaStream_t stream) {
    __half* Wd = static_cast<__half*>(ws);
    dequant_bits_kernel<<<(unsigned)device_sm_count() * 8, 256, 0, stream>>>(
        packed, reinterpret_cast<const __half*>(scales), zeros, N, (int)K, bits, group, Wd);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_tc_f16(X, M, reinterpret_cast<const uint16_t*>(Wd), N, K, Y, status, stream);
}

// ------------------------------------------------------------------------ activation preparation
// Xo[m, i] = X[m, src] (src = perm[i], or i), divided by s[src] when s is given.  A perm entry
// outside [0, K) sets W4_ERR_RANGE and yields 0.
__global__ void act_prepare_kernel(const __half* __restrict__ X, int64_t M, int K, const int32_t* __restrict__ perm,
                                   const float* __restrict__ s, __half* __restrict__ Xo, int* status) {
    const int64_t total = M * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = e / K;
        const int i = (int)(e - m * K);
        const int src = perm ? perm[i] : i;
        if (src < 0 || src >= K) {
            record_status(status, W4_ERR_RANGE);
            Xo[e] = __float2half_rn(0.0f);
            continue;
        }
        const __half x = X[m * K + src];
        Xo[e] = s ? __float2half_rn(__fdiv_rn(__half2float(x), s[src])) : x;
    }
}

cudaError_t launch_act_prepare(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, const float* s,
                               uint16_t* Xo, int* status, cudaStream_t stream) {
    const int64_t total = M * K;
    const int64_t want = (total + 255) / 256;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int blocks = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    act_prepare_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const __half*>(X), M, (int)K, perm, s,
                                                   reinterpret_cast<__half*>(Xo), status);
    return cudaGetLastError();
}

}  // namespace w4
