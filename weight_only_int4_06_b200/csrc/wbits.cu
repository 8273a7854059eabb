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
//   * the matmul for b-bit weights: for M <= 8 a fused GEMV that reads the bit stream once
//     (wb_gemv_kernel: codes dequantised in registers, fp32 sums); for larger M dequantise to fp16
//     (w = (q - z) s, exact in fp32, rounded once to fp16, as the tcgen05 INT4 GEMM does) into a
//     workspace, then the tcgen05 GEMM with an fp16 weight operand (two passes).
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

// ------------------------------------------------------------------- fused b-bit GEMV (M <= 8)
// Decode-sized M: the bit stream is read once and dequantised in registers.  One warp per weight
// row; lane l takes the 32-code chunks l, l + 32, ... of the row (a chunk is BITS whole words and
// never straddles a group: groups of 64 or 128 are 2 or 4 chunks).  Per chunk, for each activation
// row m: sum_k x_k q_k and sum_k x_k in fp32 (codes turned into fp32 exactly by the exponent trick
// 2^23 + q), and acc_m += s (sum x q - z sum x), i.e. sum_k x_k (q_k - z) s with the dequantised
// weight exact in fp32.  The lanes' sums are added by a fixed shuffle tree (deterministic).
template <int BITS>
__device__ __forceinline__ uint32_t wb_code(const uint32_t (&w)[BITS], int i) {
    const int bit = BITS * i, wi = bit >> 5, sh = bit & 31;
    const uint32_t v = (sh + BITS <= 32) ? (w[wi] >> sh) : __funnelshift_r(w[wi], w[wi + 1 < BITS ? wi + 1 : wi], sh);
    return v & ((1u << BITS) - 1u);
}

template <int BITS, int MT>
__global__ void __launch_bounds__(256) wb_gemv_kernel(const uint32_t* __restrict__ packed,
                                                      const unsigned short* __restrict__ scales,
                                                      const uint8_t* __restrict__ zeros, const __half* __restrict__ X,
                                                      __half* __restrict__ Y, int M, int N, int K, int group) {
    const int lane = threadIdx.x & 31;
    const int n = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (n >= N) return;  // whole warps
    const int wpr = K / 32 * BITS;  // words per row
    const uint32_t* prow = packed + (int64_t)n * wpr;
    const int G = K / group;
    const int n_chunks = K / 32;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    for (int ch = lane; ch < n_chunks; ch += 32) {
        uint32_t w[BITS];
#pragma unroll
        for (int j = 0; j < BITS; ++j) w[j] = __ldg(prow + (int64_t)ch * BITS + j);
        const int g = ch * 32 / group;
        const float s = __half2float(__ushort_as_half(__ldg(scales + (int64_t)n * G + g)));
        const float z = (float)__ldg(zeros + (int64_t)n * G + g);
        float q[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) q[i] = __int_as_float(0x4B000000 | (int)wb_code<BITS>(w, i)) - 8388608.0f;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m < M) {
                const uint4* xr = reinterpret_cast<const uint4*>(X + (int64_t)m * K + (int64_t)ch * 32);
                float sq = 0.0f, sx = 0.0f;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 r = __ldg(xr + v);
                    const __half2* h = reinterpret_cast<const __half2*>(&r);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 f = __half22float2(h[u]);
                        sq = fmaf(f.x, q[8 * v + 2 * u], sq);
                        sq = fmaf(f.y, q[8 * v + 2 * u + 1], sq);
                        sx += f.x + f.y;
                    }
                }
                acc[m] = fmaf(s, fmaf(-z, sx, sq), acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        float a = acc[m];
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0 && m < M) Y[(int64_t)m * N + n] = __float2half_rn(a);
    }
}

template <int BITS>
static cudaError_t launch_wb_gemv_bits(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                       const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y,
                                       cudaStream_t stream) {
    const unsigned blocks = (unsigned)((N + 7) / 8);  // 8 warps (rows) per block
    const unsigned short* sc = reinterpret_cast<const unsigned short*>(scales);
    const __half* x = reinterpret_cast<const __half*>(X);
    __half* y = reinterpret_cast<__half*>(Y);
    if (M <= 1) wb_gemv_kernel<BITS, 1><<<blocks, 256, 0, stream>>>(packed, sc, zeros, x, y, (int)M, (int)N, (int)K, group);
    else if (M <= 2) wb_gemv_kernel<BITS, 2><<<blocks, 256, 0, stream>>>(packed, sc, zeros, x, y, (int)M, (int)N, (int)K, group);
    else if (M <= 4) wb_gemv_kernel<BITS, 4><<<blocks, 256, 0, stream>>>(packed, sc, zeros, x, y, (int)M, (int)N, (int)K, group);
    else wb_gemv_kernel<BITS, 8><<<blocks, 256, 0, stream>>>(packed, sc, zeros, x, y, (int)M, (int)N, (int)K, group);
    return cudaGetLastError();
}

cudaError_t launch_wb_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, int bits, int group, uint16_t* Y,
                           void* ws, int* status, cudaStream_t stream) {
    if (M <= 8 && N < ((int64_t)1 << 31) / 32) {  // decode-sized M: the fused GEMV
        switch (bits) {
            case 2: return launch_wb_gemv_bits<2>(X, M, N, K, packed, scales, zeros, group, Y, stream);
            case 3: return launch_wb_gemv_bits<3>(X, M, N, K, packed, scales, zeros, group, Y, stream);
            case 4: return launch_wb_gemv_bits<4>(X, M, N, K, packed, scales, zeros, group, Y, stream);
            default: return launch_wb_gemv_bits<8>(X, M, N, K, packed, scales, zeros, group, Y, stream);
        }
    }
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
