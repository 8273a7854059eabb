// AWQ clip search: per-group shrinking of the quantisation range, chosen by output error.
//
// "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one percent
// that matters" (the layer keeps its function when W's channel j is multiplied by s_j and X's
// channel j divided by s_j) and the AutoAWQ pages ("activation-guided clipping"): after the
// scale search, each group's range may be shrunk so that the few large weights saturate and
// the others get a finer step, when that lowers the layer's output error on calibration data.
// The pages give no grid; the reading used here: ratios r_j = 1 - j/20 (j < n_ratios <= 10)
// multiply both ends of the group's zero-inclusive range, and for row n and group g
//     err_j = sum_t ( sum_{k in g} (X[t,k] / a_k) (w_hat_k - v_k) )^2,   v = W diag(a),
// w_hat the dequantised code of v under ratio r_j; the lowest j among the minima wins.
//
// err_j is a quadratic form in the group's 128 errors, e'^T G_g e' with e'_k = (w_hat_k - v_k)/a_k
// and G_g = X_g^T X_g the group's 128 x 128 Gram block, so the calibration rows are read once:
//   1. gram_partial_kernel: G_g over a slice of the T rows (fp32 FMA on CUDA cores, 8 x 8 outputs
//      per thread), for every (group, slice);
//   2. gram_reduce_kernel: the slices added in slice order (deterministic);
//   3. clip_kernel: one warp per (row, group): the quantiser of w4_quantize_pack under every
//      ratio, the quadratic forms against G_g in shared memory (all ratios at once, so G_g is
//      read once per row), the argmin, and the final codes/scale/zero of the chosen ratio.
#include "internal.h"
#include "quant_rtn.cuh"

namespace w4 {

constexpr int CL_MAXR = 10;
constexpr int GR_TT = 32;  // calibration rows per shared-memory chunk of the Gram kernel

// Shrink ratios r_j = 1 - j/20 (double arithmetic, one rounding to fp32).
__constant__ float kClipRatio[CL_MAXR] = {
    (float)(1.0 - 0 / 20.0), (float)(1.0 - 1 / 20.0), (float)(1.0 - 2 / 20.0), (float)(1.0 - 3 / 20.0),
    (float)(1.0 - 4 / 20.0), (float)(1.0 - 5 / 20.0), (float)(1.0 - 6 / 20.0), (float)(1.0 - 7 / 20.0),
    (float)(1.0 - 8 / 20.0), (float)(1.0 - 9 / 20.0)};

// Partial Gram block of group blockIdx.x over rows [t0, t1) of split blockIdx.y.
__global__ void __launch_bounds__(256) gram_partial_kernel(const __half* __restrict__ X, int64_t T, int K,
                                                          int rows_per_split, float* __restrict__ part) {
    __shared__ __align__(16) float xs[GR_TT][128];
    const int g = blockIdx.x, sp = blockIdx.y, G = gridDim.x;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int64_t t0 = (int64_t)sp * rows_per_split;
    const int64_t t1 = min(T, t0 + rows_per_split);
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
    for (int64_t tc = t0; tc < t1; tc += GR_TT) {
        // 32 rows x 128 halves: 512 chunks of 8, two per thread
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int idx = tid + c * 256, row = idx >> 4, ch = idx & 15;
            const int64_t t = tc + row;
            float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
            if (t < t1) {
                const uint4 r = ldg_stream(X + t * K + (int64_t)g * 128 + ch * 8);
                const __half2* h = reinterpret_cast<const __half2*>(&r);
                const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
                const float2 f2 = __half22float2(h[2]), f3 = __half22float2(h[3]);
                lo = make_float4(f0.x, f0.y, f1.x, f1.y);
                hi = make_float4(f2.x, f2.y, f3.x, f3.y);
            }
            *reinterpret_cast<float4*>(&xs[row][ch * 8]) = lo;
            *reinterpret_cast<float4*>(&xs[row][ch * 8 + 4]) = hi;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < GR_TT; ++r) {
            const float4 a0 = *reinterpret_cast<const float4*>(&xs[r][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4*>(&xs[r][ty * 8 + 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&xs[r][tx * 8]);
            const float4 b1 = *reinterpret_cast<const float4*>(&xs[r][tx * 8 + 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = part + ((size_t)sp * G + g) * 128 * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float4* o = reinterpret_cast<float4*>(out + (ty * 8 + i) * 128 + tx * 8);
        o[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        o[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
}

// gram[e] = sum over splits, in split order.
__global__ void gram_reduce_kernel(const float* __restrict__ part, int splits, int64_t n, float* __restrict__ gram) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int sp = 0; sp < splits; ++sp) s += part[(size_t)sp * n + e];
        gram[e] = s;
    }
}

constexpr int CL_WARPS = 8;
constexpr int CL_ROWS = 64;        // rows per CTA (8 per warp)

__global__ void __launch_bounds__(32 * CL_WARPS) clip_kernel(const __half* __restrict__ W, int64_t N, int K,
                                                           const float* __restrict__ act, int n_ratios,
                                                           const float* __restrict__ gram,
                                                           uint8_t* __restrict__ best_idx, float* __restrict__ err_out,
                                                           uint32_t* __restrict__ packed, __half* __restrict__ scales,
                                                           uint8_t* __restrict__ zeros, int* status) {
    extern __shared__ __align__(16) float cl_smem[];
    float* gs = cl_smem;                                   // [128][128] Gram block (symmetric)
    float* eb = cl_smem + 128 * 128;                       // [warp][ratio][128] errors e'
    const int g = blockIdx.x, G = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* gsrc = gram + (size_t)g * 128 * 128;
    for (int i = threadIdx.x; i < 128 * 128 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(gs)[i] = reinterpret_cast<const float4*>(gsrc)[i];
    __syncthreads();
    float* e = eb + warp * CL_MAXR * 128;

    // this lane's four k: 4 lane .. 4 lane + 3 of the group
    const int kb = g * 128 + 4 * lane;
    float ainv[4] = {1.0f, 1.0f, 1.0f, 1.0f}, av[4] = {1.0f, 1.0f, 1.0f, 1.0f};
    if (act) {
        const float4 a4 = *reinterpret_cast<const float4*>(act + kb);
        av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
#pragma unroll
        for (int i = 0; i < 4; ++i) ainv[i] = 1.0f / av[i];
    }

    for (int rr = 0; rr < CL_ROWS / CL_WARPS; ++rr) {
        const int64_t n = (int64_t)blockIdx.y * CL_ROWS + rr * CL_WARPS + warp;
        if (n >= N) break;  // warp-uniform
        const uint2 raw = *reinterpret_cast<const uint2*>(W + n * K + kb);
        const __half2* h = reinterpret_cast<const __half2*>(&raw);
        const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
        float v[4] = {f0.x, f0.y, f1.x, f1.y};
        if (act) {
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], av[i]);
        }
        float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
        float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);

        // errors e'_k = (w_hat_k - v_k) / a_k of every ratio, into this warp's buffer
        __syncwarp();
        for (int j = 0; j < CL_MAXR; ++j) {
            float4 ev = make_float4(0.f, 0.f, 0.f, 0.f);  // ratios beyond n_ratios: zero errors
            if (j < n_ratios) {
                const GroupQuant p = group_params(__fmul_rn(lo, kClipRatio[j]), __fmul_rn(hi, kClipRatio[j]));
                float ei[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float wq = (float)((int)quant_code(v[i], p) - p.z) * p.sf;  // exact
                    ei[i] = (wq - v[i]) * ainv[i];
                }
                ev = make_float4(ei[0], ei[1], ei[2], ei[3]);
            }
            *reinterpret_cast<float4*>(e + j * 128 + 4 * lane) = ev;
        }
        __syncwarp();
        // y = G_g e' for this lane's four rows of G, all ratios at once; then err_j = e'^T y.
        // Four k per step: G is symmetric, so rows k..k+3 at columns 4 lane.. are G[4 lane + i][k..].
        float y[4][CL_MAXR];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < CL_MAXR; ++j) y[i][j] = 0.0f;
#pragma unroll 1
        for (int kk = 0; kk < 128; kk += 4) {
            float4 gq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) gq[q] = *reinterpret_cast<const float4*>(gs + (kk + q) * 128 + 4 * lane);
#pragma unroll
            for (int j = 0; j < CL_MAXR; ++j) {
                const float4 ej = *reinterpret_cast<const float4*>(e + j * 128 + kk);  // same address in every lane
                const float ejq[4] = {ej.x, ej.y, ej.z, ej.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float gi[4] = {gq[q].x, gq[q].y, gq[q].z, gq[q].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) y[i][j] = fmaf(gi[i], ejq[q], y[i][j]);
                }
            }
        }
        float errj[CL_MAXR];
#pragma unroll
        for (int j = 0; j < CL_MAXR; ++j) {
            const float4 ev = *reinterpret_cast<const float4*>(e + j * 128 + 4 * lane);
            float s = ev.x * y[0][j];
            s = fmaf(ev.y, y[1][j], s);
            s = fmaf(ev.z, y[2][j], s);
            s = fmaf(ev.w, y[3][j], s);
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);  // same order in every lane
            errj[j] = s;
        }
        int best = 0;
        float bestv = errj[0];
#pragma unroll
        for (int j = 1; j < CL_MAXR; ++j)
            if (j < n_ratios && errj[j] < bestv) { bestv = errj[j]; best = j; }
        if (lane == 0) {
            best_idx[n * G + g] = (uint8_t)best;
            if (err_out) {
#pragma unroll
                for (int j = 0; j < CL_MAXR; ++j)
                    if (j < n_ratios) err_out[(n * G + g) * n_ratios + j] = errj[j];
            }
        }
        // the chosen ratio's codes (exactly w4_quantize_pack's quantiser on the shrunk range)
        const float rb = kClipRatio[best];
        const GroupQuant p = group_params(__fmul_rn(lo, rb), __fmul_rn(hi, rb));
        uint32_t half16 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) half16 |= quant_code(v[i], p) << (4 * i);
        const uint32_t upper = __shfl_down_sync(0xffffffffu, half16, 1);
        if ((lane & 1) == 0) packed[n * (K / 8) + g * 16 + (lane >> 1)] = half16 | (upper << 16);
        if (lane == 0) {
            scales[n * G + g] = p.s16;
            zeros[n * G + g] = (uint8_t)p.z;
            if (p.overflow) record_status(status, W4_ERR_RANGE);
        }
        __syncwarp();  // the error buffer is rewritten by the next row
    }
}

// ------------------------------------------------------------------------------------ host side
// T slices per group: as many as keep all (group, slice) CTAs in one wave of 2 CTAs per SM.
static int gram_splits(int64_t T, int G, int sms) {
    const int64_t want = (2L * sms) / G;
    const int64_t max_by_rows = (T + GR_TT - 1) / GR_TT;
    const int64_t s = want < max_by_rows ? want : max_by_rows;
    return (int)(s < 1 ? 1 : s);
}

AwqClipLayout awq_clip_layout(int64_t T, int64_t N, int64_t K, int n_ratios) {
    (void)N;
    (void)n_ratios;
    AwqClipLayout L;
    const int G = (int)(K / 128);
    L.splits = gram_splits(T, G, device_sm_count());
    const size_t blk = (size_t)G * 128 * 128 * sizeof(float);
    L.gram = 0;
    L.part = (blk + 255) & ~(size_t)255;
    L.bytes = L.part + (size_t)L.splits * blk;
    return L;
}

cudaError_t launch_awq_clip(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_ratios,
                            const float* act_scale, uint8_t* best_idx, float* err, uint32_t* packed,
                            uint16_t* scales, uint8_t* zeros, void* ws, int* status, cudaStream_t stream) {
    const int G = (int)(K / 128);
    const AwqClipLayout L = awq_clip_layout(T, N, K, n_ratios);
    unsigned char* base = static_cast<unsigned char*>(ws);
    float* gram = reinterpret_cast<float*>(base + L.gram);
    float* part = reinterpret_cast<float*>(base + L.part);
    const int rows_per_split = (int)(((T + L.splits - 1) / L.splits + GR_TT - 1) / GR_TT * GR_TT);
    gram_partial_kernel<<<dim3((unsigned)G, (unsigned)L.splits), 256, 0, stream>>>(
        reinterpret_cast<const __half*>(X), T, (int)K, rows_per_split, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)G * 128 * 128;
    gram_reduce_kernel<<<(unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, stream>>>(
        part, L.splits, n, gram);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)(128 * 128 + CL_WARPS * CL_MAXR * 128) * sizeof(float);
    e = cudaFuncSetAttribute(clip_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    clip_kernel<<<dim3((unsigned)G, (unsigned)((N + CL_ROWS - 1) / CL_ROWS)), 32 * CL_WARPS, smem, stream>>>(
        reinterpret_cast<const __half*>(W), N, (int)K, act_scale, n_ratios, gram, best_idx, err, packed,
        reinterpret_cast<__half*>(scales), zeros, status);
    return cudaGetLastError();
}

}  // namespace w4
