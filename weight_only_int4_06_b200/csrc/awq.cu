// AWQ activation-aware scale search on one linear layer.
//
// "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one percent
// that matters": channel j's scale is its mean |x| over the calibration rows to the power alpha;
// alpha is picked from a grid on [0, 1]; multiplying W's channel j by s_j and dividing X's
// channel j by s_j leaves the output unchanged, while the rounding error of the channels with
// large activations shrinks.
//
// Steps on the device (all on the caller's stream, workspace supplied by the caller):
//   1. colabs:    c_j = sum_t |X[t, j]| as an exact integer count of 2^-24 units (every fp16 value
//                 is such a multiple), so the sum is exact and order-independent;
//                 m_j = c_j * 2^-24 / T, rounded once to fp64.
//   2. scales:    s_ij = max(m_j, 1e-6)^(i / n_alpha) / sqrt(max_j s * min_j s) in fp64, then
//                 rounded to fp32 (the value that multiplies W and divides X).
//   3. per alpha: fake-quantise W * diag(s_i) with exactly the quantiser of w4_quantize_pack and
//                 emit E_i = (Wq - W * s_i) / s_i rounded to fp16, so that
//                 (X / s_i) Wq^T - X W^T = X E_i^T;
//                 then sum_{t,n} (X E_i^T)^2 with the tcgen05 GEMM (sum-of-squares epilogue,
//                 one fp64 partial per 128x256 tile).
//   4. finalize:  MSE_i = (fixed-order fp64 sum of the partials) / (T N); best = lowest index
//                 among the minima; best_s = s_best.
#include "common.cuh"
#include "internal.h"
#include "quant_rtn.cuh"

namespace w4 {

constexpr int CA_ROWS = 256;  // rows of X per CTA

// Column sums of |x| as integer numbers of 2^-24 units (exact).  A thread adds its column's
// |x| over CA_ROWS rows in fp64: every |x| is an exact multiple of 2^-24 below 2^16, so the sum of
// 256 of them stays below 2^24 and needs at most 48 significant bits — every fp64 addition is
// exact.  The sum times 2^24 is then an exact integer, added to the column's u64 total.
__device__ __forceinline__ void colabs_add(uint32_t w, double& lo, double& hi) {
    const uint32_t a = w & 0x7FFF7FFFu;  // |x| of both halves
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&a));
    lo += (double)f.x;
    hi += (double)f.y;
}

__global__ void __launch_bounds__(256) colabs_kernel(const uint4* __restrict__ X, int64_t T, int K,
                                                     unsigned long long* __restrict__ colsum) {
    const int chunks = K >> 3;  // 8 fp16 per 16-byte chunk
    const int ch = blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= chunks) return;
    const int64_t r0 = (int64_t)blockIdx.y * CA_ROWS;
    const int64_t r1 = min(T, r0 + CA_ROWS);
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ldg_stream(X + (r + u) * chunks + ch);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            colabs_add(v[u].x, acc[0], acc[1]);
            colabs_add(v[u].y, acc[2], acc[3]);
            colabs_add(v[u].z, acc[4], acc[5]);
            colabs_add(v[u].w, acc[6], acc[7]);
        }
    }
    for (; r < r1; ++r) {
        const uint4 v = ldg_stream(X + r * chunks + ch);
        colabs_add(v.x, acc[0], acc[1]);
        colabs_add(v.y, acc[2], acc[3]);
        colabs_add(v.z, acc[4], acc[5]);
        colabs_add(v.w, acc[6], acc[7]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)  // exact: an integer below 2^48
        atomicAdd(colsum + ch * 8 + i, (unsigned long long)__double2ull_rn(acc[i] * 16777216.0));
}

// One CTA per alpha.  Block-wide max/min with a fixed reduction tree.
__global__ void __launch_bounds__(1024) awq_scales_kernel(const unsigned long long* __restrict__ colsum,
                                                          int64_t T, int K, int n_alpha, float* __restrict__ s_all) {
    __shared__ double smax[32], smin[32];
    __shared__ double norm;
    const int i = blockIdx.x;
    const double alpha = (double)i / (double)n_alpha;
    const double inv_units = 5.9604644775390625e-08;  // 2^-24
    double mx = 0.0, mn = 1.0e308;
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
        const double m = (double)colsum[j] * inv_units / (double)T;
        const double s = pow(fmax(m, 1e-6), alpha);
        mx = fmax(mx, s);
        mn = fmin(mn, s);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) { smax[w] = mx; smin[w] = mn; }
    __syncthreads();
    if (w == 0) {
        const int nw = blockDim.x >> 5;
        mx = l < nw ? smax[l] : 0.0;
        mn = l < nw ? smin[l] : 1.0e308;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        if (l == 0) norm = sqrt(mx * mn);
    }
    __syncthreads();
    const double nv = norm;
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
        const double m = (double)colsum[j] * inv_units / (double)T;
        const double s = pow(fmax(m, 1e-6), alpha) / nv;
        s_all[(int64_t)i * K + j] = __double2float_rn(s);
    }
}

// E = (Wq - W*s) / s in fp16 for one alpha; the codes are those of w4_quantize_pack(W, s).
__global__ void __launch_bounds__(256) awq_fakequant_kernel(const uint4* __restrict__ W, const float* __restrict__ s,
                                                            int64_t n_groups, int G, uint4* __restrict__ E,
                                                            int* status) {
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 4, l16 = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_pairs = (n_groups + 1) >> 1;
    for (int64_t pair = warp; pair < n_pairs; pair += nwarps) {
        const int64_t f = 2 * pair + sub;
        const bool valid = f < n_groups;
        float v[8], a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { v[i] = 0.0f; a[i] = 1.0f; }
        if (valid) {
            const uint4 raw = ldg_stream(W + f * 16 + l16);
            const int64_t k0 = (f % G) * 128 + 8 * l16;
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(s + k0));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(s + k0) + 1);
            a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
            a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
            load8_scaled(raw, a, v);
        }
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
#pragma unroll
        for (int o = 8; o; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const GroupQuant p = group_params(fminf(mn, 0.0f), fmaxf(mx, 0.0f));
        if (valid) {
            uint32_t out[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float e2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int q = (int)quant_code(v[i + u], p);
                    const float wq = (float)(q - p.z) * p.sf;  // exact: |q - z| <= 15, sf has 11 bits
                    e2[u] = __fdiv_rn(__fsub_rn(wq, v[i + u]), a[i + u]);
                }
                out[i / 2] = pack_half2(e2[0], e2[1]);
            }
            E[f * 16 + l16] = make_uint4(out[0], out[1], out[2], out[3]);
            if (l16 == 0 && p.overflow) record_status(status, W4_ERR_RANGE);
        }
    }
}

// Fixed-order reduction of the per-tile partials, argmin, and the chosen scales.
__global__ void __launch_bounds__(256) awq_finalize_kernel(const double* __restrict__ part, int n_part, int n_alpha,
                                                           double denom, const float* __restrict__ s_all, int K,
                                                           double* __restrict__ mse, int32_t* __restrict__ best_idx,
                                                           float* __restrict__ best_s) {
    __shared__ double red[256];
    __shared__ double vals[64];
    __shared__ int best_sh;
    for (int i = 0; i < n_alpha; ++i) {
        double acc = 0.0;
        for (int p = threadIdx.x; p < n_part; p += blockDim.x) acc += part[(int64_t)i * n_part + p];
        red[threadIdx.x] = acc;
        __syncthreads();
        for (int w = 128; w; w >>= 1) {
            if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
            __syncthreads();
        }
        if (threadIdx.x == 0) vals[i] = red[0] / denom;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        int b = 0;
        for (int i = 0; i < n_alpha; ++i) {
            mse[i] = vals[i];
            if (vals[i] < vals[b]) b = i;
        }
        *best_idx = b;
        best_sh = b;
    }
    __syncthreads();
    const int b = best_sh;
    for (int j = threadIdx.x; j < K; j += blockDim.x) best_s[j] = s_all[(int64_t)b * K + j];
}

// ------------------------------------------------------------------------------------ host side
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

AwqLayout awq_layout(int64_t T, int64_t N, int64_t K, int n_alpha) {
    AwqLayout L;
    L.n_part = tc_sse_partials(T, N);
    size_t off = 0;
    L.colsum = off; off = align256(off + (size_t)K * 8);
    L.s_all = off; off = align256(off + (size_t)n_alpha * K * 4);
    L.E = off; off = align256(off + (size_t)N * K * 2);
    L.part = off; off = align256(off + (size_t)n_alpha * L.n_part * 8);
    L.bytes = off;
    return L;
}

cudaError_t launch_awq(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                       double* mse, int32_t* best_idx, float* best_s, void* ws, int* status, cudaStream_t stream) {
    const AwqLayout L = awq_layout(T, N, K, n_alpha);
    unsigned char* base = static_cast<unsigned char*>(ws);
    auto* colsum = reinterpret_cast<unsigned long long*>(base + L.colsum);
    float* s_all = reinterpret_cast<float*>(base + L.s_all);
    uint16_t* E = reinterpret_cast<uint16_t*>(base + L.E);
    double* part = reinterpret_cast<double*>(base + L.part);

    cudaError_t e = cudaMemsetAsync(colsum, 0, (size_t)K * 8, stream);
    if (e != cudaSuccess) return e;
    {
        const int chunks = (int)(K / 8);
        dim3 grid((chunks + 255) / 256, (unsigned)((T + CA_ROWS - 1) / CA_ROWS));
        colabs_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(X), T, (int)K, colsum);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    awq_scales_kernel<<<n_alpha, 1024, 0, stream>>>(colsum, T, (int)K, n_alpha, s_all);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t G = K / 128;
    const int64_t n_groups = N * G;
    const int64_t want = ((n_groups + 1) / 2 + 7) / 8;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int fq_blocks = (int)(want < cap ? want : cap);
    for (int i = 0; i < n_alpha; ++i) {
        awq_fakequant_kernel<<<fq_blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(W), s_all + (int64_t)i * K,
                                                             n_groups, (int)G, reinterpret_cast<uint4*>(E), status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = launch_tc_sse(X, T, E, N, K, part + (int64_t)i * L.n_part, status, stream);
        if (e != cudaSuccess) return e;
    }
    awq_finalize_kernel<<<1, 256, 0, stream>>>(part, L.n_part, n_alpha, (double)T * (double)N, s_all, (int)K, mse,
                                               best_idx, best_s);
    return cudaGetLastError();
}

// ==================================================================================================
// The search split by calibration rows (one part per rank, or any row partition): every part
// computes its exact column sums and, once the scales are known, its per-alpha sums of squares;
// the parts' column sums add exactly (integers), the parts' sums of squares add in part order.

// sse[i] = the fixed-order sum of alpha i's tile partials (the reduction of awq_finalize_kernel).
__global__ void __launch_bounds__(256) awq_sum_parts_kernel(const double* __restrict__ part, int n_part,
                                                            double* __restrict__ sse) {
    __shared__ double red[256];
    const int i = blockIdx.x;
    double acc = 0.0;
    for (int p = threadIdx.x; p < n_part; p += blockDim.x) acc += part[(int64_t)i * n_part + p];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) sse[i] = red[0];
}

// MSE_i = (sum over parts p, in order, of sse[p][i]) / denom; best = lowest index among the
// minima; best_s = s_all[best].
__global__ void __launch_bounds__(256) awq_select_kernel(const double* __restrict__ sse, int n_parts, int n_alpha,
                                                         double denom, const float* __restrict__ s_all, int K,
                                                         double* __restrict__ mse, int32_t* __restrict__ best_idx,
                                                         float* __restrict__ best_s) {
    __shared__ double vals[64];
    __shared__ int best_sh;
    if (threadIdx.x < n_alpha) {
        double acc = 0.0;
        for (int p = 0; p < n_parts; ++p) acc += sse[(int64_t)p * n_alpha + threadIdx.x];
        vals[threadIdx.x] = acc / denom;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int b = 0;
        for (int i = 0; i < n_alpha; ++i) {
            mse[i] = vals[i];
            if (vals[i] < vals[b]) b = i;
        }
        *best_idx = b;
        best_sh = b;
    }
    __syncthreads();
    const int b = best_sh;
    for (int j = threadIdx.x; j < K; j += blockDim.x) best_s[j] = s_all[(int64_t)b * K + j];
}

cudaError_t launch_awq_colsum(const uint16_t* X, int64_t T, int64_t K, uint64_t* colsum, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(colsum, 0, (size_t)K * 8, stream);
    if (e != cudaSuccess || T == 0) return e;
    const int chunks = (int)(K / 8);
    dim3 grid((chunks + 255) / 256, (unsigned)((T + CA_ROWS - 1) / CA_ROWS));
    colabs_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(X), T, (int)K,
                                            reinterpret_cast<unsigned long long*>(colsum));
    return cudaGetLastError();
}

cudaError_t launch_awq_scales_from_colsum(const uint64_t* colsum, int64_t T_total, int64_t K, int n_alpha,
                                          float* s_all, cudaStream_t stream) {
    awq_scales_kernel<<<n_alpha, 1024, 0, stream>>>(reinterpret_cast<const unsigned long long*>(colsum), T_total,
                                                    (int)K, n_alpha, s_all);
    return cudaGetLastError();
}

AwqSseLayout awq_sse_layout(int64_t T, int64_t N, int64_t K, int n_alpha) {
    AwqSseLayout L;
    L.n_part = tc_sse_partials(T, N);
    size_t off = 0;
    L.E = off; off = align256(off + (size_t)N * K * 2);
    L.part = off; off = align256(off + (size_t)n_alpha * L.n_part * 8);
    L.bytes = off;
    return L;
}

cudaError_t launch_awq_sse(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                           const float* s_all, double* sse, void* ws, int* status, cudaStream_t stream) {
    const AwqSseLayout L = awq_sse_layout(T, N, K, n_alpha);
    unsigned char* base = static_cast<unsigned char*>(ws);
    uint16_t* E = reinterpret_cast<uint16_t*>(base + L.E);
    double* part = reinterpret_cast<double*>(base + L.part);
    cudaError_t e;
    const int64_t G = K / 128;
    const int64_t n_groups = N * G;
    const int64_t want = ((n_groups + 1) / 2 + 7) / 8;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int fq_blocks = (int)(want < cap ? want : cap);
    for (int i = 0; i < n_alpha; ++i) {
        awq_fakequant_kernel<<<fq_blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(W), s_all + (int64_t)i * K,
                                                             n_groups, (int)G, reinterpret_cast<uint4*>(E), status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = launch_tc_sse(X, T, E, N, K, part + (int64_t)i * L.n_part, status, stream);
        if (e != cudaSuccess) return e;
    }
    awq_sum_parts_kernel<<<n_alpha, 256, 0, stream>>>(part, L.n_part, sse);
    return cudaGetLastError();
}

cudaError_t launch_awq_select(const double* sse, int n_parts, int n_alpha, int64_t T_total, int64_t N,
                              const float* s_all, int64_t K, double* mse, int32_t* best_idx, float* best_s,
                              cudaStream_t stream) {
    awq_select_kernel<<<1, 256, 0, stream>>>(sse, n_parts, n_alpha, (double)T_total * (double)N, s_all, (int)K, mse,
                                             best_idx, best_s);
    return cudaGetLastError();
}

// ==================================================================================================
// Gram form of the same search.  sum_{t,n} (X E_i^T)^2 = sum_n e_n^T G e_n with G = X^T X, so the T
// calibration rows are read once: G on the tensor cores, then per alpha one GEMM over K x K instead
// of T x K.  G is formed chunk by chunk: each chunk of at most GRAM_CHUNK rows is one fp32
// tensor-core product (the same accumulation length as the direct form's K-long dot products; with
// one fp32 accumulator over all 65536 calibration rows the two forms differed by a uniform 4e-4
// relative), and the chunks are summed in fp64 in chunk order.  G carries the squared activations' dynamic range (beyond
// fp16), so it is scaled symmetrically: d_k = sqrt(G_kk) (1 for a channel that is zero in every
// row), G' = D^-1 G D^-1 with entries in [-1, 1] in fp16, and E'_i = E_i D in fp16, so that
// e^T G e = e'^T G' e'.  The per-alpha GEMM E' G'^T has an epilogue that sums (E' G'^T)[n, k] E'[n, k]
// per tile; MSE_i = (fixed-order sum of the tile partials) / (T N), exactly as in the direct form.

constexpr int64_t GRAM_CHUNK = 4096;

// Rows per chunk: all of T (padded to a multiple of 64) when T fits one chunk.
static int64_t gram_chunk_rows(int64_t T) {
    const int64_t Tp = (T + 63) / 64 * 64;
    return Tp < GRAM_CHUNK ? Tp : GRAM_CHUNK;
}

// XT holds X^T chunk by chunk: chunk c is a [K, L] row-major block of rows t in [cL, cL + L), rows
// t >= T zero (L % 64 == 0: whole K-steps for the GEMM).  A CTA moves one 64 (t) x 64 (k) tile
// with 16-byte loads and stores: each thread loads 8 consecutive k of one t, scatters them into a
// [k][t] shared tile whose 16-byte chunks are XOR-swizzled by k / 8 (the 2-byte stores of a warp
// and the 16-byte loads of a quarter warp both hit distinct banks), then stores 8 consecutive t of
// one k.
constexpr int TP_TILE = 64;
__global__ void __launch_bounds__(256) transpose_pad_kernel(const uint4* __restrict__ X, int64_t T, int K,
                                                            int64_t L, int64_t Tp, uint4* __restrict__ XT) {
    __shared__ __align__(16) unsigned short tile[TP_TILE * TP_TILE];
    const int64_t t0 = (int64_t)blockIdx.x * TP_TILE;
    const int k0 = blockIdx.y * TP_TILE;
    const int64_t kc8 = K / 8;  // 16-byte chunks per row of X
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
        const int idx = threadIdx.x + rep * 256;
        const int tl = idx >> 3, kq = idx & 7;  // tile row (t) and its 8-k chunk
        const int64_t t = t0 + tl;
        const uint4 v = t < T ? ldg_stream(X + t * kc8 + (k0 >> 3) + kq) : make_uint4(0u, 0u, 0u, 0u);
        const unsigned short* h = reinterpret_cast<const unsigned short*>(&v);
        const int chunk = (tl >> 3) ^ kq;  // k / 8 == kq for all eight k of this chunk
#pragma unroll
        for (int j = 0; j < 8; ++j) tile[(kq * 8 + j) * TP_TILE + chunk * 8 + (tl & 7)] = h[j];
    }
    __syncthreads();
#pragma unroll
    for (int rep = 0; rep < 2; ++rep) {
        const int idx = threadIdx.x + rep * 256;
        const int kr = idx >> 3, tq = idx & 7;  // tile row (k) and its 8-t chunk
        const uint4 v = *reinterpret_cast<const uint4*>(tile + kr * TP_TILE + ((tq ^ (kr >> 3)) * 8));
        const int64_t t = t0 + tq * 8;  // eight consecutive t, all in one chunk (L % 64 == 0)
        if (t < Tp) {
            const int64_t c = t / L, tt = t - c * L;
            XT[((c * K + k0 + kr) * L + tt) / 8] = v;
        }
    }
}

// G64 = Gc (first chunk) or G64 += Gc in fp64, on and below the diagonal (row i, columns j <= i;
// lower = 0: every entry).  One block row of the grid per row of G.
__global__ void gram_accumulate_kernel(const float* __restrict__ Gc, int K, bool first, int lower,
                                       double* __restrict__ G64) {
    pdl_launch_dependents();  // the next chunk's product (other Gc buffer) may start beside this
    for (int i = blockIdx.x; i < K; i += gridDim.x) {
        const int jn = lower ? i + 1 : K;
        const int64_t r = (int64_t)i * K;
        for (int j = threadIdx.x; j < jn; j += blockDim.x)
            G64[r + j] = first ? (double)Gc[r + j] : G64[r + j] + (double)Gc[r + j];
    }
}

// d_k = sqrt(G_kk) (1 when G_kk is 0) and rd = 1 / d, from the fp64 G rounded once to fp32.
__global__ void gram_diag_kernel(const double* __restrict__ G64, int K, float* __restrict__ d, float* __restrict__ rd) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const double g = G64[(int64_t)k * K + k];
    const float dk = g > 0.0 ? __double2float_rn(sqrt(g)) : 1.0f;
    d[k] = dk;
    rd[k] = __frcp_rn(dk);
}

// G' = D^-1 G D^-1 in fp16, every entry; with `lower` only G's lower triangle holds values and
// entry (i, j) above the diagonal is read as its mirror (j, i), which makes G' exactly symmetric.
__global__ void gram_scale_kernel(const double* __restrict__ G64, const float* __restrict__ rd, int K, int lower,
                                  __half* __restrict__ Gp) {
    const int64_t n = (int64_t)K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / K), j = (int)(e - (int64_t)i * K);
        const double g = (lower && j > i) ? G64[(int64_t)j * K + i] : G64[e];
        Gp[e] = __double2half(g * (double)rd[i] * (double)rd[j]);
    }
}

// E' = ((Wq - W*s) / s) * d in fp16 for one alpha; the codes are those of w4_quantize_pack(W, s).
__global__ void __launch_bounds__(256) awq_fakequant_scaled_kernel(const uint4* __restrict__ W,
                                                                   const float* __restrict__ s,
                                                                   const float* __restrict__ dmul, int64_t n_groups,
                                                                   int G, uint4* __restrict__ E, int* status) {
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 4, l16 = lane & 15;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t n_pairs = (n_groups + 1) >> 1;
    for (int64_t pair = warp; pair < n_pairs; pair += nwarps) {
        const int64_t f = 2 * pair + sub;
        const bool valid = f < n_groups;
        float v[8], a[8], dm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { v[i] = 0.0f; a[i] = 1.0f; dm[i] = 1.0f; }
        if (valid) {
            const uint4 raw = ldg_stream(W + f * 16 + l16);
            const int64_t k0 = (f % G) * 128 + 8 * l16;
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(s + k0));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(s + k0) + 1);
            const float4 d0 = __ldg(reinterpret_cast<const float4*>(dmul + k0));
            const float4 d1 = __ldg(reinterpret_cast<const float4*>(dmul + k0) + 1);
            a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
            a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
            dm[0] = d0.x; dm[1] = d0.y; dm[2] = d0.z; dm[3] = d0.w;
            dm[4] = d1.x; dm[5] = d1.y; dm[6] = d1.z; dm[7] = d1.w;
            load8_scaled(raw, a, v);
        }
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
#pragma unroll
        for (int o = 8; o; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const GroupQuant p = group_params(fminf(mn, 0.0f), fmaxf(mx, 0.0f));
        if (valid) {
            uint32_t out[4];
            bool bad = false;
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float e2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int q = (int)quant_code(v[i + u], p);
                    const float wq = (float)(q - p.z) * p.sf;  // exact: |q - z| <= 15, sf has 11 bits
                    e2[u] = __fmul_rn(__fdiv_rn(__fsub_rn(wq, v[i + u]), a[i + u]), dm[i + u]);
                    if (!(fabsf(e2[u]) <= 65504.0f)) bad = true;  // E' beyond fp16: the MSE would be inf
                }
                out[i / 2] = pack_half2(e2[0], e2[1]);
            }
            E[f * 16 + l16] = make_uint4(out[0], out[1], out[2], out[3]);
            if ((l16 == 0 && p.overflow) || bad) record_status(status, W4_ERR_RANGE);
        }
    }
    // Launched as a programmatic dependent of the previous alpha's contraction (which reads the
    // other E buffer): end only after it, so that the next contraction follows both.
    pdl_wait();
}

AwqGramLayout awq_gram_layout(int64_t T, int64_t N, int64_t K, int n_alpha) {
    AwqGramLayout L;
    L.chunk = gram_chunk_rows(T);
    L.n_chunks = (T + L.chunk - 1) / L.chunk;
    L.Tp = L.chunk * L.n_chunks;
    L.n_part = tc_sse_partials(N, K);
    size_t off = 0;
    L.colsum = off; off = align256(off + (size_t)K * 8);
    L.s_all = off; off = align256(off + (size_t)n_alpha * K * 4);
    L.E = off; off = align256(off + 2 * (size_t)N * K * 2);  // two buffers: alpha i writes E[i % 2]
    L.part = off; off = align256(off + (size_t)n_alpha * L.n_part * 8);
    L.XT = off; off = align256(off + (size_t)K * (size_t)L.Tp * 2);
    L.G = off; off = align256(off + 2 * (size_t)K * K * 4);  // two buffers: chunk c writes G[c % 2]
    L.G64 = off; off = align256(off + (size_t)K * K * 8);
    L.Gp = off; off = align256(off + (size_t)K * K * 2);
    L.d = off; off = align256(off + (size_t)K * 4);
    L.rd = off; off = align256(off + (size_t)K * 4);
    L.bytes = off;
    return L;
}

cudaError_t launch_awq_gram(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                            double* mse, int32_t* best_idx, float* best_s, void* ws, int* status,
                            cudaStream_t stream) {
    const AwqGramLayout L = awq_gram_layout(T, N, K, n_alpha);
    unsigned char* base = static_cast<unsigned char*>(ws);
    auto* colsum = reinterpret_cast<unsigned long long*>(base + L.colsum);
    float* s_all = reinterpret_cast<float*>(base + L.s_all);
    uint16_t* E = reinterpret_cast<uint16_t*>(base + L.E);
    double* part = reinterpret_cast<double*>(base + L.part);
    uint16_t* XT = reinterpret_cast<uint16_t*>(base + L.XT);
    float* Gc = reinterpret_cast<float*>(base + L.G);
    double* G64 = reinterpret_cast<double*>(base + L.G64);
    __half* Gp = reinterpret_cast<__half*>(base + L.Gp);
    float* d = reinterpret_cast<float*>(base + L.d);
    float* rd = reinterpret_cast<float*>(base + L.rd);

    cudaError_t e = cudaMemsetAsync(colsum, 0, (size_t)K * 8, stream);
    if (e != cudaSuccess) return e;
    {
        const int chunks = (int)(K / 8);
        dim3 grid((chunks + 255) / 256, (unsigned)((T + CA_ROWS - 1) / CA_ROWS));
        colabs_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(X), T, (int)K, colsum);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    awq_scales_kernel<<<n_alpha, 1024, 0, stream>>>(colsum, T, (int)K, n_alpha, s_all);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    transpose_pad_kernel<<<dim3((unsigned)(L.Tp / TP_TILE), (unsigned)(K / TP_TILE)), 256, 0, stream>>>(
        reinterpret_cast<const uint4*>(X), T, (int)K, L.chunk, L.Tp, reinterpret_cast<uint4*>(XT));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const unsigned ew_blocks = (unsigned)device_sm_count() * 8;
    // G is symmetric: for K > 128 only the 256 x 256 tiles on and below the diagonal are formed
    // (half the tensor-core work, one wave at K = 4096), accumulated and read back mirrored.
    const int lower = K > 128 ? 1 : 0;
    // G = sum over chunks of X_c^T X_c.  Chunk c's product goes to Gc[c % 2]; from c = 1 on it is
    // launched as a programmatic dependent of chunk c - 1's fp64 accumulation, so the tensor-core
    // product and the memory-bound accumulation of the previous chunk overlap; the product's grid
    // ends after that accumulation, so chunk c's accumulation (a plain launch) follows both.
    for (int64_t c = 0; c < L.n_chunks; ++c) {
        const uint16_t* XTc = XT + c * K * L.chunk;
        float* Gcc = Gc + (c & 1) * K * K;
        e = lower ? launch_tc_f32_lower(XTc, K, L.chunk, Gcc, status, stream, c > 0)
                  : launch_tc_f32(XTc, K, XTc, K, L.chunk, Gcc, status, stream, c > 0);
        if (e != cudaSuccess) return e;
        gram_accumulate_kernel<<<(unsigned)(K < 4096 ? K : 4096), 256, 0, stream>>>(Gcc, (int)K, c == 0, lower, G64);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    gram_diag_kernel<<<(unsigned)((K + 255) / 256), 256, 0, stream>>>(G64, (int)K, d, rd);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gram_scale_kernel<<<ew_blocks, 256, 0, stream>>>(G64, rd, (int)K, lower, Gp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t G = K / 128;
    const int64_t n_groups = N * G;
    const int64_t want = ((n_groups + 1) / 2 + 7) / 8;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int fq_blocks = (int)(want < cap ? want : cap);
    // alpha i's errors go to E[i % 2]; from i = 1 on the fake-quantiser is a programmatic
    // dependent of alpha i - 1's contraction (which reads the other buffer), so it runs beside it.
    for (int i = 0; i < n_alpha; ++i) {
        uint16_t* Ei = E + (int64_t)(i & 1) * N * K;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)fq_blocks, 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = i > 0 ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, awq_fakequant_scaled_kernel, reinterpret_cast<const uint4*>(W),
                               (const float*)(s_all + (int64_t)i * K), (const float*)d, n_groups, (int)G,
                               reinterpret_cast<uint4*>(Ei), status);
        if (e != cudaSuccess) return e;
        e = launch_tc_dot(Ei, N, reinterpret_cast<const uint16_t*>(Gp), K, K, part + (int64_t)i * L.n_part, status,
                          stream);
        if (e != cudaSuccess) return e;
    }
    awq_finalize_kernel<<<1, 256, 0, stream>>>(part, L.n_part, n_alpha, (double)T * (double)N, s_all, (int)K, mse,
                                               best_idx, best_s);
    return cudaGetLastError();
}

}  // namespace w4
