// GPTQ quantiser emitting the library's packed INT4 format (codes, fp16 scales, 4-bit zero points).
//
// "GPTQ, AWQ and the rules of post-training quantization", section "GPTQ: pay for the error with
// the other weights": columns are quantised in a fixed order; each column's rounding error is
// absorbed by the columns still unquantised, weighted by the inverse of H = X^T X through a
// Cholesky factor, and the updates of far columns are batched per block.
//
// Arithmetic (fp64 except the quantiser's decisions, which are w4_quantize_pack's fp32 rules with
// L = 2^b - 1 steps for b-bit codes):
//   scale  = optionally AWQ's per-channel scale s first: X / s and W * s in fp64 replace X and W
//            ("GPTQ, AWQ and the rules of post-training quantization", section "What
//            activation-awareness buys and what it does not": the scaling goes before GPTQ)
//   perm   = the processing order: identity, or with act-order (desc_act, "AutoGPTQ vs The Stack
//            v2") the columns by decreasing diag(X^T X), ties in index order; H, W and the outputs
//            are taken in that order (the outputs are stored in processing order with perm)
//   H      = X^T X + lambda I,  lambda = damp * mean(diag(X^T X))
//   U      = upper triangular with H^-1 = U^T U.  With J the index reversal, chol(J H J) = L lower
//            gives H = (J L J)(J L J)^T with J L J upper, hence U = (J L J)^-1 = J L^-1 J: one
//            Cholesky and one triangular inverse, no explicit H^-1.
//   sweep  for every block of `group` columns (= one quantisation group):
//            group scale/zero from the block's current weights rounded to fp32 (RTN rule);
//            for each column k of the block, in order:
//              q_k = RTN code of fp32(w_k); e_k = (w_k - (q_k - z) s) / U_kk;
//              w_j -= e_k U_kj for the block's columns j > k;
//            then the columns right of the block: W[:, j] -= sum_k e_k U_kj  (one fp64 product).
//
// Kernels, all plain fp64 CUDA-core code (the tensor cores have no fp64 path on sm_100a beyond
// the legacy DMMA, and this step is a one-off per layer): a Gram kernel for H, a blocked
// right-looking Cholesky (32-wide panels: diagonal factor, panel solve, trailing update), a
// blocked triangular inverse, one warp per weight row for the column sweep, and a tiled
// trailing update.  Every launch is on the caller's stream; results are deterministic.
#include "common.cuh"
#include "internal.h"
#include "quant_bits.cuh"

namespace w4 {

constexpr int CH_NB = 32;  // Cholesky / inverse panel width
// A sweep block is one quantisation group (64 or 128 columns).

// ------------------------------------------------------------------------------ H = X^T X (fp64)
// One 64 x 64 tile of H per CTA (lower tiles only; each writes its mirror too).  256 threads, 4 x 4
// outputs each; X rows staged 16 at a time as fp64 (divided by the activation scale s in fp64 when
// one is given).  Every sum runs over t in increasing order, so H[i][j] and H[j][i] are the same
// bits.
constexpr int GM_T = 16;
__global__ void __launch_bounds__(256) gptq_gram_kernel(const __half* __restrict__ X, int64_t T, int K,
                                                        const float* __restrict__ s, double* __restrict__ H) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    __shared__ double xi[GM_T][64 + 1];
    __shared__ double xj[GM_T][64 + 1];
    const int tid = threadIdx.x;
    const int r = tid >> 4, c = tid & 15;
    const int i0 = ti * 64, j0 = tj * 64;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int64_t t0 = 0; t0 < T; t0 += GM_T) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = tid + 256 * u;  // 0..1023 = 16 rows x 64 columns
            const int row = e >> 6, col = e & 63;
            const int64_t t = t0 + row;
            const bool ok = t < T;
            double vi = ok && i0 + col < K ? (double)__half2float(X[t * K + i0 + col]) : 0.0;
            double vj = ok && j0 + col < K ? (double)__half2float(X[t * K + j0 + col]) : 0.0;
            if (s) {
                if (i0 + col < K) vi = __ddiv_rn(vi, (double)s[i0 + col]);
                if (j0 + col < K) vj = __ddiv_rn(vj, (double)s[j0 + col]);
            }
            xi[row][col] = vi;
            xj[row][col] = vj;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < GM_T; ++tt) {
            double a4[4], b4[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) a4[a] = xi[tt][r + 16 * a];
#pragma unroll
            for (int b = 0; b < 4; ++b) b4[b] = xj[tt][c + 16 * b];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fma(a4[a], b4[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int i = i0 + r + 16 * a, j = j0 + c + 16 * b;
            if (i < K && j < K) {
                H[(int64_t)i * K + j] = acc[a][b];
                H[(int64_t)j * K + i] = acc[a][b];
            }
        }
}

// lambda = damp * mean(diag H): one CTA, each thread a strided partial sum, then a fixed tree.
__global__ void __launch_bounds__(1024) gptq_damp_kernel(const double* __restrict__ H, int K, double damp,
                                                         double* __restrict__ lambda) {
    __shared__ double part[1024];
    double s = 0.0;
    for (int k = threadIdx.x; k < K; k += 1024) s += H[(int64_t)k * K + k];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *lambda = damp * (part[0] / (double)K);
}

// Act-order: perm[rank] = i, rank = the number of columns before i in decreasing diag(H) with
// ties in index order (NaN counts as -inf, so the order is total and perm a permutation).
__global__ void gptq_perm_kernel(const double* __restrict__ H, int K, int32_t* __restrict__ perm) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= K) return;
    auto key = [&](int k) {
        const double d = H[(int64_t)k * K + k];
        return d != d ? -INFINITY : d;
    };
    const double di = key(i);
    int rank = 0;
    for (int j = 0; j < K; ++j) {
        const double dj = key(j);
        rank += (dj > di || (dj == di && j < i)) ? 1 : 0;
    }
    perm[rank] = i;
}

// P = J H_p J + lambda I with H_p = H[perm][:, perm] (perm null: identity), i.e.
// P[i][j] = H[perm[K-1-i]][perm[K-1-j]].
__global__ void gptq_reverse_kernel(const double* __restrict__ H, int K, const int32_t* __restrict__ perm,
                                    const double* __restrict__ lambda, double* __restrict__ P) {
    const int64_t n = (int64_t)K * K;
    const double lam = *lambda;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / K), j = (int)(e - (int64_t)i * K);
        const int a = perm ? perm[K - 1 - i] : K - 1 - i;
        const int b = perm ? perm[K - 1 - j] : K - 1 - j;
        const double h = H[(int64_t)a * K + b];
        P[e] = i == j ? h + lam : h;
    }
}

// ------------------------------------------------------------------ Cholesky P = L L^T, in place
// (a) the 32 x 32 diagonal block at kb: one thread per element, one column per step.
__global__ void __launch_bounds__(CH_NB* CH_NB) chol_diag_kernel(double* __restrict__ P, int K, int kb,
                                                                 int* status) {
    __shared__ double D[CH_NB][CH_NB + 1];
    const int i = threadIdx.x / CH_NB, j = threadIdx.x % CH_NB;
    D[i][j] = i >= j ? P[(int64_t)(kb + i) * K + kb + j] : 0.0;
    __syncthreads();
    for (int c = 0; c < CH_NB; ++c) {
        if (i == c && j == c) {
            double d = D[c][c];
            if (!(d > 0.0)) {  // not positive definite (or NaN): report, keep values finite
                record_status(status, W4_ERR_NUMERIC);
                d = 1.0;
            }
            D[c][c] = sqrt(d);
        }
        __syncthreads();
        if (j == c && i > c) D[i][c] = D[i][c] / D[c][c];
        __syncthreads();
        if (j > c && i >= j) D[i][j] = D[i][j] - D[i][c] * D[j][c];
        __syncthreads();
    }
    if (i >= j) P[(int64_t)(kb + i) * K + kb + j] = D[i][j];
}

// (b) rows below the block: x L_kk^T = a by forward substitution, one thread per row.
__global__ void __launch_bounds__(128) chol_panel_kernel(double* __restrict__ P, int K, int kb) {
    __shared__ double Lk[CH_NB][CH_NB + 1];
    for (int e = threadIdx.x; e < CH_NB * CH_NB; e += blockDim.x) {
        const int a = e / CH_NB, b = e % CH_NB;
        Lk[a][b] = a >= b ? P[(int64_t)(kb + a) * K + kb + b] : 0.0;
    }
    __syncthreads();
    const int64_t row = (int64_t)kb + CH_NB + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= K) return;
    double* prow = P + row * K + kb;
    double x[CH_NB];
#pragma unroll
    for (int c = 0; c < CH_NB; ++c) x[c] = prow[c];
#pragma unroll
    for (int c = 0; c < CH_NB; ++c) {
        double s = x[c];
#pragma unroll
        for (int c2 = 0; c2 < c; ++c2) s -= x[c2] * Lk[c][c2];
        x[c] = s / Lk[c][c];
    }
#pragma unroll
    for (int c = 0; c < CH_NB; ++c) prow[c] = x[c];
}

// (c) trailing lower triangle: P[i][j] -= sum_c P[i][kb+c] P[j][kb+c] for i >= j >= kb + 32.
// 64 x 64 tiles on a square grid over the trailing part; tiles above the diagonal return.
__global__ void __launch_bounds__(256) chol_update_kernel(double* __restrict__ P, int K, int kb) {
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    const int e0 = kb + CH_NB;
    const int i0 = e0 + ti * 64, j0 = e0 + tj * 64;
    __shared__ double ai[64][CH_NB + 1];
    __shared__ double aj[64][CH_NB + 1];
    const int tid = threadIdx.x;
    for (int e = tid; e < 64 * CH_NB; e += 256) {
        const int rr = e / CH_NB, cc = e % CH_NB;
        ai[rr][cc] = i0 + rr < K ? P[(int64_t)(i0 + rr) * K + kb + cc] : 0.0;
        aj[rr][cc] = j0 + rr < K ? P[(int64_t)(j0 + rr) * K + kb + cc] : 0.0;
    }
    __syncthreads();
    const int r = tid >> 4, c = tid & 15;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
#pragma unroll 4
    for (int cc = 0; cc < CH_NB; ++cc) {
        double a4[4], b4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) a4[a] = ai[r + 16 * a][cc];
#pragma unroll
        for (int b = 0; b < 4; ++b) b4[b] = aj[c + 16 * b][cc];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = fma(a4[a], b4[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int i = i0 + r + 16 * a, j = j0 + c + 16 * b;
            if (i < K && j <= i) P[(int64_t)i * K + j] -= acc[a][b];
        }
}

// ------------------------------------------------------------- Li = L^-1 (lower), blocked by 32
// (a) every diagonal block's inverse, one CTA per block, one thread per column (forward
// substitution on the identity's column).
__global__ void __launch_bounds__(CH_NB) trinv_diag_kernel(const double* __restrict__ L, int K,
                                                           double* __restrict__ Li) {
    __shared__ double Lb[CH_NB][CH_NB + 1];
    __shared__ double Xb[CH_NB][CH_NB + 1];
    const int b0 = blockIdx.x * CH_NB;
    const int j = threadIdx.x;
    for (int i = 0; i < CH_NB; ++i) Lb[i][j] = i >= j ? L[(int64_t)(b0 + i) * K + b0 + j] : 0.0;
    __syncthreads();
    for (int i = 0; i < CH_NB; ++i) {
        double x = 0.0;
        if (i >= j) {
            double s = i == j ? 1.0 : 0.0;
            for (int c = j; c < i; ++c) s -= Lb[i][c] * Xb[c][j];
            x = s / Lb[i][i];
        }
        Xb[i][j] = x;  // column j is read and written by thread j only
    }
    for (int i = 0; i < CH_NB; ++i) Li[(int64_t)(b0 + i) * K + b0 + j] = Xb[i][j];
}

// (b) block row bi (> 0): Li[bi][bj] = -Li[bi][bi] * sum_{c = bj}^{bi-1} L[bi][c] Li[c][bj], one CTA
// per block column bj < bi.  Reads only block rows < bi and the diagonal block of Li.
__global__ void __launch_bounds__(256) trinv_row_kernel(const double* __restrict__ L, int K, int bi,
                                                        double* __restrict__ Li) {
    const int bj = blockIdx.x;
    __shared__ double la[CH_NB][CH_NB + 1];
    __shared__ double lb[CH_NB][CH_NB + 1];
    const int tid = threadIdx.x;
    const int r = tid >> 3, c0 = tid & 7;  // row r, columns c0 + 8 m
    const int64_t ri = (int64_t)bi * CH_NB;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int bc = bj; bc < bi; ++bc) {
        for (int e = tid; e < CH_NB * CH_NB; e += 256) {
            const int a = e / CH_NB, b = e % CH_NB;
            la[a][b] = L[(ri + a) * K + (int64_t)bc * CH_NB + b];
            lb[a][b] = Li[((int64_t)bc * CH_NB + a) * K + (int64_t)bj * CH_NB + b];
        }
        __syncthreads();
#pragma unroll 8
        for (int cc = 0; cc < CH_NB; ++cc) {
            const double x = la[r][cc];
#pragma unroll
            for (int m = 0; m < 4; ++m) acc[m] = fma(x, lb[cc][c0 + 8 * m], acc[m]);
        }
        __syncthreads();
    }
    // Li[bi][bj] = -Li_ii * T with T = acc
#pragma unroll
    for (int m = 0; m < 4; ++m) lb[r][c0 + 8 * m] = acc[m];
    for (int e = tid; e < CH_NB * CH_NB; e += 256) {
        const int a = e / CH_NB, b = e % CH_NB;
        la[a][b] = Li[(ri + a) * K + ri + b];
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int cc = c0 + 8 * m;
        double s = 0.0;
        for (int k = 0; k <= r; ++k) s = fma(la[r][k], lb[k][cc], s);  // Li_ii is lower triangular
        Li[(ri + r) * K + (int64_t)bj * CH_NB + cc] = -s;
    }
}

// U[i][j] = Li[K-1-i][K-1-j].
__global__ void gptq_u_kernel(const double* __restrict__ Li, int K, double* __restrict__ U) {
    const int64_t n = (int64_t)K * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / K), j = (int)(e - (int64_t)i * K);
        U[e] = Li[(int64_t)(K - 1 - i) * K + (K - 1 - j)];
    }
}

// W64[n][i] = W[n][c] * s[c] in fp64 with c = perm[i] (perm null: identity; s null: 1).  The
// product of an fp16 and an fp32 value is exact in fp64.
__global__ void gptq_w_init_kernel(const __half* __restrict__ W, int64_t N, int K, const int32_t* __restrict__ perm,
                                   const float* __restrict__ s, double* __restrict__ W64) {
    const int64_t total = N * K;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = e / K;
        const int i = (int)(e - n * K);
        const int c = perm ? perm[i] : i;
        const double w = (double)__half2float(W[n * K + c]);
        W64[e] = s ? w * (double)s[c] : w;
    }
}

// --------------------------------------------------------------------------------- column sweep
// One warp per weight row over the GROUP columns of block b.  Lane l holds columns 32 s + l of the
// block (s < GROUP / 32); column k's value is broadcast from its lane, every lane takes the same
// fp32 decision, and each lane updates its own later columns.
constexpr int SW_WARPS = 8;
template <int GROUP>
__global__ void __launch_bounds__(SW_WARPS * 32) gptq_sweep_kernel(double* __restrict__ W64, int N, int K, int b,
                                                                   int bits, const double* __restrict__ U,
                                                                   uint32_t* __restrict__ packed,
                                                                   __half* __restrict__ scales,
                                                                   uint8_t* __restrict__ zeros,
                                                                   double* __restrict__ E, int* status) {
    constexpr int V = GROUP / 32;
    __shared__ uint8_t codes[SW_WARPS][GROUP];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * SW_WARPS + warp;
    if (n >= N) return;  // whole warps only: nothing below synchronises across warps
    const int L = (1 << bits) - 1;
    double* wrow = W64 + (int64_t)n * K + b;
    double w[V];
#pragma unroll
    for (int s = 0; s < V; ++s) w[s] = wrow[32 * s + lane];
    float lo = 0.0f, hi = 0.0f;  // zero-inclusive range of the block's fp32 values
#pragma unroll
    for (int s = 0; s < V; ++s) {
        const float v = __double2float_rn(w[s]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const GroupQuant p = group_params_steps(lo, hi, L);
    const double sd = (double)p.sf;
    double ek[V];
    int qk[V];
#pragma unroll
    for (int s = 0; s < V; ++s) {
        ek[s] = 0.0;
        qk[s] = 0;
    }
#pragma unroll
    for (int s = 0; s < V; ++s) {
        for (int kk = 0; kk < 32; ++kk) {
            const int k = 32 * s + kk;  // column within the block
            const double wk = __shfl_sync(0xffffffffu, w[s], kk);
            const int q = quant_code_steps(__double2float_rn(wk), p, L);  // the quantiser's fp32 decision
            const double wh = (double)(q - p.z) * sd;
            const int64_t kg = (int64_t)b + k;
            const double e = __ddiv_rn(__dsub_rn(wk, wh), U[kg * K + kg]);
            if (lane == kk) {
                qk[s] = q;
                ek[s] = e;
            }
            const double* urow = U + kg * K + b;
#pragma unroll
            for (int s2 = s; s2 < V; ++s2) {
                const int j = 32 * s2 + lane;
                if (j > k) w[s2] = __dsub_rn(w[s2], __dmul_rn(e, urow[j]));
            }
        }
    }
#pragma unroll
    for (int s = 0; s < V; ++s) {
        codes[warp][32 * s + lane] = (uint8_t)qk[s];
        E[(int64_t)n * GROUP + 32 * s + lane] = ek[s];
    }
    __syncwarp();
    const int G = K / GROUP;
    const int nwords = GROUP * bits / 32;
    if (lane < nwords)
        packed[(int64_t)n * ((int64_t)K * bits / 32) + (int64_t)(b / GROUP) * nwords + lane] =
            stream_word(codes[warp], bits, lane);
    if (lane == 0) {
        scales[(int64_t)n * G + b / GROUP] = p.s16;
        zeros[(int64_t)n * G + b / GROUP] = (uint8_t)p.z;
        if (p.overflow) record_status(status, W4_ERR_RANGE);
    }
}

// W64[n][j] -= sum_{c < group} E[n][c] U[b + c][j] for j >= b + group: 64 x 64 output tiles, the
// sum in increasing c.
__global__ void __launch_bounds__(256) gptq_trailing_kernel(double* __restrict__ W64, int N, int K, int b, int group,
                                                            const double* __restrict__ E,
                                                            const double* __restrict__ U) {
    const int j0 = b + group + blockIdx.x * 64;
    const int n0 = blockIdx.y * 64;
    __shared__ double es[64][32 + 1];
    __shared__ double us[32][64 + 1];
    const int tid = threadIdx.x;
    const int r = tid >> 4, c = tid & 15;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.0;
    for (int c0 = 0; c0 < group; c0 += 32) {
        for (int e = tid; e < 64 * 32; e += 256) {
            const int rr = e >> 5, cc = e & 31;
            es[rr][cc] = n0 + rr < N ? E[(int64_t)(n0 + rr) * group + c0 + cc] : 0.0;
            const int ur = e >> 6, uc = e & 63;
            us[ur][uc] = j0 + uc < K ? U[(int64_t)(b + c0 + ur) * K + j0 + uc] : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int cc = 0; cc < 32; ++cc) {
            double a4[4], b4[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) a4[a] = es[r + 16 * a][cc];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) b4[bb] = us[cc][c + 16 * bb];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fma(a4[a], b4[bb], acc[a][bb]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
            const int n = n0 + r + 16 * a, j = j0 + c + 16 * bb;
            if (n < N && j < K) W64[(int64_t)n * K + j] -= acc[a][bb];
        }
}

// ------------------------------------------------------------------------------------ host side
static size_t gq_align(size_t x) { return (x + 255) & ~(size_t)255; }

GptqLayout gptq_layout(int64_t N, int64_t K) {
    GptqLayout L;
    size_t off = 0;
    L.H = off; off = gq_align(off + (size_t)K * K * 8);
    L.P = off; off = gq_align(off + (size_t)K * K * 8);
    L.W64 = off; off = gq_align(off + (size_t)N * K * 8);
    L.E = off; off = gq_align(off + (size_t)N * 128 * 8);
    L.perm = off; off = gq_align(off + (size_t)K * 4);
    L.lambda = off; off = gq_align(off + 8);
    L.bytes = off;
    return L;
}

cudaError_t launch_gptq(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int bits, int group,
                        double damp, bool act_order, const float* act_scale, uint32_t* packed, uint16_t* scales,
                        uint8_t* zeros, int32_t* perm_out, void* ws, int* status, cudaStream_t stream) {
    const GptqLayout Lo = gptq_layout(N, K);
    unsigned char* base = static_cast<unsigned char*>(ws);
    double* H = reinterpret_cast<double*>(base + Lo.H);   // H, later L^-1
    double* P = reinterpret_cast<double*>(base + Lo.P);   // J H_p J + lambda I, then L, then U
    double* W64 = reinterpret_cast<double*>(base + Lo.W64);
    double* E = reinterpret_cast<double*>(base + Lo.E);
    int32_t* perm = act_order ? reinterpret_cast<int32_t*>(base + Lo.perm) : nullptr;
    double* lambda = reinterpret_cast<double*>(base + Lo.lambda);
    const int k = (int)K, n = (int)N;
    const unsigned ew = (unsigned)device_sm_count() * 8;
    cudaError_t e;
    {
        const unsigned tiles = (unsigned)((K + 63) / 64);
        gptq_gram_kernel<<<dim3(tiles, tiles), 256, 0, stream>>>(reinterpret_cast<const __half*>(X), T, k, act_scale,
                                                                 H);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    gptq_damp_kernel<<<1, 1024, 0, stream>>>(H, k, damp, lambda);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (perm) {
        gptq_perm_kernel<<<(unsigned)((K + 255) / 256), 256, 0, stream>>>(H, k, perm);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (perm_out && (e = cudaMemcpyAsync(perm_out, perm, (size_t)K * 4, cudaMemcpyDeviceToDevice, stream)) !=
                            cudaSuccess)
            return e;
    }
    gptq_reverse_kernel<<<ew, 256, 0, stream>>>(H, k, perm, lambda, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    for (int kb = 0; kb < k; kb += CH_NB) {
        chol_diag_kernel<<<1, CH_NB * CH_NB, 0, stream>>>(P, k, kb, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int rest = k - kb - CH_NB;
        if (rest <= 0) break;
        chol_panel_kernel<<<(unsigned)((rest + 127) / 128), 128, 0, stream>>>(P, k, kb);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const unsigned t = (unsigned)((rest + 63) / 64);
        chol_update_kernel<<<dim3(t, t), 256, 0, stream>>>(P, k, kb);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // L^-1 into H's buffer (its upper triangle must read as zero)
    if ((e = cudaMemsetAsync(H, 0, (size_t)K * K * 8, stream)) != cudaSuccess) return e;
    trinv_diag_kernel<<<(unsigned)(K / CH_NB), CH_NB, 0, stream>>>(P, k, H);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    for (int bi = 1; bi < k / CH_NB; ++bi) {
        trinv_row_kernel<<<(unsigned)bi, 256, 0, stream>>>(P, k, bi, H);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    gptq_u_kernel<<<ew, 256, 0, stream>>>(H, k, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    gptq_w_init_kernel<<<ew, 256, 0, stream>>>(reinterpret_cast<const __half*>(W), N, k, perm, act_scale, W64);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    __half* sc = reinterpret_cast<__half*>(scales);
    const unsigned sweep_blocks = (unsigned)((N + SW_WARPS - 1) / SW_WARPS);
    for (int b = 0; b < k; b += group) {
        if (group == 64)
            gptq_sweep_kernel<64><<<sweep_blocks, SW_WARPS * 32, 0, stream>>>(W64, n, k, b, bits, P, packed, sc, zeros,
                                                                              E, status);
        else
            gptq_sweep_kernel<128><<<sweep_blocks, SW_WARPS * 32, 0, stream>>>(W64, n, k, b, bits, P, packed, sc,
                                                                               zeros, E, status);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int rest = k - b - group;
        if (rest <= 0) break;
        gptq_trailing_kernel<<<dim3((unsigned)((rest + 63) / 64), (unsigned)((N + 63) / 64)), 256, 0, stream>>>(
            W64, n, k, b, group, E, P);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace w4
