// Skinny W4A16 GEMM / GEMV for M <= 32 (single-token and small-batch decode).
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): for decode the layer is bound by memory traffic,
// weights are dequantised on the fly and never materialised in FP16.  Here the traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale/zero per group of 128.
//
// Design (sm_100a):
//  * The dot products run on the tensor cores with mma.sync m16n8k16 (fp16 x fp16 -> fp32): the
//    W tile is the 16-row "A" operand straight from registers, the activations are the 8-column
//    "B" operand, so no dequantised weight ever touches shared memory.  fp32 accumulation on the
//    CUDA cores would cost more ALU operations per weight than the HBM rate leaves.
//  * Dequantisation is exact and costs ~9 ALU ops per 8 weights: LOP3 with the 0x6400 exponent
//    pattern turns a nibble into the fp16 value 1024+q (or 1024+16q for the upper nibble of a
//    byte), and one f16x2 subtract / fma with (1024+z) resp. 1/16 and -(64+z) gives q - z exactly.
//    The tensor core accumulates sum_k x_k (q_k - z) for one group in fp32 (every product is
//    exact), and the group's fp16 scale multiplies that partial sum in fp32.
//  * Each packed word holds 8 consecutive k; the nibble pairs that the LOP3 trick yields are
//    (k, k+4).  The contraction does not care which k sits in which MMA slot as long as A and B
//    agree, so the activations are staged in shared memory with every 8-k chunk permuted to
//    (0,4,1,5,2,6,3,7): one 16-byte shared load then yields the B fragments of two MMAs.
//  * Tiling: a CTA owns 128 rows of W (8 warps x 16 rows) and one K split; each thread streams
//    16 bytes of two rows per group with 128-bit non-allocating loads, SK_PD groups in flight.
//    The K splits of one row tile form a thread-block cluster; partial sums meet in distributed
//    shared memory and are added in split order (deterministic, no global workspace, one launch).
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace w4 {

constexpr int SK_WARPS = 8;
constexpr int SK_BN = 16 * SK_WARPS;  // rows of W per CTA
constexpr int SK_THREADS = 32 * SK_WARPS;
constexpr int SK_PD = 4;  // groups of W per thread in flight

// 16-byte chunk swizzle of the staged activations: makes the B-fragment loads of a warp
// bank-conflict free (the row stride is padded to 16 mod 128 bytes).
__device__ __forceinline__ int sk_swz(int ch) { return ch ^ ((ch >> 2) & 2); }

// One packed word (codes n0..n7 of 8 consecutive k) -> four f16x2 registers holding q - z:
// lo0 = (n0, n4), hi0 = (n1, n5), lo1 = (n2, n6), hi1 = (n3, n7).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t zl, uint32_t zh, uint32_t& lo0,
                                             uint32_t& hi0, uint32_t& lo1, uint32_t& hi1) {
    const uint32_t kMagic = 0x64006400u;     // fp16 1024 in both halves
    const uint32_t kSixteenth = 0x2C002C00u; // fp16 1/16 in both halves
    lo0 = hsub2_u32(lop3_and_or(w, 0x000F000Fu, kMagic), zl);
    hi0 = hfma2_u32(lop3_and_or(w, 0x00F000F0u, kMagic), kSixteenth, zh);
    const uint32_t w8 = w >> 8;
    lo1 = hsub2_u32(lop3_and_or(w8, 0x000F000Fu, kMagic), zl);
    hi1 = hfma2_u32(lop3_and_or(w8, 0x00F000F0u, kMagic), kSixteenth, zh);
}

template <int NT>
__device__ __forceinline__ size_t sk_xs_bytes(int gps) {
    const size_t a = (size_t)8 * NT * (gps * 128 + 8) * 2;
    const size_t b = (size_t)8 * NT * SK_BN * 4;
    return a > b ? a : b;
}

constexpr int SK_MAX_SPLITS = 16;

template <int NT, int MINB>
__global__ void __launch_bounds__(SK_THREADS, MINB)
    skinny_kernel(const __half* __restrict__ X, int M, int N, int K, const uint4* __restrict__ packed4,
                  const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                  __half* __restrict__ Y, int splits, int gps, int weights_early) {
    constexpr int MT = 8 * NT;
    extern __shared__ __align__(16) unsigned char smem[];
    const int G = K >> 7;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, c = lane & 3;
    const int n0 = blockIdx.x * SK_BN;
    const int gb = blockIdx.y * gps;
    const int ng = min(gps, G - gb);
    const int RSh = gps * 128 + 8;  // staged activation row stride, in halves

    __half* Xs = reinterpret_cast<__half*>(smem);
    float* Part = reinterpret_cast<float*>(smem);  // reuses the activation area after the main loop

    const int ra = warp * 16 + g8, rb = ra + 8;
    const bool va = n0 + ra < N, vb = n0 + rb < N;
    const int64_t row4 = K >> 5;  // 16-byte chunks per packed row
    const uint4* pa = packed4 + (int64_t)(n0 + ra) * row4 + gb * 4 + c;
    const uint4* pb = packed4 + (int64_t)(n0 + rb) * row4 + gb * 4 + c;
    const unsigned short* sca = scales + (int64_t)(n0 + ra) * G + gb;
    const unsigned short* scb = scales + (int64_t)(n0 + rb) * G + gb;
    const uint8_t* zpa = zeros + (int64_t)(n0 + ra) * G + gb;
    const uint8_t* zpb = zeros + (int64_t)(n0 + rb) * G + gb;

    // W, scales and zero points of the first SK_PD groups go in flight first.  Weights are only
    // read ahead of the preceding kernel when the caller declared them static.
    if (!weights_early) pdl_wait();
    uint4 wa[SK_PD], wb[SK_PD];
    unsigned short sra[SK_PD], srb[SK_PD];  // raw scale bits, untouched until used
    uint8_t zra[SK_PD], zrb[SK_PD];          // raw zero points
#pragma unroll
    for (int s = 0; s < SK_PD; ++s) {
        wa[s] = make_uint4(0u, 0u, 0u, 0u);
        wb[s] = make_uint4(0u, 0u, 0u, 0u);
        sra[s] = 0; zra[s] = 0;
        srb[s] = 0; zrb[s] = 0;
        if (s < ng) {
            if (va) {
                wa[s] = ldg_stream(pa + s * 4);
                sra[s] = __ldg(sca + s); zra[s] = __ldg(zpa + s);
            }
            if (vb) {
                wb[s] = ldg_stream(pb + s * 4);
                srb[s] = __ldg(scb + s); zrb[s] = __ldg(zpb + s);
            }
        }
    }
    if (weights_early) pdl_wait();  // activations may come from the preceding kernel

    // Stage this split's activations (rows >= M are zero), 8-k chunks permuted to
    // (0,4,1,5,2,6,3,7); four loads per thread are in flight before any store.
    const int cpr = ng * 16;
    const int total = MT * cpr;
    for (int base = tid; base < total; base += 4 * SK_THREADS) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * SK_THREADS;
            r[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < total) {
                const int m = i / cpr, ch = i - m * cpr;
                if (m < M) r[u] = ldg_cached(X + (int64_t)m * K + gb * 128 + ch * 8);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * SK_THREADS;
            if (i < total) {
                const int m = i / cpr, ch = i - m * cpr;
                uint4 p;
                p.x = __byte_perm(r[u].x, r[u].z, 0x5410);
                p.y = __byte_perm(r[u].x, r[u].z, 0x7632);
                p.z = __byte_perm(r[u].y, r[u].w, 0x5410);
                p.w = __byte_perm(r[u].y, r[u].w, 0x7632);
                *reinterpret_cast<uint4*>(Xs + m * RSh + sk_swz(ch) * 8) = p;
            }
        }
    }
    __syncthreads();

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;

    const __half* xrow = Xs + g8 * RSh;
    for (int g0 = 0; g0 < ng; g0 += SK_PD) {
#pragma unroll
        for (int s = 0; s < SK_PD; ++s) {
            const int gi = g0 + s;
            if (gi < ng) {
                const uint4 A = wa[s], B = wb[s];
                const unsigned short rsa = sra[s], rsb = srb[s];
                const uint32_t za = zra[s], zb = zrb[s];
                const int gn = gi + SK_PD;
                if (gn < ng) {
                    if (va) {
                        wa[s] = ldg_stream(pa + gn * 4);
                        sra[s] = __ldg(sca + gn); zra[s] = __ldg(zpa + gn);
                    }
                    if (vb) {
                        wb[s] = ldg_stream(pb + gn * 4);
                        srb[s] = __ldg(scb + gn); zrb[s] = __ldg(zpb + gn);
                    }
                }
                const float sa = __half2float(__ushort_as_half(rsa));
                const float sb = __half2float(__ushort_as_half(rsb));
                const uint32_t zla = (0x6400u + za) * 0x10001u, zha = (0xD400u | (za << 4)) * 0x10001u;
                const uint32_t zlb = (0x6400u + zb) * 0x10001u, zhb = (0xD400u | (zb << 4)) * 0x10001u;
                const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
                const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
                float cc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) cc[nt][i] = 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t alo0, ahi0, alo1, ahi1, blo0, bhi0, blo1, bhi1;
                    dequant_word(wA[j], zla, zha, alo0, ahi0, alo1, ahi1);
                    dequant_word(wB[j], zlb, zhb, blo0, bhi0, blo1, bhi1);
                    const int ch = sk_swz(gi * 16 + c * 4 + j);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 xf = *reinterpret_cast<const uint4*>(xrow + nt * 8 * RSh + ch * 8);
                        mma_16816(cc[nt], alo0, blo0, ahi0, bhi0, xf.x, xf.y);
                        mma_16816(cc[nt], alo1, blo1, ahi1, bhi1, xf.z, xf.w);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[nt][0] = fmaf(cc[nt][0], sa, acc[nt][0]);
                    acc[nt][1] = fmaf(cc[nt][1], sa, acc[nt][1]);
                    acc[nt][2] = fmaf(cc[nt][2], sb, acc[nt][2]);
                    acc[nt][3] = fmaf(cc[nt][3], sb, acc[nt][3]);
                }
            }
        }
    }
    pdl_launch_dependents();  // the next kernel may start streaming its weights now

    __syncthreads();  // every warp is done with Xs before Part overwrites it
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m0 = nt * 8 + 2 * c;
        Part[m0 * SK_BN + ra] = acc[nt][0];
        Part[(m0 + 1) * SK_BN + ra] = acc[nt][1];
        Part[m0 * SK_BN + rb] = acc[nt][2];
        Part[(m0 + 1) * SK_BN + rb] = acc[nt][3];
    }
    if (splits == 1) {
        __syncthreads();
        for (int i = tid; i < M * SK_BN; i += SK_THREADS) {
            const int m = i / SK_BN, r = i - m * SK_BN;
            if (n0 + r < N) Y[(int64_t)m * N + n0 + r] = __float2half_rn(Part[i]);
        }
    } else {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rank = (int)cluster.block_rank();
        const int per = (SK_BN + splits - 1) / splits;
        const int r0 = rank * per;
        const int r1 = min(SK_BN, r0 + per);
        const int nr = r1 - r0;
        for (int i = tid; i < M * nr; i += SK_THREADS) {
            const int m = i / nr, r = r0 + (i - m * nr);
            float v[SK_MAX_SPLITS];
#pragma unroll
            for (int s = 0; s < SK_MAX_SPLITS; ++s)
                v[s] = s < splits ? cluster.map_shared_rank(Part, s)[m * SK_BN + r] : 0.0f;
            float sum = 0.0f;
#pragma unroll
            for (int s = 0; s < SK_MAX_SPLITS; ++s)
                if (s < splits) sum += v[s];  // split order: deterministic
            if (n0 + r < N) Y[(int64_t)m * N + n0 + r] = __float2half_rn(sum);
        }
        cluster.sync();  // keep this CTA's partials alive until every peer has read them
    }
}

// ------------------------------------------------------------------------------------ host side
static size_t skinny_smem_bytes(int mt, int gps) {
    const size_t xs_a = (size_t)mt * (gps * 128 + 8) * 2;
    const size_t xs_b = (size_t)mt * SK_BN * 4;
    const size_t xs = xs_a > xs_b ? xs_a : xs_b;
    return xs + 16;
}

bool plan_skinny(int64_t M, int64_t N, int64_t K, SkinnyPlan* plan) {
    if (M < 1 || M > 32 || K < 128 || N < 1) return false;
    const int mt = M <= 8 ? 8 : (M <= 16 ? 16 : 32);
    const int G = (int)(K / 128);
    const int n_tiles = (int)((N + SK_BN - 1) / SK_BN);
    const int sms = device_sm_count();
    const int target = (mt <= 16 ? 2 : 1) * sms;
    int S = (target + n_tiles - 1) / n_tiles;
    if (S < 1) S = 1;
    if (S > 8) S = 8;
    if (S > G) S = G;
    const size_t limit = 200 * 1024;
    for (;;) {
        const int gps = (G + S - 1) / S;
        const int s_eff = (G + gps - 1) / gps;
        const size_t smem = skinny_smem_bytes(mt, gps);
        if (smem <= limit || S >= 16 || S >= G) {
            if (smem > 227 * 1024) return false;
            plan->mt = mt;
            plan->splits = s_eff;
            plan->gps = gps;
            plan->n_tiles = n_tiles;
            plan->smem = smem;
            return true;
        }
        ++S;
    }
}

template <int NT, int MINB>
static cudaError_t launch_nt(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                             const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                             uint16_t* Y, const SkinnyPlan& p, bool weights_static, cudaStream_t stream) {
    auto kern = skinny_kernel<NT, MINB>;
    // Kernel attributes are set once per device (never inside a stream capture).
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (attr_err[dev] == cudaSuccess)
            attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.n_tiles, (unsigned)p.splits, 1);
    cfg.blockDim = dim3(SK_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned na = 0;
    if (p.splits > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = (unsigned)p.splits;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (weights_static) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const __half*>(X), (int)M, (int)N, (int)K,
                              reinterpret_cast<const uint4*>(packed),
                              reinterpret_cast<const unsigned short*>(scales), zeros,
                              reinterpret_cast<__half*>(Y), p.splits, p.gps, weights_static ? 1 : 0);
}

cudaError_t launch_skinny(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                          uint16_t* Y, const SkinnyPlan& plan, bool weights_static,
                          cudaStream_t stream) {
    switch (plan.mt) {
        case 8: return launch_nt<1, 2>(X, M, N, K, packed, scales, zeros, Y, plan, weights_static, stream);
        case 16: return launch_nt<2, 1>(X, M, N, K, packed, scales, zeros, Y, plan, weights_static, stream);
        default: return launch_nt<4, 1>(X, M, N, K, packed, scales, zeros, Y, plan, weights_static, stream);
    }
}

}  // namespace w4
