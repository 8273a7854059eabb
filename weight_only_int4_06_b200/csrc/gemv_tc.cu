// Decode GEMV / skinny GEMM (M <= 8) on the 5th-generation tensor cores, weights in TMEM.
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the GEMV kernel serves token-by-token generation,
// where the layer is bound by memory traffic and weight reuse is minimal.  The traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale and zero point per group of 128.
//
// At HBM rate a B200 SM must consume ~46 weights per cycle, so the per-weight work on the CUDA
// cores has to be minimal.  Here it is one LOP3 per two weights plus a TMEM store per 64:
//  * the 128 weight rows of a tile are the MMA's A operand and live in TMEM: each dequant thread
//    owns one row (one TMEM lane), turns 8 codes into four f16x2 registers holding the raw values
//    1024+q (low nibble of a byte) and 1024+16q (high nibble) with one LOP3 per register, and
//    stores 64 of them with one tcgen05.st;
//  * one thread issues tcgen05.mma (M=128, N=16, K=16, A from TMEM, activations as B from shared
//    memory, fp32 accumulator in TMEM), one 128 x 16 accumulator per group of 128 k;
//  * the activations are staged once with every 8-k chunk in the slot order of those registers,
//    [x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16] (rows beyond M are zero), and the exact sums
//    Sl (low-nibble slots) and Sh' (staged x/16) of each group remove the operand offsets and
//    the zero point:  sum_k x_k (q_k - z) = raw - 1024 (Sl + Sh') - z (Sl + 16 Sh');
//    the group's fp16 scale then multiplies that exact-as-fp32 sum, accumulated in fp32;
//  * the weights stream through a 3-stage TMA ring (128 rows x 256 k, 128-byte swizzle);
//  * a CTA owns 128 rows and one K split; the splits of a row tile form a thread-block cluster
//    and their partial sums are added in split order through distributed shared memory.
// Warps: 0 = TMA producer, 1 = MMA issuer, 2 = TMEM owner, 4..11 = dequant/fold (lane quarter
// warp % 4, group parity (warp - 4) / 4).  Every mbarrier wait is bounded.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace w4 {

constexpr int GT_THREADS = 384;
constexpr int GT_ROWS = 128;
constexpr uint32_t GT_WSTAGE = GT_ROWS * 128;  // 16 KB: 128 rows x 256 k
constexpr int GT_WSTAGES = 3;
constexpr int GT_NA = 3;    // TMEM A buffers, 64 columns (one group) each
constexpr int GT_ND = 4;    // TMEM D buffers, 16 columns each
constexpr uint32_t GT_TMEM_COLS = 256;
constexpr uint32_t GT_DCOL0 = GT_NA * 64;
constexpr int GT_MAXG = 12;  // groups per CTA
constexpr int GT_MAXM = 8;

struct GtLayout {
    uint32_t w, xs, corr, part, bars, total;
};

__host__ __device__ inline GtLayout gt_layout(int gps) {
    GtLayout L;
    L.w = 0;
    L.xs = GT_WSTAGES * GT_WSTAGE;
    L.corr = L.xs + (uint32_t)gps * 16 * 256;      // per 8-k chunk: rows 0-7 (128 B), rows 8-15 (128 B)
    L.part = L.corr + (uint32_t)gps * GT_MAXM * 8;  // float2 [gps][8]
    L.bars = L.part + 2 * GT_ROWS * GT_MAXM * 4;    // [parity][row][m] fp32
    L.total = L.bars + 8 * (2 * GT_WSTAGES + 2 * GT_NA + 2 * GT_ND) + 16;
    return L;
}

__device__ __forceinline__ float gt_half2_sum(uint32_t h) {  // sum of the two halves, in fp32
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    return f.x + f.y;
}

__device__ __forceinline__ void gt_deq_barrier() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

__global__ void __launch_bounds__(GT_THREADS, 2)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X,
                   const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                   __half* __restrict__ Y, int M, int N, int K, int splits, int gps, int weights_early,
                   int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_align1024(smem_raw);
    const GtLayout L = gt_layout(gps);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = K >> 7;
    const int n0 = blockIdx.x * GT_ROWS;
    const int gb = blockIdx.y * gps;
    const int ng = min(gps, G - gb);
    const int nstage = (ng + 1) >> 1;
    const uint32_t bar0 = sbase + L.bars;
    auto w_full = [&](int s) { return bar0 + 8 * s; };
    auto w_empty = [&](int s) { return bar0 + 8 * (GT_WSTAGES + s); };
    auto a_full = [&](int i) { return bar0 + 8 * (2 * GT_WSTAGES + i); };
    auto a_free = [&](int i) { return bar0 + 8 * (2 * GT_WSTAGES + GT_NA + i); };
    auto d_full = [&](int i) { return bar0 + 8 * (2 * GT_WSTAGES + 2 * GT_NA + i); };
    auto d_free = [&](int i) { return bar0 + 8 * (2 * GT_WSTAGES + 2 * GT_NA + GT_ND + i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.bars + 8 * (2 * GT_WSTAGES + 2 * GT_NA + 2 * GT_ND));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float2* corr = reinterpret_cast<float2*>(smem + L.corr);
    float* part = reinterpret_cast<float*>(smem + L.part);

    if (tid == 0) {
        for (int s = 0; s < GT_WSTAGES; ++s) {
            mbar_init(w_full(s), 1);
            mbar_init(w_empty(s), 8);
        }
        for (int i = 0; i < GT_NA; ++i) {
            mbar_init(a_full(i), 4);
            mbar_init(a_free(i), 1);
        }
        for (int i = 0; i < GT_ND; ++i) {
            mbar_init(d_full(i), 1);
            mbar_init(d_free(i), 4);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), GT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    auto fail = [&]() {
        *abort_flag = 1;
        record_status(status, W4_ERR_DEVICE_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmW);
            if (!weights_early) pdl_wait();
            int issued = 0;
            for (int st = 0; st < nstage; ++st) {
                const int s = st % GT_WSTAGES;
                const uint32_t ph = (st / GT_WSTAGES) & 1;
                // ring full: progress now depends on consumers, who first wait for the preceding kernel
                if (st == GT_WSTAGES && weights_early) pdl_wait();
                if (!mbar_wait_bounded(w_empty(s), ph ^ 1, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(w_full(s), GT_WSTAGE);
                tma_load_2d(sbase + L.w + s * GT_WSTAGE, &tmW, (gb * 128 + st * 256) / 8, n0, w_full(s));
                ++issued;
            }
            for (int st = issued - GT_WSTAGES; st < issued; ++st)  // no loads in flight at exit
                if (st >= 0) mbar_wait_bounded(w_full(st % GT_WSTAGES), (st / GT_WSTAGES) & 1, nullptr, 200000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(GT_ROWS, 16);
            int last = -1;
            for (int g = 0; g < ng; ++g) {
                const int a = g % GT_NA, d = g % GT_ND;
                if (!mbar_wait_bounded(a_full(a), (g / GT_NA) & 1, abort_flag)) { fail(); break; }
                if (!mbar_wait_bounded(d_free(d), ((g / GT_ND) & 1) ^ 1, abort_flag)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint64_t bd = noswz_kmajor_desc(sbase + L.xs + (uint32_t)(g * 16 + 2 * j) * 256, 256, 128);
                    mma_f16_ts(tmem + GT_DCOL0 + d * 16, tmem + a * 64 + j * 8, bd, idesc, j > 0);
                }
                tc_commit(a_free(a));
                tc_commit(d_full(d));
                last = g;
            }
            if (last >= 0)  // every issued MMA has completed before TMEM can be released
                mbar_wait_bounded(d_full(last % GT_ND), (last / GT_ND) & 1, nullptr, 200000000ull);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ dequant + fold
        const int q = warp & 3, h = (warp - 4) >> 2;
        const int r = q * 32 + lane;  // tile row = TMEM lane
        const int n = n0 + r;
        const int dt = tid - 128;     // 0..255
        // This row's metadata does not depend on the preceding kernel: fetch it first.
        float sv[GT_MAXG / 2], zv[GT_MAXG / 2];  // this row's scale / zero for groups h, h+2, ...
#pragma unroll
        for (int k = 0; k < GT_MAXG / 2; ++k) {
            const int g = h + 2 * k;
            sv[k] = 0.0f;
            zv[k] = 0.0f;
            if (g < ng && n < N) {
                sv[k] = __half2float(__ushort_as_half(__ldg(scales + (int64_t)n * G + gb + g)));
                zv[k] = (float)__ldg(zeros + (int64_t)n * G + gb + g);
            }
        }
        // Stage the activations of this split with the group sums that remove the operand
        // offsets (fp32, fixed tree order); B rows M..15 are zero.
        const int cpw = ng * 16;  // 8-k chunks in this split
        for (int i = dt; i < cpw * (16 - M); i += 256) {
            const int m = M + i / cpw, ch = i % cpw;
            *reinterpret_cast<uint4*>(smem + L.xs + ch * 256 + (m < 8 ? m * 16 : 128 + (m - 8) * 16)) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        for (int m = M; m < GT_MAXM; ++m)
            for (int g = dt; g < ng; g += 256) corr[g * GT_MAXM + m] = make_float2(0.0f, 0.0f);
        pdl_wait();  // the activations may be produced by the preceding kernel
        const __half2 sixteenth = __float2half2_rn(0.0625f);
        const unsigned half_mask = (lane & 16) ? 0xFFFF0000u : 0x0000FFFFu;
        constexpr int XILP = 2;
        for (int base = 0; base < M * cpw; base += 256 * XILP) {  // uniform per 16-lane half
            uint4 raw[XILP];
#pragma unroll
            for (int v = 0; v < XILP; ++v) {
                const int i = base + v * 256 + dt;
                if (i < M * cpw) raw[v] = ldg_cached(X + (int64_t)(i / cpw) * K + (int64_t)gb * 128 + (i % cpw) * 8);
            }
#pragma unroll
            for (int v = 0; v < XILP; ++v) {
                const int i = base + v * 256 + dt;
                if (i >= M * cpw) break;
                const int m = i / cpw, ch = i - m * cpw;
                const uint4 r4 = raw[v];
                uint4 p;
                p.x = __byte_perm(r4.x, r4.z, 0x5410);         // x0, x4
                uint32_t t = __byte_perm(r4.x, r4.z, 0x7632);  // x1, x5
                __half2 hh = __hmul2(*reinterpret_cast<__half2*>(&t), sixteenth);
                p.y = *reinterpret_cast<uint32_t*>(&hh);
                p.z = __byte_perm(r4.y, r4.w, 0x5410);         // x2, x6
                t = __byte_perm(r4.y, r4.w, 0x7632);           // x3, x7
                hh = __hmul2(*reinterpret_cast<__half2*>(&t), sixteenth);
                p.w = *reinterpret_cast<uint32_t*>(&hh);
                *reinterpret_cast<uint4*>(smem + L.xs + ch * 256 + m * 16) = p;  // m < 8
                float lo = gt_half2_sum(p.x) + gt_half2_sum(p.z);
                float hi = gt_half2_sum(p.y) + gt_half2_sum(p.w);
#pragma unroll
                for (int o = 8; o; o >>= 1) {
                    lo += __shfl_xor_sync(half_mask, lo, o);
                    hi += __shfl_xor_sync(half_mask, hi, o);
                }
                if ((ch & 15) == 0)  // C = 1024 (Sl + Sh'), S = Sl + 16 Sh'
                    corr[(ch >> 4) * GT_MAXM + m] = make_float2(1024.0f * (lo + hi), fmaf(16.0f, hi, lo));
            }
        }
        fence_proxy_async_shared();  // staged activations: generic-proxy writes read by the MMA
        gt_deq_barrier();  // x staged (the MMA thread reads it after the first a_full)

        float acc[GT_MAXM];
#pragma unroll
        for (int m = 0; m < GT_MAXM; ++m) acc[m] = 0.0f;
        bool dead = false;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;

        auto fold = [&](int g, int k) {
            const int d = g % GT_ND;
            if (!dead && !mbar_wait_bounded(d_full(d), (g / GT_ND) & 1, abort_flag)) { fail(); dead = true; }
            tc_fence_after();
            uint32_t v[8];
            tmem_ld_32x32b_x8(tmem + lane_base + GT_DCOL0 + d * 16, v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(d_free(d));
            float s = 0.0f, z = 0.0f;
#pragma unroll
            for (int kk = 0; kk < GT_MAXG / 2; ++kk)
                if (kk == k) { s = sv[kk]; z = zv[kk]; }
#pragma unroll
            for (int m = 0; m < GT_MAXM; ++m) {
                const float2 cs = corr[g * GT_MAXM + m];
                acc[m] = fmaf(s, __uint_as_float(v[m]) - fmaf(z, cs.y, cs.x), acc[m]);
            }
        };

        int k = 0;
        for (int g = h; g < ng; g += 2, ++k) {
            const int st = g >> 1;
            const int s = st % GT_WSTAGES;
            const int a = g % GT_NA;
            if (!dead && !mbar_wait_bounded(w_full(s), (st / GT_WSTAGES) & 1, abort_flag)) { fail(); dead = true; }
            if (!dead && !mbar_wait_bounded(a_free(a), ((g / GT_NA) & 1) ^ 1, abort_flag)) { fail(); dead = true; }
            // this row's 64 bytes of group g: chunks 4 (g & 1) .. +3 of the swizzled 128-byte row
            const unsigned char* row = smem + L.w + s * GT_WSTAGE + r * 128;
            uint4 c4[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int c = (g & 1) * 4 + cc;
                c4[cc] = *reinterpret_cast<const uint4*>(row + ((c ^ (r & 7)) << 4));
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t regs[32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint4 ch = c4[half * 2 + cc];
                    const uint32_t wd[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t w = wd[j], w8 = w >> 8;
                        uint32_t* o = regs + (cc * 4 + j) * 4;
                        o[0] = lop3_and_or(w, 0x000F000Fu, 0x64006400u);   // 1024 + n0, 1024 + n4
                        o[1] = lop3_and_or(w, 0x00F000F0u, 0x64006400u);   // 1024 + 16 n1, 1024 + 16 n5
                        o[2] = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);  // 1024 + n2, 1024 + n6
                        o[3] = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);  // 1024 + 16 n3, 1024 + 16 n7
                    }
                }
                tmem_st_32x32b_x32(tmem + lane_base + a * 64 + half * 32, regs);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(w_empty(s));  // every lane's stage loads were consumed above
                mbar_arrive(a_full(a));
            }
            if (k > 0) fold(g - 2, k - 1);
        }
        if (k > 0) fold(h + 2 * (k - 1), k - 1);
        // park this warp's partial sums (its row, its group parity)
#pragma unroll
        for (int m = 0; m < GT_MAXM; ++m) part[(h * GT_ROWS + r) * GT_MAXM + m] = acc[m];
    }

    __syncthreads();
    if (splits == 1) {
        for (int i = tid; i < GT_ROWS * M; i += GT_THREADS) {
            const int rr = i / M, m = i - rr * M;
            const float y = part[rr * GT_MAXM + m] + part[(GT_ROWS + rr) * GT_MAXM + m];
            if (n0 + rr < N) Y[(int64_t)m * N + n0 + rr] = __float2half_rn(y);
        }
    } else {
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rank = (int)cluster.block_rank();
        const int per = (GT_ROWS + splits - 1) / splits;
        const int r0 = rank * per, r1 = min(GT_ROWS, r0 + per);
        const int nr = r1 - r0;
        for (int i = tid; i < nr * M; i += GT_THREADS) {
            const int rr = r0 + i / M, m = i % M;
            float y = 0.0f;
            for (int sp = 0; sp < splits; ++sp) {  // split order: deterministic
                const float* rp = cluster.map_shared_rank(part, sp);
                y += rp[rr * GT_MAXM + m] + rp[(GT_ROWS + rr) * GT_MAXM + m];
            }
            if (n0 + rr < N) Y[(int64_t)m * N + n0 + rr] = __float2half_rn(y);
        }
        cluster.sync();  // keep this CTA's partials alive until every peer has read them
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, GT_TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------------ host side
// One wave: at most two CTAs per SM (each fits half an SM), as many (tile, split) CTAs as
// possible, fewest splits among equals.  Shapes whose splits would exceed GT_MAXG groups each
// or 16 CTAs per cluster are not planned.
bool plan_gemv_tc(int64_t M, int64_t N, int64_t K, GemvTcPlan* plan) {
    if (M < 1 || M > GT_MAXM || K < 128 || N < 8) return false;
    const int G = (int)(K / 128);
    const int n_tiles = (int)((N + GT_ROWS - 1) / GT_ROWS);
    const long slots = 2L * device_sm_count();
    long best = -1;
    for (int S = 1; S <= 16 && S <= G; ++S) {
        const int gps = (G + S - 1) / S;
        if (gps > GT_MAXG || (long)n_tiles * S > slots) continue;
        if ((G + gps - 1) / gps != S) continue;  // every split gets at least one group
        if ((long)n_tiles * S > best) {
            best = (long)n_tiles * S;
            plan->splits = S;
            plan->gps = gps;
            plan->n_tiles = n_tiles;
        }
    }
    if (best < 0) return false;
    plan->smem = (size_t)gt_layout(plan->gps).total + 1024;
    return true;
}

cudaError_t launch_gemv_tc(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, const GemvTcPlan& p,
                           bool weights_static, int* status, cudaStream_t stream) {
    CUtensorMap tm;
    if (!make_tensor_map_2d(&tm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(K / 8), (uint64_t)N, 32,
                            GT_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(gemv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 113 * 1024);
        if (attr_err[dev] == cudaSuccess)
            attr_err[dev] = cudaFuncSetAttribute(gemv_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    if (p.smem > 113 * 1024) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.n_tiles, (unsigned)p.splits, 1);
    cfg.blockDim = dim3(GT_THREADS, 1, 1);
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
    return cudaLaunchKernelEx(&cfg, gemv_tc_kernel, tm, reinterpret_cast<const __half*>(X),
                              reinterpret_cast<const unsigned short*>(scales), zeros, reinterpret_cast<__half*>(Y),
                              (int)M, (int)N, (int)K, p.splits, p.gps, weights_static ? 1 : 0, status);
}

}  // namespace w4
