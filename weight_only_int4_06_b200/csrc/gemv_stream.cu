// Single-token decode GEMV (M = 1): y = dequant(W) x, streamed at HBM rate.
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the GEMV kernel serves single-token generation,
// where the layer is bound by memory traffic and weight reuse is minimal.  The traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale and zero point per group of 128.
//
// Design (sm_100a):
//  * Persistent: one CTA per SM; CTA c owns a contiguous range of 16-row tiles over the whole K,
//    so every output is finished inside one CTA (no split-K workspace, no cluster barrier).
//  * A producer warp streams the packed tile through a GV_STAGES-deep shared-memory ring with
//    TMA (16 rows x 1024 k = 8 KB per stage), so each SM keeps ~64 KB of weights in flight no
//    matter how long the consumers take for one stage.  With static weights it starts before
//    the preceding kernel has finished (programmatic dependent launch).
//  * Eight consumer warps take one group of 128 each per stage and run mma.sync m16n8k16 with the
//    16 weight rows as the A operand.  Dequantisation is one LOP3 per two weights: the operands
//    are the raw fp16 values 1024+q (low nibble of a byte) and 1024+16q (high nibble); the
//    activations that meet high nibbles are staged pre-multiplied by 1/16, and the constant
//    offsets and the zero point are removed per group in fp32 with the exact activation sums
//        sum_k x_k (q_k - z) = raw - 1024 (Sl + Sh') - z (Sl + 16 Sh'),
//    Sl = sum of x over low-nibble slots, Sh' = sum of the staged x/16 over high-nibble slots
//    (both summed exactly in fp64).  The group's fp16 scale then multiplies that sum in fp32.
//  * Partial sums of the eight warps are added in warp order in shared memory (deterministic).
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

constexpr int GV_CWARPS = 8;                      // consumer warps (one group each per stage)
constexpr int GV_THREADS = 32 * (GV_CWARPS + 1);  // + one producer warp
constexpr int GV_KC = 128 * GV_CWARPS;            // k per stage
constexpr uint32_t GV_STAGE_BYTES = 16 * GV_KC / 2;  // 8 KB of packed codes
constexpr int GV_STAGES = 8;
constexpr int GV_PF = 8;  // units of metadata prefetched ahead

struct GvLayout {
    uint32_t ring, xs, corr, red, bars, total;
};

__host__ __device__ inline GvLayout gv_layout(int K) {
    GvLayout L;
    L.ring = 0;
    L.xs = GV_STAGES * GV_STAGE_BYTES;
    L.corr = L.xs + (uint32_t)K * 2;                            // float2 per group
    L.red = L.corr + (uint32_t)(K / 128) * 8;                   // 2 x 8 warps x 16 floats
    L.bars = (L.red + 2 * GV_CWARPS * 16 * 4 + 7) & ~7u;
    L.total = L.bars + 2 * GV_STAGES * 8 + 8;
    return L;
}

__device__ __forceinline__ void gv_named_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * GV_CWARPS) : "memory");
}

__global__ void __launch_bounds__(GV_THREADS, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X,
                       const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                       __half* __restrict__ Y, int N, int K, int n_tiles, int weights_early, int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA destinations need an aligned base: round up (the launch reserves 1 KB of slack)
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    const GvLayout L = gv_layout(K);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = K >> 7;
    const int NC = (G + GV_CWARPS - 1) / GV_CWARPS;  // stages per tile
    const int t0 = (int)(((int64_t)blockIdx.x * n_tiles) / gridDim.x);
    const int t1 = (int)(((int64_t)(blockIdx.x + 1) * n_tiles) / gridDim.x);
    const int n_units = (t1 - t0) * NC;
    auto full_bar = [&](int s) { return sbase + L.bars + 8 * s; };
    auto empty_bar = [&](int s) { return sbase + L.bars + 8 * (GV_STAGES + s); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bars + 16 * GV_STAGES);

    if (tid == 0) {
        for (int s = 0; s < GV_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), GV_CWARPS);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();  // the next kernel may claim SM space and start its own weight stream

    if (warp == GV_CWARPS) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmW);
            if (!weights_early) pdl_wait();
            int issued = 0;
            for (int u = 0; u < n_units; ++u) {
                const int s = u % GV_STAGES;
                const uint32_t ph = (u / GV_STAGES) & 1;
                // The ring is full: from here on progress depends on the consumers, who first
                // wait for the preceding kernel; start the bounded waits only after that point.
                if (u == GV_STAGES && weights_early) pdl_wait();
                if (!mbar_wait_bounded(empty_bar(s), ph ^ 1, abort_flag)) {
                    *abort_flag = 1;
                    record_status(status, W4_ERR_DEVICE_TIMEOUT);
                    break;
                }
                const int t = t0 + u / NC, kc = u % NC;
                mbar_arrive_expect_tx(full_bar(s), GV_STAGE_BYTES);
                tma_load_2d(sbase + L.ring + s * GV_STAGE_BYTES, &tmW, kc * (GV_KC / 8), t * 16, full_bar(s));
                ++issued;
            }
            for (int u = issued - GV_STAGES; u < issued; ++u)  // no loads in flight at exit
                if (u >= 0) mbar_wait_bounded(full_bar(u % GV_STAGES), (u / GV_STAGES) & 1, nullptr, 200000000ull);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Stage x: every 8-k chunk as [x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16] (the B fragments
    // of two MMAs), then the exact per-group sums that remove the operand offsets.
    pdl_wait();  // x may be produced by the preceding kernel
    __half* xs = reinterpret_cast<__half*>(smem + L.xs);
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    for (int i = tid; i < K / 8; i += 32 * GV_CWARPS) {
        const uint4 r = ldg_cached(X + (int64_t)i * 8);
        uint4 p;
        p.x = __byte_perm(r.x, r.z, 0x5410);  // x0, x4
        uint32_t h = __byte_perm(r.x, r.z, 0x7632);  // x1, x5
        __half2 hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
        p.y = *reinterpret_cast<uint32_t*>(&hh);
        p.z = __byte_perm(r.y, r.w, 0x5410);  // x2, x6
        h = __byte_perm(r.y, r.w, 0x7632);    // x3, x7
        hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
        p.w = *reinterpret_cast<uint32_t*>(&hh);
        *reinterpret_cast<uint4*>(xs + (int64_t)i * 8) = p;
    }
    gv_named_barrier();
    float2* corr = reinterpret_cast<float2*>(smem + L.corr);
    for (int g = tid; g < G; g += 32 * GV_CWARPS) {
        double lo = 0.0, hi = 0.0;  // exact: at most 128 fp16 values
        const __half* xg = xs + g * 128;
        for (int i = 0; i < 128; i += 8) {
            lo += (double)__half2float(xg[i + 0]) + (double)__half2float(xg[i + 1]) +
                  (double)__half2float(xg[i + 4]) + (double)__half2float(xg[i + 5]);
            hi += (double)__half2float(xg[i + 2]) + (double)__half2float(xg[i + 3]) +
                  (double)__half2float(xg[i + 6]) + (double)__half2float(xg[i + 7]);
        }
        corr[g] = make_float2((float)(1024.0 * (lo + hi)), (float)(lo + 16.0 * hi));
    }
    gv_named_barrier();

    const int g8 = lane >> 2, c = lane & 3;
    float* red = reinterpret_cast<float*>(smem + L.red);
    const bool xlane = g8 == 0;  // only B column 0 (the single activation row) is nonzero

    // Scale and zero point of unit v (tile t0 + v / NC, group (v % NC) * 8 + warp) for this
    // thread's two rows, fetched GV_PF units ahead.  The loaded values stay untouched in their
    // own registers until they are used, so no instruction waits on them early.
    auto meta_load = [&](int v, unsigned short& sa, unsigned short& sb, uint8_t& za, uint8_t& zb) {
        sa = 0;
        sb = 0;
        za = 0;
        zb = 0;
        if (v < n_units) {
            const int t = t0 + v / NC, gi = (v % NC) * GV_CWARPS + warp;
            if (gi < G) {
                const int na = t * 16 + g8, nb = na + 8;
                if (na < N) {
                    sa = __ldg(scales + (int64_t)na * G + gi);
                    za = __ldg(zeros + (int64_t)na * G + gi);
                }
                if (nb < N) {
                    sb = __ldg(scales + (int64_t)nb * G + gi);
                    zb = __ldg(zeros + (int64_t)nb * G + gi);
                }
            }
        }
    };
    unsigned short psa[GV_PF], psb[GV_PF];
    uint8_t pza[GV_PF], pzb[GV_PF];
#pragma unroll
    for (int p = 0; p < GV_PF; ++p) meta_load(p, psa[p], psb[p], pza[p], pzb[p]);

    float acc_a = 0.0f, acc_b = 0.0f;
    for (int u0 = 0; u0 < n_units; u0 += GV_PF) {
#pragma unroll
        for (int p = 0; p < GV_PF; ++p) {
            const int u = u0 + p;
            if (u >= n_units) break;  // uniform across the CTA
            const unsigned short sa = psa[p], sb = psb[p];
            const uint32_t za = pza[p], zb = pzb[p];
            meta_load(u + GV_PF, psa[p], psb[p], pza[p], pzb[p]);
            const int s = u % GV_STAGES;
            const uint32_t ph = (u / GV_STAGES) & 1;
            const int t = t0 + u / NC, kc = u % NC;
            const int gi = kc * GV_CWARPS + warp;
            // After a timeout every wait is skipped but the control flow (and every barrier) stays
            // the same, so no warp is left behind at a barrier.
            bool ok = !*abort_flag;
            if (ok && !mbar_wait_bounded(full_bar(s), ph, abort_flag)) {
                *abort_flag = 1;
                record_status(status, W4_ERR_DEVICE_TIMEOUT);
                ok = false;
            }
            if (ok && gi < G) {
                const unsigned char* st = smem + L.ring + s * GV_STAGE_BYTES;
                const uint4 A = *reinterpret_cast<const uint4*>(st + g8 * (GV_KC / 2) + warp * 64 + c * 16);
                const uint4 B = *reinterpret_cast<const uint4*>(st + (g8 + 8) * (GV_KC / 2) + warp * 64 + c * 16);
                const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
                const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
                float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t a = wA[j], b = wB[j], a8 = a >> 8, b8 = b >> 8;
                    uint4 xf = make_uint4(0u, 0u, 0u, 0u);
                    if (xlane) xf = *reinterpret_cast<const uint4*>(xs + gi * 128 + c * 32 + j * 8);
                    float(&cc)[4] = (j & 1) ? c1 : c0;  // two independent accumulation chains
                    mma_16816(cc, lop3_and_or(a, 0x000F000Fu, 0x64006400u), lop3_and_or(b, 0x000F000Fu, 0x64006400u),
                              lop3_and_or(a, 0x00F000F0u, 0x64006400u), lop3_and_or(b, 0x00F000F0u, 0x64006400u),
                              xf.x, xf.y);
                    mma_16816(cc, lop3_and_or(a8, 0x000F000Fu, 0x64006400u),
                              lop3_and_or(b8, 0x000F000Fu, 0x64006400u), lop3_and_or(a8, 0x00F000F0u, 0x64006400u),
                              lop3_and_or(b8, 0x00F000F0u, 0x64006400u), xf.z, xf.w);
                }
                const float2 cs = corr[gi];
                const float ra = (c0[0] + c1[0]) - fmaf((float)za, cs.y, cs.x);
                const float rb = (c0[2] + c1[2]) - fmaf((float)zb, cs.y, cs.x);
                acc_a = fmaf(__half2float(__ushort_as_half(sa)), ra, acc_a);
                acc_b = fmaf(__half2float(__ushort_as_half(sb)), rb, acc_b);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
            if (kc == NC - 1) {
                // tile done: lanes with c == 0 hold column 0 for rows g8 (acc_a) and g8 + 8 (acc_b)
                float* rt = red + ((t - t0) & 1) * (GV_CWARPS * 16);
                if (c == 0) {
                    rt[warp * 16 + g8] = acc_a;
                    rt[warp * 16 + g8 + 8] = acc_b;
                }
                gv_named_barrier();
                if (warp == 0 && lane < 16) {
                    float sum = 0.0f;
#pragma unroll
                    for (int w = 0; w < GV_CWARPS; ++w) sum += rt[w * 16 + lane];  // warp order
                    const int n = t * 16 + lane;
                    if (n < N) Y[n] = __float2half_rn(sum);
                }
                acc_a = 0.0f;
                acc_b = 0.0f;
            }
        }
    }
}

// ------------------------------------------------------------------------------------ host side
size_t gemv_stream_smem(int64_t K) {
    if (K > 65536) return SIZE_MAX;  // the activation row is staged whole in shared memory
    return (size_t)gv_layout((int)K).total + 1024;
}

cudaError_t launch_gemv_stream(const uint16_t* X, int64_t N, int64_t K, const uint32_t* packed,
                               const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, bool weights_static,
                               int* status, cudaStream_t stream) {
    CUtensorMap tm;
    if (!make_tensor_map_2d(&tm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(K / 8), (uint64_t)N,
                            GV_KC / 8, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const size_t smem = gemv_stream_smem(K);
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(gemv_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    const int n_tiles = (int)((N + 15) / 16);
    const int sms = device_sm_count();
    const int grid = n_tiles < sms ? n_tiles : sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(GV_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_static ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_stream_kernel, tm, reinterpret_cast<const __half*>(X),
                              reinterpret_cast<const unsigned short*>(scales), zeros, reinterpret_cast<__half*>(Y),
                              (int)N, (int)K, n_tiles, weights_static ? 1 : 0, status);
}

}  // namespace w4
