// Decode GEMV / skinny GEMM for M <= 8: Y = X dequant(W)^T, streamed at HBM rate.
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the GEMV kernel serves token-by-token generation,
// where the layer is bound by memory traffic and weight reuse is minimal.  The traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale and zero point per group of 128.
//
// Design (sm_100a):
//  * Persistent: one CTA per SM; CTA c owns a contiguous range of 16-row tiles over the whole K,
//    so every output is finished inside one CTA (no split-K workspace, no cluster barrier).
//  * A producer warp streams the packed tile through a GV_STAGES-deep shared-memory ring with
//    TMA (16 rows x 2048 k = 16 KB per stage), so each SM keeps ~96 KB of weights in flight no
//    matter how long one stage takes.  With static weights it starts before the preceding kernel
//    has finished (programmatic dependent launch).
//  * Sixteen consumer warps take one group of 128 each per stage and run mma.sync m16n8k16 with
//    the 16 weight rows as the A operand and the (up to 8) activation rows as B.  Dequantisation
//    is one LOP3 per two weights: the operands are the raw fp16 values 1024+q (low nibble of a
//    byte) and 1024+16q (high nibble); activations that meet high nibbles are staged pre-multiplied
//    by 1/16, and the constant offsets and the zero point are removed per group in fp32 with the
//    exact activation sums
//        sum_k x_k (q_k - z) = raw - 1024 (Sl + Sh') - z (Sl + 16 Sh'),
//    Sl = sum of x over low-nibble slots, Sh' = sum of the staged x/16 over high-nibble slots
//    (both summed exactly in fp64).  The group's fp16 scale then multiplies that sum in fp32.
//  * The activations are staged once per CTA with each 8-k chunk as
//    [x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16], so one 16-byte shared load yields the B
//    fragments of the two MMAs that consume one packed word.
//  * Partial sums of the sixteen warps are added in warp order in shared memory (deterministic).
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

constexpr int GV_CWARPS = 16;                     // consumer warps (one group each per stage)
constexpr int GV_THREADS = 32 * (GV_CWARPS + 1);  // + one producer warp
constexpr int GV_KC = 128 * GV_CWARPS;            // k per stage
constexpr uint32_t GV_STAGE_BYTES = 16 * GV_KC / 2;  // 16 KB of packed codes
constexpr int GV_STAGES = 6;
constexpr int GV_PF = 4;  // units of metadata prefetched ahead
constexpr int GV_MAXM = 8;

struct GvLayout {
    uint32_t ring, xs, corr, red, bars, total;
};

__host__ __device__ inline GvLayout gv_layout(int M, int K) {
    GvLayout L;
    L.ring = 0;
    L.xs = GV_STAGES * GV_STAGE_BYTES;
    L.corr = L.xs + (uint32_t)M * (uint32_t)K * 2;               // float2 [G][8]
    L.red = L.corr + (uint32_t)(K / 128) * GV_MAXM * 8;         // 2 x warps x 16 rows x 8 cols
    L.bars = L.red + 2 * GV_CWARPS * 16 * GV_MAXM * 4;
    L.total = L.bars + 2 * GV_STAGES * 8 + 8;
    return L;
}

__device__ __forceinline__ void gv_named_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * GV_CWARPS) : "memory");
}

__global__ void __launch_bounds__(GV_THREADS, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X,
                       const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                       __half* __restrict__ Y, int M, int N, int K, int n_tiles, int weights_early,
                       int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA destinations need an aligned base: round up (the launch reserves 1 KB of slack)
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    const GvLayout L = gv_layout(M, K);
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
            int issued = 0, t = t0, kc = 0, s = 0;
            uint32_t ph = 0;
            for (int u = 0; u < n_units; ++u) {
                // The ring is full: from here on progress depends on the consumers, who first
                // wait for the preceding kernel; start the bounded waits only after that point.
                if (u == GV_STAGES && weights_early) pdl_wait();
                if (!mbar_wait_bounded(empty_bar(s), ph ^ 1, abort_flag)) {
                    *abort_flag = 1;
                    record_status(status, W4_ERR_DEVICE_TIMEOUT);
                    break;
                }
                mbar_arrive_expect_tx(full_bar(s), GV_STAGE_BYTES);
                tma_load_2d(sbase + L.ring + s * GV_STAGE_BYTES, &tmW, kc * (GV_KC / 8), t * 16, full_bar(s));
                ++issued;
                if (++kc == NC) { kc = 0; ++t; }
                if (++s == GV_STAGES) { s = 0; ph ^= 1; }
            }
            for (int u = issued - GV_STAGES; u < issued; ++u)  // no loads in flight at exit
                if (u >= 0) mbar_wait_bounded(full_bar(u % GV_STAGES), (u / GV_STAGES) & 1, nullptr, 200000000ull);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    pdl_wait();  // the activations may be produced by the preceding kernel
    __half* xs = reinterpret_cast<__half*>(smem + L.xs);
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    const int cpr = K / 8;  // 8-k chunks per activation row
    for (int i = tid; i < M * cpr; i += 32 * GV_CWARPS) {
        const uint4 r = ldg_cached(X + (int64_t)i * 8);  // rows are contiguous: chunk i of row i / cpr
        uint4 p;
        p.x = __byte_perm(r.x, r.z, 0x5410);         // x0, x4
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
    for (int idx = tid; idx < G * GV_MAXM; idx += 32 * GV_CWARPS) {
        const int g = idx / GV_MAXM, m = idx % GV_MAXM;
        double lo = 0.0, hi = 0.0;  // exact: at most 128 fp16 values
        if (m < M) {
            const __half* xg = xs + (int64_t)m * K + g * 128;
            for (int i = 0; i < 128; i += 8) {
                lo += (double)__half2float(xg[i + 0]) + (double)__half2float(xg[i + 1]) +
                      (double)__half2float(xg[i + 4]) + (double)__half2float(xg[i + 5]);
                hi += (double)__half2float(xg[i + 2]) + (double)__half2float(xg[i + 3]) +
                      (double)__half2float(xg[i + 6]) + (double)__half2float(xg[i + 7]);
            }
        }
        corr[idx] = make_float2((float)(1024.0 * (lo + hi)), (float)(lo + 16.0 * hi));
    }
    gv_named_barrier();

    const int g8 = lane >> 2, c = lane & 3;
    float* red = reinterpret_cast<float*>(smem + L.red);
    const bool xlane = g8 < M;  // B column g8 holds activation row g8
    const __half* xrow = xs + (int64_t)(xlane ? g8 : 0) * K;
    const unsigned short* srow = scales + (int64_t)(t0 * 16 + g8) * G;
    const uint8_t* zrow = zeros + (int64_t)(t0 * 16 + g8) * G;

    // Metadata of the unit GV_PF ahead: (tile, chunk) tracked incrementally, raw loads kept in
    // their own registers until use.
    int pf_t = t0, pf_kc = 0;
    auto meta_load = [&](unsigned short& sa, unsigned short& sb, uint8_t& za, uint8_t& zb) {
        sa = 0; sb = 0; za = 0; zb = 0;
        if (pf_t < t1) {
            const int gi = pf_kc * GV_CWARPS + warp;
            if (gi < G) {
                const int na = pf_t * 16 + g8;
                const int64_t off = (int64_t)(pf_t - t0) * 16 * G + gi;
                if (na < N) { sa = __ldg(srow + off); za = __ldg(zrow + off); }
                if (na + 8 < N) { sb = __ldg(srow + off + 8 * G); zb = __ldg(zrow + off + 8 * G); }
            }
            if (++pf_kc == NC) { pf_kc = 0; ++pf_t; }
        }
    };
    unsigned short psa[GV_PF], psb[GV_PF];
    uint8_t pza[GV_PF], pzb[GV_PF];
#pragma unroll
    for (int p = 0; p < GV_PF; ++p) meta_load(psa[p], psb[p], pza[p], pzb[p]);

    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // rows (g8, g8+8) x cols (2c, 2c+1)
    int t = t0, kc = 0, s = 0;
    uint32_t ph = 0;
    for (int u0 = 0; u0 < n_units; u0 += GV_PF) {
#pragma unroll
        for (int p = 0; p < GV_PF; ++p) {
            if (u0 + p >= n_units) break;  // uniform across the CTA
            const unsigned short sa = psa[p], sb = psb[p];
            const uint32_t za = pza[p], zb = pzb[p];
            meta_load(psa[p], psb[p], pza[p], pzb[p]);
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
                const unsigned char* st = smem + L.ring + s * GV_STAGE_BYTES + warp * 64 + c * 16;
                const uint4 A = *reinterpret_cast<const uint4*>(st + g8 * (GV_KC / 2));
                const uint4 B = *reinterpret_cast<const uint4*>(st + (g8 + 8) * (GV_KC / 2));
                const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
                const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
                const __half* xg = xrow + gi * 128 + c * 32;
                float cc[4][4];  // four independent accumulation chains, one per packed word
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) cc[j][e] = 0.0f;
                    const uint32_t a = wA[j], b = wB[j], a8 = a >> 8, b8 = b >> 8;
                    uint4 xf = make_uint4(0u, 0u, 0u, 0u);
                    if (xlane) xf = *reinterpret_cast<const uint4*>(xg + j * 8);
                    mma_16816(cc[j], lop3_and_or(a, 0x000F000Fu, 0x64006400u),
                              lop3_and_or(b, 0x000F000Fu, 0x64006400u), lop3_and_or(a, 0x00F000F0u, 0x64006400u),
                              lop3_and_or(b, 0x00F000F0u, 0x64006400u), xf.x, xf.y);
                    mma_16816(cc[j], lop3_and_or(a8, 0x000F000Fu, 0x64006400u),
                              lop3_and_or(b8, 0x000F000Fu, 0x64006400u), lop3_and_or(a8, 0x00F000F0u, 0x64006400u),
                              lop3_and_or(b8, 0x00F000F0u, 0x64006400u), xf.z, xf.w);
                }
                const float4 cs = *reinterpret_cast<const float4*>(corr + gi * GV_MAXM + 2 * c);  // cols 2c, 2c+1
                const float fza = (float)za, fzb = (float)zb;
                const float fsa = __half2float(__ushort_as_half(sa)), fsb = __half2float(__ushort_as_half(sb));
                const float r0 = (cc[0][0] + cc[1][0]) + (cc[2][0] + cc[3][0]);
                const float r1 = (cc[0][1] + cc[1][1]) + (cc[2][1] + cc[3][1]);
                const float r2 = (cc[0][2] + cc[1][2]) + (cc[2][2] + cc[3][2]);
                const float r3 = (cc[0][3] + cc[1][3]) + (cc[2][3] + cc[3][3]);
                acc[0] = fmaf(fsa, r0 - fmaf(fza, cs.y, cs.x), acc[0]);  // row g8,   col 2c
                acc[1] = fmaf(fsa, r1 - fmaf(fza, cs.w, cs.z), acc[1]);  // row g8,   col 2c+1
                acc[2] = fmaf(fsb, r2 - fmaf(fzb, cs.y, cs.x), acc[2]);  // row g8+8, col 2c
                acc[3] = fmaf(fsb, r3 - fmaf(fzb, cs.w, cs.z), acc[3]);  // row g8+8, col 2c+1
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
            if (++s == GV_STAGES) { s = 0; ph ^= 1; }
            if (++kc == NC) {
                // tile done: combine the sixteen warps' partial sums in warp order
                float* rt = red + ((t - t0) & 1) * (GV_CWARPS * 16 * GV_MAXM);
                float* mine = rt + warp * (16 * GV_MAXM);
                mine[g8 * GV_MAXM + 2 * c] = acc[0];
                mine[g8 * GV_MAXM + 2 * c + 1] = acc[1];
                mine[(g8 + 8) * GV_MAXM + 2 * c] = acc[2];
                mine[(g8 + 8) * GV_MAXM + 2 * c + 1] = acc[3];
                gv_named_barrier();
                for (int o = tid; o < 16 * M; o += 32 * GV_CWARPS) {
                    const int row = o % 16, m = o / 16;
                    float sum = 0.0f;
#pragma unroll
                    for (int w = 0; w < GV_CWARPS; ++w) sum += rt[w * (16 * GV_MAXM) + row * GV_MAXM + m];
                    const int n = t * 16 + row;
                    if (n < N) Y[(int64_t)m * N + n] = __float2half_rn(sum);
                }
                acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
                kc = 0;
                ++t;
            }
        }
    }
}

// ------------------------------------------------------------------------------------ host side
size_t gemv_stream_smem(int64_t M, int64_t K) {
    if (M < 1 || M > GV_MAXM || K > 65536) return SIZE_MAX;  // activations are staged whole
    return (size_t)gv_layout((int)M, (int)K).total + 1024;
}

cudaError_t launch_gemv_stream(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                               const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, bool weights_static,
                               int* status, cudaStream_t stream) {
    CUtensorMap tm;
    if (!make_tensor_map_2d(&tm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(K / 8), (uint64_t)N,
                            GV_KC / 8, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const size_t smem = gemv_stream_smem(M, K);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
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
                              (int)M, (int)N, (int)K, n_tiles, weights_static ? 1 : 0, status);
}

}  // namespace w4
