// Tensor-core W4A16 GEMM for prefill-sized M (tcgen05 + TMEM + TMA, sm_100a).
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the batch GEMM variant dequantises INT4 weights on
// the fly instead of materialising FP16 weights.  Prefill is a dense contraction, so it runs on
// the 5th-generation tensor cores:
//
//   D[m, n] = sum_k X[m, k] * What[n, k],  What = (q - z) * s16 rounded once to fp16.
//
// One CTA computes an (MT x 128) (rows of X) x 256 (rows of W) tile: MT fp32 accumulators of
// 128 x 256 in TMEM (256 columns each) share one dequantised W tile, so with MT = 2 every
// dequantised weight feeds two MMAs.  K advances in steps of 64 through a shared-memory ring:
//   warp 0      TMA producer: X tile (MT*128 x 64 fp16, 128-byte swizzle) and the packed W tile
//               (256 rows x 32 bytes) per stage; plain (non-multicast) tile loads.
//   warp 1      one elected thread issues MT x 4 tcgen05.mma (M=128, N=256, K=16) per stage and
//               commits each stage back to the producer.
//   warp 2      allocates / frees TMEM.
//   warps 4-11  dequantise: each thread turns one packed row (64 codes) into 64 fp16 weights in
//               the UMMA K-major 128-byte-swizzle layout, then runs the epilogue (TMEM -> fp16 Y).
// Other modes (for the AWQ search) load an fp16 B operand with TMA instead of dequantising and
// replace the fp16 store (EPI 0) by a per-tile sum of squares (EPI 1), an fp32 store (EPI 2), or a
// per-tile sum of D[m, n] * A[m, n] (EPI 3, for N == K: A read back from global memory).
// w4_gemm also runs the dequantising GEMM with K cut into slices of whole groups (EPI 2 fp32
// partial tiles, summed in slice order by splitk_reduce_kernel) when its tiles fill fewer than
// half the SMs, and with a tail split (the full waves as one launch, the last, at most half full
// wave's tiles in K slices with compact partials summed by tail_reduce_kernel).
//
// Every mbarrier wait is bounded; on timeout the kernel records W4_ERR_DEVICE_TIMEOUT, stops
// issuing work, drains what it issued and frees TMEM before it exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

constexpr int TC_BN = 256;  // W rows per tile (the AWQ modes; w4_gemm also has 128-row W tiles)
constexpr int TC_BK = 64;
constexpr int TC_THREADS = 384;
constexpr int TC_DEQ_THREADS = 256;
constexpr uint32_t TC_A1_BYTES = 128 * TC_BK * 2;   // 16 KB per 128-row X tile
constexpr int TC_GROUP_M = 8;  // raster: CTAs in flight share X and W tiles through L2

// Tile of (128 MT) rows of X by BN rows of W; as many ring stages as fit (at most 6).
template <bool DEQ, int MT, int BN>
struct TcCfg {
    static constexpr int kBM = 128 * MT;
    static constexpr uint32_t kA = TC_A1_BYTES * MT;
    static constexpr uint32_t kB = BN * TC_BK * 2;  // fp16 W tile (dequantised or loaded)
    static constexpr uint32_t kP = BN * TC_BK / 2;  // packed codes of the W tile
    static constexpr uint32_t kStage = kA + kB + (DEQ ? kP : 0);
    static constexpr int kFit = (int)((227u * 1024u - 1280u) / kStage);
    static constexpr int kStages = kFit < 6 ? kFit : 6;
    static constexpr uint32_t kBarOff = kStage * kStages;
    static constexpr uint32_t kBytes = kBarOff + 256 + 1024;  // barriers + slack for 1 KB alignment
    static constexpr uint32_t kTmemCols = BN * MT;
};

__device__ __forceinline__ void tc_tile_coords(int t, int m_tiles, int n_tiles, int& mt, int& nt) {
    const int per_group = TC_GROUP_M * n_tiles;
    const int group = t / per_group;
    const int first_m = group * TC_GROUP_M;
    const int gm = min(TC_GROUP_M, m_tiles - first_m);
    const int r = t - group * per_group;
    mt = first_m + r % gm;
    nt = r / gm;
}

template <bool DEQ, int EPI, int MT, int BN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __half* __restrict__ scales, const uint8_t* __restrict__ zeros,
                   __half* __restrict__ Y, double* __restrict__ sse_part, float* __restrict__ Cf,
                   const __half* __restrict__ Adot, int M, int N, int K, int m_tiles, int n_tiles,
                   int lower, int ksplit, int tile_base, int n_compact, int* status) {
    constexpr bool SSE = EPI == 1 || EPI == 3;  // modes that reduce the tile to one fp64 partial
    using C = TcCfg<DEQ, MT, BN>;
    constexpr int S = C::kStages;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_align1024(smem_raw);
    const uint32_t sbase = smem_u32(smem);
    auto a_addr = [&](int s) { return sbase + s * C::kStage; };
    auto b_addr = [&](int s) { return sbase + s * C::kStage + C::kA; };
    auto p_addr = [&](int s) { return sbase + s * C::kStage + C::kA + C::kB; };
    const uint32_t bar0 = sbase + C::kBarOff;
    auto full_bar = [&](int s) { return bar0 + 8 * s; };
    auto deq_bar = [&](int s) { return bar0 + 8 * (S + s); };
    auto empty_bar = [&](int s) { return bar0 + 8 * (2 * S + s); };
    const uint32_t accum_bar = bar0 + 8 * (3 * S);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kBarOff + 8 * (3 * S + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kBarOff + 8 * (3 * S + 1) + 8);
    double* red = reinterpret_cast<double*>(smem + C::kBarOff + 128);  // 8 doubles for the SSE epilogue

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int mt, nt;
    // ksplit > 1: CTA b computes K slice b % ksplit of tile tile_base + b / ksplit (whole groups of
    // 128 k) and stores its fp32 partial tile into slice (b % ksplit) of Cf: [slice][M][N], or with
    // n_compact > 0 [slice][n_compact tiles][kBM][BN] (the tiles of this launch only)
    const int slice = ksplit > 1 ? (int)(blockIdx.x % ksplit) : 0;
    const int tile_id = (ksplit > 1 ? (int)(blockIdx.x / ksplit) : (int)blockIdx.x) + tile_base;
    if (lower) {  // only the tiles on or below the diagonal of a square product (one per CTA)
        const int t = tile_id;
        mt = (int)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
        while ((mt + 1) * (mt + 2) / 2 <= t) ++mt;
        while (mt * (mt + 1) / 2 > t) --mt;
        nt = t - mt * (mt + 1) / 2;
    } else {
        tc_tile_coords(tile_id, m_tiles, n_tiles, mt, nt);
    }
    const int m0 = mt * C::kBM, n0 = nt * BN;
    const int G = K >> 7;
    // this CTA's k-blocks [kb0, kb0 + nk): all K / 64 of them, or with ksplit > 1 (K a multiple of
    // 128) two per group of 128, a slice starting on a group
    const int kb0 = ksplit > 1 ? 2 * (int)(((int64_t)slice * G) / ksplit) : 0;
    const int nk = ksplit > 1 ? 2 * (int)(((int64_t)(slice + 1) * G) / ksplit) - kb0 : K / TC_BK;
    if (ksplit > 1 && EPI == 2)
        Cf += n_compact ? ((int64_t)slice * n_compact + (tile_id - tile_base)) * C::kBM * BN : (int64_t)slice * M * N;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(deq_bar(s), TC_DEQ_THREADS / 32);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(accum_bar, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // A programmatically dependent successor may launch now (it waits for this grid before it
    // reads anything this grid writes).
    pdl_launch_dependents();
    const uint32_t tmem_d = *tmem_slot;

    auto fail = [&]() {
        *abort_flag = 1;
        record_status(status, W4_ERR_DEVICE_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t tx = C::kA + (DEQ ? C::kP : C::kB);
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % S, kb = kb0 + i;
                const uint32_t ph = (i / S) & 1;
                if (!mbar_wait_bounded(empty_bar(s), ph ^ 1, abort_flag)) { fail(); break; }
                mbar_arrive_expect_tx(full_bar(s), tx);
                tma_load_2d(a_addr(s), &tmA, kb * TC_BK, m0, full_bar(s));
                if (DEQ) tma_load_2d(p_addr(s), &tmB, kb * (TC_BK / 8), n0, full_bar(s));
                else tma_load_2d(b_addr(s), &tmB, kb * TC_BK, n0, full_bar(s));
                ++issued;
            }
            // Never leave with tile loads in flight: wait (bounded) for the last stages issued.
            for (int kb = issued - S; kb < issued; ++kb) {
                if (kb < 0) continue;
                mbar_wait_bounded(full_bar(kb % S), (kb / S) & 1, nullptr, 200000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(128, BN);
            bool ok = true;
            for (int i = 0; i < nk && ok; ++i) {
                const int s = i % S;
                const uint32_t ph = (i / S) & 1;
                if (!mbar_wait_bounded(full_bar(s), ph, abort_flag)) { fail(); ok = false; break; }
                if (DEQ && !mbar_wait_bounded(deq_bar(s), ph, abort_flag)) { fail(); ok = false; break; }
                tc_fence_after();
                const uint64_t bd = sw128_kmajor_desc(b_addr(s));
#pragma unroll
                for (int j = 0; j < TC_BK / 16; ++j) {
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        const uint64_t ad = sw128_kmajor_desc(a_addr(s) + t * TC_A1_BYTES);
                        // +32 bytes along K per MMA inside the 128-byte swizzled row
                        mma_f16_ss(tmem_d + t * BN, ad + 2 * j, bd + 2 * j, idesc, (i | j) != 0);
                    }
                }
                tc_commit(empty_bar(s));
            }
            tc_commit(accum_bar);  // fires once every MMA issued above has completed
        }
    } else if (warp >= 4) {
        const int d = tid - 128;  // 0..255
        if (DEQ) {
            // -------------------------------------------------------- dequantisation
            // W tile rows are shared by 256 / BN threads, each dequantising WPT of the row's 8 words
            constexpr int WPT = 8 * BN / TC_DEQ_THREADS;
            const int r = d % BN;  // tile row (row of W)
            const int part = d / BN;
            const int n = n0 + r;
            const bool nvalid = n < N;
            uint32_t s2 = 0, zl = 0, zh = 0;
            const uint32_t b_row = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
            const unsigned short* srow = reinterpret_cast<const unsigned short*>(scales) + (int64_t)n * G;
            const uint8_t* zrow = zeros + (int64_t)n * G;
            // scale/zero of the next group are fetched one group (two stages) ahead
            uint32_t sc_next = 0, z_next = 0;
            if (nvalid) {
                sc_next = __ldg(srow + kb0 / 2);
                z_next = __ldg(zrow + kb0 / 2);
            }
            for (int i = 0; i < nk; ++i) {
                const int s = i % S, kb = kb0 + i;
                const uint32_t ph = (i / S) & 1;
                if ((kb & 1) == 0) {  // a new group of 128 every second stage
                    const int g = kb >> 1;
                    const uint32_t sb = sc_next, z = z_next;
                    if (nvalid && g + 1 < G) {
                        sc_next = __ldg(srow + g + 1);
                        z_next = __ldg(zrow + g + 1);
                    }
                    s2 = sb | (sb << 16);
                    zl = (0x6400u + z) * 0x10001u;
                    zh = (0xD400u | (z << 4)) * 0x10001u;
                }
                if (!mbar_wait_bounded(full_bar(s), ph, abort_flag)) { fail(); break; }
                const unsigned char* prow = smem + (p_addr(s) - sbase) + r * 32 + part * (WPT * 4);
                uint32_t words[WPT];
#pragma unroll
                for (int i = 0; i < WPT; i += 4) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(prow + 4 * i);
                    words[i] = w4.x; words[i + 1] = w4.y; words[i + 2] = w4.z; words[i + 3] = w4.w;
                }
                unsigned char* brow = smem + (b_addr(s) - sbase) + b_row;
#pragma unroll
                for (int cw = 0; cw < WPT; ++cw) {
                    const int c = part * WPT + cw;  // word (8 k) within the row's 64 k
                    const uint32_t w = words[cw];
                    uint32_t lo0 = hsub2_u32(lop3_and_or(w, 0x000F000Fu, 0x64006400u), zl);            // n0,n4
                    uint32_t hi0 = hfma2_u32(lop3_and_or(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zh);  // n1,n5
                    const uint32_t w8 = w >> 8;
                    uint32_t lo1 = hsub2_u32(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), zl);           // n2,n6
                    uint32_t hi1 = hfma2_u32(lop3_and_or(w8, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zh); // n3,n7
                    lo0 = hmul2_u32(lo0, s2);
                    hi0 = hmul2_u32(hi0, s2);
                    lo1 = hmul2_u32(lo1, s2);
                    hi1 = hmul2_u32(hi1, s2);
                    uint4 o;
                    o.x = __byte_perm(lo0, hi0, 0x5410);  // k0, k1
                    o.y = __byte_perm(lo1, hi1, 0x5410);  // k2, k3
                    o.z = __byte_perm(lo0, hi0, 0x7632);  // k4, k5
                    o.w = __byte_perm(lo1, hi1, 0x7632);  // k6, k7
                    *reinterpret_cast<uint4*>(brow + ((c ^ (r & 7)) << 4)) = o;
                }
                fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(deq_bar(s));
            }
        }
        // ------------------------------------------------------------ epilogue
        // warp (4 + 4*slot + q) reads TMEM lanes [32q, 32q + 32) (the quarter it may access):
        // MT == 1: columns [BN/2 * slot, BN/2 * slot + BN/2) of the single accumulator;
        // MT == 2: all BN columns of accumulator `slot`.
        const int q = warp & 3;
        const int slot = (warp - 4) >> 2;
        const int acc = MT == 1 ? 0 : slot;
        const int c_begin = MT == 1 ? slot * (BN / 2) : 0;
        const int c_count = MT == 1 ? BN / 2 : BN;
        // not cut short by the abort flag: TMEM is freed only after every issued MMA completed
        const bool ok = mbar_wait_bounded(accum_bar, 0, nullptr, 4000000000ull);
        if (!ok) fail();
        tc_fence_after();
        const int m = m0 + acc * 128 + q * 32 + lane;
        double sq = 0.0;
        if (ok && !*abort_flag) {
#pragma unroll 1
            for (int cc = 0; cc < c_count; cc += 32) {
                const int col = c_begin + cc;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + col), v);
                tmem_wait_ld();
                if (EPI == 1) {
                    float a = 0.0f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float f = __uint_as_float(v[i]);
                        a = fmaf(f, f, a);
                    }
                    sq += (double)a;
                } else if (EPI == 3) {
                    if (m < M) {  // sum of D[m, n] * A[m, n] over this thread's 32 columns
                        const int nb = n0 + col;
                        const __half* arow = Adot + (int64_t)m * K + nb;
                        float a = 0.0f;
                        if (nb + 32 <= N) {
#pragma unroll
                            for (int i = 0; i < 32; i += 8) {
                                const uint4 h8 = *reinterpret_cast<const uint4*>(arow + i);
                                const __half2* hp = reinterpret_cast<const __half2*>(&h8);
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const float2 f = __half22float2(hp[u]);
                                    a = fmaf(__uint_as_float(v[i + 2 * u]), f.x, a);
                                    a = fmaf(__uint_as_float(v[i + 2 * u + 1]), f.y, a);
                                }
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < N) a = fmaf(__uint_as_float(v[i]), __half2float(arow[i]), a);
                        }
                        sq += (double)a;
                    }
                } else if (EPI == 2 && n_compact) {  // the tile's own [kBM][BN] block: no bounds
                    float* crow = Cf + (int64_t)(m - m0) * BN + col;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(crow + i) =
                            make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                        __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                } else if (EPI == 2) {
                    if (m < M) {
                        const int nb = n0 + col;
                        float* crow = Cf + (int64_t)m * N + nb;
                        if (nb + 32 <= N) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4*>(crow + i) =
                                    make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < N) crow[i] = __uint_as_float(v[i]);
                        }
                    }
                } else if (m < M) {
                    const int nb = n0 + col;
                    __half* yrow = Y + (int64_t)m * N + nb;
                    if (nb + 32 <= N) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 o;
                            o.x = pack_half2(__uint_as_float(v[i + 0]), __uint_as_float(v[i + 1]));
                            o.y = pack_half2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                            o.z = pack_half2(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
                            o.w = pack_half2(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
                            *reinterpret_cast<uint4*>(yrow + i) = o;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (nb + i < N) yrow[i] = __float2half_rn(__uint_as_float(v[i]));
                    }
                }
            }
        }
        if (SSE) {
            // rows beyond M read zeros from TMA fill, so they add nothing
#pragma unroll
            for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (lane == 0) red[warp - 4] = sq;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (SSE && tid == 0) {
        double t = 0.0;
        for (int i = 0; i < 8; ++i) t += red[i];
        sse_part[(int64_t)mt * n_tiles + nt] = t;
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_d, C::kTmemCols);
    }
    // Launched as a programmatic dependent (pdl), this grid ends only after its predecessor has:
    // a plain launch after it then also follows the predecessor.  A no-op otherwise.
    pdl_wait();
}

// ------------------------------------------------------------------------------------ host side
// Relative time of one tile of each w4_gemm tile shape (MT x 128 rows of X, BN rows of W), in
// units of a (1 x 128) x 128 tile at the same K.  Measured on B200 at M = 4096, K = N = 4096 (many
// waves of every shape, rotating weights): 113.0, 172.9, 150.7 and 205.1 us for 256, 512, 512
// and 1024 tiles, i.e. per-tile times 2.20 : 1.69 : 1.47 : 1.00.  Larger tiles cost more per tile
// but much less per flop (each dequantised weight feeds MT MMAs, each X tile BN rows of W).
#ifndef TC_TT_2_256
#define TC_TT_2_256 2.20
#define TC_TT_1_256 1.69
#define TC_TT_2_128 1.47
#define TC_TT_1_128 1.00
#endif
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint32_t elem_bytes,
                        uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swz) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * elem_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <bool DEQ, int EPI, int MT, int BN>
static cudaError_t set_tc_attrs() {
    static std::once_flag once[64];
    static cudaError_t err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        err[dev] = cudaFuncSetAttribute(tc_gemm_kernel<DEQ, EPI, MT, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)TcCfg<DEQ, MT, BN>::kBytes);
    });
    return err[dev];
}

template <bool DEQ, int EPI, int MT, int BN = TC_BN>
static cudaError_t launch_tc(const uint16_t* X, int64_t M, const void* Bop, int64_t N, int64_t K,
                             const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, double* sse_part,
                             int* status, cudaStream_t stream, float* Cf = nullptr, bool lower = false,
                             int ksplit = 1, bool pdl = false, int tile_base = 0, int n_tiles_launch = -1,
                             int n_compact = 0) {
    using C = TcCfg<DEQ, MT, BN>;
    CUtensorMap ta, tb;
    if (!make_tensor_map_2d(&ta, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, TC_BK, C::kBM,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool okb =
        DEQ ? make_tensor_map_2d(&tb, Bop, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)(K / 8), (uint64_t)N, TC_BK / 8,
                          BN, CU_TENSOR_MAP_SWIZZLE_NONE)
            : make_tensor_map_2d(&tb, Bop, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)N, TC_BK, BN,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    if (!okb) return cudaErrorInvalidValue;
    cudaError_t e = set_tc_attrs<DEQ, EPI, MT, BN>();
    if (e != cudaSuccess) return e;
    const int m_tiles = (int)((M + C::kBM - 1) / C::kBM);
    const int n_tiles = (int)((N + BN - 1) / BN);
    if (lower && (M != N || C::kBM != BN)) return cudaErrorInvalidValue;  // square tiles of a square product
    const int all_tiles = lower ? m_tiles * (m_tiles + 1) / 2 : m_tiles * n_tiles;
    const int grid = (n_tiles_launch >= 0 ? n_tiles_launch : all_tiles) * ksplit;
    if (grid == 0) return cudaSuccess;
    // pdl: may start while the preceding kernel runs; only for operands that kernel does not
    // write (the grid still ends after it: see the kernel's last statement)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<DEQ, EPI, MT, BN>, ta, tb, reinterpret_cast<const __half*>(scales),
                              zeros, reinterpret_cast<__half*>(Y), sse_part, Cf, reinterpret_cast<const __half*>(X),
                              (int)M, (int)N, (int)K, m_tiles, n_tiles, lower ? 1 : 0, ksplit, tile_base, n_compact,
                              status);
}

// 256-row tiles once M is large enough to fill them; 128-row tiles otherwise.
static int tc_mt(int64_t M) { return M > 128 ? 2 : 1; }

// Tile shape of w4_gemm's tensor-core path: the fewest waves of one-CTA-per-SM tiles, weighed by
// each shape's per-tile time (larger tiles share every dequantised weight between more rows of X
// and every X tile between more rows of W, so they run closer to the tensor peak).
void tc_w4_pick(int64_t M, int64_t N, int* mt_out, int* bn_out) {
    const int64_t sms = device_sm_count();
    const int shapes[4][2] = {{2, 256}, {1, 256}, {2, 128}, {1, 128}};
    // relative time of one tile, from the measured per-tile rates of each shape
    const double tile_time[4] = {TC_TT_2_256, TC_TT_1_256, TC_TT_2_128, TC_TT_1_128};
    double best = -1.0;
    *mt_out = 2;
    *bn_out = 256;
    for (int i = 0; i < 4; ++i) {
        const int mt = shapes[i][0], bn = shapes[i][1];
        if (mt == 2 && M <= 128) continue;
        const int64_t tiles = ((M + 128 * mt - 1) / (128 * mt)) * ((N + bn - 1) / bn);
        const double t = (double)((tiles + sms - 1) / sms) * tile_time[i];
        if (best < 0.0 || t < best) {
            best = t;
            *mt_out = mt;
            *bn_out = bn;
        }
    }
}

// K slices of w4_gemm's tensor-core path: (128 or 256) x 256 tiles (128 rows of X up to M = 128)
// that fill fewer than half the SMs are split along K into up to 8 slices of whole groups, at
// least 8 k-blocks of 64 each, so that tiles x slices fill the SMs; 1 = no split (always for
// M <= 16, which the GEMV serves).
int tc_w4_split(int64_t M, int64_t N, int64_t K) {
    if (M <= 16) return 1;
    const int64_t sms = device_sm_count();
    const int64_t bm = M > 128 ? 256 : 128;
    const int64_t tiles = ((M + bm - 1) / bm) * ((N + 255) / 256);
    if (2 * tiles >= sms) return 1;
    int64_t s = sms / tiles;
    const int64_t max_by_k = (K / TC_BK) / 8;
    if (s > max_by_k) s = max_by_k;
    if (s > 8) s = 8;
    return s >= 2 ? (int)s : 1;
}

// Tail split of w4_gemm's tensor-core path: when the 256 x 256 tiles (the picked shape) fill whole
// waves of one CTA per SM and then at most half of one more, the full waves run as one launch and
// the last wave's `tail` tiles are cut along K into ks slices (whole groups, at least 8 k-blocks
// each, ks <= 8) that fill the SMs; their fp32 partials are added per tile in slice order.  False:
// no tail split.
bool tc_w4_tail(int64_t M, int64_t N, int64_t K, int* full, int* tail, int* ks) {
    if (M <= 128 || tc_w4_split(M, N, K) > 1) return false;
    int mt = 2, bn = 256;
    tc_w4_pick(M, N, &mt, &bn);
    if (mt != 2 || bn != 256) return false;
    const int64_t sms = device_sm_count();
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int64_t t = tiles % sms;
    if (tiles < sms || t == 0 || 2 * t > sms) return false;
    int64_t s = sms / t;
    const int64_t max_by_k = (K / TC_BK) / 8;
    if (s > max_by_k) s = max_by_k;
    if (s > 8) s = 8;
    if (s < 2) return false;
    *full = (int)(tiles - t);
    *tail = (int)t;
    *ks = (int)s;
    return true;
}

size_t tc_w4_workspace(int64_t M, int64_t N, int64_t K) {
    const int s = tc_w4_split(M, N, K);
    if (s > 1) return (size_t)s * (size_t)M * (size_t)N * 4;
    int full = 0, tail = 0, ks = 0;
    if (tc_w4_tail(M, N, K, &full, &tail, &ks)) return (size_t)ks * (size_t)tail * 256 * 256 * 4;
    return 0;
}

int tc_w4_launches(int64_t M, int64_t N, int64_t K) {
    if (tc_w4_split(M, N, K) > 1) return 2;  // the K slices, then their sum
    int full = 0, tail = 0, ks = 0;
    return tc_w4_tail(M, N, K, &full, &tail, &ks) ? 3 : 1;  // full waves, tail slices, their sum
}

// Y at the tail tiles = fp16(sum over the slices of the compact fp32 partial tiles
// P [slice][tile][256][256], in slice order): deterministic.  A programmatic dependent of the
// launch that writes the partials (it waits for that launch before reading them).
__global__ void tail_reduce_kernel(const float* __restrict__ P, int slices, int n_tail, int tile_base, int m_tiles,
                                   int n_tiles, int M, int N, __half* __restrict__ Y) {
    pdl_launch_dependents();
    pdl_wait();
    constexpr int64_t TILE = 256 * 256;
    const int64_t n4 = (int64_t)n_tail * (TILE / 4);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
        const int tl = (int)(e / (TILE / 4));
        const int local = (int)(e - (int64_t)tl * (TILE / 4)) * 4;
        int mt, nt;
        tc_tile_coords(tile_base + tl, m_tiles, n_tiles, mt, nt);
        const int m = mt * 256 + (local >> 8), n = nt * 256 + (local & 255);
        if (m >= M || n >= N) continue;  // N % 8 == 0: n < N covers all four columns
        float4 a = *reinterpret_cast<const float4*>(P + (int64_t)tl * TILE + local);
        for (int s = 1; s < slices; ++s) {
            const float4 b = *reinterpret_cast<const float4*>(P + ((int64_t)s * n_tail + tl) * TILE + local);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        uint2 o;
        o.x = pack_half2(a.x, a.y);
        o.y = pack_half2(a.z, a.w);
        *reinterpret_cast<uint2*>(Y + (int64_t)m * N + n) = o;
    }
}

// Y = fp16(sum over the slices of the fp32 partials, in slice order): deterministic.  Launched as a
// programmatic dependent of the kernel that writes the partials: it waits for that kernel's end
// before reading them, and lets its own dependent start streaming weights meanwhile.
__global__ void splitk_reduce_kernel(const float* __restrict__ P, int slices, int64_t mn, __half* __restrict__ Y) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t n4 = mn / 4;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
        float4 a = reinterpret_cast<const float4*>(P)[e];
        for (int s = 1; s < slices; ++s) {
            const float4 b = reinterpret_cast<const float4*>(P + (int64_t)s * mn)[e];
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        uint2 o;
        o.x = pack_half2(a.x, a.y);
        o.y = pack_half2(a.z, a.w);
        reinterpret_cast<uint2*>(Y)[e] = o;
    }
}

cudaError_t launch_splitk_reduce(const float* P, int slices, int64_t mn, uint16_t* Y, cudaStream_t stream) {
    if (mn % 4 != 0 || (reinterpret_cast<uintptr_t>(P) & 15) || (reinterpret_cast<uintptr_t>(Y) & 7))
        return cudaErrorInvalidValue;
    const int64_t want = (mn / 4 + 255) / 256;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, P, slices, mn, reinterpret_cast<__half*>(Y));
}

cudaError_t launch_tc_w4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                         const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, void* ws, int* status,
                         cudaStream_t stream) {
    const int ks = tc_w4_split(M, N, K);
    if (ks > 1) {  // M * N is a multiple of 8 (N % 8 == 0): whole float4s
        if (!ws) return cudaErrorInvalidValue;
        float* P = static_cast<float*>(ws);
        cudaError_t e = M > 128 ? launch_tc<true, 2, 2, 256>(X, M, packed, N, K, scales, zeros, nullptr, nullptr, status,
                                                             stream, P, false, ks)
                                : launch_tc<true, 2, 1, 256>(X, M, packed, N, K, scales, zeros, nullptr, nullptr, status,
                                                             stream, P, false, ks);
        if (e != cudaSuccess) return e;
        return launch_splitk_reduce(P, ks, M * N, Y, stream);
    }
    int full = 0, tail = 0, tks = 0;
    if (tc_w4_tail(M, N, K, &full, &tail, &tks)) {
        if (!ws) return cudaErrorInvalidValue;
        float* P = static_cast<float*>(ws);
        // the full waves, with their plain epilogue
        cudaError_t e = launch_tc<true, 0, 2, 256>(X, M, packed, N, K, scales, zeros, Y, nullptr, status, stream,
                                                   nullptr, false, 1, false, 0, full, 0);
        if (e != cudaSuccess) return e;
        // the last wave's tiles in K slices, compact partials: nothing the full waves write is read
        // here, so its CTAs start on the SMs the full waves free (programmatic dependent launch)
        e = launch_tc<true, 2, 2, 256>(X, M, packed, N, K, scales, zeros, nullptr, nullptr, status, stream, P, false,
                                       tks, true, full, tail, tail);
        if (e != cudaSuccess) return e;
        const int m_tiles = (int)((M + 255) / 256), n_tiles = (int)((N + 255) / 256);
        const int64_t want = ((int64_t)tail * 256 * 256 / 4 + 255) / 256;
        const int64_t cap = (int64_t)device_sm_count() * 8;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(want < cap ? want : cap), 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, tail_reduce_kernel, (const float*)P, tks, tail, full, m_tiles, n_tiles,
                                  (int)M, (int)N, reinterpret_cast<__half*>(Y));
    }
    int mt = 2, bn = 256;
    tc_w4_pick(M, N, &mt, &bn);
    if (mt == 2 && bn == 256)
        return launch_tc<true, 0, 2, 256>(X, M, packed, N, K, scales, zeros, Y, nullptr, status, stream);
    if (mt == 1 && bn == 256)
        return launch_tc<true, 0, 1, 256>(X, M, packed, N, K, scales, zeros, Y, nullptr, status, stream);
    if (mt == 2)
        return launch_tc<true, 0, 2, 128>(X, M, packed, N, K, scales, zeros, Y, nullptr, status, stream);
    return launch_tc<true, 0, 1, 128>(X, M, packed, N, K, scales, zeros, Y, nullptr, status, stream);
}

cudaError_t launch_tc_sse(const uint16_t* X, int64_t T, const uint16_t* E, int64_t N, int64_t K,
                          double* sse_part, int* status, cudaStream_t stream) {
    if (tc_mt(T) == 2)
        return launch_tc<false, 1, 2>(X, T, E, N, K, nullptr, nullptr, nullptr, sse_part, status, stream);
    return launch_tc<false, 1, 1>(X, T, E, N, K, nullptr, nullptr, nullptr, sse_part, status, stream);
}

cudaError_t launch_tc_f32(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, float* C,
                          int* status, cudaStream_t stream, bool pdl) {
    if (tc_mt(M) == 2)
        return launch_tc<false, 2, 2>(A, M, B, N, K, nullptr, nullptr, nullptr, nullptr, status, stream, C, false, 1,
                                      pdl);
    return launch_tc<false, 2, 1>(A, M, B, N, K, nullptr, nullptr, nullptr, nullptr, status, stream, C, false, 1, pdl);
}

cudaError_t launch_tc_f32_lower(const uint16_t* A, int64_t M, int64_t K, float* C, int* status, cudaStream_t stream,
                                bool pdl) {
    if (tc_mt(M) != 2) return cudaErrorInvalidValue;
    return launch_tc<false, 2, 2>(A, M, A, M, K, nullptr, nullptr, nullptr, nullptr, status, stream, C, true, 1, pdl);
}

cudaError_t launch_tc_f16(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, uint16_t* Y,
                          int* status, cudaStream_t stream) {
    if (tc_mt(M) == 2)
        return launch_tc<false, 0, 2>(A, M, B, N, K, nullptr, nullptr, Y, nullptr, status, stream);
    return launch_tc<false, 0, 1>(A, M, B, N, K, nullptr, nullptr, Y, nullptr, status, stream);
}

cudaError_t launch_tc_dot(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, double* part,
                          int* status, cudaStream_t stream) {
    if (N != K) return cudaErrorInvalidValue;  // the epilogue reads A[m, n] with n as a column of A
    if (tc_mt(M) == 2)
        return launch_tc<false, 3, 2>(A, M, B, N, K, nullptr, nullptr, nullptr, part, status, stream);
    return launch_tc<false, 3, 1>(A, M, B, N, K, nullptr, nullptr, nullptr, part, status, stream);
}

int tc_sse_partials(int64_t T, int64_t N) {
    const int64_t bm = 128 * tc_mt(T);
    return (int)(((T + bm - 1) / bm) * ((N + TC_BN - 1) / TC_BN));
}

}  // namespace w4
