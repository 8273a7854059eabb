// Decode GEMV / skinny GEMM for M <= 16: Y = X dequant(W)^T, streamed at HBM rate.
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the GEMV kernel serves token-by-token generation,
// where the layer is bound by memory traffic and weight reuse is minimal.  The traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale and zero point per group of 128.
//
// Design (sm_100a):
//  * One CTA per SM (or per tile when there are fewer tiles than SMs).  CTA c owns a contiguous,
//    balanced range of 16-row tiles over the whole K (CTA sizes differ by at most one tile), so
//    every output is finished inside one CTA: no split-K workspace, no cluster barrier.  Where
//    the staged activation rows of the whole K would leave a shallow ring (split mode, KS), K is
//    cut into slices of whole stages instead: blockIdx.y is the slice, each CTA stages its slice's
//    activations only, every stage brings its own scales and zero points as two 2-D TMA boxes,
//    and the slices' fp32 partials are summed in slice order by a second launch.
//  * A producer warp streams each tile through a shared-memory ring of 32 KB stages with TMA: one
//    stage is 16 rows x 32 groups (4096 k, 2 KB of each row).  A tile's scales and zero points are
//    one contiguous block of each array and ride on the tile's first stage as two bulk copies.
//    The ring is as deep as the SM's shared memory allows (6 stages at K = 4096).  With static
//    weights the kernel is launched early (programmatic dependent launch) and the producer fills
//    the ring before the preceding kernel has finished; everything that reads the activations or
//    writes Y waits for it.
//  * Sixteen consumer warps; warp w takes the two consecutive groups 2w, 2w + 1 of every stage
//    and runs mma.sync m16n8k16 with the 16 weight rows as the A operand and the (up to 8)
//    activation rows as B.  Dequantisation is one LOP3 per two weights: the operands are the raw
//    fp16 values 1024+q (low nibble of a byte) and 1024+16q (high nibble); activations that meet
//    high nibbles are staged pre-multiplied by 1/16, and the constant offsets and the zero point
//    are removed per group in fp32 with the activation sums
//        sum_k x_k (q_k - z) = raw - 1024 (Sl + Sh') - z (Sl + 16 Sh'),
//    Sl = sum of x over low-nibble slots, Sh' = sum of the staged x/16 over high-nibble slots,
//    both summed in fp32 in a fixed tree order (deterministic; their rounding is of the same order
//    as the MMA's own fp32 accumulation of the offset operands).  The group's fp16 scale then
//    multiplies that sum in fp32.
//  * Each consumer warp stages only the activations of its own groups, each 8-k chunk as
//    [x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16] so that one 16-byte shared load yields the B
//    fragments of the two MMAs that consume one packed word; no CTA-wide barrier stands between
//    the preceding kernel's end and the first MMA.  Lanes whose B column is not an activation row
//    skip the loads and feed zeros.
//  * Shared memory is read through 32-bit shared addresses with immediate offsets; a stage's
//    scales and zero points are read as vectors when the group count allows.
//  * At the end of a tile every consumer warp parks its partial sums in a shared slot and moves
//    on; a reducer warp adds the warps' partials in warp order (deterministic) and writes Y, so
//    the ring never waits for a reduction.
//  * The kernel is instantiated per activation-row bound MT (1, 2, 4, 8): columns >= MT of the
//    MMA fragments are never folded or parked.  MT = 16 (split mode, 16-group stages) feeds every
//    dequantised A fragment to two MMAs, for activation rows 0-7 and 8-15.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

// A stage is 16 rows x SG groups (SG = 16 or 32: 16 or 32 KB); consumer warp w takes the SG / 8
// consecutive groups w * SG / 8 ... of every stage.
__host__ __device__ constexpr uint32_t ds_stage_bytes(int SG) { return 16u * 64u * (uint32_t)SG; }
constexpr int DS_CW = 16;                           // consumer warps (then a producer and a reducer warp)
constexpr int DS_PWARP = DS_CW;                     // producer warp
constexpr int DS_RWARP = DS_CW + 1;                 // reducer warp
constexpr int DS_THREADS = 32 * (DS_CW + 2);
constexpr int DS_MAXM = 16;
constexpr int DS_MAXNS = 24;                        // ring stages at most
constexpr int DS_MINNS = 2;                         // ring stages at least
constexpr int DS_MAXMS = 4;                         // metadata slots at most
constexpr int DS_RSLOTS = 2;                        // partial-sum slots of the reducer
// Dynamic shared memory per CTA (alignment slack included): one CTA per SM.
constexpr uint32_t DS_FULL_SMEM = 227 * 1024;

struct DsLayout {
    uint32_t ring, meta, mslot, xs, corr, red, bars, total;
};

// Metadata of one stage in split mode: scales [16][SG] fp16, then zero points [16][SG] u8.
__host__ __device__ constexpr uint32_t ds_stage_meta_bytes(int SG) { return 48u * (uint32_t)SG; }

// Byte offsets of the shared-memory regions for `ns` ring stages and `nms` metadata slots; K is
// the staged length of k (the whole K, or one K slice in split mode, where every ring stage has a
// metadata slot of its own: nms == ns).
__host__ __device__ inline DsLayout ds_layout(int SG, int MT, int M, int K, int ns, int nms, bool ks) {
    DsLayout L;
    const uint32_t G = (uint32_t)(K / 128);
    L.ring = 0;
    L.meta = (uint32_t)ns * ds_stage_bytes(SG);
    L.mslot = ks ? ds_stage_meta_bytes(SG) : 48u * G;                   // 16 rows x groups x (2 + 1) bytes
    L.xs = L.meta + (uint32_t)nms * L.mslot;
    L.corr = L.xs + (uint32_t)M * (uint32_t)(K + 8) * 2;                // float2 [G][MT] (+ 8 spare)
    L.red = L.corr + (G * (uint32_t)MT + 8) * 8;                        // [slot][warp][16][MT] fp32
    L.bars = L.red + (uint32_t)DS_RSLOTS * DS_CW * 16 * (uint32_t)MT * 4;
    // full, empty [DS_MAXNS]; meta_empty [DS_MAXMS]; tile_full, red_empty [DS_RSLOTS]; abort flag
    L.total = L.bars + (2 * DS_MAXNS + DS_MAXMS + 2 * DS_RSLOTS) * 8 + 8;
    return L;
}

// 16-byte chunk swizzle of a staged activation row (row stride padded to 16 mod 128 bytes):
// makes the B-fragment loads of a warp bank-conflict free for up to 8 activation rows.
__device__ __forceinline__ int ds_swz(int ch) { return ch ^ ((ch >> 2) & 2); }

// Sum of the two fp16 halves of a packed pair, in fp32.
__device__ __forceinline__ float half2_sum(uint32_t h) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    return f.x + f.y;
}

constexpr int DS_XILP = 4;  // activation chunks each consumer thread loads before using any

// Shared-memory loads through 32-bit shared addresses (volatile: they stay behind the mbarrier waits).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
    return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(a));
    return r;
}
__device__ __forceinline__ unsigned short lds_u16(uint32_t a) {
    unsigned short r;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(a));
    return r;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    uint32_t r;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(r) : "r"(a));
    return r;
}

// Half h (0: low, 1: high) of a packed fp16 pair, as fp32.
__device__ __forceinline__ float ds_half(uint32_t v, int h) {
    return __half2float(__ushort_as_half((unsigned short)(h ? (v >> 16) : (v & 0xFFFFu))));
}

// One group (16 rows x 128 k) for this thread: raw tensor-core sums, then the offsets and the zero
// point removed with the group's activation sums and the scale applied, into acc.
template <int MT>
__device__ __forceinline__ void ds_group(uint32_t a_addr, uint32_t b_addr, uint32_t xg, const uint32_t (&xofs)[4],
                                         bool xlane, uint32_t corr_addr, float fsa, float fsb, float fza, float fzb,
                                         float (&acc)[4]) {
    const uint4 A = lds128(a_addr);
    const uint4 B = lds128(b_addr);
    float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
    const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = wA[j], b = wB[j], a8 = a >> 8, b8 = b >> 8;
        const uint4 xf = xlane ? lds128(xg + xofs[j]) : make_uint4(0u, 0u, 0u, 0u);
        float(&cc)[4] = (j & 1) ? c1 : c0;  // two independent accumulation chains
        mma_16816(cc, lop3_and_or(a, 0x000F000Fu, 0x64006400u), lop3_and_or(b, 0x000F000Fu, 0x64006400u),
                  lop3_and_or(a, 0x00F000F0u, 0x64006400u), lop3_and_or(b, 0x00F000F0u, 0x64006400u), xf.x, xf.y);
        mma_16816(cc, lop3_and_or(a8, 0x000F000Fu, 0x64006400u), lop3_and_or(b8, 0x000F000Fu, 0x64006400u),
                  lop3_and_or(a8, 0x00F000F0u, 0x64006400u), lop3_and_or(b8, 0x00F000F0u, 0x64006400u), xf.z, xf.w);
    }
    // rows g8 + 8 of a half tile (N % 16 == 8) hold stale metadata; never stored
    if (MT == 1) {
        const uint2 cv = lds64(corr_addr);
        const float C = __uint_as_float(cv.x), S = __uint_as_float(cv.y);
        acc[0] = fmaf(fsa, (c0[0] + c1[0]) - fmaf(fza, S, C), acc[0]);  // row g8,   col 0
        acc[2] = fmaf(fsb, (c0[2] + c1[2]) - fmaf(fzb, S, C), acc[2]);  // row g8+8, col 0
    } else {
        const uint4 cv = lds128(corr_addr);
        const float C0 = __uint_as_float(cv.x), S0 = __uint_as_float(cv.y);
        const float C1 = __uint_as_float(cv.z), S1 = __uint_as_float(cv.w);
        acc[0] = fmaf(fsa, (c0[0] + c1[0]) - fmaf(fza, S0, C0), acc[0]);  // row g8,   col 2c
        acc[1] = fmaf(fsa, (c0[1] + c1[1]) - fmaf(fza, S1, C1), acc[1]);  // row g8,   col 2c+1
        acc[2] = fmaf(fsb, (c0[2] + c1[2]) - fmaf(fzb, S0, C0), acc[2]);  // row g8+8, col 2c
        acc[3] = fmaf(fsb, (c0[3] + c1[3]) - fmaf(fzb, S1, C1), acc[3]);  // row g8+8, col 2c+1
    }
}

// KS (split mode): blockIdx.y is a K slice of `ncs` whole stages; the CTA stages the activations of
// its slice only, every stage brings its own scales and zero points (two 2-D TMA boxes of 16 rows x
// SG groups), and with several slices the reducer writes fp32 partial sums to P [slice][M][N]
// instead of Y (P null: one slice, Y directly).
// MT == 16: the same for two column blocks (activation rows 0-7 and 8-15) that share every
// dequantised A fragment; one accumulation chain per block.  acc: rows (g8, g8+8) x cols
// (2c, 2c+1) of block 0, then of block 1.
__device__ __forceinline__ void ds_group16(uint32_t a_addr, uint32_t b_addr, uint32_t xg0, uint32_t xg1,
                                           const uint32_t (&xofs)[4], bool x0, bool x1, uint32_t corr0,
                                           uint32_t corr1, float fsa, float fsb, float fza, float fzb,
                                           float (&acc)[8]) {
    const uint4 A = lds128(a_addr);
    const uint4 B = lds128(b_addr);
    float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
    const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = wA[j], b = wB[j], a8 = a >> 8, b8 = b >> 8;
        const uint4 xf0 = x0 ? lds128(xg0 + xofs[j]) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 xf1 = x1 ? lds128(xg1 + xofs[j]) : make_uint4(0u, 0u, 0u, 0u);
        uint32_t f0 = lop3_and_or(a, 0x000F000Fu, 0x64006400u), f1 = lop3_and_or(b, 0x000F000Fu, 0x64006400u);
        uint32_t f2 = lop3_and_or(a, 0x00F000F0u, 0x64006400u), f3 = lop3_and_or(b, 0x00F000F0u, 0x64006400u);
        mma_16816(c0, f0, f1, f2, f3, xf0.x, xf0.y);
        mma_16816(c1, f0, f1, f2, f3, xf1.x, xf1.y);
        f0 = lop3_and_or(a8, 0x000F000Fu, 0x64006400u);
        f1 = lop3_and_or(b8, 0x000F000Fu, 0x64006400u);
        f2 = lop3_and_or(a8, 0x00F000F0u, 0x64006400u);
        f3 = lop3_and_or(b8, 0x00F000F0u, 0x64006400u);
        mma_16816(c0, f0, f1, f2, f3, xf0.z, xf0.w);
        mma_16816(c1, f0, f1, f2, f3, xf1.z, xf1.w);
    }
    const uint4 u = lds128(corr0), v = lds128(corr1);
    acc[0] = fmaf(fsa, c0[0] - fmaf(fza, __uint_as_float(u.y), __uint_as_float(u.x)), acc[0]);
    acc[1] = fmaf(fsa, c0[1] - fmaf(fza, __uint_as_float(u.w), __uint_as_float(u.z)), acc[1]);
    acc[2] = fmaf(fsb, c0[2] - fmaf(fzb, __uint_as_float(u.y), __uint_as_float(u.x)), acc[2]);
    acc[3] = fmaf(fsb, c0[3] - fmaf(fzb, __uint_as_float(u.w), __uint_as_float(u.z)), acc[3]);
    acc[4] = fmaf(fsa, c1[0] - fmaf(fza, __uint_as_float(v.y), __uint_as_float(v.x)), acc[4]);
    acc[5] = fmaf(fsa, c1[1] - fmaf(fza, __uint_as_float(v.w), __uint_as_float(v.z)), acc[5]);
    acc[6] = fmaf(fsb, c1[2] - fmaf(fzb, __uint_as_float(v.y), __uint_as_float(v.x)), acc[6]);
    acc[7] = fmaf(fsb, c1[3] - fmaf(fzb, __uint_as_float(v.w), __uint_as_float(v.z)), acc[7]);
}

template <int MT, int SG, bool KS>
__global__ void __launch_bounds__(DS_THREADS, 1)
    decode_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
                         const __grid_constant__ CUtensorMap tmZ, const __half* __restrict__ X,
                         const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                         __half* __restrict__ Y, float* __restrict__ P, int M, int N, int K, int n_tiles, int ns,
                         int nms, int ncs, int weights_early, int* status) {
    constexpr int ROWB = SG * 64;                    // bytes of one row in a stage
    constexpr uint32_t STAGE_BYTES = 16u * ROWB;
    constexpr int GPW = SG / DS_CW;                  // groups per consumer warp per stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA destinations need an aligned base: round up (the launch reserves 1 KB of slack)
    unsigned char* smem = smem_align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = K >> 7;
    const int NC = (G + SG - 1) / SG;  // stages of the whole K
    // this CTA's stages of every tile: [kc0, kc0 + NCl)
    const int kc0 = KS ? (int)blockIdx.y * ncs : 0;
    const int NCl = KS ? min(ncs, NC - kc0) : NC;
    const int KL = KS ? ncs * SG * 128 : K;  // staged k per activation row
    const DsLayout L = ds_layout(SG, MT, M, KL, ns, nms, KS);
    const uint32_t sbase = smem_u32(smem);
    // balanced contiguous tile ranges: CTA sizes differ by at most one tile
    const int t0 = (int)(((int64_t)blockIdx.x * n_tiles) / gridDim.x);
    const int t1 = (int)(((int64_t)(blockIdx.x + 1) * n_tiles) / gridDim.x);
    const int n_units = (t1 - t0) * NCl;
    const uint32_t bar0 = sbase + L.bars;
    auto full_bar = [&](int s) { return bar0 + 8 * s; };
    auto empty_bar = [&](int s) { return bar0 + 8 * (DS_MAXNS + s); };
    auto meta_empty = [&](int i) { return bar0 + 8 * (2 * DS_MAXNS + i); };
    auto tile_full = [&](int i) { return bar0 + 8 * (2 * DS_MAXNS + DS_MAXMS + i); };
    auto red_empty = [&](int i) { return bar0 + 8 * (2 * DS_MAXNS + DS_MAXMS + DS_RSLOTS + i); };
    volatile int* abort_flag =
        reinterpret_cast<volatile int*>(smem + L.bars + 8 * (2 * DS_MAXNS + DS_MAXMS + 2 * DS_RSLOTS));
    float* red = reinterpret_cast<float*>(smem + L.red);

    if (tid == 0) {
        for (int s = 0; s < ns; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), DS_CW);
        }
        if (!KS)
            for (int i = 0; i < nms; ++i) mbar_init(meta_empty(i), DS_CW);
        for (int i = 0; i < DS_RSLOTS; ++i) {
            mbar_init(tile_full(i), 32 * DS_CW);  // every consumer lane arrives after parking
            mbar_init(red_empty(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();  // the next kernel may claim the other half of the SM and start streaming

    if (warp == DS_PWARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmW);
            if (KS) {
                prefetch_tmap(&tmS);
                prefetch_tmap(&tmZ);
            }
            if (!weights_early) pdl_wait();
            int issued = 0, t = t0, kc = 0, s = 0, ms = 0;
            uint32_t ph = 0, mph = 0;
            for (int u = 0; u < n_units; ++u) {
                // The ring is full: from here on progress depends on the consumers, who first
                // wait for the preceding kernel; start the bounded waits only after that point.
                if (u == ns && weights_early) pdl_wait();
                if ((!KS && kc == 0 && !mbar_wait_bounded(meta_empty(ms), mph ^ 1, abort_flag)) ||
                    !mbar_wait_bounded(empty_bar(s), ph ^ 1, abort_flag)) {
                    *abort_flag = 1;
                    record_status(status, W4_ERR_DEVICE_TIMEOUT);
                    break;
                }
                if constexpr (KS) {
                    // weights, scales and zero points of stage kc0 + kc of tile t (the boxes' rows past
                    // N and groups past K/128 are zero-filled and counted in full)
                    const int kg = kc0 + kc;
                    const uint32_t mdst = sbase + L.meta + (uint32_t)s * L.mslot;
                    mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES + ds_stage_meta_bytes(SG));
                    tma_load_2d(sbase + L.ring + s * STAGE_BYTES, &tmW, kg * (ROWB / 8), t * 16, full_bar(s));
                    tma_load_2d(mdst, &tmS, kg * SG, t * 16, full_bar(s));
                    tma_load_2d(mdst + 32u * SG, &tmZ, kg * SG, t * 16, full_bar(s));
                } else {
                    uint32_t sb = 0, zb = 0;
                    const int64_t mofs = (int64_t)t * 16 * G;  // first metadata entry of the tile
                    const uint32_t mdst = L.meta + ms * L.mslot;
                    if (kc == 0) {  // the tile's metadata rides on its first stage
                        const int rows = N - t * 16 < 16 ? N - t * 16 : 16;  // 8 or 16 (N % 8 == 0)
                        sb = (uint32_t)(rows * 2 * G);
                        zb = (uint32_t)(rows * G) & ~15u;
                        if (zb != (uint32_t)(rows * G))  // 8 trailing zero points (8 rows, odd G): plain copy
                            *reinterpret_cast<uint2*>(smem + mdst + 32 * G + zb) =
                                *reinterpret_cast<const uint2*>(zeros + mofs + zb);
                    }
                    mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES + sb + zb);
                    tma_load_2d(sbase + L.ring + s * STAGE_BYTES, &tmW, kc * (ROWB / 8), t * 16, full_bar(s));
                    if (sb) bulk_load_1d(sbase + mdst, scales + mofs, sb, full_bar(s));
                    if (zb) bulk_load_1d(sbase + mdst + 32 * G, zeros + mofs, zb, full_bar(s));
                }
                ++issued;
                if (++kc == NCl) {
                    kc = 0;
                    ++t;
                    if (++ms == nms) { ms = 0; mph ^= 1; }
                }
                if (++s == ns) { s = 0; ph ^= 1; }
            }
            for (int u = issued - ns; u < issued; ++u)  // no loads in flight at exit
                if (u >= 0) mbar_wait_bounded(full_bar(u % ns), (u / ns) & 1, nullptr, 200000000ull);
        }
        return;
    }

    if (warp == DS_RWARP) {
        // ------------------------------------------------------------ reducer: Y, in warp order
        pdl_wait();  // Y may be read by the preceding kernel
        int rs = 0;
        uint32_t rph = 0;
        float* Pl = KS && P ? P + (int64_t)blockIdx.y * M * N : nullptr;  // this slice's partials
        for (int t = t0; t < t1; ++t) {
            if (!mbar_wait_bounded(tile_full(rs), rph, abort_flag)) {
                *abort_flag = 1;
                record_status(status, W4_ERR_DEVICE_TIMEOUT);
                break;
            }
            const float* rsl = red + (size_t)rs * (DS_CW * 16 * MT);
#pragma unroll
            for (int o0 = 0; o0 < 16 * MT; o0 += 32) {
                const int o = o0 + lane, row = o / MT, m = o - row * MT;
                const int n = t * 16 + row;
                if (o < 16 * MT && m < M && n < N) {
                    float sum = 0.0f;
#pragma unroll
                    for (int w = 0; w < DS_CW; ++w) sum += rsl[w * (16 * MT) + o];
                    if (KS && P)
                        Pl[(int64_t)m * N + n] = sum;
                    else
                        Y[(int64_t)m * N + n] = __float2half_rn(sum);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(red_empty(rs));
            if (++rs == DS_RSLOTS) { rs = 0; rph ^= 1; }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Consumer warp w owns the GPW consecutive groups w*GPW .. w*GPW+GPW-1 of every stage: in stage
    // kc0 + kc of a tile, groups (kc0 + kc)*SG + w*GPW + e, staged at local group kc*SG + w*GPW + e.
    // It stages exactly the activations of those groups, with their offset sums, so no other warp
    // waits for them (one memory round trip after the preceding kernel has finished).  The 16
    // chunks of one group sit in 16 consecutive lanes, which reduce the sums with shuffles in a
    // fixed order.
    pdl_wait();  // the activations may be produced by the preceding kernel
    const uint32_t xs_u = sbase + L.xs;
    const uint32_t corr_u = sbase + L.corr;
    __half* xs = reinterpret_cast<__half*>(smem + L.xs);
    float2* corr = reinterpret_cast<float2*>(smem + L.corr);
    const int RS = KL + 8;  // staged row stride in halves (16 bytes of padding)
    {
        const __half2 sixteenth = __float2half2_rn(0.0625f);
        const unsigned half_mask = (lane & 16) ? 0xFFFF0000u : 0x0000FFFFu;
        const int per_warp = M * NCl * GPW * 16;  // chunks of 8 k this warp stages (a multiple of 16)
        for (int base = 0; base < per_warp; base += 32 * DS_XILP) {
            uint4 raw[DS_XILP];
#pragma unroll
            for (int v = 0; v < DS_XILP; ++v) {
                const int i = base + v * 32 + lane;
                const int q = i >> 4, e = q % GPW, r = q / GPW, kc = r % NCl, m = r / NCl;
                const int g = (kc0 + kc) * SG + warp * GPW + e;
                if (i < per_warp && g < G) raw[v] = ldg_cached(X + (int64_t)m * K + g * 128 + (i & 15) * 8);
            }
#pragma unroll
            for (int v = 0; v < DS_XILP; ++v) {
                const int i = base + v * 32 + lane;
                const int q = i >> 4, e = q % GPW, r = q / GPW, kc = r % NCl, m = r / NCl;
                const int g = (kc0 + kc) * SG + warp * GPW + e;
                if (i >= per_warp || g >= G) continue;  // uniform per 16-lane half (one group)
                const int gl = kc * SG + warp * GPW + e;  // staged (local) group
                const int ch = gl * 16 + (i & 15);        // chunk index within the staged row
                const uint4 w = raw[v];
                uint4 p;
                p.x = __byte_perm(w.x, w.z, 0x5410);         // x0, x4
                uint32_t h = __byte_perm(w.x, w.z, 0x7632);  // x1, x5
                __half2 hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
                p.y = *reinterpret_cast<uint32_t*>(&hh);
                p.z = __byte_perm(w.y, w.w, 0x5410);  // x2, x6
                h = __byte_perm(w.y, w.w, 0x7632);    // x3, x7
                hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
                p.w = *reinterpret_cast<uint32_t*>(&hh);
                *reinterpret_cast<uint4*>(xs + (int64_t)m * RS + ds_swz(ch) * 8) = p;
                float lo = half2_sum(p.x) + half2_sum(p.z);  // staged low-nibble partners
                float hi = half2_sum(p.y) + half2_sum(p.w);  // staged high-nibble partners (x/16)
#pragma unroll
                for (int o = 8; o; o >>= 1) {
                    lo += __shfl_xor_sync(half_mask, lo, o);
                    hi += __shfl_xor_sync(half_mask, hi, o);
                }
                if ((i & 15) == 0)  // C = 1024 (Sl + Sh'), S = Sl + 16 Sh'
                    corr[gl * MT + m] = make_float2(1024.0f * (lo + hi), fmaf(16.0f, hi, lo));
            }
        }
    }
    // corr entries of activation rows >= M stay unset: they only feed columns that are never stored
    __syncwarp();

    const int g8 = lane >> 2, c = lane & 3;
    const bool xlane = g8 < M;  // B column g8 holds activation row g8; other lanes use zeros
    const uint32_t xrow = xs_u + (uint32_t)(xlane ? g8 : 0) * (uint32_t)RS * 2u;
    const bool xlane1 = MT == 16 && g8 + 8 < M;  // MT == 16: column g8 of block 1 is row g8 + 8
    const uint32_t xrow1 = xs_u + (uint32_t)(xlane1 ? g8 + 8 : 0) * (uint32_t)RS * 2u;
    uint32_t xofs[4];  // swizzled byte offset of word j's chunk within a group, for this lane
#pragma unroll
    for (int j = 0; j < 4; ++j) xofs[j] = (uint32_t)ds_swz(c * 4 + j) * 16u;
    const int ccol = 2 * c < MT ? 2 * c : 0;  // first activation column of this thread's C pair
    // metadata of the warp's groups is vector-aligned (always in split mode: rows of SG groups)
    const bool mvec = GPW >= 2 && (KS || (G % GPW) == 0);
    // this thread's W bytes inside a stage: rows g8 and g8 + 8 of the warp's groups, 16 bytes at 16 c
    const uint32_t wlane = (uint32_t)(g8 * ROWB + warp * GPW * 64 + c * 16);
    int s = 0, kc = 0, ms = 0, rs = 0;
    uint32_t ph = 0, rph = 0;
    constexpr int NACC = MT == 16 ? 8 : 4;
    float acc[NACC];  // rows (g8, g8+8) x cols (2c, 2c+1) [of block 0, then block 1]
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = 0.0f;
    // one group e of the current stage
    auto group = [&](uint32_t st, uint32_t xg, uint32_t xg1, int gle, float fsa, float fsb, float fza, float fzb) {
        if constexpr (MT == 16) {
            ds_group16(st, st + 8 * ROWB, xg, xg1, xofs, xlane, xlane1, corr_u + (uint32_t)(gle * 16 + 2 * c) * 8u,
                       corr_u + (uint32_t)(gle * 16 + 8 + 2 * c) * 8u, fsa, fsb, fza, fzb, acc);
        } else {
            ds_group<MT>(st, st + 8 * ROWB, xg, xofs, xlane, corr_u + (uint32_t)(gle * MT + ccol) * 8u, fsa, fsb,
                         fza, fzb, acc);
        }
    };
    bool dead = false;
    for (int u = 0; u < n_units; ++u) {
        // After a timeout every wait is skipped; the loop still runs to the end.
        if (!dead && !mbar_wait_bounded(full_bar(s), ph, abort_flag)) {
            *abort_flag = 1;
            record_status(status, W4_ERR_DEVICE_TIMEOUT);
            dead = true;
        }
        const int g0 = (kc0 + kc) * SG + warp * GPW;  // first group of the warp in this stage
        const int gl0 = kc * SG + warp * GPW;         // its staged (local) index
        const int ng = g0 >= G ? 0 : min(GPW, G - g0);
        if (!dead && ng > 0) {
            const uint32_t st = sbase + L.ring + (uint32_t)s * STAGE_BYTES + wlane;
            const uint32_t xg = xrow + (uint32_t)gl0 * 256u, xg1 = xrow1 + (uint32_t)gl0 * 256u;
            // scales [16][mG] fp16, then zeros [16][mG] u8: the tile's (mG = K/128) or the stage's (mG = SG)
            const uint32_t mG = KS ? (uint32_t)SG : (uint32_t)G;
            const uint32_t msa = sbase + L.meta + (uint32_t)(KS ? s : ms) * L.mslot;
            const uint32_t mza = msa + 32u * mG;
            const uint32_t ia = g8 * mG + (uint32_t)(KS ? warp * GPW : g0), ib = ia + 8u * mG;
            if (ng == GPW && mvec) {
                if constexpr (GPW >= 2) {
                    // the scales and zero points of the warp's groups, packed: GPW fp16 and GPW bytes per row
                    uint32_t sa[GPW / 2], sb[GPW / 2], za, zb;
                    if constexpr (GPW == 4) {
                        const uint2 va = lds64(msa + 2u * ia), vb = lds64(msa + 2u * ib);
                        sa[0] = va.x; sa[1] = va.y; sb[0] = vb.x; sb[1] = vb.y;
                        za = lds32(mza + ia);
                        zb = lds32(mza + ib);
                    } else {
                        sa[0] = lds32(msa + 2u * ia);
                        sb[0] = lds32(msa + 2u * ib);
                        za = lds_u16(mza + ia);
                        zb = lds_u16(mza + ib);
                    }
#pragma unroll
                    for (int e = 0; e < GPW; ++e) {
                        const float fsa = ds_half(sa[e >> 1], e & 1), fsb = ds_half(sb[e >> 1], e & 1);
                        const float fza = (float)((za >> (8 * e)) & 0xFFu), fzb = (float)((zb >> (8 * e)) & 0xFFu);
                        group(st + e * 64, xg + e * 256, xg1 + e * 256, gl0 + e, fsa, fsb, fza, fzb);
                    }
                }
            } else {
                for (int e = 0; e < ng; ++e) {
                    const float fsa = __half2float(__ushort_as_half(lds_u16(msa + 2u * (ia + e))));
                    const float fsb = __half2float(__ushort_as_half(lds_u16(msa + 2u * (ib + e))));
                    const float fza = (float)lds_u8(mza + ia + e);
                    const float fzb = (float)lds_u8(mza + ib + e);
                    group(st + e * 64, xg + e * 256, xg1 + e * 256, gl0 + e, fsa, fsb, fza, fzb);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
        if (++s == ns) { s = 0; ph ^= 1; }
        if (++kc == NCl) {
            // tile done: release its metadata, park this warp's partials for the reducer
            if (!KS && lane == 0) mbar_arrive(meta_empty(ms));
            if (++ms == nms) ms = 0;
            if (!dead && !mbar_wait_bounded(red_empty(rs), rph ^ 1, abort_flag)) {
                *abort_flag = 1;
                record_status(status, W4_ERR_DEVICE_TIMEOUT);
                dead = true;
            }
            float* mine = red + (size_t)rs * (DS_CW * 16 * MT) + warp * (16 * MT);
            if (2 * c < MT) { mine[g8 * MT + 2 * c] = acc[0]; mine[(g8 + 8) * MT + 2 * c] = acc[2]; }
            if (2 * c + 1 < MT) { mine[g8 * MT + 2 * c + 1] = acc[1]; mine[(g8 + 8) * MT + 2 * c + 1] = acc[3]; }
            if constexpr (MT == 16) {
                mine[g8 * 16 + 8 + 2 * c] = acc[4];
                mine[g8 * 16 + 9 + 2 * c] = acc[5];
                mine[(g8 + 8) * 16 + 8 + 2 * c] = acc[6];
                mine[(g8 + 8) * 16 + 9 + 2 * c] = acc[7];
            }
            mbar_arrive(tile_full(rs));  // every lane: its own stores are released with it
            if (++rs == DS_RSLOTS) { rs = 0; rph ^= 1; }
#pragma unroll
            for (int i = 0; i < NACC; ++i) acc[i] = 0.0f;
            kc = 0;
        }
    }
}

// ------------------------------------------------------------------------------------ host side
static int ds_mt(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

// Groups per stage: 32 (32 KB stages, two groups per consumer warp); 16 for the 16-row
// instantiation, whose 16 staged activation rows take twice the shared memory per k.
static int ds_sg(int mt) { return mt == 16 ? 16 : 32; }

constexpr int DS_GOOD_NS = 4;   // ring depth below which the plan cuts K into slices (when it may)

// Metadata slots of the unsplit kernel: enough to run two tiles ahead of the consumers.
static int ds_nms(int64_t tpc, int NC) {
    return (int)std::min<int64_t>(DS_MAXMS, std::min<int64_t>(tpc, 2 + (int64_t)DS_MAXNS / NC));
}

// Ring stages that fit in one SM's shared memory with `ncs` stages of k staged per activation row
// (split mode) or the whole K (ncs == 0, with nms metadata slots); 0 when not even DS_MINNS fit.
static int ds_fit(int64_t M, int64_t K, int ncs, int nms) {
    const int mt = ds_mt(M), sg = ds_sg(mt);
    const bool ks = ncs > 0;
    const int KL = ks ? ncs * sg * 128 : (int)K;
    const uint32_t fixed = ds_layout(sg, mt, (int)M, KL, 0, 0, ks).total +
                           (ks ? 0u : (uint32_t)nms * 48u * (uint32_t)(K / 128)) + 1024;  // alignment slack
    const uint32_t per = ds_stage_bytes(sg) + (ks ? ds_stage_meta_bytes(sg) : 0u);
    if (fixed + (uint32_t)DS_MINNS * per > DS_FULL_SMEM) return 0;
    return (int)std::min<uint32_t>((DS_FULL_SMEM - fixed) / per, DS_MAXNS);
}

// Stages per K slice: 0 when K is not cut, -1 when the shape is not served.  A function of M and K
// alone, so the workspace query needs no device.  Split mode needs 2-D TMA boxes of the metadata
// rows (K/128 a multiple of 16: 16-byte row strides of the zero points); the slices are equal
// (their count divides the stages of K), the longest that leave DS_GOOD_NS ring stages, else one
// stage each.  Up to 8 rows, K is cut only when the whole K leaves fewer than DS_GOOD_NS stages;
// the 16-row instantiation always runs in split mode (with a single slice where K fits whole).
static int ds_split_stages(int64_t M, int64_t K) {
    const int mt = ds_mt(M), sg = ds_sg(mt);
    const int G = (int)(K / 128);
    const int NC = (G + sg - 1) / sg;
    if (mt == 16) {
        if (G % 16 != 0) return -1;
        for (int ncs = NC; ncs >= 1; --ncs)
            if (NC % ncs == 0 && ds_fit(M, K, ncs, 0) >= DS_GOOD_NS) return ncs;
        return ds_fit(M, K, 1, 0) > 0 ? 1 : -1;
    }
    const int whole = ds_fit(M, K, 0, ds_nms(DS_MAXMS, NC));
    if (whole >= DS_GOOD_NS || G % 16 != 0 || NC < 2) return whole > 0 ? 0 : -1;
    for (int ncs = NC - 1; ncs >= 1; --ncs)
        if (NC % ncs == 0 && ds_fit(M, K, ncs, 0) >= DS_GOOD_NS) return ncs;
    if (ds_fit(M, K, 1, 0) > whole) return 1;
    return whole > 0 ? 0 : -1;
}

int decode_stream_slices(int64_t M, int64_t K) {
    const int ncs = ds_split_stages(M, K);
    const int sg = ds_sg(ds_mt(M));
    const int NC = (int)((K / 128 + sg - 1) / sg);
    return ncs > 0 ? (NC + ncs - 1) / ncs : 1;
}

// 16-row launches where they measured faster than two 8-row launches on B200 (K = 8192,
// N = 8192: 25.5 vs 28.0 us at M = 16, 49.2 vs 54.3 at M = 32; a tie at N = 28672); at K = 28672
// the 16-row consumer's doubled per-byte work and 14 slices of partials make them slower (78.3 vs
// 73.2 us at M = 16), so longer K stays with 8-row launches.
int decode_stream_rows(int64_t M, int64_t K) {
    return M > 8 && K >= 128 && K % 128 == 0 && K <= 8192 && ds_split_stages(16, K) > 0 ? 16 : 8;
}

// Launch plan: ring depth and metadata slots within one SM's shared memory; one CTA per SM (or
// per tile when there are fewer tiles than SMs), the SMs shared out over the K slices.
bool plan_decode_stream(int64_t M, int64_t N, int64_t K, DecodePlan* p) {
    if (M < 1 || M > DS_MAXM || N < 8 || K < 128 || K % 128 != 0 || K > 65536 || N % 8 != 0) return false;
    const int mt = ds_mt(M), sg = ds_sg(mt);
    const int G = (int)(K / 128);
    const int NC = (G + sg - 1) / sg;
    const int64_t T = (N + 15) / 16;
    const int sms = device_sm_count();
    const int ncs = ds_split_stages(M, K);
    if (ncs < 0) return false;
    const int ks = ncs ? (NC + ncs - 1) / ncs : 1;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(T, sms / ks));
    const int64_t tpc = (T + grid - 1) / grid;  // tiles of the largest CTA
    const int units = (int)std::min<int64_t>(tpc * (ncs ? ncs : NC), DS_MAXNS);
    const int nms = ncs ? 0 : ds_nms(tpc, NC);
    const int ns = std::min(ds_fit(M, K, ncs, nms), units);
    if (ns < std::min(DS_MINNS, units) || ns < 1) return false;
    p->sg = sg;
    p->mt = mt;
    p->ns = ns;
    p->nms = ncs ? ns : nms;
    p->ks = ks;
    p->ncs = ncs;
    p->n_tiles = (int)T;
    p->grid = grid;
    const int KL = ncs ? ncs * sg * 128 : (int)K;
    p->smem = ds_layout(sg, mt, (int)M, KL, ns, p->nms, ncs > 0).total + 1024;
    return true;
}

size_t decode_stream_workspace(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || N < 1 || K < 128 || K % 128 != 0) return 0;
    // launches of up to decode_stream_rows rows; each takes its slices' fp32 partials from the start
    // of the workspace
    const int64_t rows = decode_stream_rows(M, K);
    size_t need = 0;
    for (int64_t mc : {std::min<int64_t>(M, rows), M % rows}) {
        if (mc < 1) continue;
        const int ks = decode_stream_slices(mc, K);
        if (ks > 1) need = std::max(need, (size_t)ks * (size_t)mc * (size_t)N * 4);
    }
    return need;
}

template <int MT, int SG, bool KS>
static cudaError_t ds_launch(const CUtensorMap& tm, const CUtensorMap& tmS, const CUtensorMap& tmZ, const uint16_t* X,
                             int64_t M, int64_t N, int64_t K, const uint16_t* scales, const uint8_t* zeros, uint16_t* Y,
                             float* P, const DecodePlan& p, bool weights_static, int* status, cudaStream_t stream) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(decode_stream_kernel<MT, SG, KS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DS_FULL_SMEM);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid, (unsigned)p.ks, 1);
    cfg.blockDim = dim3(DS_THREADS, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_static ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_stream_kernel<MT, SG, KS>, tm, tmS, tmZ,
                              reinterpret_cast<const __half*>(X), reinterpret_cast<const unsigned short*>(scales),
                              zeros, reinterpret_cast<__half*>(Y), P, (int)M, (int)N, (int)K, p.n_tiles, p.ns, p.nms,
                              p.ncs, weights_static ? 1 : 0, status);
}

template <bool KS>
static cudaError_t ds_launch_mt(const CUtensorMap& tm, const CUtensorMap& tmS, const CUtensorMap& tmZ,
                                const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint16_t* scales,
                                const uint8_t* zeros, uint16_t* Y, float* P, const DecodePlan& p, bool ws_,
                                int* status, cudaStream_t stream) {
    switch (p.mt) {
        case 1: return ds_launch<1, 32, KS>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, ws_, status, stream);
        case 2: return ds_launch<2, 32, KS>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, ws_, status, stream);
        case 4: return ds_launch<4, 32, KS>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, ws_, status, stream);
        case 8: return ds_launch<8, 32, KS>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, ws_, status, stream);
        default:
            if constexpr (KS)
                return ds_launch<16, 16, true>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, ws_, status, stream);
            else
                return cudaErrorInvalidValue;  // the 16-row instantiation runs in split mode only
    }
}

cudaError_t launch_decode_stream(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                 const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, void* ws,
                                 bool weights_static, int* status, cudaStream_t stream) {
    DecodePlan p;
    if (!plan_decode_stream(M, N, K, &p)) return cudaErrorInvalidValue;
    CUtensorMap tm;  // packed rows as 8-byte elements: a box of 8 SG elements is one stage's share of a row
    if (!make_tensor_map_2d(&tm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)(K / 16), (uint64_t)N,
                            (uint32_t)(8 * p.sg), 16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (p.ncs == 0) return ds_launch_mt<false>(tm, tm, tm, X, M, N, K, scales, zeros, Y, nullptr, p, weights_static,
                                               status, stream);
    // split mode: [16][SG] boxes of the scales and zero points; with several slices fp32 partials
    // in ws, then their sum
    CUtensorMap tmS, tmZ;
    const uint64_t G = (uint64_t)(K / 128);
    if (!make_tensor_map_2d(&tmS, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, G, (uint64_t)N, (uint32_t)p.sg, 16,
                            CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tensor_map_2d(&tmZ, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, G, (uint64_t)N, (uint32_t)p.sg, 16,
                            CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (p.ks == 1)
        return ds_launch_mt<true>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, nullptr, p, weights_static, status,
                                  stream);
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15)) return cudaErrorInvalidValue;
    float* P = static_cast<float*>(ws);
    cudaError_t e = ds_launch_mt<true>(tm, tmS, tmZ, X, M, N, K, scales, zeros, Y, P, p, weights_static, status, stream);
    if (e != cudaSuccess) return e;
    return launch_splitk_reduce(P, p.ks, M * N, Y, stream);
}

}  // namespace w4
