// Decode GEMV / skinny GEMM for M <= 8: Y = X dequant(W)^T, streamed at HBM rate.
//
// "AutoAWQ vs The Stack v2" (WQLinear blurb): the GEMV kernel serves token-by-token generation,
// where the layer is bound by memory traffic and weight reuse is minimal.  The traffic is the
// packed weights (0.5 B/weight) plus 3 B of scale and zero point per group of 128.
//
// Design (sm_100a):
//  * Persistent: one CTA per SM (or two half-SM CTAs, see GvCfg); CTA c owns a contiguous range
//    of 16-row tiles over the whole K, so every output is finished inside one CTA (no split-K
//    workspace, no cluster barrier).
//  * A producer warp streams the packed tile through a shared-memory ring of stages with
//    TMA: one stage is 16 rows x 4096 k (32 KB; for K = 4096 the whole tile, one contiguous
//    block of HBM).  A tile's scales and zero points are one contiguous block of each array and
//    ride on the tile's first stage as two bulk copies.  With static weights the producer starts
//    before the preceding kernel has finished (programmatic dependent launch).
//  * The consumer warps (16, or 8 in a half-SM CTA) split a stage's 32 groups of 128 between them
//    (two or four each) and run mma.sync m16n8k16 with
//    the 16 weight rows as the A operand and the (up to 8) activation rows as B.  Dequantisation
//    is one LOP3 per two weights: the operands are the raw fp16 values 1024+q (low nibble of a
//    byte) and 1024+16q (high nibble); activations that meet high nibbles are staged pre-multiplied
//    by 1/16, and the constant offsets and the zero point are removed per group in fp32 with the
//    activation sums
//        sum_k x_k (q_k - z) = raw - 1024 (Sl + Sh') - z (Sl + 16 Sh'),
//    Sl = sum of x over low-nibble slots, Sh' = sum of the staged x/16 over high-nibble slots,
//    both summed in fp32 in a fixed tree order (deterministic; their rounding is of the same order
//    as the MMA's own fp32 accumulation of the offset operands).  The group's fp16 scale then
//    multiplies that sum in fp32.
//  * The activations are staged once per CTA with each 8-k chunk as
//    [x0, x4, x1/16, x5/16, x2, x6, x3/16, x7/16], so one 16-byte shared load yields the B
//    fragments of the two MMAs that consume one packed word.  Lanes whose B column is not an
//    activation row read a block of zeros instead (no predication in the inner loop).
//  * At the end of a tile every consumer warp parks its partial sums in a shared slot and moves
//    on; a reducer warp adds the warps' partials in warp order (deterministic) and writes Y, so
//    the stage ring never waits for a reduction.
//  * The kernel is instantiated per activation-row bound MT (1, 2, 4, 8): columns >= MT of the
//    MMA fragments are never folded or parked.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace w4 {

constexpr int GV_SG = 32;                            // groups per stage
constexpr int GV_ROWB = GV_SG * 64;                  // bytes of one row in a stage (2 KB)
constexpr uint32_t GV_STAGE_BYTES = 16 * GV_ROWB;    // 32 KB of packed codes
constexpr int GV_MAXM = 8;
constexpr int GV_TSLOTS = 6;                         // tiles whose partials may be pending at once

// Partial-sum slots of the reducer: two suffice (the reducer adds a tile in far less time than the
// consumers take for the next one); eight activation rows use two to leave room for the staged
// activations, fewer rows keep more slack.
__host__ __device__ constexpr int gv_rslots(int MT) { return MT >= 8 ? 2 : GV_TSLOTS; }

struct GvLayout {
    uint32_t ring, meta, mslot, nmslot, xs, xzero, corr, red, bars, total;
};

// Two shapes of CTA: one per SM with 16 consumer warps and a 4-stage ring, or two per SM (each
// within half an SM's shared memory) with 8 consumer warps and a 2-stage ring.  Two half-SM CTAs
// let the next kernel's CTAs start streaming on an SM as soon as one of this kernel's finishes.
template <int CW_, int NS_>
struct GvCfg {
    static constexpr int CW = CW_;                 // consumer warps
    static constexpr int GPW = GV_SG / CW_;        // groups per consumer warp per stage
    static constexpr int NS = NS_;                 // ring stages
    static constexpr int PWARP = CW_;              // producer warp
    static constexpr int RWARP = CW_ + 1;          // reducer warp
    static constexpr int THREADS = 32 * (CW_ + 2);
    static constexpr int CTAS_PER_SM = CW_ == 16 ? 1 : 2;
    static constexpr int ID = CW_ == 16 ? NS_ : 0;  // 4, 3, 2: one CTA per SM; 0: two
    static constexpr int SMEM_LIMIT = CTAS_PER_SM == 1 ? 227 * 1024 : 113 * 1024;
};
using GvFull = GvCfg<16, 4>;
using GvFull3 = GvCfg<16, 3>;  // fewer stages when the staged activations leave too little room
using GvFull2 = GvCfg<16, 2>;
using GvHalf = GvCfg<8, 2>;

// A tile's metadata (16 rows x G scales, then 16 rows x G zero points) lands in a per-tile slot
// of 48 G bytes.  The producer runs at most NS stages ahead of the slowest consumer, so
// ceil(NS / stages per tile) + 1 slots let it refill a slot without waiting.
__host__ __device__ inline GvLayout gv_layout(int MT, int M, int K, int CW, int NS) {
    GvLayout L;
    const uint32_t G = (uint32_t)(K / 128);
    const uint32_t NC = (G + GV_SG - 1) / GV_SG;
    const uint32_t need = (NS + NC - 1) / NC + 1;
    L.ring = 0;
    L.meta = NS * GV_STAGE_BYTES;
    L.mslot = 48u * G;
    L.nmslot = need < (uint32_t)GV_TSLOTS ? need : (uint32_t)GV_TSLOTS;
    L.xs = L.meta + L.nmslot * L.mslot;
    L.xzero = L.xs + (uint32_t)M * (uint32_t)(K + 8) * 2;               // one group of zeros
    L.corr = L.xzero + 256;                                             // float2 [G][8]
    L.red = L.corr + G * GV_MAXM * 8;                                   // [slot][warp][16][MT] fp32
    L.bars = L.red + (uint32_t)gv_rslots(MT) * CW * 16 * (uint32_t)MT * 4;
    // full, empty [NS]; meta_empty, tile_full, red_empty [GV_TSLOTS]; abort flag
    L.total = L.bars + (2 * NS + 3 * GV_TSLOTS) * 8 + 8;
    return L;
}

// 16-byte chunk swizzle of a staged activation row (row stride padded to 16 mod 128 bytes):
// makes the B-fragment loads of a warp bank-conflict free for up to 8 activation rows.
__device__ __forceinline__ int gv_swz(int ch) { return ch ^ ((ch >> 2) & 2); }

// Sum of the two fp16 halves of a packed pair, in fp32.
__device__ __forceinline__ float half2_sum(uint32_t h) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    return f.x + f.y;
}

constexpr int GV_XILP = 4;  // activation chunks each consumer thread loads before using any

template <int CW>
__device__ __forceinline__ void gv_named_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * CW) : "memory");
}

// One group (16 rows x 128 k) of the current stage: raw MMA sums for this thread's C fragment.
__device__ __forceinline__ void gv_group_mma(const uint4 A, const uint4 B, const __half* xg, const int (&xoff)[4],
                                             float (&r)[4]) {
    float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t wA[4] = {A.x, A.y, A.z, A.w};
    const uint32_t wB[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t a = wA[j], b = wB[j], a8 = a >> 8, b8 = b >> 8;
        const uint4 xf = *reinterpret_cast<const uint4*>(xg + xoff[j]);
        float(&cc)[4] = (j & 1) ? c1 : c0;  // two independent accumulation chains
        mma_16816(cc, lop3_and_or(a, 0x000F000Fu, 0x64006400u), lop3_and_or(b, 0x000F000Fu, 0x64006400u),
                  lop3_and_or(a, 0x00F000F0u, 0x64006400u), lop3_and_or(b, 0x00F000F0u, 0x64006400u), xf.x, xf.y);
        mma_16816(cc, lop3_and_or(a8, 0x000F000Fu, 0x64006400u), lop3_and_or(b8, 0x000F000Fu, 0x64006400u),
                  lop3_and_or(a8, 0x00F000F0u, 0x64006400u), lop3_and_or(b8, 0x00F000F0u, 0x64006400u), xf.z, xf.w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = c0[e] + c1[e];
}

template <int MT, class C>
__global__ void __launch_bounds__(C::THREADS, C::CTAS_PER_SM)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X,
                       const unsigned short* __restrict__ scales, const uint8_t* __restrict__ zeros,
                       __half* __restrict__ Y, int M, int N, int K, int n_tiles, int weights_early,
                       int* status) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // TMA destinations need an aligned base: round up (the launch reserves 1 KB of slack)
    unsigned char* smem = smem_align1024(smem_raw);
    constexpr int GV_CWARPS = C::CW, GV_GPW = C::GPW, GV_STAGES = C::NS;
    const GvLayout L = gv_layout(MT, M, K, GV_CWARPS, GV_STAGES);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = K >> 7;
    const int NC = (G + GV_SG - 1) / GV_SG;  // stages per tile
    const int t0 = (int)(((int64_t)blockIdx.x * n_tiles) / gridDim.x);
    const int t1 = (int)(((int64_t)(blockIdx.x + 1) * n_tiles) / gridDim.x);
    const int n_units = (t1 - t0) * NC;
    const int nms = (int)L.nmslot;
    const uint32_t bar0 = sbase + L.bars;
    auto full_bar = [&](int s) { return bar0 + 8 * s; };
    auto empty_bar = [&](int s) { return bar0 + 8 * (GV_STAGES + s); };
    auto meta_empty = [&](int i) { return bar0 + 8 * (2 * GV_STAGES + i); };
    auto tile_full = [&](int i) { return bar0 + 8 * (2 * GV_STAGES + GV_TSLOTS + i); };
    auto red_empty = [&](int i) { return bar0 + 8 * (2 * GV_STAGES + 2 * GV_TSLOTS + i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bars + 8 * (2 * GV_STAGES + 3 * GV_TSLOTS));
    float* red = reinterpret_cast<float*>(smem + L.red);

    if (tid == 0) {
        for (int s = 0; s < GV_STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), GV_CWARPS);
        }
        for (int i = 0; i < GV_TSLOTS; ++i) {
            mbar_init(meta_empty(i), GV_CWARPS);
            mbar_init(tile_full(i), 32 * GV_CWARPS);  // every consumer lane arrives after parking
            mbar_init(red_empty(i), 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    pdl_launch_dependents();  // the next kernel may claim SM space and start its own weight stream

    if (warp == C::PWARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmW);
            if (!weights_early) pdl_wait();
            int issued = 0, t = t0, kc = 0, s = 0, ms = 0;
            uint32_t ph = 0, mph = 0;
            for (int u = 0; u < n_units; ++u) {
                // The ring is full: from here on progress depends on the consumers, who first
                // wait for the preceding kernel; start the bounded waits only after that point.
                if (u == GV_STAGES && weights_early) pdl_wait();
                if ((kc == 0 && !mbar_wait_bounded(meta_empty(ms), mph ^ 1, abort_flag)) ||
                    !mbar_wait_bounded(empty_bar(s), ph ^ 1, abort_flag)) {
                    *abort_flag = 1;
                    record_status(status, W4_ERR_DEVICE_TIMEOUT);
                    break;
                }
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
                mbar_arrive_expect_tx(full_bar(s), GV_STAGE_BYTES + sb + zb);
                tma_load_2d(sbase + L.ring + s * GV_STAGE_BYTES, &tmW, kc * (GV_ROWB / 8), t * 16, full_bar(s));
                if (sb) bulk_load_1d(sbase + mdst, scales + mofs, sb, full_bar(s));
                if (zb) bulk_load_1d(sbase + mdst + 32 * G, zeros + mofs, zb, full_bar(s));
                ++issued;
                if (++kc == NC) {
                    kc = 0;
                    ++t;
                    if (++ms == nms) { ms = 0; mph ^= 1; }
                }
                if (++s == GV_STAGES) { s = 0; ph ^= 1; }
            }
            for (int u = issued - GV_STAGES; u < issued; ++u)  // no loads in flight at exit
                if (u >= 0) mbar_wait_bounded(full_bar(u % GV_STAGES), (u / GV_STAGES) & 1, nullptr, 200000000ull);
        }
        return;
    }

    if (warp == C::RWARP) {
        // ------------------------------------------------------------ reducer: Y, in warp order
        pdl_wait();  // Y may be read by the preceding kernel
        int rs = 0;
        uint32_t rph = 0;
        for (int t = t0; t < t1; ++t) {
            if (!mbar_wait_bounded(tile_full(rs), rph, abort_flag)) {
                *abort_flag = 1;
                record_status(status, W4_ERR_DEVICE_TIMEOUT);
                break;
            }
            const float* rsl = red + (size_t)rs * (GV_CWARPS * 16 * MT);
#pragma unroll
            for (int o0 = 0; o0 < 16 * MT; o0 += 32) {
                const int o = o0 + lane, row = o / MT, m = o - row * MT;
                const int n = t * 16 + row;
                if (o < 16 * MT && m < M && n < N) {
                    float sum = 0.0f;
#pragma unroll
                    for (int w = 0; w < GV_CWARPS; ++w) sum += rsl[w * (16 * MT) + o];
                    Y[(int64_t)m * N + n] = __float2half_rn(sum);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(red_empty(rs));
            if (++rs == gv_rslots(MT)) { rs = 0; rph ^= 1; }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Stage the activations and, in the same pass, the per-group sums that remove the operand
    // offsets.  Each thread first issues all its loads of a round (one memory round trip per
    // round instead of one per chunk).  The 16 chunks of one group sit in 16 consecutive lanes,
    // which reduce them with shuffles in a fixed order.
    pdl_wait();  // the activations may be produced by the preceding kernel
    __half* xs = reinterpret_cast<__half*>(smem + L.xs);
    float2* corr = reinterpret_cast<float2*>(smem + L.corr);
    const __half2 sixteenth = __float2half2_rn(0.0625f);
    const int cpr = K / 8;  // 8-k chunks per activation row
    const int RS = K + 8;   // staged row stride in halves (16 bytes of padding)
    const int xtot = M * cpr;
    const unsigned half_mask = (lane & 16) ? 0xFFFF0000u : 0x0000FFFFu;  // the two halves may differ
    for (int base = 0; base < xtot; base += 32 * GV_CWARPS * GV_XILP) {
        uint4 raw[GV_XILP];
#pragma unroll
        for (int v = 0; v < GV_XILP; ++v) {
            const int i = base + v * 32 * GV_CWARPS + tid;
            if (i < xtot) raw[v] = ldg_cached(X + (int64_t)i * 8);  // rows are contiguous
        }
#pragma unroll
        for (int v = 0; v < GV_XILP; ++v) {
            const int i = base + v * 32 * GV_CWARPS + tid;
            if (i >= xtot) break;  // uniform per 16-lane half: xtot is a multiple of 16
            const int m = i / cpr, ch = i - m * cpr;
            const uint4 r = raw[v];
            uint4 p;
            p.x = __byte_perm(r.x, r.z, 0x5410);         // x0, x4
            uint32_t h = __byte_perm(r.x, r.z, 0x7632);  // x1, x5
            __half2 hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
            p.y = *reinterpret_cast<uint32_t*>(&hh);
            p.z = __byte_perm(r.y, r.w, 0x5410);  // x2, x6
            h = __byte_perm(r.y, r.w, 0x7632);    // x3, x7
            hh = __hmul2(*reinterpret_cast<__half2*>(&h), sixteenth);
            p.w = *reinterpret_cast<uint32_t*>(&hh);
            *reinterpret_cast<uint4*>(xs + (int64_t)m * RS + gv_swz(ch) * 8) = p;
            float lo = half2_sum(p.x) + half2_sum(p.z);  // staged low-nibble partners
            float hi = half2_sum(p.y) + half2_sum(p.w);  // staged high-nibble partners (x/16)
#pragma unroll
            for (int o = 8; o; o >>= 1) {
                lo += __shfl_xor_sync(half_mask, lo, o);
                hi += __shfl_xor_sync(half_mask, hi, o);
            }
            if ((ch & 15) == 0)  // C = 1024 (Sl + Sh'), S = Sl + 16 Sh'
                corr[(ch >> 4) * GV_MAXM + m] = make_float2(1024.0f * (lo + hi), fmaf(16.0f, hi, lo));
        }
    }
    if (tid < 16) reinterpret_cast<uint4*>(smem + L.xzero)[tid] = make_uint4(0u, 0u, 0u, 0u);
    // corr entries of activation rows >= M stay unset: they only feed columns that are never stored
    gv_named_barrier<GV_CWARPS>();

    const int g8 = lane >> 2, c = lane & 3;
    // B column g8 holds activation row g8; other lanes read one group of zeros at every k
    const bool xlane = g8 < M;
    const __half* xbase = xlane ? xs + (int64_t)g8 * RS : reinterpret_cast<const __half*>(smem + L.xzero);
    const int xstride = xlane ? 128 : 0;
    int xoff[4];  // swizzled offset (halves) of word j's chunk within a group, for this lane
#pragma unroll
    for (int j = 0; j < 4; ++j) xoff[j] = gv_swz(c * 4 + j) * 8;
    const int moa = g8 * G, mob = (g8 + 8) * G;  // this thread's two rows in a metadata slot

    // this thread's W bytes inside a stage: row g8 / g8 + 8, group (warp + 16 e), 16 bytes at 16 c
    const uint32_t wofs = (uint32_t)(g8 * GV_ROWB + warp * 64 + c * 16);
    int s = 0, kc = 0, ms = 0, rs = 0;
    uint32_t ph = 0, rph = 0;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // rows (g8, g8+8) x cols (2c, 2c+1)
    bool dead = false;
    for (int u = 0; u < n_units; ++u) {
        // After a timeout every wait is skipped; the loop still runs to the end.
        if (!dead && !mbar_wait_bounded(full_bar(s), ph, abort_flag)) {
            *abort_flag = 1;
            record_status(status, W4_ERR_DEVICE_TIMEOUT);
            dead = true;
        }
        if (!dead) {
            const unsigned char* st = smem + L.ring + s * GV_STAGE_BYTES + wofs;
            const unsigned short* msc = reinterpret_cast<const unsigned short*>(smem + L.meta + ms * L.mslot);
            const uint8_t* mzp = smem + L.meta + ms * L.mslot + 32 * G;
            const int gA = kc * GV_SG + warp;
            // groups gA + GV_CWARPS e; the last stage of a tile may hold fewer than GV_SG groups
            const int ng = gA >= G ? 0 : min(GV_GPW, (G - gA + GV_CWARPS - 1) / GV_CWARPS);
#pragma unroll
            for (int e = 0; e < GV_GPW; ++e) {
                if (e < ng) {
                    const int gi = gA + e * GV_CWARPS;
                    const uint4 A = *reinterpret_cast<const uint4*>(st + e * (GV_CWARPS * 64));
                    const uint4 B = *reinterpret_cast<const uint4*>(st + e * (GV_CWARPS * 64) + 8 * GV_ROWB);
                    float r[4];
                    gv_group_mma(A, B, xbase + gi * xstride, xoff, r);
                    // rows g8 + 8 of a half tile (N % 16 == 8) hold stale metadata; never stored
                    const float fza = (float)mzp[moa + gi], fzb = (float)mzp[mob + gi];
                    const float fsa = __half2float(__ushort_as_half(msc[moa + gi]));
                    const float fsb = __half2float(__ushort_as_half(msc[mob + gi]));
                    if (MT == 1) {
                        const float2 cs = corr[gi * GV_MAXM + 2 * c];
                        acc[0] = fmaf(fsa, r[0] - fmaf(fza, cs.y, cs.x), acc[0]);  // row g8,   col 2c
                        acc[2] = fmaf(fsb, r[2] - fmaf(fzb, cs.y, cs.x), acc[2]);  // row g8+8, col 2c
                    } else {
                        const float4 cs = *reinterpret_cast<const float4*>(corr + gi * GV_MAXM + 2 * c);
                        acc[0] = fmaf(fsa, r[0] - fmaf(fza, cs.y, cs.x), acc[0]);  // row g8,   col 2c
                        acc[1] = fmaf(fsa, r[1] - fmaf(fza, cs.w, cs.z), acc[1]);  // row g8,   col 2c+1
                        acc[2] = fmaf(fsb, r[2] - fmaf(fzb, cs.y, cs.x), acc[2]);  // row g8+8, col 2c
                        acc[3] = fmaf(fsb, r[3] - fmaf(fzb, cs.w, cs.z), acc[3]);  // row g8+8, col 2c+1
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
        if (++s == GV_STAGES) { s = 0; ph ^= 1; }
        if (++kc == NC) {
            // tile done: release its metadata, park this warp's partials for the reducer
            if (lane == 0) mbar_arrive(meta_empty(ms));
            if (++ms == nms) ms = 0;
            if (!dead && !mbar_wait_bounded(red_empty(rs), rph ^ 1, abort_flag)) {
                *abort_flag = 1;
                record_status(status, W4_ERR_DEVICE_TIMEOUT);
                dead = true;
            }
            float* mine = red + (size_t)rs * (GV_CWARPS * 16 * MT) + warp * (16 * MT);
            if (2 * c < MT) { mine[g8 * MT + 2 * c] = acc[0]; mine[(g8 + 8) * MT + 2 * c] = acc[2]; }
            if (2 * c + 1 < MT) { mine[g8 * MT + 2 * c + 1] = acc[1]; mine[(g8 + 8) * MT + 2 * c + 1] = acc[3]; }
            mbar_arrive(tile_full(rs));  // every lane: its own stores are released with it
            if (++rs == gv_rslots(MT)) { rs = 0; rph ^= 1; }
            acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
            kc = 0;
        }
    }
}

// ------------------------------------------------------------------------------------ host side
static int gv_mt(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }

template <class C>
static size_t gv_smem(int64_t M, int64_t K) {
    return (size_t)gv_layout(gv_mt(M), (int)M, (int)K, C::CW, C::NS).total + 1024;
}

// The half-SM shape when a tile is one stage (K <= 4096) and it fits half an SM; otherwise the
// full shape with the deepest ring that fits next to the staged activations (a shallower ring
// per CTA costs more than the finer overlap gains once a tile spans several stages).  0: none.
static int gv_pick(int64_t M, int64_t K) {
    if (M < 1 || M > GV_MAXM || K > 65536) return -1;  // activations are staged whole
    if (K <= GV_SG * 128 && gv_smem<GvHalf>(M, K) <= (size_t)GvHalf::SMEM_LIMIT) return GvHalf::ID;
    if (gv_smem<GvFull>(M, K) <= (size_t)GvFull::SMEM_LIMIT) return GvFull::ID;
    if (gv_smem<GvFull3>(M, K) <= (size_t)GvFull3::SMEM_LIMIT) return GvFull3::ID;
    if (gv_smem<GvFull2>(M, K) <= (size_t)GvFull2::SMEM_LIMIT) return GvFull2::ID;
    return -1;
}

size_t gemv_stream_smem(int64_t M, int64_t K) {
    switch (gv_pick(M, K)) {
        case GvHalf::ID: return gv_smem<GvHalf>(M, K) * 2;  // two CTAs share the SM
        case GvFull::ID: return gv_smem<GvFull>(M, K);
        case GvFull3::ID: return gv_smem<GvFull3>(M, K);
        case GvFull2::ID: return gv_smem<GvFull2>(M, K);
        default: return SIZE_MAX;
    }
}

template <int MT, class C>
static cudaError_t gv_launch(const CUtensorMap& tm, const uint16_t* X, int64_t M, int64_t N, int64_t K,
                             const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, bool weights_static,
                             int* status, cudaStream_t stream) {
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        attr_err[dev] = cudaFuncSetAttribute(gemv_stream_kernel<MT, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_LIMIT);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    const int n_tiles = (int)((N + 15) / 16);
    const int sms = device_sm_count();
    const int slots = C::CTAS_PER_SM * sms;
    const int grid = n_tiles < slots ? n_tiles : slots;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = gv_smem<C>(M, K);
    if (cfg.dynamicSmemBytes > (size_t)C::SMEM_LIMIT) return cudaErrorInvalidValue;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = weights_static ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemv_stream_kernel<MT, C>, tm, reinterpret_cast<const __half*>(X),
                              reinterpret_cast<const unsigned short*>(scales), zeros, reinterpret_cast<__half*>(Y),
                              (int)M, (int)N, (int)K, n_tiles, weights_static ? 1 : 0, status);
}

cudaError_t launch_gemv_stream(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                               const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, bool weights_static,
                               int* status, cudaStream_t stream) {
    CUtensorMap tm;  // packed rows as 8-byte elements: a 256-element box is 2 KB (4096 k) of a row
    if (!make_tensor_map_2d(&tm, packed, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, (uint64_t)(K / 16), (uint64_t)N,
                            GV_ROWB / 8, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int pick = gv_pick(M, K);
    if (pick < 0) return cudaErrorInvalidValue;
    const int mt = gv_mt(M);
#define GV_LAUNCH(MTV, CFG) gv_launch<MTV, CFG>(tm, X, M, N, K, scales, zeros, Y, weights_static, status, stream)
#define GV_BY_MT(CFG)                                   \
    switch (mt) {                                       \
        case 1: return GV_LAUNCH(1, CFG);               \
        case 2: return GV_LAUNCH(2, CFG);               \
        case 4: return GV_LAUNCH(4, CFG);               \
        default: return GV_LAUNCH(8, CFG);              \
    }
    switch (pick) {
        case GvHalf::ID: GV_BY_MT(GvHalf)
        case GvFull::ID: GV_BY_MT(GvFull)
        case GvFull3::ID: GV_BY_MT(GvFull3)
        default: GV_BY_MT(GvFull2)
    }
#undef GV_BY_MT
#undef GV_LAUNCH
}

}  // namespace w4
