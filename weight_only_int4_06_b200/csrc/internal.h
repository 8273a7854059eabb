// Host-side declarations shared by the translation units of libw4a16 (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cuda.h>

#include "w4a16.h"

namespace w4 {

int device_sm_count();  // SMs of the current device (cached per device)

// Quantiser (quantize.cu).
cudaError_t launch_quantize_pack(const uint16_t* W, int64_t N, int64_t K, const float* act_scale,
                                 uint32_t* packed, uint16_t* scales, uint8_t* zeros, int* status,
                                 cudaStream_t stream);

// Skinny GEMM for M <= 32 (gemm_skinny.cu).
struct SkinnyPlan {
    int mt;        // activation rows per tile: 8, 16 or 32
    int splits;    // CTAs along K that form one cluster (1..16)
    int gps;       // groups of 128 per split
    int n_tiles;   // CTAs along N (128 rows each)
    size_t smem;   // dynamic shared memory per CTA
};
bool plan_skinny(int64_t M, int64_t N, int64_t K, SkinnyPlan* plan);
// weights_static: packed/scales/zeros are not written by work still in flight on the stream, so
// the kernel is launched with programmatic dependent launch and starts streaming them before the
// preceding kernel has finished (activations are read only after it has).
cudaError_t launch_skinny(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                          uint16_t* Y, const SkinnyPlan& plan, bool weights_static,
                          cudaStream_t stream);

// Decode GEMV for M <= 16, one TMA-fed CTA per SM (decode_stream.cu).
struct DecodePlan {
    int sg;             // groups of 128 k per 16-row stage (32: 32 KB; 16 for mt = 16)
    int mt;             // activation-row bound of the instantiation: 1, 2, 4, 8 or 16
    int ns;             // ring stages
    int nms;            // metadata slots (split mode: one per ring stage)
    int ks;             // K slices (1: K is not cut)
    int ncs;            // stages per K slice (0 when K is not cut)
    int n_tiles;        // 16-row tiles in all (balanced over the CTAs of each slice)
    int grid;           // CTAs per K slice
    uint32_t smem;      // dynamic shared memory per CTA
};
bool plan_decode_stream(int64_t M, int64_t N, int64_t K, DecodePlan* plan);  // false: shape not served
// K slices of one launch of M <= 16 rows (> 1: a second, reducing launch follows).
int decode_stream_slices(int64_t M, int64_t K);
// Activation rows per launch of this path for a call of M rows: 16 where the 16-row
// instantiation serves K, else 8.
int decode_stream_rows(int64_t M, int64_t K);
// Bytes of fp32 partials a w4_gemm call of M rows on this path needs (0 when K is never cut); the
// function of M, N and K alone.
size_t decode_stream_workspace(int64_t M, int64_t N, int64_t K);
// ws: decode_stream_workspace(M, N, K) bytes, 16-byte aligned (may be null when that is 0).
cudaError_t launch_decode_stream(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                                 const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, void* ws,
                                 bool weights_static, int* status, cudaStream_t stream);
// Y [mn] fp16 = sum over `slices` fp32 partial arrays P [slices][mn], in slice order (mn % 4 == 0).
cudaError_t launch_splitk_reduce(const float* P, int slices, int64_t mn, uint16_t* Y, cudaStream_t stream);

// Decode GEMV for M <= 8 on tcgen05 with the weights as a TMEM operand (gemv_tc.cu).
struct GemvTcPlan {
    int splits;   // K splits = cluster size (1..16)
    int gps;      // groups of 128 per split (<= 12)
    int n_tiles;  // 128-row tiles
    size_t smem;  // dynamic shared memory per CTA
};
bool plan_gemv_tc(int64_t M, int64_t N, int64_t K, GemvTcPlan* plan);
cudaError_t launch_gemv_tc(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, const GemvTcPlan& plan,
                           bool weights_static, int* status, cudaStream_t stream);

// tcgen05 GEMM (gemm_tc.cu).
// ws: tc_w4_workspace(M, N, K) bytes (fp32 partial tiles of the K slices), may be null when 0.
cudaError_t launch_tc_w4(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                         const uint16_t* scales, const uint8_t* zeros, uint16_t* Y, void* ws, int* status,
                         cudaStream_t stream);
int tc_w4_split(int64_t M, int64_t N, int64_t K);         // K slices of the tensor-core path (1: none)
// Tail split: full waves of 256 x 256 tiles in one launch, the last partial wave's `tail` tiles in
// ks K slices with compact fp32 partials, summed per tile by a third launch.
bool tc_w4_tail(int64_t M, int64_t N, int64_t K, int* full, int* tail, int* ks);
size_t tc_w4_workspace(int64_t M, int64_t N, int64_t K);  // bytes of fp32 partials when split
int tc_w4_launches(int64_t M, int64_t N, int64_t K);      // kernel launches of one call
cudaError_t launch_tc_sse(const uint16_t* X, int64_t T, const uint16_t* E, int64_t N, int64_t K,
                          double* sse_part, int* status, cudaStream_t stream);
int tc_sse_partials(int64_t T, int64_t N);  // tiles of an M = T x N launch (partials of EPI 1 and 3)
// C [M, N] fp32 = A [M, K] . B [N, K]^T (both fp16, K-major, K % 64 == 0, row strides 16-byte multiples).
// Y [M, N] fp16 = A B^T with an fp16 B [N, K] (no dequantisation).
cudaError_t launch_tc_f16(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, uint16_t* Y,
                          int* status, cudaStream_t stream);
// pdl: launched as a programmatic dependent of the preceding kernel, which must not write A or B
// (the grid still ends only after that kernel has).
cudaError_t launch_tc_f32(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, float* C,
                          int* status, cudaStream_t stream, bool pdl = false);
// C [M, M] fp32 = A A^T on and below the diagonal only (256 x 256 tiles; M > 128): entries above the
// diagonal are not written.
cudaError_t launch_tc_f32_lower(const uint16_t* A, int64_t M, int64_t K, float* C, int* status, cudaStream_t stream,
                                bool pdl = false);
// Per-tile sum over (m, n) of (A . B^T)[m, n] * A[m, n] into part[tile] (requires N == K).
cudaError_t launch_tc_dot(const uint16_t* A, int64_t M, const uint16_t* B, int64_t N, int64_t K, double* part,
                          int* status, cudaStream_t stream);
// 2-D tensor map (TMA descriptor) over a row-major matrix, through the driver entry point.
bool make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint32_t elem_bytes,
                        uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swz);

// AWQ search (awq.cu).  Workspace layout (byte offsets, 256-byte aligned).
struct AwqLayout {
    size_t colsum, s_all, E, part, bytes;
    int n_part;
};
AwqLayout awq_layout(int64_t T, int64_t N, int64_t K, int n_alpha);
cudaError_t launch_awq(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                       double* mse, int32_t* best_idx, float* best_s, void* ws, int* status,
                       cudaStream_t stream);

// AWQ search split by calibration rows (awq.cu).
struct AwqSseLayout {
    size_t E, part, bytes;
    int n_part;
};
AwqSseLayout awq_sse_layout(int64_t T, int64_t N, int64_t K, int n_alpha);
cudaError_t launch_awq_colsum(const uint16_t* X, int64_t T, int64_t K, uint64_t* colsum, cudaStream_t stream);
cudaError_t launch_awq_scales_from_colsum(const uint64_t* colsum, int64_t T_total, int64_t K, int n_alpha,
                                          float* s_all, cudaStream_t stream);
cudaError_t launch_awq_sse(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                           const float* s_all, double* sse, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_awq_select(const double* sse, int n_parts, int n_alpha, int64_t T_total, int64_t N,
                              const float* s_all, int64_t K, double* mse, int32_t* best_idx, float* best_s,
                              cudaStream_t stream);

// AWQ search, Gram form (awq.cu).  Workspace layout (byte offsets, 256-byte aligned).
struct AwqGramLayout {
    size_t colsum, s_all, E, part, XT, G, G64, Gp, d, rd, bytes;
    int64_t chunk;     // rows of X per Gram chunk (a multiple of 64)
    int64_t n_chunks;
    int64_t Tp;        // chunk * n_chunks: calibration rows padded with zeros
    int n_part;
};
AwqGramLayout awq_gram_layout(int64_t T, int64_t N, int64_t K, int n_alpha);
cudaError_t launch_awq_gram(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_alpha,
                            double* mse, int32_t* best_idx, float* best_s, void* ws, int* status,
                            cudaStream_t stream);

// Other widths and column orders (wbits.cu).
cudaError_t launch_quantize_bits(const uint16_t* W, int64_t N, int64_t K, int bits, int group, const float* act_scale,
                                 uint32_t* packed, uint16_t* scales, uint8_t* zeros, int* status,
                                 cudaStream_t stream);
cudaError_t launch_wb_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, int bits, int group, uint16_t* Y,
                           void* ws, int* status, cudaStream_t stream);
cudaError_t launch_act_prepare(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, const float* s,
                               uint16_t* Xo, int* status, cudaStream_t stream);

// SM-driven copies between pinned host memory and the device (host_copy.cu).
// Device address of a pinned, mapped host buffer, or null (pageable, unknown or managed memory).
void* mapped_host_address(const void* p);
// bytes (a multiple of 16, both addresses 16-byte aligned) from src to dst, either of them a mapped
// host address; after_prior: launched as a programmatic dependent of the preceding kernel, whose
// end it awaits before reading.  The kernel lets its own dependent launch at once.
cudaError_t launch_host_copy(const void* src, void* dst, size_t bytes, bool after_prior, cudaStream_t stream);

// Self-test of the bounded waits (selftest.cu).
cudaError_t launch_selftest_wait(uint64_t limit_ns, int* status, cudaStream_t stream);

// GPTQ quantiser (gptq.cu).  Workspace layout (byte offsets, 256-byte aligned).
struct GptqLayout {
    size_t H, P, W64, E, perm, lambda, bytes;
};
GptqLayout gptq_layout(int64_t N, int64_t K);
// bits in {2, 3, 4, 8}, group in {64, 128}; perm_out (K int32) is written when act_order is set
// and perm_out is not null.
cudaError_t launch_gptq(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int bits, int group,
                        double damp, bool act_order, const float* act_scale, uint32_t* packed, uint16_t* scales,
                        uint8_t* zeros, int32_t* perm_out, void* ws, int* status, cudaStream_t stream);

// AWQ clip search (awq_clip.cu).  Workspace: Gram blocks, then per-split partial Gram blocks.
struct AwqClipLayout {
    size_t gram, part, bytes;
    int splits;
};
AwqClipLayout awq_clip_layout(int64_t T, int64_t N, int64_t K, int n_ratios);
cudaError_t launch_awq_clip(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int n_ratios,
                            const float* act_scale, uint8_t* best_idx, float* err, uint32_t* packed,
                            uint16_t* scales, uint8_t* zeros, void* ws, int* status, cudaStream_t stream);

}  // namespace w4
