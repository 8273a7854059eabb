/*
 * libw4a16 -- group-wise INT4 weight-only quantisation and the W4A16 matmul on B200 (sm_100a).
 *
 * C ABI.  Every entry point takes plain pointers and sizes; no PyTorch or CUDA types appear in
 * the signatures (a stream is passed as an opaque `void*` holding a cudaStream_t; NULL means the
 * legacy default stream).
 *
 * Conventions shared by all entry points
 * --------------------------------------
 *  - Layouts: every matrix is dense row-major with no padding between rows.
 *      X  [M, K]    fp16 (IEEE binary16 bit patterns in uint16_t)  activations
 *      W  [N, K]    fp16                                           weights
 *      packed [N, K/8] uint32: 8 four-bit codes per word, the code of the lowest k in the lowest
 *                   nibble (word j of row n holds k = 8j .. 8j+7)
 *      scales [N, K/group] fp16; zeros [N, K/group] uint8 (values 0..15)
 *      Y  [M, N]    fp16
 *    Group g of row n covers k in [group*g, group*g + group).  Dequantised weight:
 *    w[n,k] = (q[n,k] - zeros[n, k/group]) * scales[n, k/group].
 *  - Memory: all array pointers are DEVICE pointers owned by the caller (except the outputs of
 *    the *_workspace_size queries and w4_status_string, which are host memory).  The library
 *    never allocates or frees memory.  Work is enqueued asynchronously on `stream`; the only
 *    call that synchronises is w4_check_device_status.
 *  - Validation happens on the host before any launch; a rejected call enqueues nothing.
 *      W4_ERR_NULL         a required pointer is NULL
 *      W4_ERR_SHAPE        a size is negative, K % group != 0, N % 8 != 0, or a size exceeds the
 *                          library's limits (every dimension < 2^31, every matrix < 2^40 elements)
 *      W4_ERR_UNSUPPORTED  group != 128 (64 or 128 where a call says so), bits outside
 *                          {2, 3, 4, 8}, n_alpha outside 1..64, or a negative / non-finite damp
 *      W4_ERR_ALIGN        X, W, packed, Y or act_scale is not 16-byte aligned
 *      W4_ERR_WORKSPACE    ws_bytes is smaller than the size the matching query returns
 *      W4_ERR_CUDA         a CUDA launch or query failed (the CUDA error is left for the caller
 *                          to read with cudaGetLastError)
 *    Device-side conditions cannot be seen at launch time; kernels record them in a per-device
 *    status word that w4_check_device_status reads:
 *      W4_ERR_RANGE        a group's fp16 scale overflowed (|W * act_scale| too large for fp16);
 *                          the outputs of that call are unspecified
 *      W4_ERR_DEVICE_TIMEOUT  a bounded wait inside a kernel gave up; that kernel's outputs are
 *                          unspecified and the context stays usable
 *      W4_ERR_NUMERIC      gptq_quantize: the damped Hessian is not positive definite (a zero
 *                          damp with fewer calibration rows than K, or non-finite inputs); the
 *                          outputs of that call are unspecified
 *  - Results are deterministic: the same inputs give bit-identical outputs (no floating-point
 *    atomics; every reduction has a fixed order).
 *  - Thread safety: calls may come from several host threads; the only shared state is the
 *    per-device status word.
 *
 * Sources.  The method is described by the pages "GPTQ, AWQ and the rules of post-training
 * quantization" (sections "The problem both methods solve" and "AWQ: find the one percent that
 * matters"), "AutoGPTQ vs The Stack v2" (per-group quantisation with scales and zero points,
 * group size typically 128), "AutoAWQ vs The Stack v2" (INT4 storage, FP16 compute, weights
 * dequantised on the fly inside fused GEMM/GEMV kernels, picked by batch size) and "When to Use
 * AWQ vs GPTQ" (section "Practical Usage": w_bit 4, q_group_size 128).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4_OK = 0,
    W4_ERR_NULL = 1,
    W4_ERR_SHAPE = 2,
    W4_ERR_ALIGN = 3,
    W4_ERR_UNSUPPORTED = 4,
    W4_ERR_WORKSPACE = 5,
    W4_ERR_CUDA = 6,
    W4_ERR_DEVICE_TIMEOUT = 7,
    W4_ERR_RANGE = 8,
    W4_ERR_NUMERIC = 9
} w4_status;

/* Kernel families of w4_gemm_ex (w4_gemm picks one per shape). */
typedef enum {
    W4_VARIANT_AUTO = 0,
    W4_VARIANT_SKINNY = 1, /* warp-level tensor-core GEMV / skinny GEMM, split-K over a cluster */
    W4_VARIANT_TC = 2,     /* tcgen05/TMEM tensor-core GEMM with dequantisation in the smem path */
    W4_VARIANT_GEMV = 3,   /* persistent TMA-fed mma.sync GEMV, up to 8 activation rows per launch
                            * (more rows: several launches); needs 16-byte aligned scales and zeros
                            * (else W4_ERR_ALIGN; w4_gemm then uses the skinny family) */
    W4_VARIANT_GEMV_TC = 4, /* tcgen05 GEMV, weights as a TMEM operand, up to 8 rows per launch */
    /* Flag, OR-ed into the variant: packed/scales/zeros are not written by any work still in
     * flight on the stream (static weights).  The call may then use programmatic dependent launch
     * and start streaming the weights before the preceding kernel on the stream has finished;
     * X is still read only after that kernel has completed. */
    W4_FLAG_WEIGHTS_STATIC = 0x100
} w4_variant;

/*
 * w4_quantize_pack -- round-to-nearest group quantisation of W * diag(act_scale) and packing.
 *
 * Follows "GPTQ, AWQ and the rules of post-training quantization", section "The problem both
 * methods solve" (round each weight to the nearest level of a small integer format) and
 * "AutoGPTQ vs The Stack v2" (one scale and one zero point per group of 128 along K).
 * For each row n and group g, with v_k = W[n,k] * act_scale[k] (one fp32 multiply; v_k = W[n,k]
 * when act_scale is NULL):
 *     lo = min(0, min v), hi = max(0, max v)              (fp32)
 *     s32 = (hi - lo) / 15                                (fp32, IEEE round to nearest)
 *     s16 = s32 rounded to fp16 toward +infinity          (1.0 when hi == lo)
 *     z   = clamp(rint(-lo / s16), 0, 15)                 (rint: round half to even)
 *     q_k = clamp(rint(v_k / s16) + z, 0, 15)
 * Every step is one correctly rounded fp32 operation, so results are bit-identical to any
 * IEEE implementation of the same steps.
 *
 *   W          [N, K] fp16, device, 16-byte aligned.
 *   act_scale  [K] fp32, device, 16-byte aligned, or NULL.  AWQ use: quantise W*diag(s) here and
 *              feed X*diag(1/s) to w4_gemm (w4_act_prepare(X, NULL, s) forms it in one pass, or
 *              fold 1/s into the producer of X).
 *   packed     [N, K/8] uint32 out, 16-byte aligned.  scales [N, K/group] fp16 out.
 *   zeros      [N, K/group] uint8 out.   group must be 128.
 * N == 0 is a no-op.  Errors: see the conventions above; W4_ERR_RANGE is reported through the
 * device status word.
 */
w4_status w4_quantize_pack(const uint16_t* W, int64_t N, int64_t K, int group,
                           const float* act_scale, uint32_t* packed, uint16_t* scales,
                           uint8_t* zeros, void* stream);

/* Bytes of device workspace w4_gemm / w4_gemm_ex need for this shape (may be 0): fp32 partial
 * sums when the tensor-core GEMM (M > 16 with few output tiles, or a last wave at most half full)
 * or the GEMV (activation rows too long to stage whole next to a deep enough ring, K/128 a
 * multiple of 16) cut K into slices.  A function of M, N, K and group (and the device's SM count,
 * cached). */
w4_status w4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int group, size_t* bytes);

/*
 * w4_gemm -- Y = X . dequant(W)^T with fp16 inputs, fp32 accumulation and fp16 output.
 *
 * Follows "AutoAWQ vs The Stack v2" (WQLinear blurb: INT4 weights dequantised on the fly inside
 * the matmul instead of materialising FP16 weights; a GEMV kernel for single-token decode and a
 * GEMM kernel for batches, chosen by batch size).  The dequantised weights are
 * w = (q - z) * s16 as above.
 *
 *   X [M, K] fp16, packed/scales/zeros as produced by w4_quantize_pack, Y [M, N] fp16 out.
 *   ws / ws_bytes: device workspace of at least w4_gemm_workspace_size bytes, 16-byte aligned
 *   (may be NULL when that size is 0; misaligned: W4_ERR_ALIGN).  M == 0 or N == 0 is a no-op;
 *   K == 0 writes Y = 0.
 * Families (w4_gemm picks by M: GEMV, in launches of up to 8 activation rows (16 at K <= 8192),
 * for M <= 16 when scales/zeros are 16-byte aligned and the staged activation rows fit shared
 * memory or K/128 is a multiple of 16 (then K is cut into slices, their fp32 partials summed in
 * slice order by a second launch); skinny for the other M <= 16; TC above 16 rows, with K cut
 * into slices when its tiles fill fewer than half the SMs, or its last wave's tiles when that wave
 * is at most half full, the partials summed in slice order by a further launch):
 *   - GEMV: tensor-core sums of x with the raw operands 1024+q / 1024+16q, offsets and z removed
 *     per group with fp32 activation sums (fixed order), times s16 in fp32;
 *   - skinny: sum_k x_k (q_k - z) exactly per group on tensor cores in fp32, times s16 in fp32;
 *   - TC: each dequantised weight rounded once to fp16 before the fp32-accumulating MMA.
 * All accumulate in fp32, round Y once to fp16 and are deterministic (fixed reduction orders).
 */
w4_status w4_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                  const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y, void* ws,
                  size_t ws_bytes, void* stream);

/* w4_gemm with an explicit kernel family, optionally OR-ed with W4_FLAG_WEIGHTS_STATIC
 * (W4_VARIANT_AUTO alone behaves exactly like w4_gemm).  Unknown values: W4_ERR_UNSUPPORTED. */
w4_status w4_gemm_ex(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y,
                     void* ws, size_t ws_bytes, int variant, void* stream);

/*
 * w4_gemm_plan -- which kernel family a w4_gemm_ex call with these arguments runs, and how many
 * kernel launches it makes.  Nothing is enqueued and no device is touched beyond the cached
 * per-device attributes; the decision is the one w4_gemm_ex takes (the same code).
 *   variant: as for w4_gemm_ex.  scales / zeros: the metadata pointers the call will receive (the
 *   GEMV family needs both 16-byte aligned), or NULL to assume aligned ones.
 *   family_out: W4_VARIANT_GEMV, W4_VARIANT_SKINNY, W4_VARIANT_TC or W4_VARIANT_GEMV_TC (host int);
 *   W4_VARIANT_AUTO with launches_out = 0 when the call launches no kernel (M, N or K zero).
 *   launches_out: kernel launches of the call (host int).
 * Errors: those w4_gemm_ex would return for the shape and variant (W4_ERR_SHAPE when an explicit
 * family cannot serve the shape, W4_ERR_ALIGN for misaligned metadata with the explicit GEMV).
 * The pages have no counterpart to this query; it lets a caller account for the launches.
 */
w4_status w4_gemm_plan(int64_t M, int64_t N, int64_t K, int group, int variant, const void* scales,
                       const void* zeros, int* family_out, int* launches_out);

/*
 * w4_gemm_host -- w4_gemm with X and Y in host memory.
 *
 * Enqueues on `stream`: one copy of X_host [M, K] into the caller's device buffer x_dev, the
 * GEMM of w4_gemm_ex (same `variant`) into the caller's device buffer y_dev [M, N], and one copy
 * of y_dev into Y_host.  Returns once enqueued; Y_host holds the result when the stream has
 * drained.  With pinned host buffers both copies are asynchronous; with pageable ones the CUDA
 * runtime may stage them synchronously.  x_dev and y_dev: 16-byte aligned device memory the
 * caller owns (the library still allocates nothing).  Errors: as w4_gemm_ex, plus W4_ERR_CUDA if
 * a copy cannot be enqueued.
 */
w4_status w4_gemm_host(const uint16_t* X_host, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                       const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y_host,
                       uint16_t* x_dev, uint16_t* y_dev, void* ws, size_t ws_bytes, int variant,
                       void* stream);

/*
 * w4_gemm_host_batch -- several w4_gemm layers with their activations and results in host memory,
 * moved with one copy each way.
 *
 * Enqueues on `stream`: one copy of x_bytes from x_host into the caller's device buffer x_dev,
 * then for every layer i in order the GEMM of w4_gemm_ex (same `variant`) reading X_i at x_dev +
 * layers[i].x_offset and writing Y_i at y_dev + layers[i].y_offset, then one copy of y_bytes from
 * y_dev into y_host.  Returns once enqueued; y_host holds every layer's result when the stream has
 * drained.
 *   layers[i].M, N, K: the layer's shape; packed/scales/zeros: its device weights (as for w4_gemm).
 *   x_offset / y_offset: byte offsets, multiples of 16; X_i [M, K] fp16 must lie inside [0, x_bytes)
 *   and Y_i [M, N] fp16 inside [0, y_bytes).
 *   x_host, y_host: host buffers (pinned for asynchronous copies); x_dev, y_dev: 16-byte aligned
 *   device buffers the caller owns.  x_bytes may be 0 (no input copy).
 *   ws: device workspace of at least the largest w4_gemm_workspace_size of the layers.
 * Every layer is validated before anything is enqueued; errors as w4_gemm_ex (W4_ERR_SHAPE also for
 * a region outside its buffer or n_layers < 1, W4_ERR_ALIGN for an offset that is not a multiple
 * of 16), plus W4_ERR_CUDA if a copy cannot be enqueued.
 * The pages have no counterpart to this call; it exists so that a decode step pays for two copies
 * instead of two per layer.
 */
typedef struct {
    int64_t M, N, K;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint8_t* zeros;
    int64_t x_offset;
    int64_t y_offset;
} w4_gemm_layer;
w4_status w4_gemm_host_batch(const w4_gemm_layer* layers, int n_layers, int group, const void* x_host,
                             void* x_dev, size_t x_bytes, void* y_host, void* y_dev, size_t y_bytes, void* ws,
                             size_t ws_bytes, int variant, void* stream);

/* Bytes of device workspace awq_scale_search needs for this problem. */
w4_status awq_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha,
                             size_t* bytes);

/*
 * awq_scale_search -- the AWQ activation-aware per-channel scale search on one linear layer.
 *
 * Follows "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one
 * percent that matters": channel j's scale is its mean |x| over the calibration rows to the
 * power alpha, alpha is picked from a grid on [0, 1], and multiplying W's channel j by s_j while
 * dividing X's channel j by s_j leaves the layer's output unchanged.
 *     m_j      = (1/T) sum_t |X[t,j]|                        (exact sum, rounded once to fp64)
 *     alpha_i  = i / n_alpha, i = 0 .. n_alpha-1
 *     s_ij     = max(m_j, 1e-6)^alpha_i / sqrt(max_j(.) * min_j(.))   (fp64, then rounded to fp32)
 *     Wq_i     = dequant(quant(W * diag(s_i)))              (exactly w4_quantize_pack's quantiser)
 *     MSE_i    = mean over (t, n) of ((X diag(1/s_i)) Wq_i^T - X W^T)^2
 *     best     = lowest i among the minima of MSE_i
 * On the device MSE_i is evaluated as sum_{t,n} (X E_i^T)^2 / (T N) with
 * E_i = Wq_i diag(1/s_i) - W rounded to fp16, fp32 tensor-core accumulation and an fp64
 * fixed-order reduction.
 *
 *   X [T, K] fp16 calibration activations; W [N, K] fp16.
 *   mse [n_alpha] fp64 out, best_idx [1] int32 out, best_s [K] fp32 out (all device memory).
 *   ws: device workspace of at least awq_workspace_size bytes.
 * T must be >= 1 and N >= 8.  Errors: see the conventions above.
 */
w4_status awq_scale_search(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                           int group, int n_alpha, double* mse, int32_t* best_idx, float* best_s,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * awq_scale_search_noalloc -- awq_scale_search for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for integration.  Some callers cannot
 * call cudaMalloc or any allocating routine: a plugin inside an inference engine that owns all
 * device memory, a service held to a fixed memory budget, or a latency-critical path that must
 * not risk the implicit device synchronisation an allocation can cause.  This entry point takes
 * the same arguments as awq_scale_search minus the workspace: its scratch is one array of
 * W4_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that loads the library
 * holds until the process exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Limit: problems whose awq_workspace_size exceeds W4_NOALLOC_SCRATCH_BYTES are rejected
 *     with W4_ERR_WORKSPACE before anything is enqueued (e.g. T = 4096, K = N = 2048 fits;
 *     K = N = 4096 does not).
 *   - The stream must belong to the current device (else W4_ERR_CUDA, nothing enqueued); the
 *     scratch used is that device's copy of the array.
 *   - The first call on each device looks up that device's copy of the scratch array
 *     (cudaGetSymbolAddress, with the device current); make that first call before any stream
 *     capture on the device.  A lookup that fails returns W4_ERR_CUDA and is tried again by the
 *     next call.
 *   - Every call shares the one array and leaves its contents behind; the call clears what must
 *     start at zero itself.  Calls whose work overlaps on the GPU (for example on two streams)
 *     race on the array and give wrong results: serialise them.
 * Results are the same as awq_scale_search's on the same inputs.
 */
#define W4_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
w4_status awq_scale_search_noalloc(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N,
                                   int64_t K, int group, int n_alpha, double* mse,
                                   int32_t* best_idx, float* best_s, void* stream);

/*
 * The AWQ scale search split by calibration rows, for one part per rank (or any partition of the
 * rows).  awq_scale_search on all rows equals, up to the association of the fp64 sums:
 *     1. per part:  awq_colsum(X_part) -> colsum_part
 *     2. colsum = sum over parts of colsum_part (uint64 integers: exact in any order);
 *        T_total = sum of the parts' row counts
 *     3. awq_scales_from_colsum(colsum, T_total) -> s_all [n_alpha, K]  (same on every part)
 *     4. per part:  awq_sse(X_part, W, s_all) -> sse_part [n_alpha]
 *     5. awq_select(sse [n_parts, n_alpha], T_total, N, s_all) -> mse, best_idx, best_s
 * The exchange between ranks is steps 2 and 4 -> 5 (an integer all-reduce of K values and a
 * gather of n_alpha doubles per rank); no step reads another GPU's memory.
 *
 * awq_colsum: colsum [K] uint64 (device, overwritten) = sum_t |X[t, j]| * 2^24, exact (every
 *   fp16 magnitude is a whole number of 2^-24 units).  T may be 0 (all zeros).
 * awq_scales_from_colsum: s_all [n_alpha, K] fp32 = awq_scale_search's scales for alpha_i =
 *   i / n_alpha from the mean m_j = colsum_j * 2^-24 / T_total.
 * awq_sse: sse [n_alpha] fp64 = sum over this part's rows t and all n of (X E_i^T)[t, n]^2 with
 *   awq_scale_search's E_i (fp32 tensor-core accumulation, fixed-order fp64 sums).  ws: at least
 *   awq_sse_workspace_size bytes.
 * awq_select: sse [n_parts, n_alpha] fp64 (part-major); MSE_i = (sum over parts in part order) /
 *   (T_total N); best = lowest index among the minima; best_s = s_all[best].
 * All arrays are device memory; errors as for awq_scale_search.
 */
w4_status awq_colsum(const uint16_t* X, int64_t T, int64_t K, uint64_t* colsum, void* stream);
w4_status awq_scales_from_colsum(const uint64_t* colsum, int64_t T_total, int64_t K, int n_alpha,
                                 float* s_all, void* stream);
w4_status awq_sse_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha,
                                 size_t* bytes);
w4_status awq_sse(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int group,
                  int n_alpha, const float* s_all, double* sse, void* ws, size_t ws_bytes,
                  void* stream);
w4_status awq_select(const double* sse, int n_parts, int n_alpha, int64_t T_total, int64_t N,
                     const float* s_all, int64_t K, double* mse, int32_t* best_idx, float* best_s,
                     void* stream);

/* Bytes of device workspace awq_scale_search_gram needs for this problem. */
w4_status awq_gram_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha,
                                  size_t* bytes);

/*
 * awq_scale_search_gram -- awq_scale_search with the calibration rows folded into their Gram
 * matrix first.
 *
 * Same search, same arguments, same outputs ("GPTQ, AWQ and the rules of post-training
 * quantization", section "AWQ: find the one percent that matters").  The output error of a
 * weight error E is sum_{t,n} (X E^T)[t,n]^2 = sum_n e_n^T (X^T X) e_n, so X is read once to form
 * G = X^T X (fp16 inputs, fp32 tensor-core accumulation) and each alpha then costs one N x K x K
 * product instead of a T x N x K one: the faster call once T exceeds about K.  Arithmetic:
 *     G    = sum over chunks c of X_c^T X_c, X_c = rows [4096 c, 4096 c + 4096) of X: each chunk
 *            one fp32 tensor-core product, the chunks added in fp64 in chunk order
 *     d_k  = sqrt(G_kk) rounded to fp32 (1 where channel k is zero in every row)
 *     G'   = fp16(G_ij / (d_i d_j))          (entries in [-1, 1]; fp16 cannot hold G itself)
 *     E'_i = fp16(((Wq_i - W diag(s_i)) / s_i) * d)   (Wq_i exactly as in awq_scale_search)
 *     MSE_i = sum over tiles of sum_{n,k} (E'_i G'^T)[n,k] E'_i[n,k]  / (T N)
 * with fp32 accumulation inside a tile and an fp64 fixed-order sum over tiles.  The rounding of
 * G' and E' differs from the direct form's, so MSE_i agrees with awq_scale_search's to about
 * 1e-5 relative, not bit for bit; best_idx can differ only where two alphas' errors are that
 * close.  An E' entry beyond the fp16 range (a weight error far larger than the activations'
 * norm can carry) makes that alpha's MSE infinite and sets W4_ERR_RANGE in the device status.
 *
 *   X [T, K] fp16; W [N, K] fp16; mse [n_alpha] fp64, best_idx [1] int32, best_s [K] fp32 out.
 *   ws: device workspace of at least awq_gram_workspace_size bytes (it holds X^T with T padded
 *   to whole chunks, one chunk's G in fp32, G in fp64 and G' in fp16: about
 *   2 T K + 14 K^2 + 2 N K bytes).
 * T must be >= 1 and N >= 8.  Errors: see the conventions above.
 */
w4_status awq_scale_search_gram(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N,
                                int64_t K, int group, int n_alpha, double* mse, int32_t* best_idx,
                                float* best_s, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace gptq_quantize / gptq_quantize_ex need (group 64 or 128; T does not
 * change it). */
w4_status gptq_workspace_size(int64_t T, int64_t N, int64_t K, int group, size_t* bytes);

/*
 * gptq_quantize -- GPTQ: quantise W column by column, paying for each column's rounding error
 * with the columns not yet quantised, and emit w4_quantize_pack's format (so w4_gemm serves it).
 *
 * Follows "GPTQ, AWQ and the rules of post-training quantization", section "GPTQ: pay for the
 * error with the other weights" (columns in a fixed order; each column's rounding error absorbed
 * by the later columns through the inverse of H = X^T X, taken via a Cholesky factorisation;
 * updates of far columns batched):
 *     H   = X^T X + lambda I, lambda = damp * mean(diag(X^T X))   (fp64; damp 0.01 is usual)
 *     U   = the upper triangular factor with H^-1 = U^T U          (fp64)
 *     for each group of 128 columns, left to right:
 *         scale s (fp16, rounded up) and zero point z by w4_quantize_pack's rule from the group's
 *         current weights rounded to fp32;
 *         for each column k of the group: q_k = clamp(rint(fp32(w_k) / s) + z, 0, 15) (fp32,
 *         exactly w4_quantize_pack's decision); e = (w_k - (q_k - z) s) / U_kk;
 *         w_j -= e U_kj for every later column j (fp64; columns beyond the group lazily, one
 *         product per group).
 *   X [T, K] fp16 calibration activations; W [N, K] fp16 (not modified).
 *   packed [N, K/8] uint32, scales [N, K/128] fp16, zeros [N, K/128] uint8 out, as
 *   w4_quantize_pack's.
 *   damp >= 0 and finite (else W4_ERR_UNSUPPORTED); K <= 32768 (else W4_ERR_SHAPE).
 *   ws: device workspace of at least gptq_workspace_size bytes (16 K^2 + 8 N K bytes and a little).
 * A Hessian that is not positive definite sets W4_ERR_NUMERIC in the device status.  The codes
 * equal those of the same algorithm in exact arithmetic except where fp64 rounding moves a value
 * across a rounding boundary of the fp32 quantiser.
 */
w4_status gptq_quantize(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                        int group, double damp, uint32_t* packed, uint16_t* scales, uint8_t* zeros,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * gptq_quantize_ex -- gptq_quantize at other widths, group sizes and column orders.
 *
 * bits in {2, 3, 4, 8} and group in {64, 128} ("AutoGPTQ vs The Stack v2": 2/3/4/8-bit GPTQ with
 * per-group quantisation; INT3 g128 and INT2 g64 in "GPTQ, AWQ and the rules of post-training
 * quantization"), else W4_ERR_UNSUPPORTED.  The quantiser is w4_quantize_pack's with L = 2^bits - 1
 * steps; codes are packed as w4_quantize_pack_bits packs them.
 * act_order != 0 (desc_act): the columns are processed in decreasing diag(X^T X), ties in index
 * order; the outputs are stored in PROCESSING order and perm [K] int32 (device, required then)
 * receives perm[i] = the original column processed i-th.  Serve such weights with
 * w4_act_prepare(X, perm) followed by the matmul.
 * act_scale [K] fp32 (device) or NULL: AWQ's per-channel scale s applied first ("GPTQ, AWQ and
 * the rules of post-training quantization", section "What activation-awareness buys and what it
 * does not": the scaling is independent of GPTQ's update and goes before it).  GPTQ then runs on
 * X / s and W * s (both formed in fp64; s must be positive and finite) and the layer's output is
 * (X / s) . dequant(W)^T, e.g. w4_act_prepare(X, perm, s) followed by the matmul.
 *   packed [N, K*bits/32] uint32, scales / zeros [N, K/group].  K <= 32768.
 *   ws: at least gptq_workspace_size(T, N, K, group) bytes.
 * gptq_quantize(...) is gptq_quantize_ex(bits 4, group 128, act_order 0).
 */
w4_status gptq_quantize_ex(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                           int bits, int group, double damp, int act_order, const float* act_scale,
                           uint32_t* packed, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * w4_quantize_pack_bits -- w4_quantize_pack at other widths and group sizes.
 *
 * bits in {2, 3, 4, 8}, group in {64, 128} (else W4_ERR_UNSUPPORTED).  The quantiser's rules with
 * L = 2^bits - 1 steps: lo = min(0, min v), hi = max(0, max v), s32 = (hi - lo) / L, fp16 scale
 * rounded up (1 for an all-zero group), z = clamp(rint(-lo / s16), 0, L),
 * q = clamp(rint(v / s16) + z, 0, L).  Codes form one little-endian bit stream per row: code k
 * occupies bits bits*k .. bits*k + bits - 1, stream bit j is bit j % 32 of word j / 32 (a 3-bit
 * code may straddle two words; bits 4 gives exactly w4_quantize_pack's layout).
 *   W [N, K] fp16; act_scale [K] fp32 or NULL; packed [N, K*bits/32] uint32; scales [N, K/group]
 *   fp16; zeros [N, K/group] uint8.  N % 8 == 0, K % group == 0.
 */
w4_status w4_quantize_pack_bits(const uint16_t* W, int64_t N, int64_t K, int bits, int group,
                                const float* act_scale, uint32_t* packed, uint16_t* scales,
                                uint8_t* zeros, void* stream);

/* Bytes of device workspace wb_gemm needs: N * K * 2 (the dequantised weights). */
w4_status wb_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int bits, int group,
                                 size_t* bytes);

/*
 * wb_gemm -- Y = X . dequant(W)^T for w4_quantize_pack_bits' format at any supported width.
 *
 * M <= 8: one fused pass: the bit stream is read once and every weight (q - z) s is formed exactly
 * in fp32 in registers, sum_k x_k (q_k - z) s accumulated in fp32 (ws unused).  Larger M: two
 * passes: every weight is dequantised to fp16 (w = (q - z) s, exact in fp32, rounded once to fp16)
 * into ws, then the tcgen05 GEMM multiplies with fp32 accumulation.  Y is rounded once to fp16;
 * results are deterministic.  Meant for the other widths (w4_gemm serves 4-bit, group-128 weights).
 *   X [M, K] fp16, Y [M, N] fp16, ws >= wb_gemm_workspace_size bytes; all 16-byte aligned.
 */
w4_status wb_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                  const uint16_t* scales, const uint8_t* zeros, int bits, int group, uint16_t* Y,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * w4_act_prepare -- activations for act-order weights and/or an activation-side scale.
 *
 * X_out[m, i] = X[m, src], src = perm[i] (or i when perm is NULL), divided by s[src] when s is
 * not NULL: fp16(fp32(x) / s) with one IEEE division.  With act-order weights from
 * gptq_quantize_ex, X_out . dequant(W)^T (w4_gemm or wb_gemm) is the layer's output; with AWQ's
 * scale s and weights quantised as W * diag(s), it folds the division of the activations into
 * the same pass.  A perm entry outside [0, K) sets W4_ERR_RANGE and yields 0.
 *   X, X_out [M, K] fp16 (distinct buffers); perm [K] int32 or NULL; s [K] fp32 or NULL.
 */
w4_status w4_act_prepare(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, const float* s,
                         uint16_t* X_out, void* stream);

/* Bytes of device workspace awq_clip_search needs for this problem. */
w4_status awq_clip_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_ratios,
                                  size_t* bytes);

/*
 * awq_clip_search -- AWQ's activation-guided clipping: per (row, group), shrink the quantisation
 * range when that lowers the layer's output error on calibration data, then quantise.
 *
 * Follows "GPTQ, AWQ and the rules of post-training quantization", section "AWQ: find the one
 * percent that matters" (the layer computes the same function when W's channel j is multiplied
 * by s_j and X's channel j divided by s_j) and the AutoAWQ pages' "activation-guided clipping",
 * which give no grid.  Reading: ratio r_j = 1 - j/20 (double, rounded once to fp32),
 * j = 0 .. n_ratios-1, multiplies both ends of a group's zero-inclusive range (one fp32 multiply
 * each) before w4_quantize_pack's scale and zero point are derived; codes beyond the shrunk
 * range saturate.  With v = W * diag(act_scale) and w_hat the dequantised codes under r_j,
 *     err[n, g, j] = sum_t ( sum_{k in g} (X[t,k] / act_scale[k]) * (w_hat[n,k] - v[n,k]) )^2
 * (each group's own contribution to the output error), evaluated as e'^T G_g e' with the
 * group's Gram block G_g = X_g^T X_g in fp32; best = lowest j among the minima.
 *
 *   X [T, K] fp16 calibration activations (as the layer receives them before the AWQ scaling);
 *   W [N, K] fp16; act_scale [K] fp32 (the AWQ scales) or NULL for none; n_ratios 1..10.
 *   best_idx [N, K/group] uint8 out; err [N, K/group, n_ratios] fp32 out, or NULL;
 *   packed / scales / zeros out: w4_quantize_pack's format for W * diag(act_scale), each group
 *   quantised with its chosen ratio (n_ratios == 1 gives w4_quantize_pack's result exactly).
 *   ws: device workspace of at least awq_clip_workspace_size bytes.
 * T >= 1.  X, W, packed and act_scale 16-byte aligned.  Errors: see the conventions above.
 */
w4_status awq_clip_search(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                          int group, int n_ratios, const float* act_scale, uint8_t* best_idx,
                          float* err, uint32_t* packed, uint16_t* scales, uint8_t* zeros,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * w4_selftest_bounded_wait -- self-test of the library's bounded waits (no counterpart on the
 * pages).  Launches one kernel that waits on a barrier nothing ever arrives at; after limit_ns
 * (1 us .. 5 s, else W4_ERR_UNSUPPORTED) the wait gives up, W4_ERR_DEVICE_TIMEOUT is recorded in
 * the device status word and the kernel returns.  The call itself returns W4_OK once the launch is
 * enqueued; w4_check_device_status then reports the timeout, and the context stays usable.
 */
w4_status w4_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/*
 * w4_check_device_status -- synchronise `stream`, then read and clear the current device's
 * status word.  Returns W4_OK, W4_ERR_RANGE, W4_ERR_DEVICE_TIMEOUT, or W4_ERR_CUDA if the
 * synchronisation itself failed.
 */
w4_status w4_check_device_status(void* stream);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* w4_status_string(w4_status status);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
