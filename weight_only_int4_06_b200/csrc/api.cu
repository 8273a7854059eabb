// C-ABI entry points of libw4a16: argument validation, per-shape dispatch and the device status
// word.  Everything is enqueued on the caller's stream; nothing here allocates device memory.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace w4 {

// First device-side error of any call since the last w4_check_device_status (one per device).
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
int g_sm_count[kMaxDevices];
int* g_status_ptr[kMaxDevices];
cudaError_t g_dev_err[kMaxDevices];

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// Per-device set-up, done once per device with that device current.
bool device_setup(int dev) {
    std::call_once(g_dev_once[dev], [dev]() {
        cudaError_t e = cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaGetSymbolAddress((void**)&g_status_ptr[dev], g_device_status);
        g_dev_err[dev] = e;
    });
    return g_dev_err[dev] == cudaSuccess;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t)1 << 31;
constexpr int64_t kMaxElems = (int64_t)1 << 40;

bool dims_ok(int64_t a, int64_t b) {
    return a >= 0 && b >= 0 && a < kMaxDim && b < kMaxDim && (a == 0 || b <= kMaxElems / a);
}

}  // namespace

int device_sm_count() {
    const int dev = current_device();
    if (dev < 0 || !device_setup(dev)) return 148;
    return g_sm_count[dev];
}

int* device_status_ptr() {
    const int dev = current_device();
    if (dev < 0 || !device_setup(dev)) return nullptr;
    return g_status_ptr[dev];
}

// The kernel family and number of launches of one w4_gemm_ex call (shape already validated).
// AUTO: the tensor-core GEMM above 16 activation rows (with its K split when its tiles fill fewer
// than half the SMs); up to 16 rows the TMA-fed GEMV in launches of up to 8 rows (16 at
// K <= 8192) where its metadata is 16-byte aligned (it bulk-copies scales and zero points) and
// either 8 staged activation rows fit its shared memory or K/128 is a multiple of 16 (K then cut
// into slices, + 1 reducing launch), else the skinny kernel in launches of up to 32 rows.
// Measured per shape on B200 (bench.py --workload dispatch, cold L2, us): decode M = 1 GEMV
// 4.7 / 9.5 / 8.8 / 8.8 vs skinny 6.2 / 19.7 / 19.2 / 14.3; M = 4 / 8 the GEMV everywhere (12.9 /
// 15.3 at K = N = 8192, 31.8 / 37.9 at N = 28672, 32.2 / 38.5 at K = 28672; skinny 30-93, tensor
// cores 64-222); M = 16 the GEMV (25.5 / 74.6 / 75.4 vs tensor cores 30.3 / 90.2 / 83.2); M = 32
// the tensor cores (31.0 / 90.9 / 83.9 vs the GEMV's 16- or 8-row launches 49.3 / 146.5 / 147.9).
w4_status gemm_plan(int64_t M, int64_t N, int64_t K, int family, bool meta_aligned, int* chosen, int* launches) {
    if (family == W4_VARIANT_TC || (family == W4_VARIANT_AUTO && M > 16)) {
        *chosen = W4_VARIANT_TC;
        *launches = tc_w4_launches(M, N, K);  // with K slices: + their fixed-order sum
        return W4_OK;
    }
    if (family == W4_VARIANT_GEMV_TC) {
        GemvTcPlan gtp;
        if (!plan_gemv_tc(M < 8 ? M : 8, N, K, &gtp)) return W4_ERR_SHAPE;
        *chosen = W4_VARIANT_GEMV_TC;
        *launches = (int)((M + 7) / 8);
        return W4_OK;
    }
    DecodePlan dplan;
    const int64_t rows = decode_stream_rows(M, K);  // activation rows per GEMV launch
    const bool gemv_fits = plan_decode_stream(M < rows ? M : rows, N, K, &dplan);
    if (family == W4_VARIANT_GEMV && !gemv_fits) return W4_ERR_SHAPE;
    if (family == W4_VARIANT_GEMV && !meta_aligned) return W4_ERR_ALIGN;
    if (family == W4_VARIANT_GEMV || (family == W4_VARIANT_AUTO && M <= 32 && gemv_fits && meta_aligned)) {
        *chosen = W4_VARIANT_GEMV;
        *launches = 0;
        for (int64_t m0 = 0; m0 < M; m0 += rows)  // launches of up to `rows` rows, each + 1 when K is cut
            *launches += decode_stream_slices(M - m0 < rows ? M - m0 : rows, K) > 1 ? 2 : 1;
        return W4_OK;
    }
    SkinnyPlan plan;
    if (!plan_skinny(M < 32 ? M : 32, N, K, &plan)) return W4_ERR_SHAPE;
    *chosen = W4_VARIANT_SKINNY;
    *launches = (int)((M + 31) / 32);
    return W4_OK;
}

}  // namespace w4

using namespace w4;

extern "C" {

w4_status w4_quantize_pack(const uint16_t* W, int64_t N, int64_t K, int group,
                           const float* act_scale, uint32_t* packed, uint16_t* scales,
                           uint8_t* zeros, void* stream) {
    if (group != 128) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(N, K) || K % group != 0 || N % 8 != 0) return W4_ERR_SHAPE;
    if (N == 0 || K == 0) return W4_OK;
    if (!W || !packed || !scales || !zeros) return W4_ERR_NULL;
    if (!aligned16(W) || !aligned16(packed) || (act_scale && !aligned16(act_scale))) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_quantize_pack(W, N, K, act_scale, packed, scales, zeros, status,
                                         (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int group, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    if (group != 128) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    // fp32 partials when the tensor-core path splits K (prefill shapes with few tiles) or the
    // GEMV cuts K into slices (activation rows too long to stage whole next to a deep ring)
    const size_t tc = M > 16 && K > 0 && N > 0 ? tc_w4_workspace(M, N, K) : 0;
    const size_t gv = K > 0 && N > 0 ? decode_stream_workspace(M, N, K) : 0;
    *bytes = tc > gv ? tc : gv;
    return W4_OK;
}

w4_status w4_gemm_ex(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y,
                     void* ws, size_t ws_bytes, int variant, void* stream) {
    if (group != 128) return W4_ERR_UNSUPPORTED;
    const bool weights_static = (variant & W4_FLAG_WEIGHTS_STATIC) != 0;
    const int family = variant & ~W4_FLAG_WEIGHTS_STATIC;
    if (family < W4_VARIANT_AUTO || family > W4_VARIANT_GEMV_TC) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    size_t need = 0;
    w4_status st = w4_gemm_workspace_size(M, N, K, group, &need);
    if (st != W4_OK) return st;
    if (ws_bytes < need) return W4_ERR_WORKSPACE;
    if (need > 0 && !ws) return W4_ERR_NULL;
    if (need > 0 && !aligned16(ws)) return W4_ERR_ALIGN;
    if (M == 0 || N == 0) return W4_OK;
    if (!Y) return W4_ERR_NULL;
    if (!aligned16(Y)) return W4_ERR_ALIGN;
    cudaStream_t s = (cudaStream_t)stream;
    if (K == 0) {
        return cudaMemsetAsync(Y, 0, (size_t)M * (size_t)N * 2, s) == cudaSuccess ? W4_OK : W4_ERR_CUDA;
    }
    if (!X || !packed || !scales || !zeros) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(packed)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;

    int chosen = 0, launches = 0;
    st = gemm_plan(M, N, K, family, aligned16(scales) && aligned16(zeros), &chosen, &launches);
    if (st != W4_OK) return st;
    if (chosen == W4_VARIANT_TC) {
        if (tc_w4_workspace(M, N, K) > 0 && (ws_bytes < tc_w4_workspace(M, N, K) || !ws)) return W4_ERR_WORKSPACE;
        return launch_tc_w4(X, M, N, K, packed, scales, zeros, Y, ws, status, s) == cudaSuccess ? W4_OK
                                                                                                : W4_ERR_CUDA;
    }
    if (chosen == W4_VARIANT_GEMV_TC) {  // chosen explicitly only: slower than the mma.sync GEMV so far
        GemvTcPlan gtp;
        if (!plan_gemv_tc(M < 8 ? M : 8, N, K, &gtp)) return W4_ERR_SHAPE;
        for (int64_t m0 = 0; m0 < M; m0 += 8) {  // up to 8 activation rows per launch
            const int64_t mc = (M - m0) < 8 ? (M - m0) : 8;
            cudaError_t e = launch_gemv_tc(X + m0 * K, mc, N, K, packed, scales, zeros, Y + m0 * N, gtp,
                                           weights_static, status, s);
            if (e != cudaSuccess) return W4_ERR_CUDA;
        }
        return W4_OK;
    }
    if (chosen == W4_VARIANT_GEMV) {
        // up to 16 activation rows per launch (8 where the 16-row instantiation cannot serve K;
        // token-by-token decode has M == 1)
        const int64_t rows = decode_stream_rows(M, K);
        for (int64_t m0 = 0; m0 < M; m0 += rows) {
            const int64_t mc = (M - m0) < rows ? (M - m0) : rows;
            cudaError_t e = launch_decode_stream(X + m0 * K, mc, N, K, packed, scales, zeros, Y + m0 * N, ws,
                                                 weights_static, status, s);
            if (e != cudaSuccess) return W4_ERR_CUDA;
        }
        return W4_OK;
    }
    // Skinny path, in chunks of at most 32 activation rows.
    for (int64_t m0 = 0; m0 < M; m0 += 32) {
        const int64_t mc = (M - m0) < 32 ? (M - m0) : 32;
        SkinnyPlan plan;
        if (!plan_skinny(mc, N, K, &plan)) return W4_ERR_SHAPE;
        cudaError_t e = launch_skinny(X + m0 * K, mc, N, K, packed, scales, zeros, Y + m0 * N, plan,
                                      weights_static, s);
        if (e != cudaSuccess) return W4_ERR_CUDA;
    }
    return W4_OK;
}

w4_status w4_gemm_plan(int64_t M, int64_t N, int64_t K, int group, int variant, const void* scales,
                       const void* zeros, int* family_out, int* launches_out) {
    if (!family_out || !launches_out) return W4_ERR_NULL;
    if (group != 128) return W4_ERR_UNSUPPORTED;
    const int family = variant & ~W4_FLAG_WEIGHTS_STATIC;
    if (family < W4_VARIANT_AUTO || family > W4_VARIANT_GEMV_TC) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    if (M == 0 || N == 0 || K == 0) {  // no kernel (K == 0: one memset of Y)
        *family_out = W4_VARIANT_AUTO;
        *launches_out = 0;
        return W4_OK;
    }
    const bool meta_aligned = (!scales || aligned16(scales)) && (!zeros || aligned16(zeros));
    return gemm_plan(M, N, K, family, meta_aligned, family_out, launches_out);
}

w4_status w4_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                  const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y, void* ws,
                  size_t ws_bytes, void* stream) {
    return w4_gemm_ex(X, M, N, K, packed, scales, zeros, group, Y, ws, ws_bytes, W4_VARIANT_AUTO,
                      stream);
}

w4_status w4_gemm_host(const uint16_t* X_host, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                       const uint16_t* scales, const uint8_t* zeros, int group, uint16_t* Y_host, uint16_t* x_dev,
                       uint16_t* y_dev, void* ws, size_t ws_bytes, int variant, void* stream) {
    if (group != 128) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    if (M == 0 || N == 0) return W4_OK;
    if (!Y_host || !y_dev || (K > 0 && (!X_host || !x_dev))) return W4_ERR_NULL;
    cudaStream_t s = (cudaStream_t)stream;
    if (K > 0 && cudaMemcpyAsync(x_dev, X_host, (size_t)M * (size_t)K * 2, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return W4_ERR_CUDA;
    const w4_status st = w4_gemm_ex(x_dev, M, N, K, packed, scales, zeros, group, y_dev, ws, ws_bytes, variant, stream);
    if (st != W4_OK) return st;
    if (cudaMemcpyAsync(Y_host, y_dev, (size_t)M * (size_t)N * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return W4_ERR_CUDA;
    return W4_OK;
}

w4_status w4_gemm_host_batch(const w4_gemm_layer* layers, int n_layers, int group, const void* x_host, void* x_dev,
                             size_t x_bytes, void* y_host, void* y_dev, size_t y_bytes, void* ws, size_t ws_bytes,
                             int variant, void* stream) {
    if (group != 128) return W4_ERR_UNSUPPORTED;
    const int family = variant & ~W4_FLAG_WEIGHTS_STATIC;
    if (family < W4_VARIANT_AUTO || family > W4_VARIANT_GEMV_TC) return W4_ERR_UNSUPPORTED;
    if (!layers || n_layers < 1) return n_layers < 1 ? W4_ERR_SHAPE : W4_ERR_NULL;
    if ((x_bytes > 0 && (!x_host || !x_dev)) || !y_host || !y_dev) return W4_ERR_NULL;
    if ((x_dev && !aligned16(x_dev)) || !aligned16(y_dev)) return W4_ERR_ALIGN;
    // validate every layer before anything is enqueued
    for (int i = 0; i < n_layers; ++i) {
        const w4_gemm_layer& L = layers[i];
        const int64_t M = L.M, N = L.N, K = L.K;
        if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0)
            return W4_ERR_SHAPE;
        if (L.x_offset < 0 || L.y_offset < 0) return W4_ERR_SHAPE;
        if ((L.x_offset & 15) || (L.y_offset & 15)) return W4_ERR_ALIGN;
        if ((uint64_t)L.y_offset + (uint64_t)(M * N * 2) > (uint64_t)y_bytes) return W4_ERR_SHAPE;
        if (M == 0 || N == 0 || K == 0) continue;
        if ((uint64_t)L.x_offset + (uint64_t)(M * K * 2) > (uint64_t)x_bytes || !x_dev) return W4_ERR_SHAPE;
        if (!L.packed || !L.scales || !L.zeros) return W4_ERR_NULL;
        if (!aligned16(L.packed)) return W4_ERR_ALIGN;
        size_t need = 0;
        w4_status st = w4_gemm_workspace_size(M, N, K, group, &need);
        if (st != W4_OK) return st;
        if (ws_bytes < need) return W4_ERR_WORKSPACE;
        if (need > 0 && !ws) return W4_ERR_NULL;
        int chosen = 0, launches = 0;
        st = gemm_plan(M, N, K, family, aligned16(L.scales) && aligned16(L.zeros), &chosen, &launches);
        if (st != W4_OK) return st;
    }
    cudaStream_t s = (cudaStream_t)stream;
    // Pinned, mapped host buffers (16-byte multiples) are copied by the SMs: one PCIe round trip
    // each way, chained to the GEMMs by programmatic dependent launch; other host memory through
    // the copy engines.
    const void* xh = x_bytes % 16 == 0 ? mapped_host_address(x_host) : nullptr;
    void* yh = y_bytes % 16 == 0 ? mapped_host_address(y_host) : nullptr;
    if (x_bytes > 0) {
        const cudaError_t e = xh && aligned16(xh) ? launch_host_copy(xh, x_dev, x_bytes, false, s)
                                                  : cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return W4_ERR_CUDA;
    }
    for (int i = 0; i < n_layers; ++i) {
        const w4_gemm_layer& L = layers[i];
        const w4_status st =
            w4_gemm_ex(reinterpret_cast<const uint16_t*>(static_cast<const char*>(x_dev) + L.x_offset), L.M, L.N,
                       L.K, L.packed, L.scales, L.zeros, group,
                       reinterpret_cast<uint16_t*>(static_cast<char*>(y_dev) + L.y_offset), ws, ws_bytes, variant,
                       stream);
        if (st != W4_OK) return st;
    }
    if (y_bytes > 0) {
        const cudaError_t e = yh && aligned16(yh) ? launch_host_copy(y_dev, yh, y_bytes, true, s)
                                                  : cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return W4_ERR_CUDA;
    }
    return W4_OK;
}

static w4_status awq_check(int64_t T, int64_t N, int64_t K, int group, int n_alpha) {
    if (group != 128 || n_alpha < 1 || n_alpha > 64) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(T, K) || !dims_ok(N, K) || T < 1 || N < 8 || K < 128 || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    return W4_OK;
}

w4_status awq_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha,
                             size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    *bytes = awq_layout(T, N, K, n_alpha).bytes;
    return W4_OK;
}

w4_status awq_scale_search(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                           int group, int n_alpha, double* mse, int32_t* best_idx, float* best_s,
                           void* ws, size_t ws_bytes, void* stream) {
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    if (ws_bytes < awq_layout(T, N, K, n_alpha).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !mse || !best_idx || !best_s || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_awq(X, T, W, N, K, n_alpha, mse, best_idx, best_s, ws, status,
                               (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status awq_colsum(const uint16_t* X, int64_t T, int64_t K, uint64_t* colsum, void* stream) {
    if (!dims_ok(T, K) || T < 0 || K < 128 || K % 128 != 0) return W4_ERR_SHAPE;
    if ((T > 0 && !X) || !colsum) return W4_ERR_NULL;
    if ((T > 0 && !aligned16(X)) || !aligned16(colsum)) return W4_ERR_ALIGN;
    cudaError_t e = launch_awq_colsum(X, T, K, colsum, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status awq_scales_from_colsum(const uint64_t* colsum, int64_t T_total, int64_t K, int n_alpha, float* s_all,
                                 void* stream) {
    if (n_alpha < 1 || n_alpha > 64) return W4_ERR_UNSUPPORTED;
    if (T_total < 1 || K < 128 || K % 128 != 0 || K >= ((int64_t)1 << 31)) return W4_ERR_SHAPE;
    if (!colsum || !s_all) return W4_ERR_NULL;
    cudaError_t e = launch_awq_scales_from_colsum(colsum, T_total, K, n_alpha, s_all, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status awq_sse_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    *bytes = awq_sse_layout(T, N, K, n_alpha).bytes;
    return W4_OK;
}

w4_status awq_sse(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int group, int n_alpha,
                  const float* s_all, double* sse, void* ws, size_t ws_bytes, void* stream) {
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    if (ws_bytes < awq_sse_layout(T, N, K, n_alpha).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !s_all || !sse || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(s_all) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_awq_sse(X, T, W, N, K, n_alpha, s_all, sse, ws, status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status awq_select(const double* sse, int n_parts, int n_alpha, int64_t T_total, int64_t N, const float* s_all,
                     int64_t K, double* mse, int32_t* best_idx, float* best_s, void* stream) {
    if (n_alpha < 1 || n_alpha > 64) return W4_ERR_UNSUPPORTED;
    if (n_parts < 1 || T_total < 1 || N < 1 || K < 1 || K >= ((int64_t)1 << 31)) return W4_ERR_SHAPE;
    if (!sse || !s_all || !mse || !best_idx || !best_s) return W4_ERR_NULL;
    cudaError_t e = launch_awq_select(sse, n_parts, n_alpha, T_total, N, s_all, K, mse, best_idx, best_s,
                                      (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status awq_gram_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_alpha, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    *bytes = awq_gram_layout(T, N, K, n_alpha).bytes;
    return W4_OK;
}

w4_status awq_scale_search_gram(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K,
                                int group, int n_alpha, double* mse, int32_t* best_idx, float* best_s,
                                void* ws, size_t ws_bytes, void* stream) {
    w4_status st = awq_check(T, N, K, group, n_alpha);
    if (st != W4_OK) return st;
    if (ws_bytes < awq_gram_layout(T, N, K, n_alpha).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !mse || !best_idx || !best_s || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_awq_gram(X, T, W, N, K, n_alpha, mse, best_idx, best_s, ws, status,
                                    (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

// group 64 or 128 (the Cholesky's 32-wide panels need K % 32 == 0, which K % group == 0 gives)
static w4_status gptq_shape(int64_t T, int64_t N, int64_t K, int group) {
    if (!dims_ok(T, K) || !dims_ok(N, K) || T < 1 || N < 8 || K < group || K > 32768 || K % group != 0 ||
        N % 8 != 0)
        return W4_ERR_SHAPE;
    return W4_OK;
}

static w4_status gptq_check(int64_t T, int64_t N, int64_t K, int group) {
    if (group != 128) return W4_ERR_UNSUPPORTED;
    return gptq_shape(T, N, K, group);
}

w4_status gptq_workspace_size(int64_t T, int64_t N, int64_t K, int group, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    if (group != 64 && group != 128) return W4_ERR_UNSUPPORTED;
    w4_status st = gptq_shape(T, N, K, group);
    if (st != W4_OK) return st;
    *bytes = gptq_layout(N, K).bytes;
    return W4_OK;
}

w4_status gptq_quantize(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int group,
                        double damp, uint32_t* packed, uint16_t* scales, uint8_t* zeros, void* ws,
                        size_t ws_bytes, void* stream) {
    w4_status st = gptq_check(T, N, K, group);
    if (st != W4_OK) return st;
    if (!(damp >= 0.0) || !(damp < 1.0e300)) return W4_ERR_UNSUPPORTED;  // rejects NaN and inf too
    if (ws_bytes < gptq_layout(N, K).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !packed || !scales || !zeros || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(packed) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_gptq(X, T, W, N, K, 4, 128, damp, false, nullptr, packed, scales, zeros, nullptr, ws,
                                status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

static bool bits_ok(int bits, int group) {
    return (bits == 2 || bits == 3 || bits == 4 || bits == 8) && (group == 64 || group == 128);
}

w4_status gptq_quantize_ex(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int bits,
                           int group, double damp, int act_order, const float* act_scale, uint32_t* packed,
                           uint16_t* scales, uint8_t* zeros, int32_t* perm, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!bits_ok(bits, group)) return W4_ERR_UNSUPPORTED;
    w4_status st = gptq_shape(T, N, K, group);
    if (st != W4_OK) return st;
    if (!(damp >= 0.0) || !(damp < 1.0e300)) return W4_ERR_UNSUPPORTED;
    if (ws_bytes < gptq_layout(N, K).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !packed || !scales || !zeros || !ws || (act_order && !perm)) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(packed) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_gptq(X, T, W, N, K, bits, group, damp, act_order != 0, act_scale, packed, scales, zeros,
                                act_order ? perm : nullptr, ws, status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_quantize_pack_bits(const uint16_t* W, int64_t N, int64_t K, int bits, int group,
                                const float* act_scale, uint32_t* packed, uint16_t* scales, uint8_t* zeros,
                                void* stream) {
    if (!bits_ok(bits, group)) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(N, K) || K % group != 0 || N % 8 != 0) return W4_ERR_SHAPE;
    if (N == 0 || K == 0) return W4_OK;
    if (!W || !packed || !scales || !zeros) return W4_ERR_NULL;
    if (!aligned16(W) || !aligned16(packed) || (act_scale && !aligned16(act_scale))) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_quantize_bits(W, N, K, bits, group, act_scale, packed, scales, zeros, status,
                                         (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status wb_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int bits, int group, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    if (!bits_ok(bits, group)) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0) return W4_ERR_SHAPE;
    *bytes = (size_t)N * (size_t)K * 2;
    return W4_OK;
}

w4_status wb_gemm(const uint16_t* X, int64_t M, int64_t N, int64_t K, const uint32_t* packed,
                  const uint16_t* scales, const uint8_t* zeros, int bits, int group, uint16_t* Y, void* ws,
                  size_t ws_bytes, void* stream) {
    if (!bits_ok(bits, group)) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(M, K) || !dims_ok(N, K) || !dims_ok(M, N) || K % group != 0 || N % 8 != 0) return W4_ERR_SHAPE;
    if (M == 0 || N == 0) return W4_OK;
    if (K == 0) return W4_ERR_SHAPE;
    if (ws_bytes < (size_t)N * (size_t)K * 2) return W4_ERR_WORKSPACE;
    if (!X || !packed || !scales || !zeros || !Y || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(Y) || !aligned16(ws)) return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_wb_gemm(X, M, N, K, packed, scales, zeros, bits, group, Y, ws, status,
                                   (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_act_prepare(const uint16_t* X, int64_t M, int64_t K, const int32_t* perm, const float* s,
                         uint16_t* X_out, void* stream) {
    if (!dims_ok(M, K)) return W4_ERR_SHAPE;
    if (M == 0 || K == 0) return W4_OK;
    if (!X || !X_out) return W4_ERR_NULL;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_act_prepare(X, M, K, perm, s, X_out, status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

static w4_status clip_check(int64_t T, int64_t N, int64_t K, int group, int n_ratios) {
    if (group != 128 || n_ratios < 1 || n_ratios > 10) return W4_ERR_UNSUPPORTED;
    if (!dims_ok(T, K) || !dims_ok(N, K) || T < 1 || N < 8 || K < 128 || K % group != 0 || N % 8 != 0)
        return W4_ERR_SHAPE;
    return W4_OK;
}

w4_status awq_clip_workspace_size(int64_t T, int64_t N, int64_t K, int group, int n_ratios, size_t* bytes) {
    if (!bytes) return W4_ERR_NULL;
    w4_status st = clip_check(T, N, K, group, n_ratios);
    if (st != W4_OK) return st;
    *bytes = awq_clip_layout(T, N, K, n_ratios).bytes;
    return W4_OK;
}

w4_status awq_clip_search(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N, int64_t K, int group,
                          int n_ratios, const float* act_scale, uint8_t* best_idx, float* err, uint32_t* packed,
                          uint16_t* scales, uint8_t* zeros, void* ws, size_t ws_bytes, void* stream) {
    w4_status st = clip_check(T, N, K, group, n_ratios);
    if (st != W4_OK) return st;
    if (ws_bytes < awq_clip_layout(T, N, K, n_ratios).bytes) return W4_ERR_WORKSPACE;
    if (!X || !W || !best_idx || !packed || !scales || !zeros || !ws) return W4_ERR_NULL;
    if (!aligned16(X) || !aligned16(W) || !aligned16(packed) || !aligned16(ws) ||
        (act_scale && !aligned16(act_scale)))
        return W4_ERR_ALIGN;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_awq_clip(X, T, W, N, K, n_ratios, act_scale, best_idx, err, packed, scales, zeros, ws,
                                    status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_check_device_status(void* stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return W4_ERR_CUDA;
    int* p = device_status_ptr();
    if (!p) return W4_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return W4_ERR_CUDA;
    if (v != 0 && cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return W4_ERR_CUDA;
    return (w4_status)v;
}

w4_status w4_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1000u || limit_ns > 5000000000ull) return W4_ERR_UNSUPPORTED;
    int* status = device_status_ptr();
    if (!status) return W4_ERR_CUDA;
    cudaError_t e = launch_selftest_wait(limit_ns, status, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

const char* w4_status_string(w4_status status) {
    switch (status) {
        case W4_OK: return "ok";
        case W4_ERR_NULL: return "a required pointer is NULL";
        case W4_ERR_SHAPE: return "unsupported or inconsistent shape";
        case W4_ERR_ALIGN: return "pointer is not 16-byte aligned";
        case W4_ERR_UNSUPPORTED: return "unsupported parameter (group must be 128; n_alpha 1..64)";
        case W4_ERR_WORKSPACE: return "workspace too small";
        case W4_ERR_CUDA: return "CUDA launch or query failed";
        case W4_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
        case W4_ERR_RANGE: return "fp16 group scale overflow";
        case W4_ERR_NUMERIC: return "matrix not positive definite (GPTQ Hessian)";
    }
    return "unknown status";
}

}  // extern "C"
