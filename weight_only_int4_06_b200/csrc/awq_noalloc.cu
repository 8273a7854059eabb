// awq_scale_search_noalloc: the AWQ scale search for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine): a plugin running inside an
// inference engine that owns every byte of device memory, a service held to a fixed memory
// budget, or a latency-critical path that must not risk the implicit device synchronisation an
// allocation can cause.  awq_scale_search needs a caller-supplied workspace; this entry point
// instead uses one scratch array compiled into the library, so the caller passes only inputs and
// outputs.
//
// The scratch is a file-scope __device__ array of W4_NOALLOC_SCRATCH_BYTES.  Every GPU that loads
// the library holds it until the process exits.  In host code the array's name is only a host-side
// stand-in, so its device address is looked up with cudaGetSymbolAddress once per device (with
// that device current) on the first call that succeeds there, and that address is what the
// kernels receive.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace w4 {

static __device__ __align__(256) unsigned char g_awq_scratch[W4_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDev = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDev];  // set once the lookup has succeeded on that device

// Device address of `dev`'s copy of the scratch array; `dev` must be the current device.  A failed
// lookup is not remembered: the next call tries again.
void* scratch_on(int dev) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_awq_scratch) == cudaSuccess) {
            g_scratch_ptr[dev] = p;
        } else {
            (void)cudaGetLastError();  // leave no error behind for the caller's next check
        }
    }
    return g_scratch_ptr[dev];
}
}  // namespace

}  // namespace w4

using namespace w4;

extern "C" w4_status awq_scale_search_noalloc(const uint16_t* X, int64_t T, const uint16_t* W, int64_t N,
                                              int64_t K, int group, int n_alpha, double* mse,
                                              int32_t* best_idx, float* best_s, void* stream) {
    size_t need = 0;
    const w4_status st = awq_workspace_size(T, N, K, group, n_alpha, &need);
    if (st != W4_OK) return st;
    if (need > (size_t)W4_NOALLOC_SCRATCH_BYTES) return W4_ERR_WORKSPACE;  // problem too large for the scratch
    // The scratch used is the copy on the stream's device, which must be the current device (the
    // kernels are launched there, and only there can the symbol's address be looked up).
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return W4_ERR_CUDA;
    if (stream) {
        int sdev = -1;
        if (cudaStreamGetDevice((cudaStream_t)stream, &sdev) != cudaSuccess) {
            (void)cudaGetLastError();
            return W4_ERR_CUDA;
        }
        if (sdev != dev) return W4_ERR_CUDA;  // a stream of another device: nothing enqueued
    }
    void* scratch = scratch_on(dev);
    if (!scratch) return W4_ERR_CUDA;
    return awq_scale_search(X, T, W, N, K, group, n_alpha, mse, best_idx, best_s, scratch,
                            (size_t)W4_NOALLOC_SCRATCH_BYTES, stream);
}
