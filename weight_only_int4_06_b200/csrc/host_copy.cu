// Copies between pinned host memory and the device made by the SMs instead of the copy engines.
//
// A decode step moves a few tens of KB each way; a copy-engine transfer of that size costs several
// microseconds of setup and leaves a gap before and after the kernels around it.  A kernel that
// reads (or writes) the host buffer through its mapped device address takes one PCIe round trip,
// and it joins the programmatic-dependent-launch chain of the GEMMs: the inbound copy lets the
// first GEMM launch at once (its producer streams weights while the activations arrive; its
// consumers wait for this kernel's end), and the outbound copy is launched early and waits for
// the last GEMM's end before it reads the results.
#include "common.cuh"
#include "internal.h"

namespace w4 {

__global__ void __launch_bounds__(256) host_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                        int64_t n16, int after_prior) {
    pdl_launch_dependents();
    if (after_prior) pdl_wait();  // the data is written by the preceding kernel
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

void* mapped_host_address(const void* p) {
    if (!p) return nullptr;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // a pointer the runtime does not know: not an error of this call
        return nullptr;
    }
    // pinned (page-locked) host memory the runtime has mapped for the device; anything else
    // (pageable or managed memory) goes through the copy engines
    if (a.type != cudaMemoryTypeHost || !a.devicePointer) return nullptr;
    return a.devicePointer;
}

cudaError_t launch_host_copy(const void* src, void* dst, size_t bytes, bool after_prior, cudaStream_t stream) {
    if (bytes == 0) return cudaSuccess;
    if ((bytes & 15) || (reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
        return cudaErrorInvalidValue;
    const int64_t n16 = (int64_t)(bytes / 16);
    const int64_t want = (n16 + 255) / 256;
    const int64_t cap = device_sm_count();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_prior ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, host_copy_kernel, reinterpret_cast<const uint4*>(src),
                              reinterpret_cast<uint4*>(dst), n16, after_prior ? 1 : 0);
}

}  // namespace w4
