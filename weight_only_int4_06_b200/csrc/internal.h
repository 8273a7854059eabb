// Host-side declarations shared by the translation units of libw4a16 (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

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
cudaError_t launch_skinny(const uint16_t* X, int64_t M, int64_t N, int64_t K,
                          const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                          uint16_t* Y, const SkinnyPlan& plan, cudaStream_t stream);

}  // namespace w4
