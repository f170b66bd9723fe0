// bcnorm.cuh -- the BC-norm prologue's row scale, shared by the CUDA-core
// kernels: 1 / sqrt(mean_n v_n^2 + eps) of one (token, head, rank) row of B or
// C, computed by one warp (every lane gets the result).  The norm and the
// head-specific biases it precedes are those of "Знакомство с Mamba-3",
// section "Архитектура и нормализация".
#pragma once
#include <cuda_runtime.h>

namespace m3 {

template <typename Get>
__device__ __forceinline__ float bcn_row_scale_warp(Get get, int n, float eps) {
    float ss = 0.f;
    for (int i = threadIdx.x & 31; i < n; i += 32) {
        const float v = get(i);
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    return rsqrtf(ss / (float)n + eps);
}

}  // namespace m3
