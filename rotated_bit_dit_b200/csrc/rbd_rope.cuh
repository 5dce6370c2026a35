// Launchers of the Q/K RMSNorm + RoPE step (defined in rbd_rope.cu).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace rbd {

cudaError_t launch_qk_norm_rope(const uint16_t* x, int64_t ldx, int T, int H, const uint16_t* gamma,
                                const float* cos_t, const float* sin_t, float eps, uint16_t* y, int64_t ldy,
                                cudaStream_t st);
cudaError_t launch_rope_tables(const int32_t* pos, int T, double base, float* cos_t, float* sin_t,
                               cudaStream_t st);

}  // namespace rbd
