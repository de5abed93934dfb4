// State initialisation and the RMS-norm x gate epilogue (sm_100a).
#pragma once

#include "sdm_device.cuh"

namespace sdm {

// M[b] <- M0 for every batch row: the learned initial state shared by all rows
// (SDM explainer, section 3.1, "learned initial state"). Bandwidth-bound
// 16-byte copies; blockIdx.y is the batch row.
__global__ void __launch_bounds__(256) k_state_init(const uint4* __restrict__ M0, uint4* __restrict__ M,
                                                    int64_t units_per_row) {
  uint4* dst = M + static_cast<int64_t>(blockIdx.y) * units_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < units_per_row;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = M0[i];
}

// y <- g * y / sqrt(mean(y^2) + eps) over d_v for each token-head (SDM
// explainer, section 3.1 step 3: RMS-Norm, then element-wise gating). One warp
// per row; the sum of squares is reduced in a fixed order.
template <typename Tin>
__global__ void __launch_bounds__(256) k_rmsnorm_gate(float* __restrict__ y, const Tin* __restrict__ g,
                                                      int64_t n_rows, int d_v, float eps) {
  const int lane = lane_id();
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / kWarp);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + threadIdx.x / kWarp;
       row < n_rows; row += warps) {
    float* yr = y + row * d_v;
    const Tin* gr = g + row * d_v;
    float ss = 0.f;
    for (int c = lane; c < d_v; c += kWarp) ss = fmaf(yr[c], yr[c], ss);
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / static_cast<float>(d_v) + eps);
    for (int c = lane; c < d_v; c += kWarp) yr[c] = to_f32<Tin>(gr[c]) * yr[c] * inv;
  }
}

}  // namespace sdm
