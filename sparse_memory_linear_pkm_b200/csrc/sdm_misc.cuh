// State initialisation and the RMS-norm x gate epilogue (sm_100a).
#pragma once

#include "sdm_device.cuh"

namespace sdm {

// M[b] <- M0 for every batch row: the learned initial state shared by all rows
// (SDM explainer, section 3.1, "learned initial state"). Bandwidth-bound
// 16-byte copies; blockIdx.y is the batch row.
static __global__ void __launch_bounds__(256) k_state_init(const uint4* __restrict__ M0, uint4* __restrict__ M,
                                                    int64_t units_per_row) {
  uint4* dst = M + static_cast<int64_t>(blockIdx.y) * units_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < units_per_row;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = M0[i];
}

// y[i] += other[i] for n float4s: the read sums of the second slot part of the
// pipelined recurrence added to the first part's.
static __global__ void __launch_bounds__(256) k_add_f4(float4* __restrict__ y, const float4* __restrict__ other,
                                                       int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = y[i];
    const float4 b = other[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    y[i] = a;
  }
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

// Sum of squares of each row of y over its d_v columns (one warp per row, a
// fixed order). When the d_v columns of a layer are split across devices,
// adding the devices' sums gives the full row's sum for the RMS norm.
static __global__ void __launch_bounds__(256) k_row_sumsq(const float* __restrict__ y, int64_t n_rows, int d_v,
                                                          float* __restrict__ ss) {
  const int lane = lane_id();
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / kWarp);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + threadIdx.x / kWarp;
       row < n_rows; row += warps) {
    const float* yr = y + row * d_v;
    float s = 0.f;
    for (int c = lane; c < d_v; c += kWarp) s = fmaf(yr[c], yr[c], s);
    s = warp_sum(s);
    if (lane == 0) ss[row] = s;
  }
}

// The RMS-norm x gate on a column slice of rows of d_total values, given the
// full rows' sums of squares: y <- g * y / sqrt(ss / d_total + eps).
template <typename Tin>
__global__ void __launch_bounds__(256) k_rmsnorm_gate_rows(float* __restrict__ y, const Tin* __restrict__ g,
                                                           const float* __restrict__ ss, int64_t n_rows, int d_v,
                                                           int d_total, float eps) {
  const int lane = lane_id();
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / kWarp);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + threadIdx.x / kWarp;
       row < n_rows; row += warps) {
    float* yr = y + row * d_v;
    const Tin* gr = g + row * d_v;
    const float inv = 1.0f / sqrtf(ss[row] / static_cast<float>(d_total) + eps);
    for (int c = lane; c < d_v; c += kWarp) yr[c] = to_f32<Tin>(gr[c]) * yr[c] * inv;
  }
}

// Backward of the RMS-norm x gate for dL/dout (x: the row before the
// epilogue, r = sqrt(mean(x^2) + eps), out = g x / r):
//   dL/dx_j = g_j dout_j / r - x_j sum_i(g_i dout_i x_i) / (d_v r^3),  dL/dg_i = dout_i x_i / r.
// One warp per row; both row sums are reduced in a fixed order.
template <typename Tin>
__global__ void __launch_bounds__(256) k_rmsnorm_gate_backward(const float* __restrict__ x, const Tin* __restrict__ g,
                                                               const float* __restrict__ dout, int64_t n_rows, int d_v,
                                                               float eps, float* __restrict__ dx,
                                                               float* __restrict__ dg) {
  const int lane = lane_id();
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / kWarp);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + threadIdx.x / kWarp;
       row < n_rows; row += warps) {
    const float* xr = x + row * d_v;
    const Tin* gr = g + row * d_v;
    const float* dr = dout + row * d_v;
    float ss = 0.f, dot = 0.f;
    for (int c = lane; c < d_v; c += kWarp) {
      ss = fmaf(xr[c], xr[c], ss);
      dot = fmaf(to_f32<Tin>(gr[c]) * dr[c], xr[c], dot);
    }
    ss = warp_sum(ss);
    dot = warp_sum(dot);
    const float rms = sqrtf(ss / static_cast<float>(d_v) + eps);
    const float inv = 1.0f / rms;
    const float corr = dot * inv * inv * inv / static_cast<float>(d_v);
    for (int c = lane; c < d_v; c += kWarp) {
      const float gc = to_f32<Tin>(gr[c]);
      dx[row * d_v + c] = gc * dr[c] * inv - xr[c] * corr;
      dg[row * d_v + c] = dr[c] * xr[c] * inv;
    }
  }
}

// Slot utilisation: counts[b, h, i] += number of (t, k) with idx[b, t, h, k]
// == i. A monitor of how the selection spreads over the N slots (uneven
// addressing, the collapse onto few slots that the explainer page's
// "亮点与局限" and "工程落地关键点" sections warn about). grid
// (ceil(T / tokens_per_cta), B*H), 256 threads. With N <= kCountSmemSlots a
// CTA counts in shared memory and adds its nonzero bins to global memory at
// the end; otherwise it adds to global memory directly. The work is HBM-bound
// (4 bytes of index per count), so each thread keeps kCountUnroll 16-byte
// index loads in flight before it counts them. Indices outside [0, N) are
// skipped and flagged.
constexpr int kCountSmemSlots = 16384;
constexpr int kCountUnroll = 4;

template <bool kLocal>
__device__ __forceinline__ void count_one(int slot, int N, int* bins, int32_t* out, unsigned* err) {
  if (static_cast<unsigned>(slot) >= static_cast<unsigned>(N)) {
    atomicOr(err, kErrIndexOutOfRange);
    return;
  }
  if (kLocal) atomicAdd(&bins[slot], 1);
  else atomicAdd(&out[slot], 1);
}

template <bool kLocal, bool kVec>
__global__ void __launch_bounds__(256) k_slot_counts(const int32_t* __restrict__ idx, int T, int H, int K, int N,
                                                     int tokens_per_cta, int32_t* __restrict__ counts,
                                                     unsigned* err) {
  extern __shared__ int bins[];
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * tokens_per_cta;
  const int t1 = min(T, t0 + tokens_per_cta);
  int32_t* out = counts + static_cast<int64_t>(bh) * N;
  if (kLocal) {
    for (int i = threadIdx.x; i < N; i += blockDim.x) bins[i] = 0;
    __syncthreads();
  }
  // token t's K indices start at row(t) * K, rows H apart
  const int64_t row0 = (static_cast<int64_t>(b) * T + t0) * H + h;
  if (kVec) {
    const int kv = K / 4;  // int4 per token
    const int n = (t1 - t0) * kv;
    for (int x0 = threadIdx.x; x0 < n; x0 += blockDim.x * kCountUnroll) {
      int4 v[kCountUnroll];
#pragma unroll
      for (int u = 0; u < kCountUnroll; ++u) {
        const int x = x0 + u * blockDim.x;
        if (x < n) {
          const int t = x / kv, j = x - t * kv;
          v[u] = __ldcs(reinterpret_cast<const int4*>(idx + (row0 + static_cast<int64_t>(t) * H) * K) + j);
        } else {
          v[u] = make_int4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kCountUnroll; ++u) {
        if (x0 + u * blockDim.x < n) {
          count_one<kLocal>(v[u].x, N, bins, out, err);
          count_one<kLocal>(v[u].y, N, bins, out, err);
          count_one<kLocal>(v[u].z, N, bins, out, err);
          count_one<kLocal>(v[u].w, N, bins, out, err);
        }
      }
    }
  } else {
    const int n = (t1 - t0) * K;
    for (int x0 = threadIdx.x; x0 < n; x0 += blockDim.x * kCountUnroll) {
      int v[kCountUnroll];
#pragma unroll
      for (int u = 0; u < kCountUnroll; ++u) {
        const int x = x0 + u * blockDim.x;
        if (x < n) {
          const int t = x / K, k = x - t * K;
          v[u] = __ldcs(idx + (row0 + static_cast<int64_t>(t) * H) * K + k);
        }
      }
#pragma unroll
      for (int u = 0; u < kCountUnroll; ++u)
        if (x0 + u * blockDim.x < n) count_one<kLocal>(v[u], N, bins, out, err);
    }
  }
  if (kLocal) {
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      if (bins[i] != 0) atomicAdd(&out[i], bins[i]);
  }
}

}  // namespace sdm
