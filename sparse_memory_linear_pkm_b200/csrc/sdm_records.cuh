// Per-token staging records for the recurrence kernels (sm_100a).
//
// The recurrence walks tokens in order for one (b, h). It stages, per token,
// one contiguous record with everything the write and the read need except v:
//   int32 slot_w[Wp] | f32 k_w[Wp] | int32 slot_r[Rp] | f32 q_r[Rp] |
//   int16 fwd[Fp]    | f32 alpha, beta, 0, 0
// (Wp, Rp rounded up to 4 entries, Fp = W+R rounded up to 8, so a record is a
// multiple of 16 bytes; Fp = 0 when the consumer needs no hazard plan). Records are laid out [B, H, T] so a run of tokens of
// one (b, h) is one contiguous bulk copy.
//
// fwd[e] is the hazard plan of the streaming kernel, which gathers the state
// rows of token t+P while token t computes. A row gathered early is stale if a
// token in between writes that slot, so the plan names the most recent such
// write: fwd = (k << 9) | j means "take token t-k's freshly written row for
// its write entry j" (k in [1, P-1] for write entries, [0, P-1] for read
// entries, k = 0 being the read-after-write inside one token), fwd = -1 means
// the gathered row is current. Built with one small open-addressing table of
// write slots per token in shared memory.
//
// Slot indices outside [0, N) are replaced by -1 (skipped by the kernels) and
// flagged in the device error word; the padding entries also carry slot -1.
#pragma once

#include "sdm_device.cuh"

namespace sdm {

struct RecLayout {
  int Wp, Rp, Fp;
  int off_slot_w, off_k_w, off_slot_r, off_q_r, off_fwd, off_ab;
  int words;  // record stride in 32-bit words (multiple of 4)
};

constexpr uint32_t kEmptyCell = 0xFFFFFFFFu;
constexpr int kRecTokensPerBlock = 32;

__device__ __forceinline__ uint32_t slot_hash(uint32_t slot, int log2_cells) {
  return (slot * 2654435761u) >> (32 - log2_cells);
}

template <typename Tin>
__global__ void __launch_bounds__(256) k_build_records(
    const int32_t* __restrict__ idx_w, const float* __restrict__ w_w, const int32_t* __restrict__ idx_r,
    const float* __restrict__ w_r, const Tin* __restrict__ alpha, const Tin* __restrict__ beta, int T, int H,
    int N, int W, int R, int P, int log2_cells, RecLayout rl, uint32_t* __restrict__ rec, unsigned* err) {
  extern __shared__ uint32_t cells[];  // one table per token in [t_first, t_end), P > 0 only
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * kRecTokensPerBlock;
  const int t_end = min(T, t0 + kRecTokensPerBlock);
  const int t_first = P > 0 ? max(0, t0 - (P - 1)) : t0;
  const int n_cells = 1 << log2_cells;

  if (P > 0) {
    const int n_tab = t_end - t_first;
    for (int i = threadIdx.x; i < n_tab * n_cells; i += blockDim.x) cells[i] = kEmptyCell;
    __syncthreads();
    for (int x = threadIdx.x; x < n_tab * W; x += blockDim.x) {
      const int tt = t_first + x / W, j = x % W;
      const int slot = idx_w[((static_cast<int64_t>(b) * T + tt) * H + h) * W + j];
      if (slot < 0 || slot >= N) continue;
      const uint32_t packed = static_cast<uint32_t>(slot) * 512u + static_cast<uint32_t>(j);
      uint32_t* tab = cells + (tt - t_first) * n_cells;
      uint32_t pos = slot_hash(static_cast<uint32_t>(slot), log2_cells);
      for (int probe = 0; probe < n_cells; ++probe) {  // at most W < n_cells entries per table
        const uint32_t prev = atomicCAS(&tab[pos], kEmptyCell, packed);
        if (prev == kEmptyCell || (prev >> 9) == static_cast<uint32_t>(slot)) break;
        pos = (pos + 1) & (n_cells - 1);
      }
    }
    __syncthreads();
  }

  const int E = W + R;
  for (int x = threadIdx.x; x < (t_end - t0) * E; x += blockDim.x) {
    const int t = t0 + x / E, e = x % E;
    const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
    uint32_t* r = rec + (static_cast<int64_t>(bh) * T + t) * rl.words;
    int slot;
    float wt;
    if (e < W) {
      slot = idx_w[th * W + e];
      wt = w_w[th * W + e];
    } else {
      slot = idx_r[th * R + (e - W)];
      wt = w_r[th * R + (e - W)];
    }
    if (slot < 0 || slot >= N) {
      atomicOr(err, kErrIndexOutOfRange);
      slot = -1;
    }
    int code = -1;
    if (P > 0 && slot >= 0) {
      for (int k = (e < W ? 1 : 0); k < P && code < 0; ++k) {
        const int tt = t - k;
        if (tt < 0) break;
        const uint32_t* tab = cells + (tt - t_first) * n_cells;
        uint32_t pos = slot_hash(static_cast<uint32_t>(slot), log2_cells);
        for (int probe = 0; probe < n_cells; ++probe) {
          const uint32_t cur = tab[pos];
          if (cur == kEmptyCell) break;
          if ((cur >> 9) == static_cast<uint32_t>(slot)) {
            code = (k << 9) | static_cast<int>(cur & 511u);
            break;
          }
          pos = (pos + 1) & (n_cells - 1);
        }
      }
    }
    if (e < W) {
      r[rl.off_slot_w + e] = static_cast<uint32_t>(slot);
      r[rl.off_k_w + e] = __float_as_uint(wt);
    } else {
      r[rl.off_slot_r + e - W] = static_cast<uint32_t>(slot);
      r[rl.off_q_r + e - W] = __float_as_uint(wt);
    }
    if (rl.Fp > 0) reinterpret_cast<int16_t*>(r + rl.off_fwd)[e] = static_cast<int16_t>(code);
  }
  // Padding entries (W..Wp, R..Rp) carry slot -1.
  const int npad = (rl.Wp - W) + (rl.Rp - R);
  for (int x = threadIdx.x; x < (t_end - t0) * npad; x += blockDim.x) {
    const int t = t0 + x / npad, e = x % npad;
    uint32_t* r = rec + (static_cast<int64_t>(bh) * T + t) * rl.words;
    if (e < rl.Wp - W) {
      r[rl.off_slot_w + W + e] = 0xFFFFFFFFu;
      r[rl.off_k_w + W + e] = 0u;
    } else {
      r[rl.off_slot_r + R + e - (rl.Wp - W)] = 0xFFFFFFFFu;
      r[rl.off_q_r + R + e - (rl.Wp - W)] = 0u;
    }
  }
  for (int t = t0 + static_cast<int>(threadIdx.x); t < t_end; t += blockDim.x) {
    const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
    uint32_t* r = rec + (static_cast<int64_t>(bh) * T + t) * rl.words;
    r[rl.off_ab] = __float_as_uint(to_f32<Tin>(alpha[th]));
    r[rl.off_ab + 1] = __float_as_uint(to_f32<Tin>(beta[th]));
    r[rl.off_ab + 2] = 0u;
    r[rl.off_ab + 3] = 0u;
  }
}

}  // namespace sdm
