// Backward of the sparse gated delta recurrence and of the selection weights
// (sm_100a): the derivatives a training step needs.
//
// The SDM explainer (papers.ananclaw.com), section 3.4 "高效训练", says only
// that a memory-efficient backward exists. These kernels take the derivatives
// of the forward of section 3.1 steps 2-3 for a fixed selection, in the
// factored form the forward kernels compute (a_i = alpha (1 - beta k_i),
// c_i = beta k_i, M[i] <- a_i M[i] + c_i v):
//
//   read  y_t = sum_j q_j M_t[j]:   dq_j = <dy_t, M_t[j]>,  G[j] += q_j dy_t
//   write (per write slot i, G = dL/dM_t[i], m = M_{t-1}[i]):
//         da_i = <G, m>, dc_i = <G, v_t>,  dv_t += c_i G,  G <- a_i G
//         dk_i = beta (dc_i - alpha da_i)
//         dalpha_t = sum_i (1 - beta k_i) da_i
//         dbeta_t  = sum_i k_i (dc_i - alpha da_i)
//
// with G = dL/dM running backwards over the tokens from dL/dM_T, the read of a
// token before its write. Every column of d_v is independent given the
// per-token scalars, so one warp carries one 4-column tile of one (b, h) with
// its state M and adjoint G resident in shared memory. Memory-efficient by
// recomputation: a first forward pass stores the tile every C tokens
// (checkpoints); then, chunk by chunk from the end, the warp reloads the
// chunk's checkpoint, recomputes the chunk forward keeping the values each
// write overwrites (the log), and sweeps the chunk backwards, restoring the
// overwritten values as it goes. The recomputed trajectory is the forward
// kernels' bit for bit (same fp32 operations in the same order).
//
// dv is complete per tile; dk, dq, dalpha and dbeta are sums over all columns,
// so each tile writes its partial sums and k_scan_backward_reduce adds the
// tiles in a fixed order (bit-reproducible).
#pragma once

#include "sdm_device.cuh"
#include "sdm_records.cuh"

namespace sdm {

struct BwdArgs {
  int B, T, H, N, d_v, W, R;
  int C;      // tokens per checkpoint chunk
  int ntile;  // d_v / 4
  RecLayout rl;
  const uint32_t* rec;  // [B, H, T, rl.words] per-token records (slots, weights, alpha, beta; no hazard plan)
  const void* v;        // [B, T, H, d_v] Tin
  const float* M_in;  // rows of (b, h) at M_in + b * M_in_b_stride + h * N * d_v
  int64_t M_in_b_stride;
  const float* dy;  // [B, T, H, d_v]
  float* dM;        // [B, H, N, d_v] in: dL/dM_T, out: dL/dM_0
  float* dv;        // [B, T, H, d_v]
  float* part;      // [B, T, H, ntile, W + R + 2] per-tile partial sums
  float* ckpt;      // per tile: (ceil(T / C) - 1) * N * 4
  float* logbuf;    // per tile: C * W * 4
  unsigned* err;
};

// 8-byte global -> shared asynchronous copy (generic proxy); both addresses
// 8-byte aligned.
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}

// Tile geometry: a warp owns kBwdCols = 4 columns of one (b, h); lane l
// handles entry e0 + l of a token (32 entries per warp instruction) and its 4
// columns as one float4, so the sums over the tile's columns stay inside the
// lane. State and adjoint rows are 16 bytes in shared memory.
constexpr int kBwdCols = 4;

// Staging: per token, a ring stage in shared memory holds
//   log  [W][4] f32     the values its W writes overwrote (reverse sweep only)
//   rec  [rl.words]     its record: slots, weights, alpha, beta
//   v    [4] Tin        this tile's columns of v_t (padded to 16 bytes)
//   dy   [4] f32        this tile's columns of dy_t (reverse sweep only)
// filled by cp.async kBwdStages - 1 tokens ahead of use, so the token loop
// itself issues no global loads.
constexpr int kBwdStages = 4;
constexpr int kBwdUnroll = 2;  // entries per lane handled together (W, R <= 64 in one round)

struct BwdStage {
  int log, rec, v, dy, words;  // word offsets and the stage size (all multiples of 4)
};
__host__ __device__ inline BwdStage bwd_stage(int W, int rec_words) {
  BwdStage st;
  st.log = 0;
  st.rec = W * kBwdCols;
  st.v = st.rec + rec_words;
  st.dy = st.v + 4;
  st.words = st.dy + 4;
  return st;
}

// Per-token view of a filled stage.
struct BwdTok {
  const float4* log;
  const uint32_t* rec;
  float alpha, beta;
  float4 v, dy;
};

// Sums eight values over the warp with nine shuffles (reduce-scatter: each
// exchange sends the half of the values the partner keeps). Lane l returns the
// warp sum of value (l >> 2) & 7; lanes 4j .. 4j+3 hold value j. The order of
// the additions is fixed, so the sums are reproducible.
__device__ __forceinline__ float warp_sum8_transposed(float x0, float x1, float x2, float x3, float x4, float x5,
                                                      float x6, float x7, int lane) {
  const bool h16 = (lane & 16) != 0, h8 = (lane & 8) != 0, h4 = (lane & 4) != 0;
  const float y0 = (h16 ? x4 : x0) + __shfl_xor_sync(0xffffffffu, h16 ? x0 : x4, 16);
  const float y1 = (h16 ? x5 : x1) + __shfl_xor_sync(0xffffffffu, h16 ? x1 : x5, 16);
  const float y2 = (h16 ? x6 : x2) + __shfl_xor_sync(0xffffffffu, h16 ? x2 : x6, 16);
  const float y3 = (h16 ? x7 : x3) + __shfl_xor_sync(0xffffffffu, h16 ? x3 : x7, 16);
  const float z0 = (h8 ? y2 : y0) + __shfl_xor_sync(0xffffffffu, h8 ? y0 : y2, 8);
  const float z1 = (h8 ? y3 : y1) + __shfl_xor_sync(0xffffffffu, h8 ? y1 : y3, 8);
  float w = (h4 ? z1 : z0) + __shfl_xor_sync(0xffffffffu, h4 ? z0 : z1, 4);
  w += __shfl_xor_sync(0xffffffffu, w, 2);
  w += __shfl_xor_sync(0xffffffffu, w, 1);
  return w;
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return __fmaf_rn(a.w, b.w, __fmaf_rn(a.z, b.z, __fmaf_rn(a.y, b.y, a.x * b.x)));
}

// Runs body(t, token) over n tokens t = t_first + i * step of one (b, h) and
// column tile, each with its stage filled (log rows from log_src when given,
// dy when with_dy).
template <typename Tin, class Body>
__device__ __forceinline__ void bwd_token_pass(const BwdArgs& a, int b, int h, int tile, int lane, int t_first,
                                               int step, int n, float* ring, const float* log_src, int log_t0,
                                               bool with_dy, Body body) {
  const BwdStage L = bwd_stage(a.W, a.rl.words);
  const int n_log = log_src != nullptr ? a.W : 0;  // 16-byte pieces: one row each
  const int n_rec = a.rl.words / 4;
  const int bh = b * a.H + h;
  auto issue = [&](int i) {
    if (i < n) {
      const int t = t_first + i * step;
      const int64_t th = (static_cast<int64_t>(b) * a.T + t) * a.H + h;
      float* st = ring + (i % kBwdStages) * L.words;
      const uint32_t* rsrc = a.rec + (static_cast<int64_t>(bh) * a.T + t) * a.rl.words;
      for (int x = lane; x < n_rec; x += kWarp) cp_async16(st + L.rec + 4 * x, rsrc + 4 * x);
      if (n_log > 0) {
        const float* lsrc = log_src + static_cast<int64_t>(t - log_t0) * a.W * kBwdCols;
        for (int x = lane; x < n_log; x += kWarp) cp_async16(st + L.log + 4 * x, lsrc + 4 * x);
      }
      if (lane == kWarp - 1) {
        const Tin* vsrc = static_cast<const Tin*>(a.v) + th * a.d_v + tile * kBwdCols;
        if constexpr (sizeof(Tin) == 4) cp_async16(st + L.v, vsrc);
        else cp_async8(st + L.v, vsrc);
      } else if (lane == kWarp - 2 && with_dy) {
        cp_async16(st + L.dy, a.dy + th * a.d_v + tile * kBwdCols);
      }
    }
    cp_async_commit();  // empty groups past the end keep the count uniform
  };
#pragma unroll
  for (int i = 0; i < kBwdStages - 1; ++i) issue(i);
  for (int i = 0; i < n; ++i) {
    issue(i + kBwdStages - 1);
    cp_async_wait<kBwdStages - 1>();
    __syncwarp();
    const float* st = ring + (i % kBwdStages) * L.words;
    BwdTok k;
    k.log = reinterpret_cast<const float4*>(st + L.log);
    k.rec = reinterpret_cast<const uint32_t*>(st + L.rec);
    k.alpha = __uint_as_float(k.rec[a.rl.off_ab]);
    k.beta = __uint_as_float(k.rec[a.rl.off_ab + 1]);
    const Tin* vv = reinterpret_cast<const Tin*>(st + L.v);
    k.v = make_float4(to_f32<Tin>(vv[0]), to_f32<Tin>(vv[1]), to_f32<Tin>(vv[2]), to_f32<Tin>(vv[3]));
    k.dy = with_dy ? *reinterpret_cast<const float4*>(st + L.dy) : make_float4(0.f, 0.f, 0.f, 0.f);
    body(t_first + i * step, k);
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncwarp();
}

// The forward write of one token on the tile (the forward kernels' exact fp32
// operations: m <- fma(alpha (1 - beta k), m, (beta k) v)). With `log`, the
// overwritten rows are kept at log[e].
__device__ __forceinline__ void bwd_forward_token(const BwdArgs& a, const BwdTok& k, float4* Ms, float4* log,
                                                  int lane) {
  const int32_t* slot = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_w);
  const float* ww = reinterpret_cast<const float*>(k.rec + a.rl.off_k_w);
  // kBwdUnroll entries per lane at once: their loads first, then the stores
  // (the slots of one token are distinct, so the order is free).
  for (int e0 = lane; e0 < a.W; e0 += kWarp * kBwdUnroll) {
    int s[kBwdUnroll];
    float4 m[kBwdUnroll];
    float aw[kBwdUnroll], cw[kBwdUnroll];
#pragma unroll
    for (int u = 0; u < kBwdUnroll; ++u) {
      const int e = e0 + u * kWarp;
      s[u] = e < a.W ? slot[e] : -1;
      cw[u] = s[u] >= 0 ? k.beta * ww[e] : 0.0f;
      aw[u] = k.alpha * (1.0f - cw[u]);
      m[u] = s[u] >= 0 ? Ms[s[u]] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kBwdUnroll; ++u) {
      if (s[u] < 0) continue;
      if (log != nullptr) log[e0 + u * kWarp] = m[u];
      Ms[s[u]] = make_float4(__fmaf_rn(aw[u], m[u].x, __fmul_rn(cw[u], k.v.x)),
                             __fmaf_rn(aw[u], m[u].y, __fmul_rn(cw[u], k.v.y)),
                             __fmaf_rn(aw[u], m[u].z, __fmul_rn(cw[u], k.v.z)),
                             __fmaf_rn(aw[u], m[u].w, __fmul_rn(cw[u], k.v.w)));
    }
  }
}

template <typename Tin>
__global__ void __launch_bounds__(32) k_scan_backward(BwdArgs a) {
  extern __shared__ __align__(16) float bsm[];
  const int N = a.N;
  float4* Ms = reinterpret_cast<float4*>(bsm);  // [N] state rows of the tile
  float4* Gs = Ms + N;                          // [N] adjoint rows
  float* ring = reinterpret_cast<float*>(Gs + N);

  const int lane = threadIdx.x;
  const int tile = blockIdx.x % a.ntile;
  const int bh = blockIdx.x / a.ntile;
  const int b = bh / a.H, h = bh % a.H;
  const int col0 = tile * kBwdCols;
  const int64_t tile_id = blockIdx.x;
  const int nC = (a.T + a.C - 1) / a.C;
  float4* ckpt = reinterpret_cast<float4*>(a.ckpt) + tile_id * static_cast<int64_t>(nC > 1 ? nC - 1 : 0) * N;
  float4* logb = reinterpret_cast<float4*>(a.logbuf) + tile_id * static_cast<int64_t>(a.C) * a.W;
  const float* Min = a.M_in + b * a.M_in_b_stride + static_cast<int64_t>(h) * N * a.d_v + col0;
  auto load_min = [&]() {
    for (int row = lane; row < N; row += kWarp)
      Ms[row] = *reinterpret_cast<const float4*>(Min + static_cast<int64_t>(row) * a.d_v);
  };

  // --------------------------------------------- pass 1: checkpoints --
  // (only when the sequence has more than one chunk)
  load_min();
  __syncwarp();
  if (nC > 1)
    bwd_token_pass<Tin>(a, b, h, tile, lane, 0, 1, a.T, ring, nullptr, 0, false, [&](int t, const BwdTok& k) {
    if (t > 0 && t % a.C == 0) {
      float4* dst = ckpt + static_cast<int64_t>(t / a.C - 1) * N;
      for (int row = lane; row < N; row += kWarp) dst[row] = Ms[row];
    }
    bwd_forward_token(a, k, Ms, nullptr, lane);
  });

  // ---------------------------------- pass 2: chunks from the end --
  float* Gout = a.dM + (static_cast<int64_t>(b) * a.H + h) * N * a.d_v + col0;
  for (int row = lane; row < N; row += kWarp)
    Gs[row] = *reinterpret_cast<const float4*>(Gout + static_cast<int64_t>(row) * a.d_v);
  const int PW = a.W + a.R + 2;
  for (int kc = nC - 1; kc >= 0; --kc) {
    const int t0 = kc * a.C, t1 = min(a.T, t0 + a.C);
    // State at the chunk start.
    if (kc == 0) {
      load_min();
    } else {
      const float4* src = ckpt + static_cast<int64_t>(kc - 1) * N;
      for (int row = lane; row < N; row += kWarp) Ms[row] = src[row];
    }
    __syncwarp();
    // Recompute the chunk forward, logging overwritten rows.
    bwd_token_pass<Tin>(a, b, h, tile, lane, t0, 1, t1 - t0, ring, nullptr, 0, false, [&](int t, const BwdTok& k) {
      bwd_forward_token(a, k, Ms, logb + static_cast<int64_t>(t - t0) * a.W, lane);
    });
    // The log rows were written by other lanes; the reverse pass reads them
    // back through cp.async.
    __threadfence_block();
    __syncwarp();
    // Backward sweep over the chunk.
    bwd_token_pass<Tin>(
        a, b, h, tile, lane, t1 - 1, -1, t1 - t0, ring, reinterpret_cast<const float*>(logb), t0, true,
        [&](int t, const BwdTok& k) {
          const int64_t th = (static_cast<int64_t>(b) * a.T + t) * a.H + h;
          const int32_t* sw_ = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_w);
          const float* ww = reinterpret_cast<const float*>(k.rec + a.rl.off_k_w);
          const int32_t* ir = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_r);
          const float* wr = reinterpret_cast<const float*>(k.rec + a.rl.off_q_r);
          float* prt = a.part + (th * a.ntile + tile) * PW;
          // Read of token t (state after its write): dq and the adjoint.
          for (int e0 = lane; e0 < a.R; e0 += kWarp * kBwdUnroll) {
            int s[kBwdUnroll];
            float4 m[kBwdUnroll], g[kBwdUnroll];
            float q[kBwdUnroll];
#pragma unroll
            for (int u = 0; u < kBwdUnroll; ++u) {
              const int e = e0 + u * kWarp;
              s[u] = e < a.R ? ir[e] : -1;
              q[u] = s[u] >= 0 ? wr[e] : 0.0f;
              m[u] = s[u] >= 0 ? Ms[s[u]] : make_float4(0.f, 0.f, 0.f, 0.f);
              g[u] = s[u] >= 0 ? Gs[s[u]] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kBwdUnroll; ++u) {
              const int e = e0 + u * kWarp;
              if (e >= a.R) continue;
              prt[a.W + e] = s[u] >= 0 ? dot4(k.dy, m[u]) : 0.0f;
              if (s[u] >= 0)
                Gs[s[u]] = make_float4(__fmaf_rn(q[u], k.dy.x, g[u].x), __fmaf_rn(q[u], k.dy.y, g[u].y),
                                       __fmaf_rn(q[u], k.dy.z, g[u].z), __fmaf_rn(q[u], k.dy.w, g[u].w));
            }
          }
          __syncwarp();
          // Write of token t, undone: derivatives, adjoint decay, state restore.
          float4 dv = make_float4(0.f, 0.f, 0.f, 0.f);
          float dal = 0.0f, dbe = 0.0f;
          for (int e0 = lane; e0 < a.W; e0 += kWarp * kBwdUnroll) {
            int s[kBwdUnroll];
            float4 g[kBwdUnroll], m[kBwdUnroll];
            float kw[kBwdUnroll];
#pragma unroll
            for (int u = 0; u < kBwdUnroll; ++u) {
              const int e = e0 + u * kWarp;
              s[u] = e < a.W ? sw_[e] : -1;
              kw[u] = s[u] >= 0 ? ww[e] : 0.0f;
              g[u] = s[u] >= 0 ? Gs[s[u]] : make_float4(0.f, 0.f, 0.f, 0.f);
              m[u] = s[u] >= 0 ? k.log[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kBwdUnroll; ++u) {
              const int e = e0 + u * kWarp;
              if (e >= a.W) continue;
              float dk = 0.0f;
              if (s[u] >= 0) {
                const float cw = k.beta * kw[u];
                const float aw = k.alpha * (1.0f - cw);
                const float da = dot4(g[u], m[u]), dc = dot4(g[u], k.v);
                const float r = dc - k.alpha * da;
                dk = k.beta * r;
                dal = __fmaf_rn(1.0f - cw, da, dal);
                dbe = __fmaf_rn(kw[u], r, dbe);
                dv.x = __fmaf_rn(cw, g[u].x, dv.x);
                dv.y = __fmaf_rn(cw, g[u].y, dv.y);
                dv.z = __fmaf_rn(cw, g[u].z, dv.z);
                dv.w = __fmaf_rn(cw, g[u].w, dv.w);
                Gs[s[u]] = make_float4(aw * g[u].x, aw * g[u].y, aw * g[u].z, aw * g[u].w);
                Ms[s[u]] = m[u];
              }
              prt[e] = dk;
            }
          }
          // Warp sums of dv (4 values), dalpha and dbeta: value j ends in lane 4 j.
          const float sum = warp_sum8_transposed(dv.x, dv.y, dv.z, dv.w, dal, dbe, 0.0f, 0.0f, lane);
          if ((lane & 3) == 0) {
            const int j = lane >> 2;
            if (j < 4) a.dv[th * a.d_v + col0 + j] = sum;
            else if (j < 6) prt[a.W + a.R + (j - 4)] = sum;
          }
        });
  }
  __syncwarp();
  for (int row = lane; row < N; row += kWarp) *reinterpret_cast<float4*>(Gout + static_cast<int64_t>(row) * a.d_v) = Gs[row];
}

// Sums the per-tile partials in tile order: dw_w, dw_r [B,T,H,W|R], dalpha,
// dbeta [B,T,H]. One thread per output value.
__global__ void __launch_bounds__(256) k_scan_backward_reduce(const float* __restrict__ part, int64_t n_th, int W,
                                                              int R, int ntile, float* __restrict__ dw_w,
                                                              float* __restrict__ dw_r, float* __restrict__ dalpha,
                                                              float* __restrict__ dbeta) {
  const int PW = W + R + 2;
  const int64_t total = n_th * PW;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t th = x / PW;
    const int e = static_cast<int>(x % PW);
    const float* p = part + th * ntile * PW + e;
    float s = 0.0f;
    for (int k = 0; k < ntile; ++k) s += p[static_cast<int64_t>(k) * PW];
    if (e < W) dw_w[th * W + e] = s;
    else if (e < W + R) dw_r[th * R + (e - W)] = s;
    else if (e == W + R) dalpha[th] = s;
    else dbeta[th] = s;
  }
}

// Derivative of the softmax weights of one selection with respect to its
// scores (SDM explainer 3.1 step 1; the weights are the softmax of the K
// selected sums sigma_k = s1[a_k] + s2[b_k], slot = a * sqrt_n + b):
//   dsigma_k = w_k (dw_k - sum_j w_j dw_j);  ds1[a] += dsigma_k;  ds2[b] += dsigma_k.
// One warp per token-head; each lane owns score entries x = lane, lane + 32, ...
// of the 2 sqrt_n row and sums its contributions over k in order
// (deterministic). dscores rows are written whole (zeros where unused).
__global__ void __launch_bounds__(256) k_pkm_topk_backward(const int32_t* __restrict__ idx,
                                                           const float* __restrict__ w,
                                                           const float* __restrict__ dw, int64_t n_units,
                                                           int sqrt_n, int K, float* __restrict__ dscores,
                                                           unsigned* err) {
  extern __shared__ float pk[];  // per warp: dsigma[K] | a[K] | b[K]
  const int wib = threadIdx.x / kWarp, lane = lane_id();
  float* dsig = pk + wib * 3 * K;
  int* ra = reinterpret_cast<int*>(dsig + K);
  int* rb = ra + K;
  const int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + wib;
  if (u >= n_units) return;
  const int N = sqrt_n * sqrt_n;
  float mean = 0.0f;
  for (int k = lane; k < K; k += kWarp) mean = __fmaf_rn(w[u * K + k], dw[u * K + k], mean);
  mean = warp_sum(mean);
  for (int k = lane; k < K; k += kWarp) {
    const int s = idx[u * K + k];
    const bool ok = s >= 0 && s < N;
    if (!ok) atomicOr(err, kErrIndexOutOfRange);
    dsig[k] = ok ? w[u * K + k] * (dw[u * K + k] - mean) : 0.0f;
    ra[k] = ok ? s / sqrt_n : -1;
    rb[k] = ok ? s % sqrt_n : -1;
  }
  __syncwarp();
  float* out = dscores + u * 2 * sqrt_n;
  for (int x = lane; x < 2 * sqrt_n; x += kWarp) {
    const int* key = x < sqrt_n ? ra : rb;
    const int want = x < sqrt_n ? x : x - sqrt_n;
    float acc = 0.0f;
    for (int k = 0; k < K; ++k)
      if (key[k] == want) acc += dsig[k];
    out[x] = acc;
  }
}

}  // namespace sdm
