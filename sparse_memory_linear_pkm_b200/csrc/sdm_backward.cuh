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
// per-token scalars, so one warp carries one CW-column tile of one (b, h) with
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

namespace sdm {

struct BwdArgs {
  int B, T, H, N, d_v, W, R;
  int C;      // tokens per checkpoint chunk
  int ntile;  // d_v / CW
  const int32_t* idx_w;
  const float* w_w;
  const int32_t* idx_r;
  const float* w_r;
  const void* v;      // [B, T, H, d_v] Tin
  const void* alpha;  // [B, T, H] Tin
  const void* beta;   // [B, T, H] Tin
  const float* M_in;  // rows of (b, h) at M_in + b * M_in_b_stride + h * N * d_v
  int64_t M_in_b_stride;
  const float* dy;  // [B, T, H, d_v]
  float* dM;        // [B, H, N, d_v] in: dL/dM_T, out: dL/dM_0
  float* dv;        // [B, T, H, d_v]
  float* part;      // [B, T, H, ntile, W + R + 2] per-tile partial sums
  float* ckpt;      // per tile: (ceil(T / C) - 1) * N * CW
  float* logbuf;    // per tile: C * W * CW
  unsigned* err;
};

// 4-byte global -> shared asynchronous copy (generic proxy).
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}

// Per-token selection metadata staged in shared memory:
// idx_w[W] | w_w[W] | idx_r[R] | w_r[R] (32-bit words).
__device__ __forceinline__ void stage_token_meta(const BwdArgs& a, int64_t th, int32_t* buf, int lane) {
  for (int x = lane; x < a.W; x += kWarp) {
    cp_async4(buf + x, a.idx_w + th * a.W + x);
    cp_async4(buf + a.W + x, a.w_w + th * a.W + x);
  }
  int32_t* r = buf + 2 * a.W;
  for (int x = lane; x < a.R; x += kWarp) {
    cp_async4(r + x, a.idx_r + th * a.R + x);
    cp_async4(r + a.R + x, a.w_r + th * a.R + x);
  }
  cp_async_commit();
}

// Per-lane token scalars: alpha, beta and this lane's column of v and dy.
struct BwdTok {
  float alpha, beta, v, dy;
};

template <typename Tin>
__device__ __forceinline__ BwdTok load_token(const BwdArgs& a, int64_t th, int col, bool with_dy) {
  BwdTok k;
  k.alpha = to_f32<Tin>(static_cast<const Tin*>(a.alpha)[th]);
  k.beta = to_f32<Tin>(static_cast<const Tin*>(a.beta)[th]);
  k.v = to_f32<Tin>(static_cast<const Tin*>(a.v)[th * a.d_v + col]);
  k.dy = with_dy ? a.dy[th * a.d_v + col] : 0.0f;
  return k;
}

// The forward write of one token on the tile (the forward kernels' exact fp32
// operations). With `log`, the overwritten values are kept at log[e * CW + c].
template <int CW>
__device__ __forceinline__ void bwd_forward_token(const BwdArgs& a, const int32_t* meta, const BwdTok& k, float* Ms,
                                                  float* log, int e4, int c) {
  constexpr int EPG = kWarp / CW;
  const float* ww = reinterpret_cast<const float*>(meta + a.W);
  for (int e0 = 0; e0 < a.W; e0 += EPG) {
    const int e = e0 + e4;
    if (e < a.W) {
      const int s = meta[e];
      if (static_cast<unsigned>(s) < static_cast<unsigned>(a.N)) {
        const float cw = k.beta * ww[e];
        const float aw = k.alpha * (1.0f - cw);
        const float m = Ms[s * CW + c];
        if (log != nullptr) log[e * CW + c] = m;
        Ms[s * CW + c] = __fmaf_rn(aw, m, __fmul_rn(cw, k.v));
      }
    }
  }
}

template <typename Tin, int CW>
__global__ void __launch_bounds__(32) k_scan_backward(BwdArgs a) {
  constexpr int EPG = kWarp / CW;
  extern __shared__ __align__(16) float bsm[];
  const int N = a.N;
  float* Ms = bsm;                                         // [N][CW] state tile
  float* Gs = bsm + static_cast<size_t>(N) * CW;           // [N][CW] adjoint tile
  int32_t* meta0 = reinterpret_cast<int32_t*>(Gs + static_cast<size_t>(N) * CW);
  const int meta_words = 2 * (a.W + a.R);
  auto metab = [&](int i) { return meta0 + i * meta_words; };  // two staging buffers

  const int lane = threadIdx.x;
  const int e4 = lane / CW, c = lane % CW;
  const int tile = blockIdx.x % a.ntile;
  const int bh = blockIdx.x / a.ntile;
  const int b = bh / a.H, h = bh % a.H;
  const int col = tile * CW + c;
  const int64_t tile_id = blockIdx.x;
  const int nC = (a.T + a.C - 1) / a.C;
  float* ckpt = a.ckpt + tile_id * static_cast<int64_t>(nC > 1 ? nC - 1 : 0) * N * CW;
  float* logb = a.logbuf + tile_id * static_cast<int64_t>(a.C) * a.W * CW;
  const float* Min = a.M_in + b * a.M_in_b_stride + static_cast<int64_t>(h) * N * a.d_v;
  auto th_of = [&](int t) { return (static_cast<int64_t>(b) * a.T + t) * a.H + h; };

  // --------------------------------------------- pass 1: checkpoints --
  for (int row = e4; row < N; row += EPG) Ms[row * CW + c] = Min[static_cast<int64_t>(row) * a.d_v + col];
  __syncwarp();
  if (a.T > 0) stage_token_meta(a, th_of(0), metab(0), lane);
  BwdTok nxt = a.T > 0 ? load_token<Tin>(a, th_of(0), col, false) : BwdTok{};
  for (int t = 0; t < a.T; ++t) {
    if (t > 0 && t % a.C == 0) {
      float* dst = ckpt + static_cast<int64_t>(t / a.C - 1) * N * CW;
      for (int row = e4; row < N; row += EPG) dst[row * CW + c] = Ms[row * CW + c];
    }
    const BwdTok cur = nxt;
    if (t + 1 < a.T) {
      stage_token_meta(a, th_of(t + 1), metab((t + 1) & 1), lane);
      nxt = load_token<Tin>(a, th_of(t + 1), col, false);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const int32_t* meta = metab(t & 1);
    if (c == 0) {  // out-of-range slots are skipped everywhere and flagged here, once
      for (int e = e4; e < a.W; e += EPG)
        if (static_cast<unsigned>(meta[e]) >= static_cast<unsigned>(N)) atomicOr(a.err, kErrIndexOutOfRange);
      for (int e = e4; e < a.R; e += EPG)
        if (static_cast<unsigned>(meta[2 * a.W + e]) >= static_cast<unsigned>(N)) atomicOr(a.err, kErrIndexOutOfRange);
    }
    bwd_forward_token<CW>(a, meta, cur, Ms, nullptr, e4, c);
    __syncwarp();
  }

  // ---------------------------------- pass 2: chunks from the end --
  float* Gout = a.dM + (static_cast<int64_t>(b) * a.H + h) * N * a.d_v;
  for (int row = e4; row < N; row += EPG) Gs[row * CW + c] = Gout[static_cast<int64_t>(row) * a.d_v + col];
  const int PW = a.W + a.R + 2;
  for (int kc = nC - 1; kc >= 0; --kc) {
    const int t0 = kc * a.C, t1 = min(a.T, t0 + a.C);
    // State at the chunk start.
    __syncwarp();
    if (kc == 0) {
      for (int row = e4; row < N; row += EPG) Ms[row * CW + c] = Min[static_cast<int64_t>(row) * a.d_v + col];
    } else {
      const float* src = ckpt + static_cast<int64_t>(kc - 1) * N * CW;
      for (int row = e4; row < N; row += EPG) Ms[row * CW + c] = src[row * CW + c];
    }
    __syncwarp();
    // Recompute the chunk forward, logging overwritten values.
    stage_token_meta(a, th_of(t0), metab(0), lane);
    nxt = load_token<Tin>(a, th_of(t0), col, false);
    for (int t = t0; t < t1; ++t) {
      const BwdTok cur = nxt;
      if (t + 1 < t1) {
        stage_token_meta(a, th_of(t + 1), metab((t + 1 - t0) & 1), lane);
        nxt = load_token<Tin>(a, th_of(t + 1), col, false);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      bwd_forward_token<CW>(a, metab((t - t0) & 1), cur, Ms, logb + static_cast<int64_t>(t - t0) * a.W * CW, e4,
                            c);
      __syncwarp();
    }
    // Backward sweep over the chunk.
    stage_token_meta(a, th_of(t1 - 1), metab(0), lane);
    nxt = load_token<Tin>(a, th_of(t1 - 1), col, true);
    for (int t = t1 - 1; t >= t0; --t) {
      const int64_t th = th_of(t);
      const BwdTok k = nxt;
      const int slot_buf = (t1 - 1 - t) & 1;
      if (t - 1 >= t0) {
        stage_token_meta(a, th_of(t - 1), metab(slot_buf ^ 1), lane);
        nxt = load_token<Tin>(a, th_of(t - 1), col, true);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncwarp();
      const int32_t* meta = metab(slot_buf);
      const float* ww = reinterpret_cast<const float*>(meta + a.W);
      const int32_t* ir = meta + 2 * a.W;
      const float* wr = reinterpret_cast<const float*>(ir + a.R);
      float* prt = a.part + (th * a.ntile + tile) * PW;
      // Read of token t (state after its write): dq and the adjoint.
      for (int e0 = 0; e0 < a.R; e0 += EPG) {
        const int e = e0 + e4;
        const int s = e < a.R ? ir[e] : -1;
        const bool ok = static_cast<unsigned>(s) < static_cast<unsigned>(N);
        float p = ok ? k.dy * Ms[s * CW + c] : 0.0f;
#pragma unroll
        for (int o = 1; o < CW; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if (ok) Gs[s * CW + c] = __fmaf_rn(wr[e], k.dy, Gs[s * CW + c]);
        if (c == 0 && e < a.R) prt[a.W + e] = p;
      }
      __syncwarp();
      // Write of token t, undone: derivatives, adjoint decay, state restore.
      const float* lg = logb + static_cast<int64_t>(t - t0) * a.W * CW;
      float dv_acc = 0.0f, dal = 0.0f, dbe = 0.0f;
      for (int e0 = 0; e0 < a.W; e0 += EPG) {
        const int e = e0 + e4;
        const int s = e < a.W ? meta[e] : -1;
        const bool ok = static_cast<unsigned>(s) < static_cast<unsigned>(N);
        const float kw = ok ? ww[e] : 0.0f;
        const float cw = k.beta * kw;
        const float aw = k.alpha * (1.0f - cw);
        const float g = ok ? Gs[s * CW + c] : 0.0f;
        const float m = ok ? lg[e * CW + c] : 0.0f;
        float da = g * m, dc = g * k.v;
#pragma unroll
        for (int o = 1; o < CW; o <<= 1) {
          da += __shfl_xor_sync(0xffffffffu, da, o);
          dc += __shfl_xor_sync(0xffffffffu, dc, o);
        }
        const float r = dc - k.alpha * da;
        if (c == 0 && e < a.W) prt[e] = k.beta * r;
        dal = __fmaf_rn(1.0f - cw, da, dal);
        dbe = __fmaf_rn(kw, r, dbe);
        dv_acc = __fmaf_rn(cw, g, dv_acc);
        if (ok) {
          Gs[s * CW + c] = aw * g;
          Ms[s * CW + c] = m;
        }
      }
#pragma unroll
      for (int o = CW; o < kWarp; o <<= 1) {
        dv_acc += __shfl_xor_sync(0xffffffffu, dv_acc, o);
        dal += __shfl_xor_sync(0xffffffffu, dal, o);
        dbe += __shfl_xor_sync(0xffffffffu, dbe, o);
      }
      if (e4 == 0) a.dv[th * a.d_v + col] = dv_acc;
      if (lane == 0) {
        prt[a.W + a.R] = dal;
        prt[a.W + a.R + 1] = dbe;
      }
      __syncwarp();
    }
  }
  __syncwarp();
  for (int row = e4; row < N; row += EPG) Gout[static_cast<int64_t>(row) * a.d_v + col] = Gs[row * CW + c];
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
