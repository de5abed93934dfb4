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
// per-token scalars, so one CTA carries one column tile of one (b, h) with its
// state M and adjoint G: 4 columns in shared memory, shared by two warps that
// split each token's entries, or, for states too large for shared memory,
// 32 columns in global memory with one warp. Memory-efficient by
// recomputation: a first forward pass stores the tile every C tokens
// (checkpoints); then, chunk by chunk from the end, the CTA reloads the
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
  int ntile;  // d_v / (4 U)
  RecLayout rl;
  const uint32_t* rec;  // [B, H, T, rl.words] per-token records (slots, weights, alpha, beta; no hazard plan)
  const void* v;        // [B, T, H, d_v] Tin
  const float* M_in;  // rows of (b, h) at M_in + b * M_in_b_stride + h * N * d_v
  int64_t M_in_b_stride;
  const float* dy;  // [B, T, H, d_v]
  float* dM;        // [B, H, N, d_v] in: dL/dM_T, out: dL/dM_0
  float* dv;        // [B, T, H, d_v]
  float* part;      // [B, T, H, ntile, W + R + 2] per-tile partial sums
  float* ckpt;      // per tile: (ceil(T / C) - 1) * N * 4 U
  const float* ckpt_ext;  // or the forward's checkpoints: [ceil(T / C) - 1][B, H, N, d_v] (then no pass 1)
  float* logbuf;    // per tile: C * W * 4 U
  float* Mwork;     // [B, H, N, d_v] working state when the tiles live in global memory
  unsigned* err;
};

// 8-byte global -> shared asynchronous copy (generic proxy); both addresses
// 8-byte aligned.
__device__ __forceinline__ void cp_async8(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}

// Tile geometry: a warp owns 4 U columns of one (b, h); lane l handles entries
// l and l + 32 of a token and walks the U 16-byte units of each entry's row
// segment, so the sums over the tile's columns stay inside the lane. U = 1
// keeps the state and adjoint tiles in shared memory (16 bytes per slot);
// U = 8 (or 4) keeps them in global memory, where a lane's row segment is a
// whole 128-byte line and wide tiles keep the per-tile partial sums few.
constexpr int kBwdStages = 4;

struct BwdStage {
  int log, rec, v, vf, dy, words;  // word offsets and the stage size (all multiples of 4)
};
// log [W][4U] f32 | rec [words] | v [4U] Tin (raw) | vf [4U] f32 | dy [4U] f32
__host__ __device__ inline BwdStage bwd_stage(int W, int rec_words, int U, int in_bytes) {
  BwdStage st;
  st.log = 0;
  st.rec = W * 4 * U;
  st.v = st.rec + rec_words;
  st.vf = st.v + ((U * in_bytes + 3) & ~3);
  st.dy = st.vf + 4 * U;
  st.words = st.dy + 4 * U;
  return st;
}

// Per-token view of a filled stage.
struct BwdTok {
  const float4* log;  // row e of the log at log[e * U]
  const uint32_t* rec;
  const float4* v;    // U units of v_t (fp32; U > 1)
  float4 v0;          // v_t itself when U = 1
  const float4* dy;   // U units of dy_t
  float alpha, beta;
};

// Sums V values (V = 8 or 32) over the warp with V - 1 + log2(32 / V)
// shuffles (reduce-scatter: each exchange sends the half of the values the
// partner keeps). Value j ends in lanes j * (32 / V) .. j * (32 / V) + 32 / V - 1.
// The order of the additions is fixed, so the sums are reproducible.
// One reduce-scatter step: lanes with bit o set keep the upper half of the
// n values and receive their partner's upper half; the others the lower.
template <int n>
__device__ __forceinline__ void halve_exchange(float* x, int o, int lane) {
  const bool hi = (lane & o) != 0;
#pragma unroll
  for (int j = 0; j < n / 2; ++j) {
    const float keep = hi ? x[j + n / 2] : x[j];
    const float send = hi ? x[j] : x[j + n / 2];
    x[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}
template <int V>
__device__ __forceinline__ float warp_sum_transposed(float (&x)[V], int lane) {
  static_assert(V == 8 || V == 32, "8 or 32 values");
  if constexpr (V == 32) {
    halve_exchange<32>(x, 16, lane);
    halve_exchange<16>(x, 8, lane);
    halve_exchange<8>(x, 4, lane);
    halve_exchange<4>(x, 2, lane);
    halve_exchange<2>(x, 1, lane);
  } else {
    halve_exchange<8>(x, 16, lane);
    halve_exchange<4>(x, 8, lane);
    halve_exchange<2>(x, 4, lane);
    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 2);
    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 1);
  }
  return x[0];
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return __fmaf_rn(a.w, b.w, __fmaf_rn(a.z, b.z, __fmaf_rn(a.y, b.y, a.x * b.x)));
}

// The NWB warps that share one tile meet here (memory ordering included).
template <int NWB>
__device__ __forceinline__ void tile_sync() {
  if constexpr (NWB == 1) __syncwarp();
  else asm volatile("bar.sync 1, %0;\n" ::"n"(NWB * kWarp) : "memory");
}

// Runs body(t, token) over n tokens t = t_first + i * step of one (b, h) and
// column tile, each with its stage filled (log rows from log_src when given,
// dy when with_dy).
template <typename Tin, int U, int NWB, class Body>
__device__ __forceinline__ void bwd_token_pass(const BwdArgs& a, int b, int h, int tile, int tid, int t_first,
                                               int step, int n, float* ring, const float* log_src, int log_t0,
                                               bool with_dy, Body body) {
  const BwdStage L = bwd_stage(a.W, a.rl.words, U, static_cast<int>(sizeof(Tin)));
  const int n_log = log_src != nullptr ? a.W * U : 0;  // 16-byte pieces
  const int n_rec = a.rl.words / 4;
  constexpr int kVBytes = 4 * U * static_cast<int>(sizeof(Tin));
  const int bh = b * a.H + h;
  auto issue = [&](int i) {
    if (i < n) {
      const int t = t_first + i * step;
      const int64_t th = (static_cast<int64_t>(b) * a.T + t) * a.H + h;
      float* st = ring + (i % kBwdStages) * L.words;
      const uint32_t* rsrc = a.rec + (static_cast<int64_t>(bh) * a.T + t) * a.rl.words;
      constexpr int NT = NWB * kWarp;
      for (int x = tid; x < n_rec; x += NT) cp_async16(st + L.rec + 4 * x, rsrc + 4 * x);
      if (n_log > 0) {
        const float* lsrc = log_src + static_cast<int64_t>(t - log_t0) * a.W * 4 * U;
        for (int x = tid; x < n_log; x += NT) cp_async16(st + L.log + 4 * x, lsrc + 4 * x);
      }
      const char* vsrc = reinterpret_cast<const char*>(static_cast<const Tin*>(a.v) + th * a.d_v + tile * 4 * U);
      if constexpr (kVBytes >= 16) {
        for (int x = tid; x < kVBytes / 16; x += NT)
          cp_async16(reinterpret_cast<char*>(st + L.v) + 16 * x, vsrc + 16 * x);
      } else {
        if (tid == NT - 1) cp_async8(st + L.v, vsrc);
      }
      if (with_dy) {
        const float* dsrc = a.dy + th * a.d_v + tile * 4 * U;
        for (int x = tid; x < U; x += NT) cp_async16(st + L.dy + 4 * x, dsrc + 4 * x);
      }
    }
    cp_async_commit();  // empty groups past the end keep the count uniform
  };
#pragma unroll
  for (int i = 0; i < kBwdStages - 1; ++i) issue(i);
  for (int i = 0; i < n; ++i) {
    issue(i + kBwdStages - 1);
    cp_async_wait<kBwdStages - 1>();
    tile_sync<NWB>();
    float* st = ring + (i % kBwdStages) * L.words;
    if constexpr (U > 1) {  // v widened to fp32 once per token in shared memory
      if (tid < 4 * U) st[L.vf + tid] = to_f32<Tin>(reinterpret_cast<const Tin*>(st + L.v)[tid]);
      tile_sync<NWB>();
    }
    BwdTok k;
    k.log = reinterpret_cast<const float4*>(st + L.log);
    k.rec = reinterpret_cast<const uint32_t*>(st + L.rec);
    k.v = reinterpret_cast<const float4*>(st + L.vf);
    if constexpr (U == 1) {  // one unit: widened straight into registers
      const Tin* vv = reinterpret_cast<const Tin*>(st + L.v);
      k.v0 = make_float4(to_f32<Tin>(vv[0]), to_f32<Tin>(vv[1]), to_f32<Tin>(vv[2]), to_f32<Tin>(vv[3]));
    }
    k.dy = reinterpret_cast<const float4*>(st + L.dy);
    k.alpha = __uint_as_float(k.rec[a.rl.off_ab]);
    k.beta = __uint_as_float(k.rec[a.rl.off_ab + 1]);
    body(t_first + i * step, k);
    tile_sync<NWB>();
  }
  cp_async_wait<0>();
  tile_sync<NWB>();
}

// The rows of one tile: in shared memory (stride 4 U floats) or in a global
// [N, d_v] array (stride d_v); row(s)[u] is unit u of slot s.
struct BwdRows {
  float* base;
  int64_t stride;
  __device__ __forceinline__ float4* row(int s) const { return reinterpret_cast<float4*>(base + s * stride); }
};

// The forward write of one token on the tile (the forward kernels' exact fp32
// operations: m <- fma(alpha (1 - beta k), m, (beta k) v)). With `log`, the
// overwritten units are kept at log[e * U + u].
template <int U, int NWB>
__device__ __forceinline__ void bwd_forward_token(const BwdArgs& a, const BwdTok& k, const BwdRows& Ms, float4* log,
                                                  int tid) {
  constexpr int UNR = U == 1 && NWB == 1 ? 2 : 1;  // entries per lane in flight together
  constexpr int NT = NWB * kWarp;
  const int32_t* slot = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_w);
  const float* ww = reinterpret_cast<const float*>(k.rec + a.rl.off_k_w);
  for (int e0 = tid; e0 < a.W; e0 += NT * UNR) {
    int s[UNR];
    float4 m[UNR][U];
    float aw[UNR], cw[UNR];
#pragma unroll
    for (int q = 0; q < UNR; ++q) {
      const int e = e0 + q * NT;
      s[q] = e < a.W ? slot[e] : -1;
      cw[q] = s[q] >= 0 ? k.beta * ww[e] : 0.0f;
      aw[q] = k.alpha * (1.0f - cw[q]);
#pragma unroll
      for (int u = 0; u < U; ++u) m[q][u] = s[q] >= 0 ? Ms.row(s[q])[u] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < UNR; ++q) {
      if (s[q] < 0) continue;
      const int e = e0 + q * NT;
      float4* r = Ms.row(s[q]);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float4 vv = U == 1 ? k.v0 : k.v[u];
        if (log != nullptr) log[e * U + u] = m[q][u];
        r[u] = make_float4(__fmaf_rn(aw[q], m[q][u].x, __fmul_rn(cw[q], vv.x)),
                           __fmaf_rn(aw[q], m[q][u].y, __fmul_rn(cw[q], vv.y)),
                           __fmaf_rn(aw[q], m[q][u].z, __fmul_rn(cw[q], vv.z)),
                           __fmaf_rn(aw[q], m[q][u].w, __fmul_rn(cw[q], vv.w)));
      }
    }
  }
}

// kGlobal: the state and adjoint tiles live in global memory (a working copy
// of the state in a.Mwork and dL/dM in place in a.dM) instead of shared
// memory, for states too large to keep on chip; everything else is the same.
// NWB warps share one tile (NWB = 2 only with shared-memory tiles): each
// takes every NWB-th group of 32 entries of a token, and they meet at named
// barriers between the phases of a token.
template <typename Tin, int U, bool kGlobal, int NWB>
__global__ void __launch_bounds__(NWB * 32) k_scan_backward(BwdArgs a) {
  static_assert(NWB == 1 || (U == 1 && !kGlobal), "two warps per tile only for shared-memory tiles");
  extern __shared__ __align__(16) float bsm[];
  __shared__ float red[8];  // the second warp's sums of dv, dalpha, dbeta
  constexpr int UNR = U == 1 && NWB == 1 ? 2 : 1;
  constexpr int NT = NWB * kWarp;
  const int N = a.N;
  const int tid = threadIdx.x;
  const int lane = tid % kWarp, wid = tid / kWarp;
  const int tile = blockIdx.x % a.ntile;
  const int bh = blockIdx.x / a.ntile;
  const int b = bh / a.H, h = bh % a.H;
  const int col0 = tile * 4 * U;
  const int64_t tile_id = blockIdx.x;
  const int nC = (a.T + a.C - 1) / a.C;
  float4* ckpt = reinterpret_cast<float4*>(a.ckpt) + tile_id * static_cast<int64_t>(nC > 1 ? nC - 1 : 0) * N * U;
  float4* logb = reinterpret_cast<float4*>(a.logbuf) + tile_id * static_cast<int64_t>(a.C) * a.W * U;
  const float* Min = a.M_in + b * a.M_in_b_stride + static_cast<int64_t>(h) * N * a.d_v + col0;
  float* Gout = a.dM + (static_cast<int64_t>(b) * a.H + h) * N * a.d_v + col0;
  BwdRows Ms, Gs;
  float* ring;
  if constexpr (kGlobal) {
    Ms = BwdRows{a.Mwork + (static_cast<int64_t>(b) * a.H + h) * N * a.d_v + col0, a.d_v};
    Gs = BwdRows{Gout, a.d_v};
    ring = bsm;
  } else {
    Ms = BwdRows{bsm, 4 * U};
    Gs = BwdRows{bsm + static_cast<size_t>(N) * 4 * U, 4 * U};
    ring = bsm + 2 * static_cast<size_t>(N) * 4 * U;
  }
  // Tile-wide copies, one 16-byte unit per lane and step.
  auto copy_in = [&](const BwdRows& dst, const float* src, int64_t src_stride) {
    for (int x = tid; x < N * U; x += NT) {
      const int row = x / U, u = x % U;
      dst.row(row)[u] = reinterpret_cast<const float4*>(src + row * src_stride)[u];
    }
  };

  // --------------------------------------------- pass 1: checkpoints --
  // (only when the sequence has more than one chunk)
  copy_in(Ms, Min, a.d_v);
  tile_sync<NWB>();
  if (nC > 1 && a.ckpt_ext == nullptr)
    bwd_token_pass<Tin, U, NWB>(a, b, h, tile, tid, 0, 1, a.T, ring, nullptr, 0, false, [&](int t, const BwdTok& k) {
      if (t > 0 && t % a.C == 0) {
        float4* dst = ckpt + static_cast<int64_t>(t / a.C - 1) * N * U;
        for (int x = tid; x < N * U; x += NT) dst[x] = Ms.row(x / U)[x % U];
      }
      bwd_forward_token<U, NWB>(a, k, Ms, nullptr, tid);
    });

  // ---------------------------------- pass 2: chunks from the end --
  if constexpr (!kGlobal) copy_in(Gs, Gout, a.d_v);
  const int PW = a.W + a.R + 2;
  for (int kc = nC - 1; kc >= 0; --kc) {
    const int t0 = kc * a.C, t1 = min(a.T, t0 + a.C);
    // State at the chunk start.
    if (kc == 0) {
      copy_in(Ms, Min, a.d_v);
    } else if (a.ckpt_ext != nullptr) {
      copy_in(Ms, a.ckpt_ext + (static_cast<int64_t>(kc - 1) * a.B * a.H + bh) * N * a.d_v + col0, a.d_v);
    } else {
      const float* src = reinterpret_cast<const float*>(ckpt + static_cast<int64_t>(kc - 1) * N * U);
      copy_in(Ms, src, 4 * U);
    }
    tile_sync<NWB>();
    // Recompute the chunk forward, logging overwritten units.
    bwd_token_pass<Tin, U, NWB>(a, b, h, tile, tid, t0, 1, t1 - t0, ring, nullptr, 0, false,
                                [&](int t, const BwdTok& k) {
                                  bwd_forward_token<U, NWB>(a, k, Ms, logb + static_cast<int64_t>(t - t0) * a.W * U,
                                                            tid);
                                });
    // The log rows were written by other threads; the reverse pass reads them
    // back through cp.async.
    __threadfence_block();
    tile_sync<NWB>();
    // Backward sweep over the chunk.
    bwd_token_pass<Tin, U, NWB>(
        a, b, h, tile, tid, t1 - 1, -1, t1 - t0, ring, reinterpret_cast<const float*>(logb), t0, true,
        [&](int t, const BwdTok& k) {
          const int64_t th = (static_cast<int64_t>(b) * a.T + t) * a.H + h;
          const int32_t* sw_ = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_w);
          const float* ww = reinterpret_cast<const float*>(k.rec + a.rl.off_k_w);
          const int32_t* ir = reinterpret_cast<const int32_t*>(k.rec + a.rl.off_slot_r);
          const float* wr = reinterpret_cast<const float*>(k.rec + a.rl.off_q_r);
          float* prt = a.part + (th * a.ntile + tile) * PW;
          // Read of token t (state after its write): dq and the adjoint.
          for (int e0 = tid; e0 < a.R; e0 += NT * UNR) {
            int s[UNR];
            float q[UNR];
            float4 m[UNR][U], g[UNR][U];
#pragma unroll
            for (int qq = 0; qq < UNR; ++qq) {
              const int e = e0 + qq * NT;
              s[qq] = e < a.R ? ir[e] : -1;
              q[qq] = s[qq] >= 0 ? wr[e] : 0.0f;
#pragma unroll
              for (int u = 0; u < U; ++u) {
                m[qq][u] = s[qq] >= 0 ? Ms.row(s[qq])[u] : make_float4(0.f, 0.f, 0.f, 0.f);
                g[qq][u] = s[qq] >= 0 ? Gs.row(s[qq])[u] : make_float4(0.f, 0.f, 0.f, 0.f);
              }
            }
#pragma unroll
            for (int qq = 0; qq < UNR; ++qq) {
              const int e = e0 + qq * NT;
              if (e >= a.R) continue;
              float p = 0.0f;
              if (s[qq] >= 0) {
                float4* gr = Gs.row(s[qq]);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                  const float4 d = k.dy[u];
                  p += dot4(d, m[qq][u]);
                  gr[u] = make_float4(__fmaf_rn(q[qq], d.x, g[qq][u].x), __fmaf_rn(q[qq], d.y, g[qq][u].y),
                                      __fmaf_rn(q[qq], d.z, g[qq][u].z), __fmaf_rn(q[qq], d.w, g[qq][u].w));
                }
              }
              prt[a.W + e] = p;
            }
          }
          tile_sync<NWB>();
          // Write of token t, undone: derivatives, adjoint decay, state restore.
          float4 dv[U];
#pragma unroll
          for (int u = 0; u < U; ++u) dv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          float dal = 0.0f, dbe = 0.0f;
          for (int e0 = tid; e0 < a.W; e0 += NT * UNR) {
            int s[UNR];
            float kw[UNR];
            float4 g[UNR][U], m[UNR][U];
#pragma unroll
            for (int qq = 0; qq < UNR; ++qq) {
              const int e = e0 + qq * NT;
              s[qq] = e < a.W ? sw_[e] : -1;
              kw[qq] = s[qq] >= 0 ? ww[e] : 0.0f;
#pragma unroll
              for (int u = 0; u < U; ++u) {
                g[qq][u] = s[qq] >= 0 ? Gs.row(s[qq])[u] : make_float4(0.f, 0.f, 0.f, 0.f);
                m[qq][u] = s[qq] >= 0 ? k.log[e * U + u] : make_float4(0.f, 0.f, 0.f, 0.f);
              }
            }
#pragma unroll
            for (int qq = 0; qq < UNR; ++qq) {
              const int e = e0 + qq * NT;
              if (e >= a.W) continue;
              float dk = 0.0f;
              if (s[qq] >= 0) {
                const float cw = k.beta * kw[qq];
                const float aw = k.alpha * (1.0f - cw);
                float da = 0.0f, dc = 0.0f;
                float4* gr = Gs.row(s[qq]);
                float4* mr = Ms.row(s[qq]);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                  const float4 gg = g[qq][u];
                  da += dot4(gg, m[qq][u]);
                  dc += dot4(gg, U == 1 ? k.v0 : k.v[u]);
                  dv[u].x = __fmaf_rn(cw, gg.x, dv[u].x);
                  dv[u].y = __fmaf_rn(cw, gg.y, dv[u].y);
                  dv[u].z = __fmaf_rn(cw, gg.z, dv[u].z);
                  dv[u].w = __fmaf_rn(cw, gg.w, dv[u].w);
                  gr[u] = make_float4(aw * gg.x, aw * gg.y, aw * gg.z, aw * gg.w);
                  mr[u] = m[qq][u];
                }
                const float r = dc - k.alpha * da;
                dk = k.beta * r;
                dal = __fmaf_rn(1.0f - cw, da, dal);
                dbe = __fmaf_rn(kw[qq], r, dbe);
              }
              prt[e] = dk;
            }
          }
          // Warp sums of dv (4 U values), dalpha and dbeta.
          if constexpr (U == 1) {
            float x[8] = {dv[0].x, dv[0].y, dv[0].z, dv[0].w, dal, dbe, 0.0f, 0.0f};
            float sum = warp_sum_transposed<8>(x, lane);  // value j in lanes 4j .. 4j+3
            const int j = lane >> 2;
            if constexpr (NWB == 2) {  // the second warp hands its sums to the first
              if (wid == 1 && (lane & 3) == 0 && j < 6) red[j] = sum;
              tile_sync<NWB>();
              if ((lane & 3) == 0 && j < 6) sum += red[j];
            }
            if (wid == 0 && (lane & 3) == 0) {
              if (j < 4) a.dv[th * a.d_v + col0 + j] = sum;
              else if (j < 6) prt[a.W + a.R + (j - 4)] = sum;
            }
          } else {
            float x[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              x[4 * u] = u < U ? dv[u < U ? u : 0].x : 0.0f;
              x[4 * u + 1] = u < U ? dv[u < U ? u : 0].y : 0.0f;
              x[4 * u + 2] = u < U ? dv[u < U ? u : 0].z : 0.0f;
              x[4 * u + 3] = u < U ? dv[u < U ? u : 0].w : 0.0f;
            }
            if constexpr (U < 8) {  // spare slots carry dalpha and dbeta
              x[4 * U] = dal;
              x[4 * U + 1] = dbe;
            }
            const float sum = warp_sum_transposed<32>(x, lane);  // value j in lane j
            if (lane < 4 * U) a.dv[th * a.d_v + col0 + lane] = sum;
            if constexpr (U < 8) {
              if (lane == 4 * U || lane == 4 * U + 1) prt[a.W + a.R + (lane - 4 * U)] = sum;
            } else {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                dal += __shfl_xor_sync(0xffffffffu, dal, o);
                dbe += __shfl_xor_sync(0xffffffffu, dbe, o);
              }
              if (lane == 0) {
                prt[a.W + a.R] = dal;
                prt[a.W + a.R + 1] = dbe;
              }
            }
          }
        });
  }
  tile_sync<NWB>();
  if constexpr (!kGlobal) {
    for (int x = tid; x < N * U; x += NT)
      reinterpret_cast<float4*>(Gout + static_cast<int64_t>(x / U) * a.d_v)[x % U] = Gs.row(x / U)[x % U];
  }
}

// Sums the per-tile partials in tile order: dw_w, dw_r [B,T,H,W|R], dalpha,
// dbeta [B,T,H]. One thread per output value.
static __global__ void __launch_bounds__(256) k_scan_backward_reduce(const float* __restrict__ part, int64_t n_th, int W,
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
static __global__ void __launch_bounds__(256) k_pkm_topk_backward(const int32_t* __restrict__ idx,
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
