// The sparse gated delta recurrence (sm_100a).
//
// SDM explainer (papers.ananclaw.com), section 3.1 step 2: for each selected
// write slot i, M~ = alpha_t M[i] and M[i] = M~ + beta_t k_i (v_t - M~); other
// slots keep their value. Step 3: y_t = sum over read slots of q_i M_t[i], on
// the state after the write. (Technical Summary: Sparse Delta Memory, Core
// Mechanism 3-4.) The kernels use the equivalent factored form
// M[i] = (alpha_t (1 - beta_t k_i)) M[i] + (beta_t k_i) v_t in fp32 and round
// to the state dtype on every store.
//
// Every column of d_v evolves independently given the per-token scalars, so a
// CTA owns one (b, h) and a tile of C columns and walks all T tokens. Within a
// token the W writes touch distinct slots and run in parallel, one thread per
// (entry, 16-byte unit); a barrier separates them from the R reads, whose
// partial sums are reduced in a fixed order (bit-reproducible y). Per-token
// records and v rows are staged a chunk of L tokens at a time with 1-D bulk
// copies (no multicast) into a double buffer tracked by mbarriers.
//
//   k_scan_resident  : the (b, h) column tile of the state lives in shared
//                      memory (fp32) for the whole sequence; M_in is read once
//                      and M_out written once. Two barriers per token.
//   k_scan_streaming : the state stays in global memory. The rows of token t+P
//                      are gathered (cp.async, 16 B per thread) while token t
//                      computes, into a ring of 2P stages; the hazard plan in
//                      the record forwards rows written by the tokens in
//                      between from their stage. Written rows are stored back
//                      to global memory at once.
#pragma once

#include "sdm_device.cuh"
#include "sdm_records.cuh"

namespace sdm {

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / kWarp;

struct ScanArgs {
  int B, T, H, N, d_v, W, R;
  RecLayout rl;
  const uint32_t* rec;  // [B, H, T, rl.words]
  const void* v;        // [B, T, H, d_v] in dtype
  const void* M_in;     // resident: initial state rows of (b, h) at M_in + b*M_in_b_stride + h*N*d_v
  int64_t M_in_b_stride;
  void* M;              // [B, H, N, d_v] final state (resident) / state in place (streaming)
  float* y;             // [B, T, H, d_v]
  unsigned* err;
};

// Loads VE consecutive input elements (VE * sizeof(Tin) bytes, aligned) as fp32.
template <typename Tin, int VE>
__device__ __forceinline__ void load_in_vec(const Tin* p, float* out) {
  if constexpr (sizeof(Tin) == 4) {
    static_assert(VE % 4 == 0, "fp32 vectors of 4");
#pragma unroll
    for (int i = 0; i < VE; i += 4) {
      const float4 f = *reinterpret_cast<const float4*>(p + i);
      out[i] = f.x; out[i + 1] = f.y; out[i + 2] = f.z; out[i + 3] = f.w;
    }
  } else {
    static_assert(VE % 4 == 0, "bf16 vectors of 4");
#pragma unroll
    for (int i = 0; i < VE; i += 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p + i);
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
      out[i] = fa.x; out[i + 1] = fa.y; out[i + 2] = fb.x; out[i + 3] = fb.y;
    }
  }
}

// 16 bytes of state elements <-> fp32.
template <typename Tst>
__device__ __forceinline__ void unpack16(const uint4& u, float* out) {
  if constexpr (sizeof(Tst) == 4) {
    out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
  } else {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
}
template <typename Tst>
__device__ __forceinline__ uint4 pack16(const float* in) {
  uint4 u;
  if constexpr (sizeof(Tst) == 4) {
    u.x = __float_as_uint(in[0]); u.y = __float_as_uint(in[1]);
    u.z = __float_as_uint(in[2]); u.w = __float_as_uint(in[3]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
  }
  return u;
}

// Issues the bulk copies of chunk c (records + v rows of up to L tokens) into
// buffer c & 1. Called by one thread.
template <typename Tin, int C, int L>
__device__ __forceinline__ void issue_chunk(const ScanArgs& a, int bh, int b, int h, int c0, int c,
                                            uint32_t* recbuf, Tin* vbuf, uint64_t* bars) {
  const int bi = c & 1;
  const int t0 = c * L;
  const int nt = min(L, a.T - t0);
  const uint32_t rec_bytes = static_cast<uint32_t>(nt) * a.rl.words * 4u;
  const uint32_t v_bytes = C * sizeof(Tin);
  mbar_arrive_expect_tx(&bars[bi], rec_bytes + nt * v_bytes);
  bulk_g2s(recbuf + static_cast<size_t>(bi) * L * a.rl.words,
           a.rec + (static_cast<int64_t>(bh) * a.T + t0) * a.rl.words, rec_bytes, &bars[bi]);
  const Tin* v = static_cast<const Tin*>(a.v);
  for (int i = 0; i < nt; ++i) {
    const Tin* src = v + ((static_cast<int64_t>(b) * a.T + t0 + i) * a.H + h) * a.d_v + c0;
    bulk_g2s(vbuf + (static_cast<size_t>(bi) * L + i) * C, src, v_bytes, &bars[bi]);
  }
}

// ------------------------------------------------------------ resident ----

template <typename Tin, typename Tst, int C, int L>
__global__ void __launch_bounds__(kScanThreads) k_scan_resident(ScanArgs a) {
  constexpr int U = C / 4;  // 16-byte units of an fp32 row segment
  static_assert(kScanThreads % U == 0, "a thread keeps one unit column");
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = a.N, W = a.W, R = a.R, T = a.T;
  const int words = a.rl.words;
  float* S = reinterpret_cast<float*>(smem);  // [N][C]
  uint32_t* recbuf = reinterpret_cast<uint32_t*>(smem + static_cast<size_t>(N) * C * 4);
  Tin* vbuf = reinterpret_cast<Tin*>(recbuf + 2 * L * words);
  float* ypart = reinterpret_cast<float*>(vbuf + 2 * L * C);  // [2][warps][C]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ypart + 2 * kScanWarps * C);

  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int c0 = blockIdx.y * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = tid % U;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  // Initial state tile.
  {
    constexpr int VE = 16 / sizeof(Tst);
    const Tst* Min = static_cast<const Tst*>(a.M_in) + b * a.M_in_b_stride +
                     static_cast<int64_t>(h) * N * a.d_v + c0;
    for (int x = tid; x < N * (C / VE); x += kScanThreads) {
      const int row = x / (C / VE), u = x % (C / VE);
      float f[VE];
      unpack16<Tst>(*reinterpret_cast<const uint4*>(Min + static_cast<int64_t>(row) * a.d_v + u * VE), f);
#pragma unroll
      for (int i = 0; i < VE; ++i) S[row * C + u * VE + i] = f[i];
    }
  }
  __syncthreads();
  const int n_chunks = (T + L - 1) / L;
  if (tid == 0 && n_chunks > 0) {
    issue_chunk<Tin, C, L>(a, bh, b, h, c0, 0, recbuf, vbuf, bars);
    if (n_chunks > 1) issue_chunk<Tin, C, L>(a, bh, b, h, c0, 1, recbuf, vbuf, bars);
  }
  float* y_bh = a.y + static_cast<int64_t>(h) * a.d_v + c0;

  for (int c = 0; c < n_chunks; ++c) {
    const int bi = c & 1;
    const bool ok = mbar_wait_bounded(&bars[bi], (c >> 1) & 1, a.err);
    if (__syncthreads_or(!ok)) return;
    const uint32_t* recs = recbuf + static_cast<size_t>(bi) * L * words;
    const Tin* vs = vbuf + static_cast<size_t>(bi) * L * C;
    const int nt = min(L, T - c * L);
    for (int i = 0; i < nt; ++i) {
      const int t = c * L + i;
      const uint32_t* rec = recs + i * words;
      const float alpha = __uint_as_float(rec[a.rl.off_ab]);
      const float beta = __uint_as_float(rec[a.rl.off_ab + 1]);
      // Write: W distinct slots, one (entry, unit) per thread.
      for (int x = tid; x < W * U; x += kScanThreads) {
        const int e = x / U;
        const int slot = static_cast<int>(rec[a.rl.off_slot_w + e]);
        if (slot < 0) continue;
        const float cw = beta * __uint_as_float(rec[a.rl.off_k_w + e]);
        const float aw = alpha * (1.0f - cw);
        float vv[4];
        load_in_vec<Tin, 4>(vs + i * C + 4 * q, vv);
        float4* p = reinterpret_cast<float4*>(S + slot * C + 4 * q);
        float4 m = *p;
        m.x = round_to<Tst>(fmaf(aw, m.x, cw * vv[0]));
        m.y = round_to<Tst>(fmaf(aw, m.y, cw * vv[1]));
        m.z = round_to<Tst>(fmaf(aw, m.z, cw * vv[2]));
        m.w = round_to<Tst>(fmaf(aw, m.w, cw * vv[3]));
        *p = m;
      }
      __syncthreads();
      // Read after the write.
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int x = tid; x < R * U; x += kScanThreads) {
        const int r = x / U;
        const int slot = static_cast<int>(rec[a.rl.off_slot_r + r]);
        if (slot < 0) continue;
        const float qw = __uint_as_float(rec[a.rl.off_q_r + r]);
        const float4 m = *reinterpret_cast<const float4*>(S + slot * C + 4 * q);
        acc[0] = fmaf(qw, m.x, acc[0]);
        acc[1] = fmaf(qw, m.y, acc[1]);
        acc[2] = fmaf(qw, m.z, acc[2]);
        acc[3] = fmaf(qw, m.w, acc[3]);
      }
#pragma unroll
      for (int o = U; o < kWarp; o <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
      float* yp = ypart + (t & 1) * kScanWarps * C;
      if (lane < U) *reinterpret_cast<float4*>(yp + warp * C + 4 * lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      __syncthreads();
      if (tid < C) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kScanWarps; ++w) s += yp[w * C + tid];
        y_bh[(static_cast<int64_t>(b) * T + t) * a.H * a.d_v + tid] = s;
      }
    }
    // Every thread is past the last read of buffer bi (barrier above).
    if (tid == 0 && c + 2 < n_chunks) {
      fence_proxy_async_smem();
      issue_chunk<Tin, C, L>(a, bh, b, h, c0, c + 2, recbuf, vbuf, bars);
    }
  }
  __syncthreads();
  {
    constexpr int VE = 16 / sizeof(Tst);
    Tst* Mout = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * N * a.d_v + c0;
    for (int x = tid; x < N * (C / VE); x += kScanThreads) {
      const int row = x / (C / VE), u = x % (C / VE);
      *reinterpret_cast<uint4*>(Mout + static_cast<int64_t>(row) * a.d_v + u * VE) =
          pack16<Tst>(S + row * C + u * VE);
    }
  }
}

// ----------------------------------------------------------- streaming ----

template <typename Tin, typename Tst, int C, int P, int L>
__global__ void __launch_bounds__(kScanThreads) k_scan_streaming(ScanArgs a) {
  constexpr int VE = 16 / sizeof(Tst);  // state elements per 16-byte unit
  constexpr int U = C / VE;             // units per row segment
  constexpr int S = 2 * P;              // stage ring
  static_assert(kScanThreads % U == 0, "a thread keeps one unit column");
  static_assert(L > P, "a chunk must be staged before its tokens are gathered");
  extern __shared__ __align__(16) unsigned char smem[];
  const int W = a.W, R = a.R, T = a.T, E = W + R;
  const int words = a.rl.words;
  Tst* stage = reinterpret_cast<Tst*>(smem);  // [S][E][C]
  uint32_t* recbuf = reinterpret_cast<uint32_t*>(smem + static_cast<size_t>(S) * E * C * sizeof(Tst));
  Tin* vbuf = reinterpret_cast<Tin*>(recbuf + 2 * L * words);
  float* ypart = reinterpret_cast<float*>(vbuf + 2 * L * C);  // [2][warps][C]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ypart + 2 * kScanWarps * C);

  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int c0 = blockIdx.y * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = tid % U;
  Tst* Mbh = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * a.N * a.d_v + c0;
  float* y_bh = a.y + static_cast<int64_t>(h) * a.d_v + c0;

  auto rec_of = [&](int t) -> const uint32_t* {
    return recbuf + (static_cast<size_t>((t / L) & 1) * L + (t % L)) * words;
  };
  auto fwd_of = [&](const uint32_t* rec, int e) -> int {
    return reinterpret_cast<const int16_t*>(rec + a.rl.off_fwd)[e];
  };
  auto row_ptr = [&](int t, int e) -> Tst* { return stage + (static_cast<size_t>(t % S) * E + e) * C; };
  // Gathers the rows of token t that the plan does not forward.
  auto gather = [&](int t) {
    const uint32_t* rec = rec_of(t);
    for (int x = tid; x < E * U; x += kScanThreads) {
      const int e = x / U, u = x % U;
      const int slot = static_cast<int>(e < W ? rec[a.rl.off_slot_w + e] : rec[a.rl.off_slot_r + e - W]);
      if (slot >= 0 && fwd_of(rec, e) < 0)
        cp_async16(row_ptr(t, e) + u * VE, Mbh + static_cast<int64_t>(slot) * a.d_v + u * VE);
    }
  };

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_chunks = (T + L - 1) / L;
  if (n_chunks == 0) return;
  if (tid == 0) {
    issue_chunk<Tin, C, L>(a, bh, b, h, c0, 0, recbuf, vbuf, bars);
    if (n_chunks > 1) issue_chunk<Tin, C, L>(a, bh, b, h, c0, 1, recbuf, vbuf, bars);
  }
  {
    const bool ok = mbar_wait_bounded(&bars[0], 0, a.err);
    if (__syncthreads_or(!ok)) return;
  }
#pragma unroll 1
  for (int t = 0; t < P; ++t) {
    if (t < T) gather(t);
    cp_async_commit();
  }

#pragma unroll 1
  for (int t = 0; t < T; ++t) {
    cp_async_wait<P - 1>();
    __syncthreads();  // rows of t landed and visible; reads of t-1 done
    if (t > 0 && t % L == 0 && tid == 0 && t / L + 1 < n_chunks) {
      fence_proxy_async_smem();
      issue_chunk<Tin, C, L>(a, bh, b, h, c0, t / L + 1, recbuf, vbuf, bars);
    }
    if (t > 0 && tid < C) {
      const float* yp = ypart + ((t - 1) & 1) * kScanWarps * C;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kScanWarps; ++w) s += yp[w * C + tid];
      y_bh[(static_cast<int64_t>(b) * T + (t - 1)) * a.H * a.d_v + tid] = s;
    }
    const uint32_t* rec = rec_of(t);
    const Tin* vrow = vbuf + (static_cast<size_t>((t / L) & 1) * L + (t % L)) * C;
    const float alpha = __uint_as_float(rec[a.rl.off_ab]);
    const float beta = __uint_as_float(rec[a.rl.off_ab + 1]);
    // Write.
    for (int x = tid; x < W * U; x += kScanThreads) {
      const int e = x / U;
      const int slot = static_cast<int>(rec[a.rl.off_slot_w + e]);
      if (slot < 0) continue;
      const int f = fwd_of(rec, e);
      const Tst* src = f < 0 ? row_ptr(t, e) : row_ptr(t - (f >> 9), f & 511);
      float m[VE], vv[VE];
      unpack16<Tst>(*reinterpret_cast<const uint4*>(src + q * VE), m);
      load_in_vec<Tin, VE>(vrow + q * VE, vv);
      const float cw = beta * __uint_as_float(rec[a.rl.off_k_w + e]);
      const float aw = alpha * (1.0f - cw);
#pragma unroll
      for (int j = 0; j < VE; ++j) m[j] = fmaf(aw, m[j], cw * vv[j]);
      const uint4 packed = pack16<Tst>(m);
      *reinterpret_cast<uint4*>(row_ptr(t, e) + q * VE) = packed;
      *reinterpret_cast<uint4*>(Mbh + static_cast<int64_t>(slot) * a.d_v + q * VE) = packed;
    }
    __syncthreads();  // writes of t visible to the reads of t
    // Read after the write.
    float acc[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) acc[j] = 0.f;
    for (int x = tid; x < R * U; x += kScanThreads) {
      const int r = x / U;
      const int slot = static_cast<int>(rec[a.rl.off_slot_r + r]);
      if (slot < 0) continue;
      const int f = fwd_of(rec, W + r);
      const Tst* src = f < 0 ? row_ptr(t, W + r) : row_ptr(t - (f >> 9), f & 511);
      float m[VE];
      unpack16<Tst>(*reinterpret_cast<const uint4*>(src + q * VE), m);
      const float qw = __uint_as_float(rec[a.rl.off_q_r + r]);
#pragma unroll
      for (int j = 0; j < VE; ++j) acc[j] = fmaf(qw, m[j], acc[j]);
    }
#pragma unroll
    for (int o = U; o < kWarp; o <<= 1)
#pragma unroll
      for (int j = 0; j < VE; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    if (lane < U) {
      float* yp = ypart + (t & 1) * kScanWarps * C + warp * C + lane * VE;
#pragma unroll
      for (int j = 0; j < VE; ++j) yp[j] = acc[j];
    }
    // Gather token t + P (its chunk must have landed).
    if (t + P < T) {
      if ((t + P) % L == 0) {
        const int c = (t + P) / L;
        const bool ok = mbar_wait_bounded(&bars[c & 1], (c >> 1) & 1, a.err);
        if (__syncthreads_or(!ok)) {
          cp_async_wait<0>();
          return;
        }
      }
      gather(t + P);
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();
  if (T > 0 && tid < C) {
    const float* yp = ypart + ((T - 1) & 1) * kScanWarps * C;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) s += yp[w * C + tid];
    y_bh[(static_cast<int64_t>(b) * T + (T - 1)) * a.H * a.d_v + tid] = s;
  }
}

}  // namespace sdm
