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
// CTA owns one (b, h) and a tile of C columns and walks all T tokens. A row
// segment of the tile is U 16-byte units; lane q%U of a warp handles unit q
// of one entry and a warp instruction covers 32/U entries, so each entry's
// metadata is read once per U lanes and v_t stays in registers for the whole
// token. The W writes of a token touch distinct slots and run in parallel; the
// R reads follow them, and their partial sums are reduced in a fixed order
// (bit-reproducible y). Per-token records and v rows are staged a
// chunk of L tokens at a time by 1-D bulk copies (no multicast) into a double
// buffer tracked by mbarriers with bounded waits.
//
//   k_scan_resident  : the (b, h) column tile of the state lives in shared
//                      memory (fp32) for the whole sequence; M_in is read once
//                      and M_out written once. Each warp carries its own
//                      column tile through the tokens (no barrier per token).
//   k_scan_streaming : the state stays in global memory. The rows of token t+P
//                      are gathered (16-byte cp.async per lane) into a
//                      ring of P+1 load stages while token t computes; the
//                      hazard plan in the record forwards rows written by the
//                      tokens in between from a ring of P written-row stages.
//                      Written rows are stored back to global memory at once.
#pragma once

#include "sdm_device.cuh"
#include "sdm_records.cuh"

namespace sdm {


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
  static_assert(VE % 4 == 0, "vectors of 4");
  if constexpr (sizeof(Tin) == 4) {
#pragma unroll
    for (int i = 0; i < VE; i += 4) {
      const float4 f = *reinterpret_cast<const float4*>(p + i);
      out[i] = f.x; out[i + 1] = f.y; out[i + 2] = f.z; out[i + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < VE; i += 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p + i);
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
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

// m[j] <- aw * m[j] + cw * v[j] for j < VE, two fp32 lanes per instruction.
template <int VE>
__device__ __forceinline__ void delta_update(float* m, const float* v, float aw, float cw) {
  const float2 a2 = make_float2(aw, aw), c2 = make_float2(cw, cw);
#pragma unroll
  for (int j = 0; j < VE; j += 2) {
    const float2 t = __fmul2_rn(c2, make_float2(v[j], v[j + 1]));
    const float2 r = __ffma2_rn(a2, make_float2(m[j], m[j + 1]), t);
    m[j] = r.x;
    m[j + 1] = r.y;
  }
}
// acc[j] += qw * m[j] for j < VE.
template <int VE>
__device__ __forceinline__ void weighted_add(float* acc, const float* m, float qw) {
  const float2 q2 = make_float2(qw, qw);
#pragma unroll
  for (int j = 0; j < VE; j += 2) {
    const float2 r = __ffma2_rn(q2, make_float2(m[j], m[j + 1]), make_float2(acc[j], acc[j + 1]));
    acc[j] = r.x;
    acc[j + 1] = r.y;
  }
}

// Stores four fp32 values as four consecutive state elements (16 or 8 bytes).
template <typename Tst>
__device__ __forceinline__ void store_vec4(Tst* p, const float4& f) {
  if constexpr (sizeof(Tst) == 4) {
    *reinterpret_cast<float4*>(p) = f;
  } else {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x, f.y), hi = __floats2bfloat162_rn(f.z, f.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
  }
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

// Per-token metadata one lane group of the resident kernel needs first: its
// first block of EB write entries and of EB read entries, alpha, beta and its
// four columns of v.
template <int EB>
struct ResidentMeta {
  int ws[EB], rs[EB];
  float wk[EB], rq[EB];
  float alpha, beta;
  float v[4];
};

// EB consecutive 32-bit words (EB = 2 or 4, 8- or 16-byte aligned).
template <int EB>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t* out) {
  if constexpr (EB == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    out[0] = u.x; out[1] = u.y; out[2] = u.z; out[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    out[0] = u.x; out[1] = u.y;
  }
}

// Block g of the write and of the read entries of one staged record; a lane
// group without a block gets empty entries (slot -1, coefficient 0).
template <typename Tin, int EB>
__device__ __forceinline__ void load_meta(ResidentMeta<EB>& m, const RecLayout& rl, const uint32_t* rec,
                                          const Tin* vrow, int g, int W, int R) {
  if (g * EB < W) {
    load_words<EB>(rec + rl.off_slot_w + g * EB, reinterpret_cast<uint32_t*>(m.ws));
    load_words<EB>(rec + rl.off_k_w + g * EB, reinterpret_cast<uint32_t*>(m.wk));
  } else {
#pragma unroll
    for (int j = 0; j < EB; ++j) { m.ws[j] = -1; m.wk[j] = 0.f; }
  }
  if (g * EB < R) {
    load_words<EB>(rec + rl.off_slot_r + g * EB, reinterpret_cast<uint32_t*>(m.rs));
    load_words<EB>(rec + rl.off_q_r + g * EB, reinterpret_cast<uint32_t*>(m.rq));
  } else {
#pragma unroll
    for (int j = 0; j < EB; ++j) { m.rs[j] = -1; m.rq[j] = 0.f; }
  }
  const float2 ab = *reinterpret_cast<const float2*>(rec + rl.off_ab);
  m.alpha = ab.x;
  m.beta = ab.y;
  load_in_vec<Tin, 4>(vrow, m.v);
}

__device__ __forceinline__ void load_row4(const float4* p, float* m) {
  const float4 r = *p;
  m[0] = r.x; m[1] = r.y; m[2] = r.z; m[3] = r.w;
}
template <typename Tst>
__device__ __forceinline__ void store_row4(float4* p, const float* m) {
  *p = make_float4(round_to<Tst>(m[0]), round_to<Tst>(m[1]), round_to<Tst>(m[2]), round_to<Tst>(m[3]));
}

// Sums acc[0:4) (four columns of unit q = lane % U) over the 32 / U entry
// groups of the warp and stores the four column sums at y[0:4) of unit q.
// Reduce-scatter over the two highest lane bits (each lane keeps half, then a
// quarter of its values), plain butterfly over the lower group bits; the
// order is fixed, so y does not depend on timing.
template <int U>
__device__ __forceinline__ void reduce_store_y(const float* acc, float* y, int lane) {
  static_assert(U <= 8, "at least four entry groups");
  const bool hi = lane & 16, hi2 = lane & 8;
  float k0 = hi ? acc[2] : acc[0], k1 = hi ? acc[3] : acc[1];
  const float s0 = hi ? acc[0] : acc[2], s1 = hi ? acc[1] : acc[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
  float k = hi2 ? k1 : k0;
  k += __shfl_xor_sync(0xffffffffu, hi2 ? k0 : k1, 8);
#pragma unroll
  for (int o = 4; o >= U; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
  if ((lane & (7 & ~(U - 1))) == 0) y[(hi ? 2 : 0) + (hi2 ? 1 : 0)] = k;
}

// A resident warp tile (N rows of CW fp32 columns) into checkpoint k of
// the state ([k][B,H,N,d_v]) at columns col..col+CW of (b, h) = bh. Kept out
// of line: it runs once per checkpoint chunk, outside the per-token chain.
template <int CW>
__device__ __noinline__ void resident_store_checkpoint(float* ckpt, int64_t bhs, int N, int d_v, const float* tile,
                                                       int k, int bh, int col, int lane) {
  float* dst = ckpt + (static_cast<int64_t>(k) * bhs + bh) * N * d_v + col;
  for (int x = lane; x < N * (CW / 4); x += kWarp) {
    const int row = x / (CW / 4), c = (x % (CW / 4)) * 4;
    *reinterpret_cast<float4*>(dst + static_cast<int64_t>(row) * d_v + c) =
        *reinterpret_cast<const float4*>(tile + static_cast<size_t>(row) * CW + c);
  }
}

// Shared-memory bytes of k_scan_resident (host and device agree on this).
__host__ __device__ constexpr size_t resident_smem_bytes(int N, int CW, int NWARP, int L, int words, int s_in) {
  return static_cast<size_t>(NWARP) * (N + 2) * CW * 4 + static_cast<size_t>(2) * L * words * 4 +
         static_cast<size_t>(2) * L * CW * NWARP * s_in + 2 * 8;
}

// Each warp owns a CW-column tile of one (b, h) and carries it through all T
// tokens on its own: lane q % U holds four fp32 columns (one 16-byte unit) of
// the entry block g = lane / U, so one warp instruction covers G = 32 / U
// entries. The tile never leaves the warp, so tokens need no block barrier;
// the only block barriers are the two per staged chunk of L tokens. The read
// sum of a token is reduced over the G entry groups with a fixed butterfly,
// so y does not depend on timing.
// kCkpt builds also store the backward's checkpoints: the state before tokens
// ckpt_C, 2 ckpt_C, ... into ckpt ([n-1][B,H,N,d_v] fp32). (Kernel
// parameters of their own: growing ScanArgs changed this kernel's code.)
template <typename Tin, typename Tst, int CW, int NWARP, int L, int EB, bool kCkpt = false>
__global__ void __launch_bounds__(NWARP * kWarp) k_scan_resident(ScanArgs a, float* ckpt, int ckpt_C) {
  constexpr int NT = NWARP * kWarp;
  constexpr int C = CW * NWARP;  // columns of the CTA
  constexpr int U = CW / 4;      // lanes per entry
  constexpr int G = kWarp / U;   // entry blocks per warp instruction
  static_assert(CW == 4 || CW == 8 || CW == 16 || CW == 32, "warp tile of 4..32 fp32 columns");
  static_assert(EB == 2 || EB == 4, "entry blocks of 2 or 4");
  extern __shared__ __align__(16) unsigned char smem[];
  const int N = a.N, W = a.W, R = a.R, T = a.T;
  const int words = a.rl.words;
  float* S = reinterpret_cast<float*>(smem);  // [NWARP][N + 2][CW]
  uint32_t* recbuf = reinterpret_cast<uint32_t*>(smem + static_cast<size_t>(NWARP) * (N + 2) * CW * 4);
  Tin* vbuf = reinterpret_cast<Tin*>(recbuf + 2 * L * words);
  uint64_t* bars = reinterpret_cast<uint64_t*>(vbuf + 2 * L * C);

  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int c0 = blockIdx.y * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane / U, q = lane % U;
  // Warp tile: rows 0..N-1 hold the state; row N absorbs writes of skipped
  // entries (never read) and row N+1 stays zero for skipped reads, so the
  // entry loops need no branches.
  float4* Sw = reinterpret_cast<float4*>(S + static_cast<size_t>(warp) * (N + 2) * CW) + q;  // row r at Sw[r * U]
  const int sink_w = N, zero_r = N + 1;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  {  // initial state tile, four columns at a time
    const Tst* Min = static_cast<const Tst*>(a.M_in) + b * a.M_in_b_stride +
                     static_cast<int64_t>(h) * N * a.d_v + c0;
    for (int x = tid; x < N * (C / 4); x += NT) {
      const int row = x / (C / 4), col = (x % (C / 4)) * 4;
      float f[4];
      load_in_vec<Tst, 4>(Min + static_cast<int64_t>(row) * a.d_v + col, f);
      *reinterpret_cast<float4*>(S + (static_cast<size_t>(col / CW) * (N + 2) + row) * CW + col % CW) =
          make_float4(f[0], f[1], f[2], f[3]);
    }
    for (int x = tid; x < NWARP * 2 * CW; x += NT)
      S[(static_cast<size_t>(x / (2 * CW)) * (N + 2) + N) * CW + x % (2 * CW)] = 0.f;
  }
  __syncthreads();
  const int n_chunks = (T + L - 1) / L;
  if (tid == 0 && n_chunks > 0) {
    issue_chunk<Tin, C, L>(a, bh, b, h, c0, 0, recbuf, vbuf, bars);
    if (n_chunks > 1) issue_chunk<Tin, C, L>(a, bh, b, h, c0, 1, recbuf, vbuf, bars);
  }
  if (n_chunks > 0) {
    // Software pipeline over tokens: the metadata of token t+1 is loaded
    // while token t computes, and the y reduction of token t-1 overlaps the
    // row loads of token t. Two tokens per iteration, so the metadata
    // registers alternate without copies.
    const int vcol = warp * CW + 4 * q;  // this lane's first column within the CTA tile
    const int64_t y_step = static_cast<int64_t>(a.H) * a.d_v;
    float* y_t = a.y + static_cast<int64_t>(b) * T * y_step + static_cast<int64_t>(h) * a.d_v + c0 + vcol;
    auto rec_of = [&](int t) { return recbuf + (static_cast<size_t>((t / L) & 1) * L + t % L) * words; };
    auto vrow_of = [&](int t) { return vbuf + (static_cast<size_t>((t / L) & 1) * L + t % L) * C + vcol; };
    auto chunk_ok = [&](int cc) {
      const bool ok = mbar_wait_bounded(&bars[cc & 1], (cc >> 1) & 1, a.err);
      return !__syncthreads_or(!ok);
    };
    if (!chunk_ok(0)) return;
    ResidentMeta<EB> ma, mb;
    load_meta<Tin, EB>(ma, a.rl, rec_of(0), vrow_of(0), g, W, R);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    bool failed = false;

    // Checkpoints (kCkpt builds only): the token before which the next one
    // is taken.
    int next_ckpt = ckpt_C;
    // One token: returns false when a staging wait gave up.
    auto step = [&](int t, const ResidentMeta<EB>& cur, ResidentMeta<EB>& nxt) -> bool {
      if constexpr (kCkpt) {
        if (t == next_ckpt) {  // the warp's tile is past token t - 1
          resident_store_checkpoint<CW>(ckpt, static_cast<int64_t>(a.B) * a.H, N, a.d_v,
                                        S + static_cast<size_t>(warp) * (N + 2) * CW, t / ckpt_C - 1, bh,
                                        c0 + warp * CW, lane);
          next_ckpt += ckpt_C;
        }
      }
      // 1. row loads of the first write block
      int wrow[EB];
      float m[EB][4];
#pragma unroll
      for (int j = 0; j < EB; ++j) {
        wrow[j] = cur.ws[j] < 0 ? sink_w : cur.ws[j];
        load_row4(Sw + wrow[j] * U, m[j]);
      }
      // 2. y of token t-1 (independent of the loads in flight)
      if (t > 0) reduce_store_y<U>(acc, y_t - y_step, lane);
      // 3. metadata of token t+1
      if (t + 1 < T) {
        if ((t + 1) % L == 0 && !chunk_ok((t + 1) / L)) return false;
        load_meta<Tin, EB>(nxt, a.rl, rec_of(t + 1), vrow_of(t + 1), g, W, R);
      }
      // 4. write: the W slots of a token are distinct, so a block is loaded
      // before any of it is stored; blocks past the first (W > EB * G) are
      // loaded here.
#pragma unroll
      for (int j = 0; j < EB; ++j) {
        const float cw = cur.beta * cur.wk[j];
        delta_update<4>(m[j], cur.v, cur.alpha * (1.0f - cw), cw);
        store_row4<Tst>(Sw + wrow[j] * U, m[j]);
      }
      for (int jb = g + G; jb * EB < W; jb += G) {
        const uint32_t* rec = rec_of(t);
        int sl[EB];
        float kk[EB];
        load_words<EB>(rec + a.rl.off_slot_w + jb * EB, reinterpret_cast<uint32_t*>(sl));
        load_words<EB>(rec + a.rl.off_k_w + jb * EB, reinterpret_cast<uint32_t*>(kk));
#pragma unroll
        for (int j = 0; j < EB; ++j) {
          sl[j] = sl[j] < 0 ? sink_w : sl[j];
          load_row4(Sw + sl[j] * U, m[j]);
        }
#pragma unroll
        for (int j = 0; j < EB; ++j) {
          const float cw = cur.beta * kk[j];
          delta_update<4>(m[j], cur.v, cur.alpha * (1.0f - cw), cw);
          store_row4<Tst>(Sw + sl[j] * U, m[j]);
        }
      }
      __syncwarp();  // rows written by one lane group are read by another
      // 5. read after the write
#pragma unroll
      for (int j = 0; j < EB; ++j) load_row4(Sw + (cur.rs[j] < 0 ? zero_r : cur.rs[j]) * U, m[j]);
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = 0.f;
#pragma unroll
      for (int j = 0; j < EB; ++j) weighted_add<4>(acc, m[j], cur.rq[j]);
      for (int jb = g + G; jb * EB < R; jb += G) {
        const uint32_t* rec = rec_of(t);
        int sl[EB];
        float qq[EB];
        load_words<EB>(rec + a.rl.off_slot_r + jb * EB, reinterpret_cast<uint32_t*>(sl));
        load_words<EB>(rec + a.rl.off_q_r + jb * EB, reinterpret_cast<uint32_t*>(qq));
#pragma unroll
        for (int j = 0; j < EB; ++j) load_row4(Sw + (sl[j] < 0 ? zero_r : sl[j]) * U, m[j]);
#pragma unroll
        for (int j = 0; j < EB; ++j) weighted_add<4>(acc, m[j], qq[j]);
      }
      __syncwarp();  // this token's reads precede the next token's writes
      // 6. at the end of a chunk every warp is past its buffer: refill it
      if (t % L == L - 1) {
        __syncthreads();
        if (tid == 0 && t / L + 2 < n_chunks) {
          fence_proxy_async_smem();
          issue_chunk<Tin, C, L>(a, bh, b, h, c0, t / L + 2, recbuf, vbuf, bars);
        }
      }
      y_t += y_step;
      return true;
    };

#pragma unroll 1
    for (int t = 0; t < T; t += 2) {
      if (!step(t, ma, mb)) { failed = true; break; }
      if (t + 1 < T && !step(t + 1, mb, ma)) { failed = true; break; }
    }
    if (failed) return;
    reduce_store_y<U>(acc, y_t - y_step, lane);
  }
  __syncthreads();
  {
    Tst* Mout = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * N * a.d_v + c0;
    for (int x = tid; x < N * (C / 4); x += NT) {
      const int row = x / (C / 4), col = (x % (C / 4)) * 4;
      store_vec4<Tst>(Mout + static_cast<int64_t>(row) * a.d_v + col,
                      *reinterpret_cast<const float4*>(S + (static_cast<size_t>(col / CW) * (N + 2) + row) * CW + col % CW));
    }
  }
}

// ----------------------------------------------------------- streaming ----

// Sums a[0:VE) (the VE columns of one 16-byte unit, held by the U lanes of
// every entry group) over the 32 / U entry groups of the warp and stores the
// column sums at y[0:VE): reduce-scatter while a lane still holds more than
// one value, butterfly after that; the order is fixed, so y does not depend
// on timing.
template <int VE, int U>
__device__ __forceinline__ void reduce_store_unit(float (&a)[VE], float* y, int lane) {
  int n = VE, off = 0, bmask = 0;
#pragma unroll
  for (int o = 16; o >= U; o >>= 1) {
    if (n > 1) {
      const bool hi = lane & o;
      const int h = n / 2;
#pragma unroll
      for (int j = 0; j < VE / 2; ++j) {
        if (j < h) {
          const float keep = hi ? a[j + h] : a[j];
          const float send = hi ? a[j] : a[j + h];
          a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      off += hi ? h : 0;
      n = h;
    } else {
      a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
      bmask |= o;
    }
  }
  if ((lane & bmask) == 0) {
#pragma unroll
    for (int j = 0; j < VE; ++j)
      if (j < n) y[off + j] = a[j];
  }
}

// Shared-memory bytes of the stage rings of k_scan_streaming.
__host__ __device__ constexpr size_t streaming_stage_bytes(int P, int E, int W, int C, int s_state) {
  return (static_cast<size_t>(P + 1) * E + static_cast<size_t>(P + 1) * W) * C * s_state;
}

// The state stays in global memory. A CTA of NW warps owns one (b, h) and C
// columns. The rows of token t+P are gathered (one 16-byte cp.async per lane
// and unit) into a ring of P+1 load stages right after token t's barrier, so
// the copies overlap token t's compute; the hazard plan forwards rows that
// tokens t+P-1 .. t write from a ring of P+1 written-row stages. A read of a
// slot written by the same token recomputes that write from its source row
// (plan code k = 0), so the writes and reads of a token have no dependency
// between warps: one block barrier per token orders token t's rows before
// token t+1 and before the gathers that token t+1 issues. Written rows go
// straight back to global memory. Warp partial sums of y are reduced in a
// fixed order one token later.
template <typename Tin, typename Tst, int C, int P, int L, int NW>
__global__ void __launch_bounds__(NW * kWarp, 1) k_scan_streaming(ScanArgs a) {
  constexpr int NT = NW * kWarp;
  constexpr int VE = 16 / sizeof(Tst);  // state elements per 16-byte unit
  constexpr int U = C / VE;             // units per row segment
  constexpr int G = kWarp / U;          // entries per warp instruction
  constexpr int GS = G * NW;            // entries per block instruction
  constexpr int SL = P + 1;             // load stages
  constexpr int SW = P + 1;             // written-row stages
  constexpr uint32_t RS = C * sizeof(Tst);
  static_assert(L > P, "a chunk must be staged before its tokens are gathered");
  static_assert(kWarp % U == 0, "a row segment spans a divisor of the warp");
  static_assert(C <= NT, "one thread per column sums y");
  extern __shared__ __align__(16) unsigned char smem[];
  const int W = a.W, R = a.R, T = a.T, E = W + R;
  const int words = a.rl.words;
  unsigned char* lstage = smem;                                    // [SL][E][RS]
  unsigned char* wstage = smem + static_cast<size_t>(SL) * E * RS;  // [SW][W][RS]
  uint32_t* recbuf = reinterpret_cast<uint32_t*>(smem + streaming_stage_bytes(P, E, W, C, sizeof(Tst)));
  Tin* vbuf = reinterpret_cast<Tin*>(recbuf + 2 * L * words);
  float* ypart = reinterpret_cast<float*>(vbuf + 2 * L * C);  // [2][NW][C]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ypart + 2 * NW * C);

  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int c0 = blockIdx.y * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane / U, q = lane % U;
  const int e0 = g + G * warp;
  Tst* Mbh = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * a.N * a.d_v + c0 + q * VE;
  const int64_t y_step = static_cast<int64_t>(a.H) * a.d_v;
  float* y_bh = a.y + static_cast<int64_t>(b) * T * y_step + static_cast<int64_t>(h) * a.d_v + c0;

  auto rec_of = [&](int t) -> const uint32_t* {
    return recbuf + (static_cast<size_t>((t / L) & 1) * L + (t % L)) * words;
  };
  auto fwd_of = [&](const uint32_t* rec, int e) -> int {
    return reinterpret_cast<const int16_t*>(rec + a.rl.off_fwd)[e];
  };
  // Row unit of entry e of token t: gathered, or forwarded from an earlier
  // token's written row (code (k << 9) | j, k >= 1).
  auto source = [&](int t, const uint32_t* rec, int e) -> const unsigned char* {
    const int f = fwd_of(rec, e);
    if (f < 0) return lstage + (static_cast<size_t>(t % SL) * E + e) * RS + q * 16;
    return wstage + (static_cast<size_t>((t - (f >> 9)) % SW) * W + (f & 511)) * RS + q * 16;
  };
  // Gathers the rows of token t that the plan does not forward: one 16-byte
  // cp.async per (entry, unit), one commit group per call.
  auto gather = [&](int t) {
    const uint32_t* rec = rec_of(t);
    unsigned char* ls = lstage + static_cast<size_t>(t % SL) * E * RS + q * 16;
    for (int e = e0; e < E; e += GS) {
      const int slot = static_cast<int>(e < W ? rec[a.rl.off_slot_w + e] : rec[a.rl.off_slot_r + e - W]);
      if (slot >= 0 && fwd_of(rec, e) < 0) cp_async16(ls + e * RS, Mbh + static_cast<int64_t>(slot) * a.d_v);
    }
    cp_async_commit();
  };
  auto chunk_ok = [&](int cc) {
    const bool ok = mbar_wait_bounded(&bars[cc & 1], (cc >> 1) & 1, a.err);
    return !__syncthreads_or(!ok);
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
  if (!chunk_ok(0)) return;
  for (int t = 0; t < P; ++t) {
    if (t < T) gather(t);
    else cp_async_commit();
  }

#pragma unroll 1
  for (int t = 0; t < T; ++t) {
    cp_async_wait<P - 1>();
    __syncthreads();  // token t's rows landed; token t-1's rows written and visible
    if (t > 0 && t % L == 0 && tid == 0 && t / L + 1 < n_chunks) {
      fence_proxy_async_smem();
      issue_chunk<Tin, C, L>(a, bh, b, h, c0, t / L + 1, recbuf, vbuf, bars);
    }
    if (t > 0 && tid < C) {  // y of token t-1: fixed-order sum of the warp partials
      const float* yp = ypart + ((t - 1) & 1) * NW * C + tid;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) sum += yp[w * C];
      y_bh[(t - 1) * y_step + tid] = sum;
    }
    // Gather token t+P into the load stage token t-1 used (free after the barrier).
    if (t + P < T) {
      if ((t + P) % L == 0 && !chunk_ok((t + P) / L)) {
        cp_async_wait<0>();
        return;
      }
      gather(t + P);
    } else {
      cp_async_commit();
    }
    const uint32_t* rec = rec_of(t);
    const float2 ab = *reinterpret_cast<const float2*>(rec + a.rl.off_ab);
    float vv[VE];
    load_in_vec<Tin, VE>(vbuf + (static_cast<size_t>((t / L) & 1) * L + (t % L)) * C + q * VE, vv);
    unsigned char* wrow = wstage + static_cast<size_t>(t % SW) * W * RS + q * 16;
    // Entries e < W are writes, the rest reads; with reads of this token's
    // written slots recomputed from the write's source row, the two kinds are
    // independent, so every lane group takes the same share of either.
    float acc[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) acc[j] = 0.f;
    for (int e = e0; e < E; e += GS) {
      if (e < W) {
        const int slot = static_cast<int>(rec[a.rl.off_slot_w + e]);
        if (slot < 0) continue;
        float m[VE];
        unpack16<Tst>(*reinterpret_cast<const uint4*>(source(t, rec, e)), m);
        const float cw = ab.y * __uint_as_float(rec[a.rl.off_k_w + e]);
        delta_update<VE>(m, vv, ab.x * (1.0f - cw), cw);
        const uint4 packed = pack16<Tst>(m);
        *reinterpret_cast<uint4*>(wrow + e * RS) = packed;
        *reinterpret_cast<uint4*>(Mbh + static_cast<int64_t>(slot) * a.d_v) = packed;
      } else {
        const int r = e - W;
        const int slot = static_cast<int>(rec[a.rl.off_slot_r + r]);
        if (slot < 0) continue;
        const int f = fwd_of(rec, e);
        float m[VE];
        if (f >= 0 && (f >> 9) == 0) {  // written by this token: recompute that write
          const int j = f & 511;
          unpack16<Tst>(*reinterpret_cast<const uint4*>(source(t, rec, j)), m);
          const float cw = ab.y * __uint_as_float(rec[a.rl.off_k_w + j]);
          delta_update<VE>(m, vv, ab.x * (1.0f - cw), cw);
          unpack16<Tst>(pack16<Tst>(m), m);  // the stored (rounded) value
        } else {
          unpack16<Tst>(*reinterpret_cast<const uint4*>(source(t, rec, e)), m);
        }
        weighted_add<VE>(acc, m, __uint_as_float(rec[a.rl.off_q_r + r]));
      }
    }
    reduce_store_unit<VE, U>(acc, ypart + (t & 1) * NW * C + warp * C + q * VE, lane);
  }
  cp_async_wait<0>();
  __syncthreads();
  if (T > 0 && tid < C) {
    const float* yp = ypart + ((T - 1) & 1) * NW * C + tid;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sum += yp[w * C];
    y_bh[(T - 1) * y_step + tid] = sum;
  }
}

}  // namespace sdm
