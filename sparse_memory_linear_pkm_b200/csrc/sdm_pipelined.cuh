// The sparse gated delta recurrence for states far larger than the chip,
// when few (b, h) sequences are in flight (sm_100a).
//
// SDM explainer (papers.ananclaw.com), section 3.1: step 2 writes the W
// selected slots, M~ = alpha_t M[i], M[i] = M~ + beta_t k_i (v_t - M~); step 3
// reads y_t = sum_r q_r M_t[r] after the write. The kernel uses the factored
// form M[i] = (alpha_t (1 - beta_t k_i)) M[i] + (beta_t k_i) v_t in fp32 and
// rounds to the state dtype on every store, like the other recurrence
// kernels.
//
// Why a third kernel. Every token touches W + R random state rows, and one
// B200 SM moves at most about one random 128-byte row per 3 ns, however the
// copies are issued (measured with cp.async from 4-16 warps and with TMA
// gather4: ~40 GB/s per SM). The long-context workload has only B*H = 2
// sequences, so a grid of one CTA per (b, h) and 128-byte column tile fills
// 64 SMs and cannot pass ~2.5 TB/s. Here each (b, h) column tile is split
// over `parts` CTAs by a hash bit of the slot index: a part owns a fixed
// half of the slots, so it alone writes and reads them and the parts need no
// synchronisation; each adds its partial read sum into y (with two parts the
// sum 0 + a + b does not depend on their order, so y stays reproducible).
//
// Within a CTA (warp roles; one token a step, or two with S = 2):
//   * producer warps request each token's rows with TMA row gathers (four
//     128-byte rows an instruction, two instructions a warp at W = R = 64)
//     into a ring of P stages, up to P - 1 tokens ahead, and reload the
//     record and v chunks; before reusing a stage they wait on a per-token
//     `done` mbarrier, once per token pair (tokens finish in order). An SM
//     takes one random 128-byte row per ~6-7 cycles however it is asked, and
//     the issuing thread waits for the acceptance, so the requests live in
//     warps of their own;
//   * the control warp waits for the next token's rows and records, sums the
//     read lanes' partial sums of the previous token in a fixed order and
//     stores them to y (part 0) or to a scratch copy that a separate pass adds
//     into y (part 1; plain stores, no atomics), and arrives on `done`;
//   * write warps apply the write to the part's write entries (each lane owns
//     one 16-byte unit of a row), store the rows to global memory and keep
//     them in a ring of written-row stages;
//   * read warps sum the part's read entries, each lane its unit over its
//     entry group, and store those partial sums for the control warp;
//   * the control warp and the consumers meet at one named barrier a step
//     (barrier.cta.red.or: a failed wait in the control warp ends them all).
// Write warps fence their global stores (fence.proxy.async.global) before
// the next barrier, so the TMA gathers issued after `done` read them. A row
// gathered early is stale when one of the P - 1 tokens before its use wrote
// it; the hazard plan in the records names that write (token t - k, write
// entry j of this part) and the row is taken from the written-row ring
// instead; a read of a slot written by the same token (k = 0) recomputes that
// write from its source.
#pragma once

#include <cuda.h>

#include "sdm_device.cuh"
#include "sdm_fp8.cuh"
#include "sdm_scan.cuh"

namespace sdm {

// Four rows of a 2-D tensor map (row coordinates r0..r3, column x) into
// consecutive boxes at dst, completing on bar (TMA row gather, no multicast).
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, int x, int r0, int r1, int r2, int r3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];\n" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}
// Orders this thread's earlier generic-proxy global writes before later
// async-proxy (TMA) reads of the same memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

// Per-token record of one part (32-bit words):
//   uint16 src_w[Wp] | uint16 src_r[Rp] | float2 awcw[Wp] | f32 q_r[Rp] |
//   int32 slot_w[Wp] | int32 slot_r[Rp] | int32 nw, int32 nr, 0, 0
// The part's write and read entries are compacted to the front in selection
// order (nw, nr of them); the rest is padding (slot -1, coefficients 0).
// Everything a consumer lane needs is precomputed by the record build:
//   src    the row of the kernel's stage space (shared memory, RS bytes a row)
//          the entry's source row sits in: rows [0, P E) are the gather
//          stages (stage s, entry e at s E + e; writes first, reads from Wp),
//          rows P E + s Wp + j the written-row ring (token t - k's write j,
//          s = (t - k) mod P) when a token in between wrote the slot (the
//          hazard plan); a read of a slot written by the same token carries
//          0x8000 | j: that write recomputed from its own source;
//   awcw   the write's factored coefficients a = alpha (1 - beta k), c = beta k;
//   q_r    the read weight; slot_*: the rows the part gathers and stores.
struct PipeLayout {
  int Wp, Rp;
  int off_src_w, off_src_r, off_awcw, off_q_r, off_slot_w, off_slot_r, off_meta;
  int words;
};

__host__ __device__ inline PipeLayout pipe_layout(int W, int R) {
  PipeLayout pl{};
  pl.Wp = (W + 7) / 8 * 8;
  pl.Rp = (R + 7) / 8 * 8;
  pl.off_src_w = 0;
  pl.off_src_r = pl.Wp / 2;
  pl.off_awcw = pl.off_src_r + pl.Rp / 2;
  pl.off_q_r = pl.off_awcw + 2 * pl.Wp;
  pl.off_slot_w = pl.off_q_r + pl.Rp;
  pl.off_slot_r = pl.off_slot_w + pl.Wp;
  pl.off_meta = pl.off_slot_r + pl.Rp;
  pl.words = pl.off_meta + 4;
  return pl;
}

// Source codes (16 bits): a row of the stage space below 0x2000, or a flag
// with a write entry j in the low 9 bits.
constexpr uint32_t kSrcSameToken = 0x8000u;  // reads: recompute this token's write j
constexpr uint32_t kSrcPrevToken = 0x4000u;  // second token of a two-token step: recompute the first token's write j
constexpr uint32_t kSkipStore = 0x2000u;     // first token's write: the second token rewrites the slot, no HBM store
constexpr uint32_t kRowMask = 0x1FFFu;
constexpr uint32_t kEntryMask = 0x1FFu;
constexpr int kTokW = 3;  // two-token step: write units of each token per pass of a write lane
constexpr int kTokR = 3;  // two-token step: read entries of each token per pass of a read lane

// 16 bytes of state (8 bf16 or 4 fp32 values) as fp32, by bit operations.
template <typename Tst>
__device__ __forceinline__ void unpack_unit(const uint4& u, float* m) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if constexpr (sizeof(Tst) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[2 * i] = __uint_as_float(w[i] << 16);
      m[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = __uint_as_float(w[i]);
  }
}
// m <- a m + c v on VE values, two lanes of fp32 per instruction (per element
// the same roundings as the other recurrence kernels: a product, then a fused
// multiply-add).
template <int VE>
__device__ __forceinline__ void write_unit(float* m, const float* v, float a, float c) {
  const float2 a2 = make_float2(a, a), c2 = make_float2(c, c);
#pragma unroll
  for (int j = 0; j < VE; j += 2) {
    const float2 r = __ffma2_rn(a2, make_float2(m[j], m[j + 1]), __fmul2_rn(c2, make_float2(v[j], v[j + 1])));
    m[j] = r.x;
    m[j + 1] = r.y;
  }
}
template <int VE>
__device__ __forceinline__ void read_unit(float* acc, const float* m, float q) {
  const float2 q2 = make_float2(q, q);
#pragma unroll
  for (int j = 0; j < VE; j += 2) {
    const float2 r = __ffma2_rn(q2, make_float2(m[j], m[j + 1]), make_float2(acc[j], acc[j + 1]));
    acc[j] = r.x;
    acc[j + 1] = r.y;
  }
}

// Part of a slot: a hash bit, so that structured selections (e.g. slots that
// share a grid column) still spread over both parts.
__device__ __forceinline__ int slot_part(uint32_t slot, int parts) {
  return parts == 1 ? 0 : static_cast<int>((slot * 0x9E3779B1u) >> 31);
}

constexpr int kPipeTokensPerBlock = 32;

// Written stages of the pipelined kernel: P + S - 1, so that the S tokens
// of a step never write a stage that one of them still reads.
__host__ __device__ constexpr int pipe_wstages(int P, int S) { return P + S - 1; }

// Shared-memory bytes of k_build_pipe_records.
__host__ __device__ constexpr size_t pipe_records_smem(int W, int R, int P, int log2_cells, int parts) {
  return static_cast<size_t>(kPipeTokensPerBlock + P) * ((size_t{1} << log2_cells) * 4 + W * 2) +
         static_cast<size_t>(kPipeTokensPerBlock) * R * 2 + 4 + static_cast<size_t>(kPipeTokensPerBlock) * parts * 8;
}

// Records of one (b, h) and 32 tokens for every part: compaction of each
// part's write and read entries (warp ballots, in selection order), the
// hazard plan against the written slots of the P - 1 tokens before (one
// open-addressing table per token, slot -> compacted write entry), and, when
// y_zero is given, zeros for those tokens' y rows (the recurrence adds the
// parts' sums into it). With S = 2 the recurrence takes tokens in pairs
// (2s, 2s + 1): the second token's entries that the first one wrote become
// kSrcPrevToken, and the first token's writes of slots the second one
// rewrites get kSkipStore. Slot indices outside [0, N) are left out and set
// the device error word.
template <typename Tin>
__global__ void __launch_bounds__(256) k_build_pipe_records(
    const int32_t* __restrict__ idx_w, const float* __restrict__ w_w, const int32_t* __restrict__ idx_r,
    const float* __restrict__ w_r, const Tin* __restrict__ alpha, const Tin* __restrict__ beta, int T, int H, int N,
    int W, int R, int P, int S, int parts, int log2_cells, PipeLayout pl, uint32_t* __restrict__ rec,
    float* __restrict__ y_zero, int d_v, unsigned* err) {
  const int E = pl.Wp + pl.Rp;  // rows of one gather stage
  const int Q = pipe_wstages(P, S);
  extern __shared__ uint32_t sm[];
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int t0 = blockIdx.x * kPipeTokensPerBlock;
  const int t_end = min(T, t0 + kPipeTokensPerBlock);
  const int t_first = max(0, t0 - (P - 1));
  const int t_tab_end = min(T, t_end + (S - 1));  // the tables reach the second token of the last pair
  const int n_tab = t_tab_end - t_first, n_own = t_end - t0;
  const int n_cells = 1 << log2_cells;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* cells = sm;                                               // [n_tab][n_cells]
  int16_t* jcw = reinterpret_cast<int16_t*>(cells + n_tab * n_cells);  // [n_tab][W]
  int16_t* rcr = jcw + n_tab * W;                                     // [n_own][R]
  const int n16 = n_tab * W + n_own * R;
  int* cnt = reinterpret_cast<int*>(jcw + ((n16 + 1) & ~1));          // [n_own][parts][2]

  for (int i = threadIdx.x; i < n_tab * n_cells; i += blockDim.x) cells[i] = kEmptyCell;
  __syncthreads();

  // 1. compaction (one warp per token) and the tables of written slots
  for (int tt = t_first + warp; tt < t_tab_end; tt += blockDim.x / 32) {
    const int64_t th = (static_cast<int64_t>(b) * T + tt) * H + h;
    uint32_t* tab = cells + (tt - t_first) * n_cells;
    int base[2] = {0, 0};
    for (int j0 = 0; j0 < W; j0 += 32) {
      const int j = j0 + lane;
      const int slot = j < W ? idx_w[th * W + j] : -1;
      const bool valid = j < W && slot >= 0 && slot < N;
      const int part = valid ? slot_part(static_cast<uint32_t>(slot), parts) : -1;
      int jc = -1;
      for (int p = 0; p < parts; ++p) {
        const unsigned m = __ballot_sync(0xffffffffu, part == p);
        if (part == p) jc = base[p] + __popc(m & lanemask_lt());
        base[p] += __popc(m);
      }
      if (j < W) jcw[(tt - t_first) * W + j] = static_cast<int16_t>(jc);
      if (valid) {
        const uint32_t packed = static_cast<uint32_t>(slot) * 512u + static_cast<uint32_t>(jc);
        uint32_t pos = slot_hash(static_cast<uint32_t>(slot), log2_cells);
        for (int probe = 0; probe < n_cells; ++probe) {  // at most W < n_cells entries per table
          const uint32_t prev = atomicCAS(&tab[pos], kEmptyCell, packed);
          if (prev == kEmptyCell || (prev >> 9) == static_cast<uint32_t>(slot)) break;
          pos = (pos + 1) & (n_cells - 1);
        }
      }
    }
    if (tt >= t0 && tt < t_end) {
      int rbase[2] = {0, 0};
      for (int r0 = 0; r0 < R; r0 += 32) {
        const int r = r0 + lane;
        const int slot = r < R ? idx_r[th * R + r] : -1;
        const bool valid = r < R && slot >= 0 && slot < N;
        const int part = valid ? slot_part(static_cast<uint32_t>(slot), parts) : -1;
        int rc = -1;
        for (int p = 0; p < parts; ++p) {
          const unsigned m = __ballot_sync(0xffffffffu, part == p);
          if (part == p) rc = rbase[p] + __popc(m & lanemask_lt());
          rbase[p] += __popc(m);
        }
        if (r < R) rcr[(tt - t0) * R + r] = static_cast<int16_t>(rc);
      }
      if (lane < parts) {
        cnt[((tt - t0) * parts + lane) * 2] = base[lane];
        cnt[((tt - t0) * parts + lane) * 2 + 1] = rbase[lane];
      }
    }
  }
  __syncthreads();

  // 2. entries: compacted position, hazard plan, source row
  const int WR = W + R;
  for (int x = threadIdx.x; x < n_own * WR; x += blockDim.x) {
    const int t = t0 + x / WR, e = x % WR;
    const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
    int slot, c;
    float wt;
    if (e < W) {
      slot = idx_w[th * W + e];
      wt = w_w[th * W + e];
      c = jcw[(t - t_first) * W + e];
    } else {
      slot = idx_r[th * R + e - W];
      wt = w_r[th * R + e - W];
      c = rcr[(t - t0) * R + e - W];
    }
    if (c < 0) {
      atomicOr(err, kErrIndexOutOfRange);
      continue;
    }
    const int part = slot_part(static_cast<uint32_t>(slot), parts);
    int code = -1;
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
    uint32_t* r = rec + ((static_cast<int64_t>(bh) * parts + part) * T + t) * pl.words;
    // the entry's source row in the stage space (see PipeLayout)
    uint32_t src;
    if (code < 0) src = static_cast<uint32_t>((t % P) * E + (e < W ? c : pl.Wp + c));
    else if ((code >> 9) == 0) src = kSrcSameToken | static_cast<uint32_t>(code & 511);
    else if ((code >> 9) == 1 && S == 2 && (t & 1)) src = kSrcPrevToken | static_cast<uint32_t>(code & 511);
    else src = static_cast<uint32_t>(P * E + ((t - (code >> 9)) % Q) * pl.Wp + (code & 511));
    if (e < W && S == 2 && !(t & 1) && t + 1 < T) {  // does the pair's second token rewrite the slot?
      const uint32_t* tab = cells + (t + 1 - t_first) * n_cells;
      uint32_t pos = slot_hash(static_cast<uint32_t>(slot), log2_cells);
      for (int probe = 0; probe < n_cells; ++probe) {
        const uint32_t cur = tab[pos];
        if (cur == kEmptyCell) break;
        if ((cur >> 9) == static_cast<uint32_t>(slot)) {
          src |= kSkipStore;
          break;
        }
        pos = (pos + 1) & (n_cells - 1);
      }
    }
    if (e < W) {
      const float a_t = to_f32<Tin>(alpha[th]), b_t = to_f32<Tin>(beta[th]);
      const float cw = b_t * wt;
      r[pl.off_slot_w + c] = static_cast<uint32_t>(slot);
      reinterpret_cast<float2*>(r + pl.off_awcw)[c] = make_float2(a_t * (1.0f - cw), cw);
      reinterpret_cast<uint16_t*>(r + pl.off_src_w)[c] = static_cast<uint16_t>(src);
    } else {
      r[pl.off_slot_r + c] = static_cast<uint32_t>(slot);
      r[pl.off_q_r + c] = __float_as_uint(wt);
      reinterpret_cast<uint16_t*>(r + pl.off_src_r)[c] = static_cast<uint16_t>(src);
    }
  }

  // 3. padding after the compacted entries, and the counts, alpha and beta
  const int EP = pl.Wp + pl.Rp;
  for (int x = threadIdx.x; x < n_own * parts * EP; x += blockDim.x) {
    const int t = t0 + x / (parts * EP), rem = x % (parts * EP), part = rem / EP, pos = rem % EP;
    const int* cn = cnt + ((t - t0) * parts + part) * 2;
    uint32_t* r = rec + ((static_cast<int64_t>(bh) * parts + part) * T + t) * pl.words;
    if (pos < pl.Wp) {
      if (pos >= cn[0]) {  // padding: a gathered row of its own, coefficients that keep it
        r[pl.off_slot_w + pos] = 0xFFFFFFFFu;
        reinterpret_cast<float2*>(r + pl.off_awcw)[pos] = make_float2(0.f, 0.f);
        reinterpret_cast<uint16_t*>(r + pl.off_src_w)[pos] = static_cast<uint16_t>((t % P) * E + pos);
      }
    } else if (pos - pl.Wp >= cn[1]) {
      const int i = pos - pl.Wp;
      r[pl.off_slot_r + i] = 0xFFFFFFFFu;
      r[pl.off_q_r + i] = 0u;
      reinterpret_cast<uint16_t*>(r + pl.off_src_r)[i] = static_cast<uint16_t>((t % P) * E + pos);
    }
  }
  for (int x = threadIdx.x; x < n_own * parts; x += blockDim.x) {
    const int t = t0 + x / parts, part = x % parts;
    const int* cn = cnt + ((t - t0) * parts + part) * 2;
    uint32_t* r = rec + ((static_cast<int64_t>(bh) * parts + part) * T + t) * pl.words;
    r[pl.off_meta] = static_cast<uint32_t>(cn[0]);
    r[pl.off_meta + 1] = static_cast<uint32_t>(cn[1]);
    r[pl.off_meta + 2] = 0u;
    r[pl.off_meta + 3] = 0u;
  }

  // 4. zeros for the y rows the parts add into
  if (y_zero != nullptr) {
    const int q4 = d_v / 4;
    for (int x = threadIdx.x; x < n_own * q4; x += blockDim.x) {
      const int t = t0 + x / q4;
      float4* row = reinterpret_cast<float4*>(y_zero + ((static_cast<int64_t>(b) * T + t) * H + h) * d_v);
      row[x % q4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

struct PipeArgs {
  CUtensorMap state_map;  // M as rows [B*H*N, d_v] of the state dtype (fp8: code bytes), box C columns x 1 row
  CUtensorMap exps_map;   // fp8 state: the block exponents as rows [B*H*N, d_v/16] of bytes, box 16 x 1 row
  int8_t* exps;           // fp8 state: the block exponents [B, H, N, d_v/16] (after the codes)
  int B, T, H, N, d_v, W, R, parts;
  PipeLayout pl;
  const uint32_t* rec;  // [B, H, parts, T, pl.words]
  const void* v;        // [B, T, H, d_v] in dtype
  void* M;              // [B, H, N, d_v] state dtype, updated in place
  float* y;             // [B, T, H, d_v]: part 0's read sums
  float* y_other;       // [B, T, H, d_v]: part 1's read sums (parts == 2), added into y afterwards
  unsigned* err;
};

// Shared-memory bytes of k_scan_pipelined (host and device agree on this).
// fp8 state: the block exponents of the stage rows, 16 bytes a row (the TMA
// box of 16 exponents that covers the row's C columns) in groups of four rows
// 128 bytes apart (the landing spot of one four-row gather).
__host__ __device__ constexpr size_t pipe_exp_bytes(int P, int Wp, int Rp, int S) {
  return static_cast<size_t>((P * (Wp + Rp) + pipe_wstages(P, S) * Wp + 3) / 4) * 128;
}

// Entries one consumer-warp instruction covers: 32 lanes over the 16-byte
// units of a C-column row segment.
__host__ __device__ constexpr int pipe_entry_groups(int C, int s_state) { return 32 * 16 / (C * s_state); }

__host__ __device__ constexpr size_t pipe_smem_bytes(int P, int L, int Wp, int Rp, int words, int C, int s_state,
                                                     int s_in, int NWR, int S, bool fp8 = false) {
  return static_cast<size_t>(P) * (Wp + Rp) * C * s_state + static_cast<size_t>(pipe_wstages(P, S)) * Wp * C * s_state +
         (fp8 ? pipe_exp_bytes(P, Wp, Rp, S) : 0) +
         static_cast<size_t>(2) * L * words * 4 + static_cast<size_t>(2) * L * C * s_in +
         static_cast<size_t>(2) * S * NWR * pipe_entry_groups(C, s_state) * C * 4 + (2 * P + 2) * 8 + 128;
}

template <typename Tin, typename Tst, int C, int P, int L, int NWW, int NWR, int NP, int S>
__global__ void __launch_bounds__((NP + 1 + NWW + NWR) * kWarp, 1) k_scan_pipelined(const __grid_constant__ PipeArgs a) {
  constexpr int NT = (NP + 1 + NWW + NWR) * kWarp;
  constexpr bool kFp8 = std::is_same<Tst, Fp8Blk>::value;  // block-scaled fp8 state: 16 codes and one exponent a unit
  static_assert(!kFp8 || S == 1, "the fp8 state takes one token per step");
  constexpr int VE = 16 / sizeof(Tst);  // state elements per 16-byte unit
  constexpr int U = C / VE;             // units per row segment
  constexpr int RS = C * sizeof(Tst);   // bytes of a row segment
  constexpr int G = kWarp / U;          // entries per consumer-warp instruction
  static_assert(G == pipe_entry_groups(C, sizeof(Tst)), "the host sizes the read partials by the same count");
  static_assert(U >= 1 && U <= kWarp && kWarp % U == 0, "a row segment spans a divisor of the warp");
  static_assert(NT % U == 0, "gather lanes cover whole rows");
  static_assert(L >= P, "a chunk of records is staged before its tokens are gathered");
  static_assert(S == 1 || (S == 2 && L % 2 == 0 && P >= 5), "one or two tokens per step; pairs never straddle a chunk");
  constexpr int Q = pipe_wstages(P, S);  // written stages
  static_assert(P >= 3, "rows are gathered P - 1 >= 2 tokens ahead");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  // TMA boxes land at 128-byte aligned rows
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const PipeLayout pl = a.pl;
  const int Wp = pl.Wp, E = pl.Wp + pl.Rp, words = pl.words, T = a.T;
  unsigned char* lstage = smem;                                                    // [P][E][RS]
  unsigned char* wstage = lstage + static_cast<size_t>(P) * E * RS;               // [Q][Wp][RS]
  unsigned char* xstage = wstage + static_cast<size_t>(Q) * Wp * RS;              // fp8: exponents of the stage rows
  uint32_t* recbuf = reinterpret_cast<uint32_t*>(xstage + (kFp8 ? pipe_exp_bytes(P, Wp, pl.Rp, S) : 0));  // [2][L][words]
  Tin* vbuf = reinterpret_cast<Tin*>(recbuf + 2 * L * words);                      // [2][L][C]
  float* ybuf = reinterpret_cast<float*>(vbuf + 2 * L * C);                        // [2][S][NWR][G][C] read partials
  uint64_t* cbar = reinterpret_cast<uint64_t*>(ybuf + 2 * S * NWR * G * C);       // [2] record chunks
  uint64_t* full = cbar + 2;                                                       // [P] gathered stages
  uint64_t* done = full + P;  // [P] the consumers are through with a token, its stores fenced

  const int part = blockIdx.x % a.parts, bh = blockIdx.x / a.parts;
  const int b = bh / a.H, h = bh % a.H;
  const int c0 = blockIdx.y * C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  Tst* Mbh = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * a.N * a.d_v + c0;
  const uint32_t* rec_g = a.rec + (static_cast<int64_t>(bh) * a.parts + part) * T * words;
  const int64_t tok_step = static_cast<int64_t>(a.H) * a.d_v;  // [B, T, H, d_v] rows of one (b, h)
  float* y_bh = (part == 0 ? a.y : a.y_other) + static_cast<int64_t>(b) * T * tok_step +
                static_cast<int64_t>(h) * a.d_v + c0;
  const Tin* v_bh = static_cast<const Tin*>(a.v) + static_cast<int64_t>(b) * T * tok_step + static_cast<int64_t>(h) * a.d_v + c0;

  if (tid == 0) {
    for (int st = 0; st < P; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&done[st], 1);
    }
    mbar_init(&cbar[0], 1);
    mbar_init(&cbar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_chunks = (T + L - 1) / L;
  if (n_chunks == 0) return;
  int last_chunk = -1;  // thread 0: the last chunk whose copies it issued
  auto load_chunk = [&](int c) {  // thread 0: records and v rows of tokens [cL, cL + L)
    const int bi = c & 1, t0 = c * L, nt = min(L, T - t0);
    const uint32_t rb = static_cast<uint32_t>(nt) * words * 4u, vb = C * sizeof(Tin);
    mbar_arrive_expect_tx(&cbar[bi], rb + nt * vb);
    bulk_g2s(recbuf + static_cast<size_t>(bi) * L * words, rec_g + static_cast<int64_t>(t0) * words, rb, &cbar[bi]);
    for (int i = 0; i < nt; ++i)
      bulk_g2s(vbuf + (static_cast<size_t>(bi) * L + i) * C, v_bh + static_cast<int64_t>(t0 + i) * tok_step, vb,
               &cbar[bi]);
    last_chunk = c;
  };
  auto rec_of = [&](int t) { return recbuf + (static_cast<size_t>((t / L) & 1) * L + t % L) * words; };
  auto chunk_wait = [&](int c) { return mbar_wait_bounded(&cbar[c & 1], (c >> 1) & 1, a.err); };
  // Token u's rows of this part into stage u % P with TMA row gathers, four
  // rows an instruction (padding rows of a partial group read a neighbour row
  // or the zero fill; they are never used), issued by the producer warps'
  // lanes; thread 0 arms the stage's barrier with the token's bytes.
  auto gather = [&](int u) {
    const uint32_t* rec = rec_of(u);
    const int nw = static_cast<int>(rec[pl.off_meta]), nr = static_cast<int>(rec[pl.off_meta + 1]);
    const int gw = (nw + 3) / 4, gr = (nr + 3) / 4;
    uint64_t* bar = &full[u % P];
    if (tid == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(gw + gr) * 4u * (RS + (kFp8 ? 16 : 0)));
    const int row0 = bh * a.N;
    for (int g = warp + NP * lane; g < gw + gr; g += NP * kWarp) {
      const bool wr = g < gw;
      const int e = wr ? 4 * g : 4 * (g - gw);
      const uint4 sl = *reinterpret_cast<const uint4*>(rec + (wr ? pl.off_slot_w : pl.off_slot_r) + e);
      const int r = (u % P) * E + (wr ? e : Wp + e);  // stage row of the group's first row (a multiple of 4)
      const int r0 = row0 + static_cast<int>(sl.x), r1 = row0 + static_cast<int>(sl.y);
      const int r2 = row0 + static_cast<int>(sl.z), r3 = row0 + static_cast<int>(sl.w);
      tma_gather4(lstage + static_cast<size_t>(r) * RS, &a.state_map, c0, r0, r1, r2, r3, bar);
      // fp8: the 16-exponent box (16-byte aligned) that holds this tile's U exponents
      if constexpr (kFp8) tma_gather4(xstage + static_cast<size_t>(r >> 2) * 128, &a.exps_map, (c0 / 16) & ~15, r0, r1, r2, r3, bar);
    }
  };
  int last_gathered = -1;  // producer threads: the last token whose rows they requested
  auto finish = [&]() {  // a producer's copies in flight land before it exits
    if (tid == 0)
      for (int c = max(0, last_chunk - 1); c <= last_chunk; ++c) mbar_wait_bounded(&cbar[c & 1], (c >> 1) & 1, a.err);
    for (int u = max(0, last_gathered - P + 1); u <= last_gathered; ++u)
      mbar_wait_bounded(&full[u % P], (u / P) & 1, a.err);
  };

  // Warp roles: NP producers (row gathers, record chunks), one control warp,
  // NWW writers, NWR readers. The control warp and the consumers (writers and
  // readers) meet at one barrier per token; the control warp does all the
  // waiting on copies and signalling, so that the consumers' chain from one
  // barrier to the next holds only their own loads, arithmetic and stores.
  // The producers run up to P - 1 tokens ahead, paced by mbarriers.
  const bool producer = warp < NP;
  const bool control = warp == NP;
  const bool writer = warp > NP && warp <= NP + NWW;
  const int cw = warp - NP - 1;  // consumer warp index: writers, then readers
  // Consumer lanes take unit lane % U of entries lane / U + k G: one warp
  // instruction covers every unit of G rows, all 32 banks.
  const int qw = lane % U;
  constexpr int stride_w = NWW * kWarp;  // write units per pass of the write warps
  constexpr int stride_r = G * NWR;      // read entries per pass of the read warps
  const int base_w = cw * kWarp + lane;
  const int base_r = (cw - NWW) * G + lane / U;
  auto row_at = [&](uint32_t src) { return *reinterpret_cast<const uint4*>(smem + static_cast<size_t>(src) * RS + qw * 16); };
  // The state as fp32 and back, per 16-byte unit: bf16 / fp32 by bits, the
  // fp8 state with the unit's block exponent (this tile's U exponents sit at
  // xoff .. xoff + U - 1 of a row's 16-byte exponent box).
  const int xoff = (c0 / 16) & 15;
  auto exp_byte = [&](uint32_t row) -> unsigned char& {
    return xstage[static_cast<size_t>(row >> 2) * 128 + (row & 3) * 16 + xoff + qw];
  };
  auto load_row = [&](uint32_t src, float (&m)[VE]) {
    if constexpr (kFp8) fp8blk_unpack16(row_at(src), static_cast<int8_t>(exp_byte(src)), m);
    else unpack_unit<Tst>(row_at(src), m);
  };
  auto as_stored = [&](float (&m)[VE]) {  // m rounded as the state holds it
    if constexpr (kFp8) {
      uint4 q;
      const int e = fp8blk_pack16(m, &q);
      fp8blk_unpack16(q, e, m);
    } else {
      unpack_unit<Tst>(pack16<Tst>(m), m);
    }
  };
  int8_t* Mx = kFp8 ? a.exps + static_cast<int64_t>(bh) * a.N * (a.d_v / 16) + c0 / 16 + qw : nullptr;
  // m, rounded to the state type, into written-stage row wrow and, unless
  // slot < 0, into the state in HBM
  auto store_row = [&](const float (&m)[VE], uint32_t wrow, int64_t slot) {
    unsigned char* dst = smem + static_cast<size_t>(wrow) * RS + qw * 16;
    if constexpr (kFp8) {
      uint4 q;
      const int e = fp8blk_pack16(m, &q);
      *reinterpret_cast<uint4*>(dst) = q;
      exp_byte(wrow) = static_cast<unsigned char>(static_cast<int8_t>(e));
      if (slot >= 0) {
        *reinterpret_cast<uint4*>(Mbh + qw * VE + slot * a.d_v) = q;
        Mx[slot * (a.d_v / 16)] = static_cast<int8_t>(e);
      }
    } else {
      const uint4 pk = pack16<Tst>(m);
      *reinterpret_cast<uint4*>(dst) = pk;
      if (slot >= 0) *reinterpret_cast<uint4*>(Mbh + qw * VE + slot * a.d_v) = pk;
    }
  };
  // Token t on this consumer thread. Every row it reads is complete: the
  // token's gathered stage and the written stages of the tokens before it.
  auto compute = [&](int t) {
    const uint32_t* rec = rec_of(t);
    const int nw = static_cast<int>(rec[pl.off_meta]), nr = static_cast<int>(rec[pl.off_meta + 1]);
    const uint16_t* sw = reinterpret_cast<const uint16_t*>(rec + pl.off_src_w);
    const float2* ac = reinterpret_cast<const float2*>(rec + pl.off_awcw);
    float vv[VE];
    load_in_vec<Tin, VE>(vbuf + (static_cast<size_t>((t / L) & 1) * L + t % L) * C + qw * VE, vv);
    // the write of entry j on this thread's unit of its source row (fp32 math, state rounding by the caller)
    auto written = [&](int j, float (&m)[VE]) {
      load_row(sw[j] & kRowMask, m);
      const float2 c = ac[j];
      write_unit<VE>(m, vv, c.x, c.y);
    };
    if (writer) {
      const uint32_t wbase = static_cast<uint32_t>(P * E + (t % Q) * Wp);  // this token's written stage
      const uint32_t* slw = rec + pl.off_slot_w;
      const int n = nw * U;
      for (int p0 = base_w; p0 < n; p0 += 2 * stride_w) {  // two independent units per pass
        const int p1 = p0 + stride_w;
        const bool has1 = p1 < n;
        const int j0 = p0 / U, j1 = has1 ? p1 / U : j0;
        float m0[VE], m1[VE];
        written(j0, m0);
        written(j1, m1);
        store_row(m0, wbase + j0, slw[j0]);
        if (has1) store_row(m1, wbase + j1, slw[j1]);
      }
    } else {
      const uint16_t* sr = reinterpret_cast<const uint16_t*>(rec + pl.off_src_r);
      const float* qr = reinterpret_cast<const float*>(rec + pl.off_q_r);
      // a read of a slot this token writes: that write, rounded as stored
      auto same_token = [&](uint32_t src, float (&m)[VE]) {
        written(static_cast<int>(src & kEntryMask), m);
        as_stored(m);
      };
      float acc[VE];
#pragma unroll
      for (int j = 0; j < VE; ++j) acc[j] = 0.f;
      for (int i0 = base_r; i0 < nr; i0 += 2 * stride_r) {
        const int i1 = i0 + stride_r;
        const bool has1 = i1 < nr;
        const uint32_t src0 = sr[i0], src1 = sr[has1 ? i1 : i0];
        // both rows first (a flagged code's low bits still name a row in
        // shared memory), the rare recomputation after: no branch between them
        float m0[VE], m1[VE];
        load_row(src0 & kRowMask, m0);
        load_row(src1 & kRowMask, m1);
        if ((src0 | src1) & kSrcSameToken) {
          if (src0 & kSrcSameToken) same_token(src0, m0);
          if (src1 & kSrcSameToken) same_token(src1, m1);
        }
        read_unit<VE>(acc, m0, qr[i0]);
        read_unit<VE>(acc, m1, has1 ? qr[i1] : 0.0f);
      }
      // this lane's sums of its unit over its entry group; the control warp adds
      // the NWR * G groups of a column in a fixed order
      float* yb = ybuf + ((static_cast<size_t>(t & 1) * NWR + (cw - NWW)) * G + lane / U) * C + qw * VE;
#pragma unroll
      for (int j = 0; j < VE; j += 4) *reinterpret_cast<float4*>(yb + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
    }
  };
  // Tokens ta and ta + 1 (if hb) on this consumer thread, interleaved. Rows
  // that the first token writes and the second one reads or rewrites are
  // recomputed from the first token's source (as stored, rounded to the state
  // type), so the two tokens need no barrier between them; per token, every
  // value and every sum comes out as in the one-token step.
  auto compute_pair = [&](int ta, bool hb) {
    const int tb = ta + 1;
    const uint32_t* recA = rec_of(ta);
    const uint32_t* recB = hb ? rec_of(tb) : recA;
    const uint16_t* swA = reinterpret_cast<const uint16_t*>(recA + pl.off_src_w);
    const uint16_t* swB = reinterpret_cast<const uint16_t*>(recB + pl.off_src_w);
    const float2* acA = reinterpret_cast<const float2*>(recA + pl.off_awcw);
    const float2* acB = reinterpret_cast<const float2*>(recB + pl.off_awcw);
    float vA[VE], vB[VE];
    load_in_vec<Tin, VE>(vbuf + (static_cast<size_t>((ta / L) & 1) * L + ta % L) * C + qw * VE, vA);
    load_in_vec<Tin, VE>(vbuf + (static_cast<size_t>(((hb ? tb : ta) / L) & 1) * L + (hb ? tb : ta) % L) * C + qw * VE, vB);
    auto writtenA = [&](int j, float (&m)[VE]) {  // the first token's write j (unrounded)
      load_row(swA[j] & kRowMask, m);
      const float2 c = acA[j];
      write_unit<VE>(m, vA, c.x, c.y);
    };
    auto writtenB = [&](int j, float (&m)[VE]) {  // the second token's write j (unrounded)
      const uint32_t src = swB[j];
      if (src & kSrcPrevToken) {
        writtenA(static_cast<int>(src & kEntryMask), m);
        as_stored(m);
      } else {
        load_row(src & kRowMask, m);
      }
      const float2 c = acB[j];
      write_unit<VE>(m, vB, c.x, c.y);
    };
    if (writer) {
      const uint32_t wbA = static_cast<uint32_t>(P * E + (ta % Q) * Wp);  // the two tokens' written stages
      const uint32_t wbB = static_cast<uint32_t>(P * E + (tb % Q) * Wp);
      const uint32_t* slwA = recA + pl.off_slot_w;
      const uint32_t* slwB = recB + pl.off_slot_w;
      const int nA = static_cast<int>(recA[pl.off_meta]) * U;
      const int nB = hb ? static_cast<int>(recB[pl.off_meta]) * U : 0;
      for (int p0 = base_w; p0 < max(nA, nB); p0 += kTokW * stride_w) {
        // every unit computed from a record entry (past the counts: padding
        // entries, in-bounds rows, zero coefficients); only the stores are
        // conditional
        int j[kTokW];
        uint32_t srcB[kTokW];
        float mA[kTokW][VE], mB[kTokW][VE];
#pragma unroll
        for (int k = 0; k < kTokW; ++k) {
          j[k] = min((p0 + k * stride_w) / U, Wp - 1);
          srcB[k] = swB[j[k]];
          load_row(swA[j[k]] & kRowMask, mA[k]);
          load_row(srcB[k] & kRowMask, mB[k]);
        }
#pragma unroll
        for (int k = 0; k < kTokW; ++k) {
          if (srcB[k] & kSrcPrevToken) {  // rare: the first token's write of the slot, as stored
            writtenA(static_cast<int>(srcB[k] & kEntryMask), mB[k]);
            as_stored(mB[k]);
          }
        }
#pragma unroll
        for (int k = 0; k < kTokW; ++k) {
          const float2 ca = acA[j[k]], cb = acB[j[k]];
          write_unit<VE>(mA[k], vA, ca.x, ca.y);
          write_unit<VE>(mB[k], vB, cb.x, cb.y);
        }
#pragma unroll
        for (int k = 0; k < kTokW; ++k) {
          const int p = p0 + k * stride_w;
          if (p < nA)
            store_row(mA[k], wbA + j[k], (swA[j[k]] & kSkipStore) ? int64_t{-1} : static_cast<int64_t>(slwA[j[k]]));
          if (p < nB) store_row(mB[k], wbB + j[k], slwB[j[k]]);
        }
      }
    } else {
      const uint16_t* srA = reinterpret_cast<const uint16_t*>(recA + pl.off_src_r);
      const uint16_t* srB = reinterpret_cast<const uint16_t*>(recB + pl.off_src_r);
      const float* qrA = reinterpret_cast<const float*>(recA + pl.off_q_r);
      const float* qrB = reinterpret_cast<const float*>(recB + pl.off_q_r);
      const int nA = static_cast<int>(recA[pl.off_meta + 1]);
      const int nB = hb ? static_cast<int>(recB[pl.off_meta + 1]) : 0;
      float accA[VE], accB[VE];
#pragma unroll
      for (int j = 0; j < VE; ++j) accA[j] = accB[j] = 0.f;
      for (int i0 = base_r; i0 < max(nA, nB); i0 += kTokR * stride_r) {
        int i[kTokR];
        uint32_t sA[kTokR], sB[kTokR];
        float mA[kTokR][VE], mB[kTokR][VE];
#pragma unroll
        for (int k = 0; k < kTokR; ++k) {
          i[k] = min(i0 + k * stride_r, pl.Rp - 1);
          sA[k] = srA[i[k]];
          sB[k] = srB[i[k]];
          load_row(sA[k] & kRowMask, mA[k]);
          load_row(sB[k] & kRowMask, mB[k]);
        }
#pragma unroll
        for (int k = 0; k < kTokR; ++k) {  // rare: reads of rows this step writes, as stored
          if (sA[k] & kSrcSameToken) {
            writtenA(static_cast<int>(sA[k] & kEntryMask), mA[k]);
            as_stored(mA[k]);
          }
          if (sB[k] & (kSrcSameToken | kSrcPrevToken)) {
            if (sB[k] & kSrcSameToken) writtenB(static_cast<int>(sB[k] & kEntryMask), mB[k]);
            else writtenA(static_cast<int>(sB[k] & kEntryMask), mB[k]);
            as_stored(mB[k]);
          }
        }
#pragma unroll
        for (int k = 0; k < kTokR; ++k) {  // rows past a token's count may hold anything: not summed
          const int ik = i0 + k * stride_r;
          if (ik < nA) read_unit<VE>(accA, mA[k], qrA[i[k]]);
          if (ik < nB) read_unit<VE>(accB, mB[k], qrB[i[k]]);
        }
      }
      float* yb = ybuf + ((static_cast<size_t>((ta / 2) & 1) * 2 * NWR + (cw - NWW)) * G + lane / U) * C + qw * VE;
#pragma unroll
      for (int j = 0; j < VE; j += 4) {
        *reinterpret_cast<float4*>(yb + j) = make_float4(accA[j], accA[j + 1], accA[j + 2], accA[j + 3]);
        *reinterpret_cast<float4*>(yb + NWR * G * C + j) = make_float4(accB[j], accB[j + 1], accB[j + 2], accB[j + 3]);
      }
    }
  };

  if (producer) {
    if (tid == 0) {
      load_chunk(0);
      if (n_chunks > 1) load_chunk(1);
    }
#pragma unroll 1
    for (int u = 0; u < T; ++u) {
      // Stage u % P held token u - P: the consumers are through with it, and
      // the writes of every token up to u - P were fenced (the hazard plan
      // forwards rows written by tokens u - P + 1 .. u - 1 from shared memory).
      // Tokens finish in order, so one wait serves two: an even token waits for
      // token u - P + 1, which also frees the stage of the odd token after it.
      const int need = u < P ? -1 : (u % 2 == 0 ? u - P + 1 : (u - 1 < P ? u - P : -1));
      bool ok = need < 0 || mbar_wait_backoff(&done[need % P], (need / P) & 1, a.err);
      if (ok && u % L == 0) ok = chunk_wait(u / L);
      if (!ok) break;
      const int c = u / L;
      if (tid == 0 && u % L == P - 1 && c >= 1 && c + 1 < n_chunks) {
        fence_proxy_async_smem();
        load_chunk(c + 1);  // the consumers are through with chunk c - 1 (token cL - 1 is done)
      }
      gather(u);
      last_gathered = u;
    }
    finish();
    return;
  }
  constexpr int kBarThreads = (1 + NWW + NWR) * kWarp;  // the control warp and the consumers
  const int n_steps = (T + S - 1) / S;                  // a step: S consecutive tokens
  if (control) {
    // y of token u: the read lanes' partial sums, added in (read warp, entry
    // group) order, two adjacent columns a lane
    auto put_y = [&](int u) {
      static_assert(C % 2 == 0 && C <= 2 * kWarp, "one column pair a lane");
      if (2 * lane < C) {
        const float* yb = ybuf + (static_cast<size_t>((u / S) & 1) * S + u % S) * NWR * G * C + 2 * lane;
        float2 acc = *reinterpret_cast<const float2*>(yb);
#pragma unroll
        for (int k = 1; k < NWR * G; ++k) {
          const float2 p = *reinterpret_cast<const float2*>(yb + k * C);
          acc.x += p.x;
          acc.y += p.y;
        }
        *reinterpret_cast<float2*>(y_bh + static_cast<int64_t>(u) * tok_step + 2 * lane) = acc;
      }
    };
    auto ready = [&](int u) {  // token u's records and rows are in shared memory
      const bool ok = u % L != 0 || chunk_wait(u / L);
      return ok && mbar_wait_bounded(&full[u % P], (u / P) & 1, a.err);
    };
    bool ok = true;
    for (int u = 0; u < S && u < T; ++u) ok = ok && ready(u);
#pragma unroll 1
    for (int st = 0; st < n_steps; ++st) {
      if (named_barrier_or(1, kBarThreads, !ok)) return;  // step st - 1 is complete, step st's rows have landed
      if (st > 0) {
        for (int u = (st - 1) * S; u < st * S; ++u) put_y(u);
        __syncwarp();
        if (lane == 0)
          for (int u = (st - 1) * S; u < st * S; ++u) mbar_arrive(&done[u % P]);
      }
      for (int u = (st + 1) * S; u < (st + 2) * S && u < T; ++u) ok = ok && ready(u);
    }
    if (!named_barrier_or(1, kBarThreads, !ok))
      for (int u = (n_steps - 1) * S; u < T; ++u) put_y(u);
    return;
  }
  // consumers
#pragma unroll 1
  for (int st = 0; st < n_steps; ++st) {
    // the state rows this thread stored in step st - 1 become visible to the
    // gathers that the producers issue after the control warp's signal
    if (writer && st > 0) fence_proxy_async_global();
    if (named_barrier_or(1, kBarThreads, false)) return;
    if constexpr (S == 1) compute(st);
    else compute_pair(2 * st, 2 * st + 1 < T);
  }
  named_barrier_or(1, kBarThreads, false);
}

}  // namespace sdm
