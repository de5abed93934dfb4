// One decode step of the SDM layer in one launch (sm_100a).
//
// For T = 1 (a new token per batch row, the state carried across calls) the
// whole layer is small and latency-bound: selection of k' and q' (SDM
// explainer, section 3.1 step 1), the gated delta write (step 2), the read
// after the write (step 3) and the optional RMS-norm x gate. One CTA per
// (b, h) does all of it: warp 0 selects the W write slots (the register-path
// selection of pkm_topk_fast.cuh, same order and weights as sdm_pkm_topk);
// then warps 0 and 2..7 update the 16-byte units of the W written rows in
// global memory (m <- fma(alpha (1 - beta k), m, (beta k) v), rounded to the
// state dtype on store, as the recurrence kernels do) while warp 1 selects the
// R read slots; after a barrier the R read rows are summed into y, each
// column's entries split into groups whose partial sums are added in group
// order. Slots of one token are distinct, so the writes need no ordering
// among themselves and their loads can all be issued before any store.
#pragma once

#include <type_traits>

#include "pkm_topk_fast.cuh"
#include "sdm_fp8.cuh"
#include "sdm_scan.cuh"

namespace sdm {

constexpr int kDecodeThreads = 256;

struct DecodeArgs {
  int H, N, d_v, K;  // K = W = R
  float eps;
  FastTopkLayout L;
  const void* kp;     // [B, 1, H, 2 sqrtN] Tin
  const void* qp;     // [B, 1, H, 2 sqrtN] Tin
  const void* v;      // [B, 1, H, d_v] Tin
  const void* alpha;  // [B, 1, H] Tin
  const void* beta;   // [B, 1, H] Tin
  const void* g;      // [B, 1, H, d_v] Tin or null
  void* M;            // [B, H, N, d_v] Tst, updated in place (fp8: the codes)
  int8_t* exps;       // fp8 state only: [B, H, N, d_v / 16] block exponents
  float* y;           // [B, 1, H, d_v]
  uint32_t sel_off;   // byte offsets in shared memory
  uint32_t part_off;
  unsigned* err;
};

// Shared memory: candidate table | 2 selection scratches | idx_w, w_w, idx_r,
// w_r [K] each | read partial sums [groups][d_v].
template <typename Tin, typename Tst, int E, int EH, int EPL, int CP>
__global__ void __launch_bounds__(kDecodeThreads) k_decode_step(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid / kWarp;
  const int bh = blockIdx.x;  // = b * H + h = the token-head of this step
  const int K = a.K, N = a.N, d_v = a.d_v;
  uint16_t* tab = reinterpret_cast<uint16_t*>(smem);
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + a.sel_off);  // [2K]: write slots, then read slots
  float* sw = reinterpret_cast<float*>(sidx + 2 * K);             // [2K]: their weights
  float* part = reinterpret_cast<float*>(smem + a.part_off);

  if (warp == 0) fast_topk_build_table(tab, a.L.Kh, K, lane_id());
  __syncthreads();
  // state columns per 16-byte unit (the fp8 tag is one byte per value)
  constexpr int VE = std::is_same<Tst, Fp8Blk>::value ? 16 : 16 / static_cast<int>(sizeof(Tst));
  const int UR = d_v / VE;                                 // units per row
  Tst* Mbh = static_cast<Tst*>(a.M) + static_cast<int64_t>(bh) * N * d_v;
  if (warp == 1) {
    // The read selection runs while the other warps apply the writes.
    unsigned char* ws = smem + a.L.table_bytes + a.L.warp_bytes;
    fast_topk_unit<Tin, E, EH, EPL, CP>(static_cast<const Tin*>(a.qp) + static_cast<int64_t>(bh) * 2 * a.L.n, a.L,
                                        tab, ws, sidx + K, sw + K);
  } else {
    if (warp == 0)
      fast_topk_unit<Tin, E, EH, EPL, CP>(static_cast<const Tin*>(a.kp) + static_cast<int64_t>(bh) * 2 * a.L.n,
                                          a.L, tab, smem + a.L.table_bytes, sidx, sw);
    // Warps 0 and 2..7 meet once the write slots are known.
    asm volatile("bar.sync 1, %0;\n" ::"r"(kDecodeThreads - kWarp) : "memory");
    const Tin* vrow = static_cast<const Tin*>(a.v) + static_cast<int64_t>(bh) * d_v;
    const float alpha = to_f32<Tin>(static_cast<const Tin*>(a.alpha)[bh]);
    const float beta = to_f32<Tin>(static_cast<const Tin*>(a.beta)[bh]);
    const int tw = warp == 0 ? tid : tid - kWarp;  // 0 .. 223
    constexpr int kWriters = kDecodeThreads - kWarp;
    constexpr int kBatch = 8;  // units loaded before any is stored (the rows are distinct)
    // Write: unit u of row idx_w[e], for every (e, u).
    for (int x0 = tw; x0 < K * UR; x0 += kWriters * kBatch) {
      uint4 raw[kBatch];
      int sl[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int x = x0 + j * kWriters;
        sl[j] = -1;
        if (x < K * UR) {
          const int e = x / UR, u = x - e * UR;
          const int s = sidx[e];
          if (static_cast<unsigned>(s) < static_cast<unsigned>(N)) {
            sl[j] = s;
            raw[j] = *reinterpret_cast<const uint4*>(Mbh + static_cast<int64_t>(s) * d_v + u * VE);
          } else {
            atomicOr(a.err, kErrIndexOutOfRange);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (sl[j] < 0) continue;
        const int x = x0 + j * kWriters;
        const int e = x / UR, u = x - e * UR;
        const float cw = beta * sw[e];
        const float aw = alpha * (1.0f - cw);
        float m[VE], vv[VE];
        load_in_vec<Tin, VE>(vrow + u * VE, vv);
        uint4* dst = reinterpret_cast<uint4*>(Mbh + static_cast<int64_t>(sl[j]) * d_v + u * VE);
        if constexpr (std::is_same<Tst, Fp8Blk>::value) {
          int8_t* ex = a.exps + (static_cast<int64_t>(bh) * N + sl[j]) * (d_v / 16) + u;
          fp8blk_unpack16(raw[j], *ex, m);
#pragma unroll
          for (int i = 0; i < VE; ++i) m[i] = __fmaf_rn(aw, m[i], __fmul_rn(cw, vv[i]));
          uint4 q;
          *ex = static_cast<int8_t>(fp8blk_pack16(m, &q));
          *dst = q;
        } else {
          unpack16<Tst>(raw[j], m);
#pragma unroll
          for (int i = 0; i < VE; ++i) m[i] = __fmaf_rn(aw, m[i], __fmul_rn(cw, vv[i]));
          *dst = pack16<Tst>(m);
        }
      }
    }
  }
  __syncthreads();

  // Read: groups of entries per unit, partial sums in shared memory.
  const int groups = UR >= kDecodeThreads ? 1 : kDecodeThreads / UR;
  for (int x = tid; x < groups * UR; x += kDecodeThreads) {
    const int gi = x / UR, u = x - gi * UR;
    float acc[VE];
#pragma unroll
    for (int j = 0; j < VE; ++j) acc[j] = 0.0f;
    for (int e = gi; e < K; e += groups) {
      const int s = sidx[K + e];
      if (static_cast<unsigned>(s) >= static_cast<unsigned>(N)) {
        atomicOr(a.err, kErrIndexOutOfRange);
        continue;
      }
      const float q = sw[K + e];
      float m[VE];
      const uint4 raw = *reinterpret_cast<const uint4*>(Mbh + static_cast<int64_t>(s) * d_v + u * VE);
      if constexpr (std::is_same<Tst, Fp8Blk>::value)
        fp8blk_unpack16(raw, a.exps[(static_cast<int64_t>(bh) * N + s) * (d_v / 16) + u], m);
      else
        unpack16<Tst>(raw, m);
#pragma unroll
      for (int j = 0; j < VE; ++j) acc[j] = __fmaf_rn(q, m[j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < VE; ++j) part[gi * d_v + u * VE + j] = acc[j];
  }
  __syncthreads();
  float* yrow = a.y + static_cast<int64_t>(bh) * d_v;
  float ss = 0.0f;
  for (int c = tid; c < d_v; c += kDecodeThreads) {
    float acc = 0.0f;
    for (int gi = 0; gi < groups; ++gi) acc += part[gi * d_v + c];
    part[c] = acc;  // group 0's slot is read only by this thread
    ss = __fmaf_rn(acc, acc, ss);
  }
  if (a.g == nullptr) {
    for (int c = tid; c < d_v; c += kDecodeThreads) yrow[c] = part[c];
    return;
  }
  // RMS-norm x gate over the row (the epilogue kernel's formula).
  __shared__ float red[kDecodeThreads / kWarp];
  ss = warp_sum(ss);
  if (lane_id() == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int w = 0; w < kDecodeThreads / kWarp; ++w) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(d_v) + a.eps);
  const Tin* grow = static_cast<const Tin*>(a.g) + static_cast<int64_t>(bh) * d_v;
  for (int c = tid; c < d_v; c += kDecodeThreads) yrow[c] = to_f32<Tin>(grow[c]) * part[c] * inv;
}

}  // namespace sdm
