// Product-key top-k slot selection (sm_100a).
//
// SDM explainer (papers.ananclaw.com), section 3.1 step 1; Technical Summary:
// Sparse Delta Memory, Core Mechanism 2: the score vector x of length 2*sqrtN
// is split into s1 = x[0:sqrtN] and s2 = x[sqrtN:]; slot i = a*sqrtN + b has
// score s1[a] + s2[b]; the top-K slots follow from
// topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)), so the N sums are never formed.
//
// One warp owns one token-head:
//   1. per half, the top-Kh (Kh = min(K, sqrtN)) values by (value desc, index
//      asc): radix select of the Kh-th largest order key (4 passes of 8-bit
//      digits over a shared histogram), ballot compaction, rank sort;
//   2. candidates: per-half ranks (ra, rb) with (ra+1)(rb+1) <= K -- any other
//      pair is preceded by at least K pairs, so it cannot be selected;
//   3. exact pair scores as fp32 TwoSum (hi, lo); radix select on hi, ties in
//      hi resolved by (lo desc, slot asc), then a rank sort of the K winners.
//      (hi, lo) compared lexicographically orders the exact real sums because
//      round-to-nearest is monotone;
//   4. softmax of the K selected scores (fp32 hi), written in selection order.
#pragma once

#include "sdm_device.cuh"

namespace sdm {

// Byte offsets of one warp's scratch area and the sizes that drive it.
struct TopkLayout {
  int n;   // sqrtN
  int K;   // slots to select
  int Kh;  // per-half selection size, min(K, n)
  int C;   // candidate pairs with (ra+1)(rb+1) <= K
  uint32_t table_bytes;  // block-shared candidate table, at offset 0
  uint32_t warp_bytes;
  uint32_t vals, hist, hkey, hval, hidx, c_hi, c_lo, c_slot, tie, f_hi, f_lo, f_slot;
};

// k-th largest (1-based) of the keys key(e), e in [0, n), with the number of
// keys strictly greater than it. All lanes of the warp call it together.
template <class KeyFn>
__device__ __forceinline__ void warp_radix_kth_largest(KeyFn key, int n, int k, uint32_t* hist,
                                                       uint32_t& thr, int& n_greater) {
  const int lane = lane_id();
  uint32_t prefix = 0, mask = 0;
  int rem = k, gt = 0;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += kWarp) hist[i] = 0;
    __syncwarp();
    for (int e = lane; e < n; e += kWarp) {
      const uint32_t kk = key(e);
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 255u], 1u);
    }
    __syncwarp();
    // Lane l owns bins 255-8l .. 248-8l, visited from the top.
    uint32_t c[8];
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = hist[255 - 8 * lane - j];
      s += c[j];
    }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t excl = incl - s;
    const bool mine = excl < static_cast<uint32_t>(rem) && static_cast<uint32_t>(rem) <= incl;
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    int digit = 0;
    uint32_t above = 0;
    if (mine) {
      uint32_t acc = excl;
      bool found = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!found && acc + c[j] >= static_cast<uint32_t>(rem)) {
          digit = 255 - 8 * lane - j;
          above = acc;
          found = true;
        }
        acc += c[j];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    rem -= static_cast<int>(above);
    gt += static_cast<int>(above);
    prefix |= static_cast<uint32_t>(digit) << shift;
    mask |= 0xFFu << shift;
    __syncwarp();
  }
  thr = prefix;
  n_greater = gt;
}

// Top-Kh of one half v[0:n) by (value desc, index asc), sorted, into
// hval/hidx[0:Kh). hkey is scratch of Kh 64-bit keys.
__device__ __forceinline__ void warp_half_topk(const float* v, int n, int Kh, uint32_t* hist,
                                               uint64_t* hkey, float* hval, int32_t* hidx) {
  const int lane = lane_id();
  // key64 = ord(value) : (0xFFFFFFFF - index); larger key = earlier in the order.
  if (Kh == n) {
    for (int e = lane; e < n; e += kWarp)
      hkey[e] = (static_cast<uint64_t>(ord_f32(v[e])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
  } else {
    uint32_t thr;
    int ngt;
    warp_radix_kth_largest([&](int e) { return ord_f32(v[e]); }, n, Kh, hist, thr, ngt);
    const int rem = Kh - ngt;
    int cnt = 0, eq_seen = 0;
    const uint32_t lt = lanemask_lt();
    for (int e0 = 0; e0 < n; e0 += kWarp) {
      const int e = e0 + lane;
      const bool valid = e < n;
      const uint32_t k = valid ? ord_f32(v[e]) : 0u;
      const bool gt = valid && k > thr;
      const bool eq = valid && k == thr;
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      const bool take = gt || (eq && eq_seen + __popc(be & lt) < rem);
      const uint32_t bt = __ballot_sync(0xffffffffu, take);
      if (take)
        hkey[cnt + __popc(bt & lt)] =
            (static_cast<uint64_t>(k) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
      cnt += __popc(bt);
      eq_seen += __popc(be);
    }
  }
  __syncwarp();
  for (int i = lane; i < Kh; i += kWarp) {
    const uint64_t ki = hkey[i];
    int rank = 0;
    for (int j = 0; j < Kh; ++j) rank += hkey[j] > ki;
    hval[rank] = unord_f32(static_cast<uint32_t>(ki >> 32));
    hidx[rank] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(ki));
  }
  __syncwarp();
}

template <typename Tin>
__global__ void __launch_bounds__(128) k_pkm_topk_general(const Tin* __restrict__ scores, int64_t n_units,
                                                  TopkLayout L, int32_t* __restrict__ idx_out,
                                                  float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warps = blockDim.x / kWarp;
  const int warp = threadIdx.x / kWarp;
  const int lane = lane_id();
  const int n = L.n, K = L.K, Kh = L.Kh, C = L.C;

  // Candidate table: rows ra in [0, Kh) of length min(Kh, K / (ra + 1)).
  uint16_t* tab = reinterpret_cast<uint16_t*>(smem);
  if (warp == 0) {
    int base = 0;
    for (int r0 = 0; r0 < Kh; r0 += kWarp) {
      const int ra = r0 + lane;
      const int len = ra < Kh ? min(Kh, K / (ra + 1)) : 0;
      int incl = len;
#pragma unroll
      for (int o = 1; o < kWarp; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int start = base + incl - len;
      for (int rb = 0; rb < len; ++rb) {
        tab[2 * (start + rb)] = static_cast<uint16_t>(ra);
        tab[2 * (start + rb) + 1] = static_cast<uint16_t>(rb);
      }
      base += __shfl_sync(0xffffffffu, incl, kWarp - 1);
    }
  }
  __syncthreads();

  unsigned char* ws = smem + L.table_bytes + static_cast<size_t>(warp) * L.warp_bytes;
  float* vals = reinterpret_cast<float*>(ws + L.vals);
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  uint64_t* hkey = reinterpret_cast<uint64_t*>(ws + L.hkey);
  float* hval = reinterpret_cast<float*>(ws + L.hval);
  int32_t* hidx = reinterpret_cast<int32_t*>(ws + L.hidx);
  uint32_t* c_hi = reinterpret_cast<uint32_t*>(ws + L.c_hi);
  uint32_t* c_lo = reinterpret_cast<uint32_t*>(ws + L.c_lo);
  int32_t* c_slot = reinterpret_cast<int32_t*>(ws + L.c_slot);
  uint16_t* tie = reinterpret_cast<uint16_t*>(ws + L.tie);
  uint32_t* f_hi = reinterpret_cast<uint32_t*>(ws + L.f_hi);
  uint32_t* f_lo = reinterpret_cast<uint32_t*>(ws + L.f_lo);
  int32_t* f_slot = reinterpret_cast<int32_t*>(ws + L.f_slot);
  const uint32_t lt = lanemask_lt();

  for (int64_t unit = static_cast<int64_t>(blockIdx.x) * warps + warp; unit < n_units;
       unit += static_cast<int64_t>(gridDim.x) * warps) {
    const Tin* x = scores + unit * 2 * n;
    for (int e = lane; e < 2 * n; e += kWarp) vals[e] = canon_zero(to_f32<Tin>(x[e]));
    __syncwarp();

    // 1. per-half top-Kh, sorted.
    warp_half_topk(vals, n, Kh, hist, hkey, hval, hidx);
    warp_half_topk(vals + n, n, Kh, hist, hkey, hval + Kh, hidx + Kh);

    // 2-3. candidate pairs with exact scores.
    for (int c = lane; c < C; c += kWarp) {
      const int ra = tab[2 * c], rb = tab[2 * c + 1];
      float hi, lo;
      two_sum(hval[ra], hval[Kh + rb], hi, lo);
      c_hi[c] = ord_f32(canon_zero(hi));
      c_lo[c] = ord_f32(canon_zero(lo));
      c_slot[c] = hidx[ra] * n + hidx[Kh + rb];
    }
    __syncwarp();
    uint32_t thr;
    int ngt;
    warp_radix_kth_largest([&](int c) { return c_hi[c]; }, C, K, hist, thr, ngt);
    int nf = 0, ntie = 0;
    for (int c0 = 0; c0 < C; c0 += kWarp) {
      const int c = c0 + lane;
      const bool valid = c < C;
      const uint32_t k = valid ? c_hi[c] : 0u;
      const bool gt = valid && k > thr;
      const bool eq = valid && k == thr;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt);
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      if (gt) {
        const int p = nf + __popc(bg & lt);
        f_hi[p] = k;
        f_lo[p] = c_lo[c];
        f_slot[p] = c_slot[c];
      }
      if (eq) tie[ntie + __popc(be & lt)] = static_cast<uint16_t>(c);
      nf += __popc(bg);
      ntie += __popc(be);
    }
    __syncwarp();
    // The tie group (equal hi) supplies the remaining K - nf by (lo desc, slot asc).
    const int rem = K - nf;
    for (int i = lane; i < ntie; i += kWarp) {
      const int ci = tie[i];
      const uint32_t lo_i = c_lo[ci];
      const int s_i = c_slot[ci];
      int rank = i;
      if (ntie > rem) {
        rank = 0;
        for (int j = 0; j < ntie; ++j) {
          const int cj = tie[j];
          const uint32_t lo_j = c_lo[cj];
          rank += (lo_j > lo_i) || (lo_j == lo_i && c_slot[cj] < s_i);
        }
      }
      if (rank < rem) {
        f_hi[nf + rank] = thr;
        f_lo[nf + rank] = lo_i;
        f_slot[nf + rank] = s_i;
      }
    }
    __syncwarp();

    // 4. selection order and softmax of the selected fp32 scores.
    uint32_t top_hi = 0;
    for (int i = lane; i < K; i += kWarp) top_hi = max(top_hi, f_hi[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) top_hi = max(top_hi, __shfl_xor_sync(0xffffffffu, top_hi, o));
    const float top = unord_f32(top_hi);
    float z = 0.0f;
    for (int i = lane; i < K; i += kWarp) z += expf(unord_f32(f_hi[i]) - top);
    z = warp_sum(z);
    const float inv_z = 1.0f / z;
    int32_t* io = idx_out + unit * K;
    float* wo = w_out + unit * K;
    for (int i = lane; i < K; i += kWarp) {
      const uint64_t ki = (static_cast<uint64_t>(f_hi[i]) << 32) | f_lo[i];
      const int si = f_slot[i];
      int rank = 0;
      for (int j = 0; j < K; ++j) {
        const uint64_t kj = (static_cast<uint64_t>(f_hi[j]) << 32) | f_lo[j];
        rank += (kj > ki) || (kj == ki && f_slot[j] < si);
      }
      io[rank] = si;
      wo[rank] = expf(unord_f32(f_hi[i]) - top) * inv_z;
    }
    __syncwarp();
  }
}

}  // namespace sdm
