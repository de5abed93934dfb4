// Product-key top-k selection, register path for K <= 64 (sm_100a).
//
// Same definition as k_pkm_topk_general (SDM explainer, section 3.1 step 1;
// Technical Summary: Sparse Delta Memory, Core Mechanism 2): slot a*sqrtN + b
// scores s1[a] + s2[b], order (exact sum desc, slot asc), the top K found as
// topk(topk(s1) (+) topk(s2)).
//
// One warp per token-head, working sets in registers:
//   * each half: if sqrtN <= SZ (SZ = 32 or 64, the sort width) every value
//     goes straight into a bitonic sort; otherwise a radix select finds the
//     Kh-th largest order key and exactly Kh values are compacted (equal
//     values: lowest index first) for the sort. Sort keys are
//     ord(value):(~index), i.e. (value desc, index asc);
//   * candidates (ra, rb) with (ra+1)(rb+1) <= K, exact sums as fp32 TwoSum
//     (hi, lo); the radix select on ord(hi) picks the K winners; if its
//     boundary splits a group of equal hi, that group is ranked by
//     (lo desc, slot asc);
//   * a bitonic sort of the winners by ord(hi):(~slot), carrying ord(lo);
//     neighbours with equal hi and different lo (possible only when sums are
//     inexact in fp32) are re-ranked by (hi, lo, slot);
//   * softmax of the K selected fp32 scores.
// The radix select starts from a lower bound on the answer (the smallest, over
// lanes, of each lane's ceil(k/32)-th largest key) and takes up to 8 bits per
// pass from the highest bit where the bound and the maximum differ, stopping
// once the boundary bin is taken whole.
#pragma once

#include "sdm_device.cuh"

namespace sdm {

constexpr int kFastTopkWarps = 8;
constexpr int kFastTopkMaxK = 64;

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Descending bitonic sort of 32*E 64-bit keys, each carrying a 32-bit payload;
// position p = lane*E + s. For E <= 2 the stage loops stay rolled (one copy
// of the compare-exchange body instead of one per stage keeps the kernel
// small enough for the instruction caches); wider sorts are unrolled.
template <int E, bool PAYLOAD>
__device__ __forceinline__ void warp_bitonic_desc(uint64_t (&k)[E], uint32_t (&pl)[E]) {
  const int lane = lane_id();
  constexpr int SZ = kWarp * E;
  if constexpr (E <= 2) {
#pragma unroll 1
    for (int kk = 2; kk <= SZ; kk <<= 1) {
#pragma unroll 1
      for (int j = kk >> 1; j > 0; j >>= 1) {
        if (E == 2 && j == 1) {  // partners in the same lane: positions 2*lane and 2*lane+1
          const bool desc = ((lane * E) & kk) == 0;
          const uint64_t a = k[0], b = k[E - 1];
          const bool swap = desc ? (a < b) : (a > b);
          k[0] = swap ? b : a;
          k[E - 1] = swap ? a : b;
          if (PAYLOAD) {
            const uint32_t pa = pl[0], pb = pl[E - 1];
            pl[0] = swap ? pb : pa;
            pl[E - 1] = swap ? pa : pb;
          }
        } else {
#pragma unroll
          for (int s = 0; s < E; ++s) {
            const int p = lane * E + s;
            const uint64_t other = shfl_xor_u64(k[s], j / E);
            const bool keep_max = ((p & j) == 0) == ((p & kk) == 0);
            const bool take_other = keep_max ? (other > k[s]) : (other < k[s]);
            if (PAYLOAD) {
              const uint32_t opl = __shfl_xor_sync(0xffffffffu, pl[s], j / E);
              pl[s] = take_other ? opl : pl[s];
            }
            k[s] = take_other ? other : k[s];
          }
        }
      }
    }
  } else {
#pragma unroll
    for (int kk = 2; kk <= SZ; kk <<= 1) {
#pragma unroll
      for (int j = kk >> 1; j > 0; j >>= 1) {
        if (j < E) {
#pragma unroll
          for (int s = 0; s < E; ++s) {
            const int t = s ^ j;
            if (t > s) {
              const bool desc = ((lane * E + s) & kk) == 0;
              const uint64_t a = k[s], b = k[t];
              const bool swap = desc ? (a < b) : (a > b);
              k[s] = swap ? b : a;
              k[t] = swap ? a : b;
              if (PAYLOAD) {
                const uint32_t pa = pl[s], pb = pl[t];
                pl[s] = swap ? pb : pa;
                pl[t] = swap ? pa : pb;
              }
            }
          }
        } else {
#pragma unroll
          for (int s = 0; s < E; ++s) {
            const int p = lane * E + s;
            const uint64_t other = shfl_xor_u64(k[s], j / E);
            const bool keep_max = ((p & j) == 0) == ((p & kk) == 0);
            const bool take_other = keep_max ? (other > k[s]) : (other < k[s]);
            if (PAYLOAD) {
              const uint32_t opl = __shfl_xor_sync(0xffffffffu, pl[s], j / E);
              pl[s] = take_other ? opl : pl[s];
            }
            k[s] = take_other ? other : k[s];
          }
        }
      }
    }
  }
}

// How to take exactly k of the keys: every key with (key >> shift) >
// (thr >> shift), plus the first take_eq (in the caller's element order) of
// the bin_count keys with (key >> shift) == (thr >> shift). Key 0 marks an
// absent element, never taken.
struct SelectPlan {
  uint32_t thr;
  int shift;
  int take_eq;
  int bin_count;
  uint32_t floor;  // keys below it were not counted and are never taken
};

// Lower bound on the k-th largest key (k <= 64): every lane holds at least
// ceil(k/32) keys >= its ceil(k/32)-th largest, so at least k keys are >= the
// smallest of those over the warp.
template <int P>
__device__ __forceinline__ uint32_t warp_kth_floor(const uint32_t (&key)[P], int k) {
  uint32_t m1 = 0u, m2 = 0u;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const uint32_t x = key[i];
    m2 = x > m1 ? m1 : max(m2, x);
    m1 = max(m1, x);
  }
  uint32_t f = k <= kWarp ? m1 : m2;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) f = min(f, __shfl_xor_sync(0xffffffffu, f, o));
  return f;
}

// Plan for the top k of the present keys, given floor_key <= the k-th
// largest (keys below it are ignored).
template <int P>
__device__ __forceinline__ SelectPlan warp_select_plan(const uint32_t (&key)[P], int k, uint32_t* hist,
                                                       uint32_t floor_key) {
  const int lane = lane_id();
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < P; ++i) mx = max(mx, key[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const uint32_t lo_key = max(floor_key, 1u);
  SelectPlan sp;
  if (mx == lo_key) {  // every key that can be taken is equal
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < P; ++i) cnt += __popc(__ballot_sync(0xffffffffu, key[i] == mx));
    sp.thr = mx;
    sp.shift = 0;
    sp.take_eq = k;
    sp.bin_count = cnt;
    sp.floor = lo_key;
    return sp;
  }
  int hb = 31 - __clz(mx ^ lo_key);  // keys in [lo_key, mx] agree above bit hb
  uint32_t prefix = hb == 31 ? 0u : (mx >> (hb + 1)) << (hb + 1);
  uint32_t above_mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
  int rem = k;
#pragma unroll 1
  for (;;) {
    const int shift = max(hb - 7, 0);
    const int width = hb - shift + 1;
    const uint32_t dmask = (1u << width) - 1u;
    const int nb = 1 << width;
    if (nb == 256) {
      reinterpret_cast<uint4*>(hist)[lane] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(hist)[lane + kWarp] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      for (int i = lane; i < nb; i += kWarp) hist[i] = 0u;
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < P; ++i)
      if (key[i] >= lo_key && (key[i] & above_mask) == prefix) atomicAdd(&hist[(key[i] >> shift) & dmask], 1u);
    __syncwarp();
    // Counts from the top bin down: lane l holds bins nb-1-8l .. nb-8-8l.
    uint32_t c[8];
    if (nb == 256) {
      const uint4 a = reinterpret_cast<const uint4*>(hist)[2 * (kWarp - 1 - lane) + 1];
      const uint4 b = reinterpret_cast<const uint4*>(hist)[2 * (kWarp - 1 - lane)];
      c[0] = a.w; c[1] = a.z; c[2] = a.y; c[3] = a.x;
      c[4] = b.w; c[5] = b.z; c[6] = b.y; c[7] = b.x;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int bb = nb - 1 - 8 * lane - j;
        c[j] = bb >= 0 ? hist[bb] : 0u;
      }
    }
    uint32_t s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += c[j];
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const uint32_t excl = incl - s;
    const bool mine = excl < static_cast<uint32_t>(rem) && static_cast<uint32_t>(rem) <= incl;
    const int src = (__ffs(__ballot_sync(0xffffffffu, mine)) - 1) & 31;
    int digit = 0;
    uint32_t above = 0, cnt = 0;
    if (mine) {
      uint32_t acc = excl;
      bool found = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!found && acc + c[j] >= static_cast<uint32_t>(rem)) {
          digit = nb - 1 - 8 * lane - j;
          above = acc;
          cnt = c[j];
          found = true;
        }
        acc += c[j];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    cnt = __shfl_sync(0xffffffffu, cnt, src);
    __syncwarp();
    rem -= static_cast<int>(above);
    prefix |= static_cast<uint32_t>(digit) << shift;
    above_mask |= dmask << shift;
    if (static_cast<int>(cnt) == rem || shift == 0) {
      sp.thr = prefix;
      sp.shift = shift;
      sp.take_eq = rem;
      sp.bin_count = static_cast<int>(cnt);
      sp.floor = lo_key;
      return sp;
    }
    hb = shift - 1;
  }
}

// Per-half top-Kh by (value desc, index asc), sorted, into hv/hx[0:Kh).
// x: the half's n input values in global memory (-0 is taken as +0).
template <typename Tin, int E, int EPL>
__device__ __forceinline__ void warp_half_select_body(const Tin* __restrict__ x, int n, int Kh, uint32_t* hist,
                                                      uint64_t* sel, float* hv, int32_t* hx) {
  constexpr int SZ = kWarp * E;  // this half's sort width
  const int lane = lane_id();
  uint64_t k[E];
  uint32_t unused[E];
  if (n <= SZ) {
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int e = lane * E + s;
      k[s] = e < n ? (static_cast<uint64_t>(ord_f32(canon_zero(to_f32<Tin>(x[e])))) << 32) |
                         (0xFFFFFFFFu - static_cast<uint32_t>(e))
                   : 0ull;
    }
  } else {
    uint32_t hw[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = i * kWarp + lane;
      hw[i] = e < n ? ord_f32(canon_zero(to_f32<Tin>(x[e]))) : 0u;
    }
    const SelectPlan sp = warp_select_plan<EPL>(hw, Kh, hist, warp_kth_floor<EPL>(hw, Kh));
    const uint32_t lt = lanemask_lt();
    const uint32_t tb = sp.thr >> sp.shift;
    int cnt = 0, eq_seen = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = i * kWarp + lane;
      const uint32_t kb = hw[i] >> sp.shift;
      const bool gt = hw[i] != 0u && kb > tb;
      const bool eq = hw[i] >= sp.floor && kb == tb;
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      const bool take = gt || (eq && eq_seen + __popc(be & lt) < sp.take_eq);  // equal: lowest index first
      const uint32_t bt = __ballot_sync(0xffffffffu, take);
      if (take)
        sel[cnt + __popc(bt & lt)] = (static_cast<uint64_t>(hw[i]) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
      cnt += __popc(bt);
      eq_seen += __popc(be);
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      k[s] = p < Kh ? sel[p] : 0ull;
    }
    __syncwarp();
  }
  warp_bitonic_desc<E, false>(k, unused);
#pragma unroll
  for (int s = 0; s < E; ++s) {
    const int r = lane * E + s;
    if (r < Kh) {
      hv[r] = unord_f32(static_cast<uint32_t>(k[s] >> 32));
      hx[r] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k[s]));
    }
  }
  __syncwarp();
}

// The wide paths (4 or more values per lane, sqrtN >= 128) share one
// out-of-line copy between a selection's two halves: fully unrolled over the
// lane's values, two inlined copies do not fit the instruction caches (at
// sqrtN = 512 the kernel stalled mostly on instruction fetch; one shared copy
// takes its time from 83 to 65 ms per layer step, and 3.90 to 3.77 ms at 128).
constexpr int kHalfSelectOutOfLine = 4;
template <typename Tin, int E, int EPL>
__device__ __noinline__ void warp_half_select_call(const Tin* __restrict__ x, int n, int Kh, uint32_t* hist,
                                                   uint64_t* sel, float* hv, int32_t* hx) {
  warp_half_select_body<Tin, E, EPL>(x, n, Kh, hist, sel, hv, hx);
}
template <typename Tin, int E, int EPL>
__device__ __forceinline__ void warp_half_select(const Tin* __restrict__ x, int n, int Kh, uint32_t* hist,
                                                 uint64_t* sel, float* hv, int32_t* hx) {
  if constexpr (EPL >= kHalfSelectOutOfLine) warp_half_select_call<Tin, E, EPL>(x, n, Kh, hist, sel, hv, hx);
  else warp_half_select_body<Tin, E, EPL>(x, n, Kh, hist, sel, hv, hx);
}

// Per-warp shared scratch (byte offsets): hist 256 words | sel 64 keys |
// hv, hx 2*64 each | tie 2 words per candidate (rare paths).
struct FastTopkLayout {
  int n, K, Kh, C;
  uint32_t table_bytes, warp_bytes;
  uint32_t hist, sel, hv, hx, tie;
};

// Builds the candidate table tab[c] = (ra, rb) for the pairs (ra+1)(rb+1) <= K
// of the per-half ranks; run by one warp.
__device__ __forceinline__ void fast_topk_build_table(uint16_t* tab, int Kh, int K, int lane) {
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

// One selection by one warp: the top K slots of the score vector x[0 : 2n]
// in selection order (io) and their softmax weights (wo); ws is the warp's
// scratch of L.warp_bytes in shared memory.
template <typename Tin, int E, int EH, int EPL, int CP>
__device__ __forceinline__ void fast_topk_unit(const Tin* __restrict__ x, const FastTopkLayout& L,
                                               const uint16_t* tab, unsigned char* ws, int32_t* io, float* wo) {
  const int lane = lane_id();
  const int n = L.n, K = L.K, Kh = L.Kh, C = L.C;
  constexpr int SZ = kWarp * kFastTopkMaxK / kWarp;  // stride of the two halves in hv/hx
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  uint64_t* sel = reinterpret_cast<uint64_t*>(ws + L.sel);
  float* hv = reinterpret_cast<float*>(ws + L.hv);
  int32_t* hx = reinterpret_cast<int32_t*>(ws + L.hx);
  uint32_t* tie = reinterpret_cast<uint32_t*>(ws + L.tie);
  const uint32_t lt = lanemask_lt();
  warp_half_select<Tin, EH, EPL>(x, n, Kh, hist, sel, hv, hx);
  warp_half_select<Tin, EH, EPL>(x + n, n, Kh, hist, sel, hv + SZ, hx + SZ);

  // Candidates with exact scores: ck = ord(hi), cl = ~slot, clo = ord(lo).
  uint32_t ck[CP], cl[CP], clo[CP];
#pragma unroll
  for (int j = 0; j < CP; ++j) {
    const int c = j * kWarp + lane;
    ck[j] = 0u;
    cl[j] = 0u;
    clo[j] = 0u;
    if (c < C) {
      const int ra = tab[2 * c], rb = tab[2 * c + 1];
      float hi, lo;
      two_sum(hv[ra], hv[SZ + rb], hi, lo);
      ck[j] = ord_f32(canon_zero(hi));
      clo[j] = ord_f32(canon_zero(lo));
      cl[j] = 0xFFFFFFFFu - static_cast<uint32_t>(hx[ra] * n + hx[SZ + rb]);
    }
  }
  // Winners by hi; a boundary that splits equal hi ranks that group by
  // (lo desc, slot asc). Exact fp32 sums of bf16 inputs tie often, but such
  // groups are small.
  const SelectPlan sp = warp_select_plan<CP>(ck, K, hist, warp_kth_floor<CP>(ck, K));
  const uint32_t tb = sp.thr >> sp.shift;
  const bool split = sp.take_eq < sp.bin_count;  // only at shift 0, i.e. equal hi
  int tie_rank[CP];
#pragma unroll
  for (int j = 0; j < CP; ++j) tie_rank[j] = 0;
  if (split) {
    int g = 0;
#pragma unroll
    for (int j = 0; j < CP; ++j) {
      const bool eq = j * kWarp + lane < C && ck[j] == sp.thr;
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      if (eq) {
        const int p = g + __popc(be & lt);
        tie[2 * p] = clo[j];
        tie[2 * p + 1] = cl[j];
      }
      g += __popc(be);
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < CP; ++j) {
      if (j * kWarp + lane < C && ck[j] == sp.thr) {
        int r = 0;
        for (int q = 0; q < g; ++q) {
          const uint32_t lq = tie[2 * q], sq = tie[2 * q + 1];
          r += (lq > clo[j]) || (lq == clo[j] && sq > cl[j]);
        }
        tie_rank[j] = r;
      }
    }
    __syncwarp();
  }
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < CP; ++j) {
    const int c = j * kWarp + lane;
    const uint32_t kb = ck[j] >> sp.shift;
    const bool take = c < C && (kb > tb || (kb == tb && ck[j] >= sp.floor && (!split || tie_rank[j] < sp.take_eq)));
    const uint32_t bt = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int p = cnt + __popc(bt & lt);
      sel[p] = (static_cast<uint64_t>(ck[j]) << 32) | cl[j];
      hist[p] = clo[j];
    }
    cnt += __popc(bt);
  }
  __syncwarp();
  // Order the K winners by ord(hi):(~slot), descending: each winner's rank is
  // the number of winner keys above it (keys are distinct: the slot is part
  // of the key), counted against all K keys read two at a time from shared
  // memory; then every winner moves to its rank.
  uint64_t k[E];
  uint32_t kl[E];
  {
    uint64_t mine[E];
    uint32_t mlo[E];
    int rank[E];
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      mine[s] = p < K ? sel[p] : 0ull;
      mlo[s] = p < K ? hist[p] : 0u;
      rank[s] = 0;
    }
    const ulonglong2* sel2 = reinterpret_cast<const ulonglong2*>(sel);
    for (int j = 0; j < K; j += 2) {
      const ulonglong2 two = sel2[j >> 1];
      const uint64_t second = j + 1 < K ? two.y : 0ull;  // past K: stale, never above a winner
#pragma unroll
      for (int s = 0; s < E; ++s) rank[s] += (two.x > mine[s]) + (second > mine[s]);
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < E; ++s) {
      if (lane * E + s < K) {
        sel[rank[s]] = mine[s];
        hist[rank[s]] = mlo[s];
      }
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      k[s] = p < K ? sel[p] : 0ull;
      kl[s] = p < K ? hist[p] : 0u;
    }
    __syncwarp();
  }
  // Neighbours with equal hi but different lo need the (lo desc, slot asc) order.
  bool fix = false;
  {
    const uint32_t nh = __shfl_down_sync(0xffffffffu, static_cast<uint32_t>(k[0] >> 32), 1);
    const uint32_t nl = __shfl_down_sync(0xffffffffu, kl[0], 1);
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      if (p + 1 < K) {
        const uint32_t h1 = s + 1 < E ? static_cast<uint32_t>(k[(s + 1) % E] >> 32) : nh;
        const uint32_t l1 = s + 1 < E ? kl[(s + 1) % E] : nl;
        fix = fix || (static_cast<uint32_t>(k[s] >> 32) == h1 && kl[s] != l1);
      }
    }
  }
  const bool any_fix = __any_sync(0xffffffffu, fix);
  // Softmax of the selected scores (order independent).
  const float top = unord_f32(__shfl_sync(0xffffffffu, static_cast<uint32_t>(k[0] >> 32), 0));
  float ev[E];
  float z = 0.f;
#pragma unroll
  for (int s = 0; s < E; ++s) {
    const int p = lane * E + s;
    ev[s] = p < K ? expf(unord_f32(static_cast<uint32_t>(k[s] >> 32)) - top) : 0.f;
    z += ev[s];
  }
  z = warp_sum(z);
  const float inv_z = 1.0f / z;
  if (!any_fix) {
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      if (p < K) {
        io[p] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k[s]));
        wo[p] = ev[s] * inv_z;
      }
    }
  } else {
    // Rare: rank each winner by (hi desc, lo desc, slot asc).
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      if (p < K) {
        sel[p] = k[s];
        tie[p] = kl[s];
      }
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < E; ++s) {
      const int p = lane * E + s;
      if (p < K) {
        const uint32_t h = static_cast<uint32_t>(k[s] >> 32), lw = static_cast<uint32_t>(k[s]);
        int r = 0;
        for (int q = 0; q < K; ++q) {
          const uint32_t hq = static_cast<uint32_t>(sel[q] >> 32), lq = static_cast<uint32_t>(sel[q]);
          r += hq > h || (hq == h && (tie[q] > kl[s] || (tie[q] == kl[s] && lq > lw)));
        }
        io[r] = static_cast<int32_t>(0xFFFFFFFFu - lw);
        wo[r] = ev[s] * inv_z;
      }
    }
  }
}

// E: winners sort width / 32; EH: half sort width / 32 (1 when sqrtN <= 32);
// EPL: half values per lane when sqrtN > 32*EH; CP: candidates per lane.
template <typename Tin, int E, int EH, int EPL, int CP>
__global__ void __launch_bounds__(kFastTopkWarps * kWarp) k_pkm_topk_fast(const Tin* __restrict__ scores,
                                                                          int64_t n_units, FastTopkLayout L,
                                                                          int32_t* __restrict__ idx_out,
                                                                          float* __restrict__ w_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x / kWarp;
  uint16_t* tab = reinterpret_cast<uint16_t*>(smem);  // candidate c -> (ra, rb)
  if (warp == 0) fast_topk_build_table(tab, L.Kh, L.K, lane_id());
  __syncthreads();
  unsigned char* ws = smem + L.table_bytes + static_cast<size_t>(warp) * L.warp_bytes;
  for (int64_t unit = static_cast<int64_t>(blockIdx.x) * kFastTopkWarps + warp; unit < n_units;
       unit += static_cast<int64_t>(gridDim.x) * kFastTopkWarps) {
    fast_topk_unit<Tin, E, EH, EPL, CP>(scores + unit * 2 * L.n, L, tab, ws, idx_out + unit * L.K,
                                        w_out + unit * L.K);
    __syncwarp();
  }
}

}  // namespace sdm
