// Sparse Delta Memory (SDM) recurrent core -- CPU ORACLE.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously-correct
// definition that the CUDA path is checked against. Only the tests, the smoke
// check and the benchmark's CPU-baseline leg may load it. It shares no code,
// header, table or helper with the CUDA library, and the library never calls it.
//
// Sources (web pages about arXiv 2607.07386, "Sparse Delta Memory: Scaling the
// State of Linear RNNs through Sparsity"), cited below by these short names:
//   [explainer]  papers.ananclaw.com explainer "Sparse Delta Memory：通过稀疏性扩展
//                线性 RNN 的状态容量", section 3.1 "SDM 层的三步流程" (steps 1-3),
//                section 3.2 (IsoFLOP), section 3.3 (equation 6).
//   [summary]    gist.science "Technical Summary: Sparse Delta Memory (SDM)",
//                Methodology / Core Mechanism items 1-4 and "IsoFLOP Design".
//
// What it computes, step by step, in the pages' order:
//   1. Selection ([explainer] 3.1 step 1; [summary] Core Mechanism 2). The score
//      vector x of length 2*sqrtN is split into s1 = x[0:sqrtN], s2 = x[sqrtN:].
//      The N = sqrtN^2 slot scores are the outer SUM s1[a] + s2[b]; slot number
//      i = a*sqrtN + b (row-major over the sqrtN x sqrtN grid). All N scores are
//      materialised and the first K of the order (exact real sum descending,
//      slot ascending) are kept. The exact sum is held as a double TwoSum pair
//      (hi, lo) -- fp32 operands are exact in double, TwoSum makes hi+lo the
//      exact real sum -- and compared lexicographically, which equals comparing
//      the real sums because round-to-nearest is monotone.
//   2. Sparse weights: softmax over the K selected scores, in double. The pages
//      use the weights k^(i), q^(i) without defining them; this reading is the
//      softmax of the selected scores with ties broken by lowest slot index.
//   3. Write ([explainer] 3.1 step 2; [summary] Core Mechanism 3), for every
//      selected write slot i, literally:  Mt = alpha*M[i];
//      M[i] = Mt + beta*k_i*(v - Mt); other slots untouched. Math in double,
//      rounded to the state dtype (fp32, or bf16 round-to-nearest-even) on store.
//   4. Read after the write ([explainer] 3.1 step 3; [summary] Core Mechanism 4):
//      y_t = sum over read slots of q_i * M_t[i], in double.
//   5. Optional epilogue ([explainer] 3.1 step 3): y <- g * y / sqrt(mean(y^2)+eps).
//   6. Backward (the derivatives for training): reverse-mode through steps 2-4
//      for a fixed selection, by the chain rule on the pages' own formulas
//      ([explainer] 3.4 "高效训练" says only that a memory-efficient backward
//      exists and leaves its details to an appendix the pages do not show).
//   7. A block-scaled fp8 state (E4M3 values, one power-of-two scale per 16
//      row values; see "block-scaled fp8 state" below): the recurrence of
//      steps 3-4 on the decoded state, each written row computed in double by
//      the pages' two-step write and then re-quantised.
//
// Parity status: selection, weights, write, read and epilogue are each pinned by
// tests that do not re-run this file's formulas (exact-rational brute force,
// closed forms, invariants, hand-worked fixtures, planted-mistake checks); the
// backward is pinned by central finite differences of the double-precision
// forward, a hand-derived one-slot closed form, and planted-mistake checks; the
// fp8 state by an exact-rational model of E4M3, block invariants and scan
// identities.
//
// ORACLE_MUTANT (default 0) plants one known mistake per value so the tests
// can show that the pins catch it; it is never set outside those tests.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

namespace {

// One materialised slot score: exact sum hi + lo of s1[a] + s2[b].
struct SlotScore {
  double hi;
  double lo;
  int32_t slot;
};

// Knuth's TwoSum: hi = fl(x + y), lo = the exact rounding error, so hi + lo == x + y.
inline void two_sum(double x, double y, double* hi, double* lo) {
  const double s = x + y;
  const double bb = s - x;
  *hi = s;
  *lo = (x - (s - bb)) + (y - bb);
}

// The selection order: exact sum descending, then slot ascending (ties -> lowest slot).
inline bool precedes(const SlotScore& p, const SlotScore& q) {
#if ORACLE_MUTANT == 3
  if (p.hi != q.hi) return p.hi > q.hi;  // planted: the low part is ignored
#else
  if (p.hi != q.hi) return p.hi > q.hi;
  if (p.lo != q.lo) return p.lo > q.lo;
#endif
#if ORACLE_MUTANT == 2
  return p.slot > q.slot;  // planted: ties go to the highest slot
#else
  return p.slot < q.slot;
#endif
}

// Runs fn(i) for i in [0, n) on up to n_threads threads.
template <class Fn>
void parallel_for(int64_t n, int n_threads, Fn fn) {
  if (n_threads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  const int nt = static_cast<int>(std::min<int64_t>(n_threads, n));
  for (int t = 0; t < nt; ++t) {
    pool.emplace_back([&]() {
      for (;;) {
        const int64_t i = next.fetch_add(1);
        if (i >= n) break;
        fn(i);
      }
    });
  }
  for (auto& th : pool) th.join();
}

// Rounds a double to the nearest bf16 value (ties to even), returned as float.
// bf16 keeps 8 significant bits and fp32's exponent range; its smallest
// subnormal step is 2^-133.
float round_to_bf16(double x) {
  if (x == 0.0 || !std::isfinite(x)) return static_cast<float>(x);
  int e = 0;
  std::frexp(x, &e);  // x = m * 2^e with 0.5 <= |m| < 1
  int q = e - 8;      // weight of the last kept bit
  if (q < -133) q = -133;
  const double r = std::nearbyint(std::ldexp(x, -q));  // default mode: nearest-even
  return static_cast<float>(std::ldexp(r, q));
}

inline float round_state(double x, bool bf16) {
  return bf16 ? round_to_bf16(x) : static_cast<float>(x);
}

// Selection for one score vector x[0 : 2*sqrt_n): writes K slots (selection
// order) and their softmax weights.
void select_one(const float* x, int32_t sqrt_n, int32_t K, std::vector<SlotScore>& grid,
                int32_t* idx, double* w) {
  const int64_t n = static_cast<int64_t>(sqrt_n) * sqrt_n;
  const float* s1 = x;           // first half  -> grid row a
  const float* s2 = x + sqrt_n;  // second half -> grid column b
  grid.resize(static_cast<size_t>(n));
  for (int32_t a = 0; a < sqrt_n; ++a) {
    for (int32_t b = 0; b < sqrt_n; ++b) {
      SlotScore& e = grid[static_cast<size_t>(a) * sqrt_n + b];
      two_sum(static_cast<double>(s1[a]), static_cast<double>(s2[b]), &e.hi, &e.lo);
#if ORACLE_MUTANT == 1
      e.slot = b * sqrt_n + a;  // planted: grid numbered column-major
#else
      e.slot = a * sqrt_n + b;
#endif
    }
  }
  // Library sort primitive: partial_sort returns exactly the first K elements
  // of the full sort because `precedes` is a strict total order.
  std::partial_sort(grid.begin(), grid.begin() + K, grid.end(), precedes);
  double mx = -INFINITY;
  for (int32_t k = 0; k < K; ++k) mx = std::max(mx, grid[k].hi + grid[k].lo);
  double z = 0.0;
  for (int32_t k = 0; k < K; ++k) {
    idx[k] = grid[k].slot;
    w[k] = std::exp((grid[k].hi + grid[k].lo) - mx);
    z += w[k];
  }
  for (int32_t k = 0; k < K; ++k) {
#if ORACLE_MUTANT == 8
    w[k] = 1.0 / K;  // planted: uniform weights
#else
    w[k] = w[k] / z;
#endif
  }
}

// The epilogue on one row ([explainer] 3.1 step 3, "RMS-Norm" then the
// element-wise gate g): y <- g * y / sqrt(mean(y^2) + eps), in double.
template <class G>
void rmsnorm_gate_row(double* y, const G* g, int32_t d_v, double eps) {
  double ss = 0.0;
  for (int32_t c = 0; c < d_v; ++c) ss += y[c] * y[c];
#if ORACLE_MUTANT == 9
  const double inv = 1.0 / std::sqrt(ss + eps);  // planted: sum instead of mean
#else
  const double inv = 1.0 / std::sqrt(ss / d_v + eps);
#endif
  for (int32_t c = 0; c < d_v; ++c) y[c] = static_cast<double>(g[c]) * y[c] * inv;
}

// ------------------------------------------------- block-scaled fp8 state --
// A reduced-precision state ([explainer] "工程落地关键点", item 2: at N = 10^7
// the state needs int8/fp8 quantisation; the pages fix no format). Reading:
// OCP FP8 E4M3 values (sign, 4 exponent bits with bias 7, 3 mantissa bits;
// subnormals down to 2^-9; no infinities; largest finite 448; S.1111.111 is
// NaN and never produced) with one power-of-two scale 2^e per 16 consecutive
// values of a state row (block scaling in the manner of the OCP MX formats,
// with blocks of 16). Every value is rounded to nearest-even onto the E4M3
// grid after division by 2^e; for a block with largest magnitude m > 0, e is
// the smallest integer for which that rounding of m / 2^e is at most 448,
// i.e. the smallest e with m <= 464 * 2^e (464 lies halfway between 448 and
// the next step, 480, and rounds to the even 448). So m / 2^e lies in
// (232, 464], no value of a block is ever clamped, and re-quantising a
// decoded block returns the same codes and exponent (its rounded maximum lies
// in [240, 448]). An all-zero block has e = 0.

// E4M3 code of a double (round to nearest, ties to even; clamped to 448).
uint8_t round_e4m3(double x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(x);
#if ORACLE_MUTANT == 21
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7F);  // planted: overflow to the NaN code
#else
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7E);
#endif
  // Grid spacing for |x| in [2^k, 2^(k+1)): 2^(k-3) for k >= -6, 2^-9 below (subnormals).
  int k = 0;
  if (a > 0.0) {
    std::frexp(a, &k);
    k -= 1;  // a in [2^k, 2^(k+1))
  }
  const int q = std::max(k, -6) - 3;  // weight of the last mantissa bit
#if ORACLE_MUTANT == 20
  const double r = std::trunc(std::ldexp(a, -q));  // planted: rounding toward zero
#else
  const double r = std::nearbyint(std::ldexp(a, -q));  // default mode: nearest-even
#endif
  double v = std::ldexp(r, q);
  if (v > 448.0) v = 448.0;
  // Encode v (exactly representable now).
  if (v == 0.0) return sign;
  int ev = 0;
  std::frexp(v, &ev);
  ev -= 1;  // v in [2^ev, 2^(ev+1))
  if (ev < -6) {  // subnormal: v = m * 2^-9, m in 1..7
    const int m = static_cast<int>(std::ldexp(v, 9));
    return static_cast<uint8_t>(sign | m);
  }
  const int mant = static_cast<int>(std::ldexp(v, -ev) * 8.0) - 8;  // 0..7
  return static_cast<uint8_t>(sign | ((ev + 7) << 3) | mant);
}

double decode_e4m3(uint8_t c) {
  const double sign = (c & 0x80) ? -1.0 : 1.0;
  const int e = (c >> 3) & 0x0F, m = c & 0x07;
  if (e == 0) return sign * std::ldexp(static_cast<double>(m), -9);
  return sign * std::ldexp(1.0 + m / 8.0, e - 7);
}

// Scale exponent of a block of n values (see above): the smallest e with
// max|x| <= 464 * 2^e.
template <class X>
int block_exponent(const X* x, int n) {
  double mx = 0.0;
  for (int i = 0; i < n; ++i) mx = std::max(mx, std::fabs(static_cast<double>(x[i])));
  if (mx == 0.0) return 0;
  int k = 0;
  std::frexp(mx, &k);  // mx in [2^(k-1), 2^k)
  int e = (k - 1) - 8;  // mx / 2^e in [256, 512)
#if ORACLE_MUTANT == 19
  return e;  // planted: a block maximum above 464 * 2^e is clipped to 448 * 2^e
#else
  if (std::ldexp(mx, -e) > 464.0) ++e;  // (464, 512) would saturate: one binade up, (232, 256)
  return e;
#endif
}

// Quantises one block of 16 values: codes[16], returns the exponent (kept in
// the int8 range; blocks beyond it use the nearest exponent).
template <class X>
int quantize_block(const X* x, uint8_t* codes) {
  const int e = std::max(-127, std::min(127, block_exponent(x, 16)));
  for (int i = 0; i < 16; ++i) codes[i] = round_e4m3(std::ldexp(static_cast<double>(x[i]), -e));
  return e;
}

// Stores a freshly computed state value: rounded to fp32 (or to bf16 and kept
// as an exact fp32) in a float state; kept exactly in a double state.
template <class S>
inline S store_state(double x, bool bf16);
template <>
inline float store_state<float>(double x, bool bf16) {
  return round_state(x, bf16);
}
template <>
inline double store_state<double>(double x, bool) {
  return x;
}

// The recurrence over a given selection (the body of oracle_scan and
// oracle_scan_f64; S is the state's storage type, I the type of v, alpha, beta).
template <class S, class I>
int scan_impl(int32_t B, int32_t T, int32_t H, int64_t N, int32_t d_v, int32_t W, int32_t R,
              const int32_t* idx_w, const double* w_w, const int32_t* idx_r, const double* w_r,
              const I* v, const I* alpha, const I* beta, const float* g,
              double eps, int32_t state_bf16, S* M, double* y, int32_t n_threads,
              int64_t* op_count) {
  if (B < 0 || T < 0 || H < 0 || N < 1 || d_v < 1 || W < 0 || R < 0) return -1;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * W; ++e)
    if (idx_w[e] < 0 || idx_w[e] >= N) return -2;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * R; ++e)
    if (idx_r[e] < 0 || idx_r[e] >= N) return -2;
  const bool bf16 = state_bf16 != 0;
  // Columns of d_v evolve independently, so the work splits over (b, h, column block).
  const int32_t col_block = 64;
  const int32_t n_cb = (d_v + col_block - 1) / col_block;
  std::atomic<int64_t> ops(0);
  parallel_for(static_cast<int64_t>(B) * H * n_cb, std::max(1, n_threads), [&](int64_t u) {
    const int32_t cb = static_cast<int32_t>(u % n_cb);
    const int32_t h = static_cast<int32_t>((u / n_cb) % H);
    const int32_t b = static_cast<int32_t>(u / (static_cast<int64_t>(n_cb) * H));
    const int32_t c0 = cb * col_block;
    const int32_t c1 = std::min(d_v, c0 + col_block);
    S* Mbh = M + (static_cast<int64_t>(b) * H + h) * N * d_v;
    int64_t local_ops = 0;
    for (int32_t t = 0; t < T; ++t) {
      const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;  // token-head
      const double a_t = alpha[th];
      const double b_t = beta[th];
      const I* v_t = v + th * d_v;
      double* y_t = y + th * d_v;
      auto do_reads = [&]() {
        for (int32_t c = c0; c < c1; ++c) {
          double acc = 0.0;
          for (int32_t r = 0; r < R; ++r) {
            const int64_t i = idx_r[th * R + r];
            acc += w_r[th * R + r] * static_cast<double>(Mbh[i * d_v + c]);
          }
          y_t[c] = acc;
        }
        local_ops += static_cast<int64_t>(2) * R * (c1 - c0);
      };
#if ORACLE_MUTANT == 6
      do_reads();  // planted: read before the write
#endif
      // Step 2: gated delta write on the selected write slots only.
      for (int32_t j = 0; j < W; ++j) {
        const int64_t i = idx_w[th * W + j];
        const double k_i = w_w[th * W + j];
        for (int32_t c = c0; c < c1; ++c) {
          const double m_prev = Mbh[i * d_v + c];
#if ORACLE_MUTANT == 4
          const double m_tilde = m_prev;  // planted: forget gate dropped
#else
          const double m_tilde = a_t * m_prev;
#endif
          const double v_c = v_t[c];
#if ORACLE_MUTANT == 5
          const double m_new = m_tilde - b_t * k_i * (v_c - m_tilde);  // planted: sign
#elif ORACLE_MUTANT == 7
          const double m_new = m_tilde + b_t * (v_c - m_tilde);  // planted: k dropped
#else
          const double m_new = m_tilde + b_t * k_i * (v_c - m_tilde);
#endif
#if ORACLE_MUTANT == 10
          Mbh[i * d_v + c] = static_cast<S>(m_new);  // planted: no state rounding
#else
          Mbh[i * d_v + c] = store_state<S>(m_new, bf16);
#endif
        }
        local_ops += static_cast<int64_t>(4) * (c1 - c0);
      }
#if ORACLE_MUTANT == 11
      // planted: the forget gate also decays one unselected slot
      {
        int64_t other = (idx_w[th * W] + 1) % N;
        bool selected = false;
        for (int32_t j = 0; j < W; ++j) selected = selected || idx_w[th * W + j] == other;
        if (!selected)
          for (int32_t c = c0; c < c1; ++c)
            Mbh[other * d_v + c] = store_state<S>(a_t * Mbh[other * d_v + c], bf16);
      }
#endif
      // Step 3: sparse read of the state after this token's write.
#if ORACLE_MUTANT != 6
      do_reads();
#endif
    }
    ops.fetch_add(local_ops);
  });
  // Optional epilogue: RMS-norm over d_v per token-head, then the element-wise gate.
  if (g != nullptr) {
    parallel_for(static_cast<int64_t>(B) * T * H, std::max(1, n_threads), [&](int64_t th) {
      rmsnorm_gate_row(y + th * d_v, g + th * d_v, d_v, eps);
    });
  }
  if (op_count != nullptr) *op_count = ops.load();
  return 0;
}

}  // namespace

extern "C" {

int oracle_abi_version() { return 1; }

float oracle_round_to_bf16(double x) { return round_to_bf16(x); }

// Top-K slot selection for n_units independent score vectors.
//   scores : [n_units, 2*sqrt_n] fp32 (bf16 inputs are widened exactly by the caller)
//   idx_out: [n_units, K] int32, selection order;  w_out: [n_units, K] softmax weights
// Returns 0, or -1 for invalid sizes.
int oracle_pkm_topk(const float* scores, int64_t n_units, int32_t sqrt_n, int32_t K,
                    int32_t* idx_out, double* w_out, int32_t n_threads) {
  if (sqrt_n < 1 || K < 1 || static_cast<int64_t>(K) > static_cast<int64_t>(sqrt_n) * sqrt_n ||
      n_units < 0)
    return -1;
  const int nt = std::max(1, n_threads);
  const int64_t chunk = 64;
  const int64_t n_chunks = (n_units + chunk - 1) / chunk;
  parallel_for(n_chunks, nt, [&](int64_t c) {
    std::vector<SlotScore> grid;
    const int64_t u_end = std::min(n_units, (c + 1) * chunk);
    for (int64_t u = c * chunk; u < u_end; ++u) {
      select_one(scores + u * 2 * sqrt_n, sqrt_n, K, grid, idx_out + u * K, w_out + u * K);
    }
  });
  return 0;
}

// The recurrence over a given selection.
//   idx_w, w_w : [B,T,H,W]   idx_r, w_r : [B,T,H,R]
//   v          : [B,T,H,d_v] alpha, beta : [B,T,H]   g: [B,T,H,d_v] or NULL
//   M          : [B,H,N,d_v] in/out (fp32 array; with state_bf16 every stored
//                value is rounded to bf16 and kept as an exact fp32)
//   y          : [B,T,H,d_v] out, double
//   op_count   : if not NULL, receives the number of scalar multiply/add
//                operations the write and read steps performed
// Returns 0, or -1 for invalid sizes, or -2 when an index is outside [0, N).
int oracle_scan(int32_t B, int32_t T, int32_t H, int64_t N, int32_t d_v, int32_t W, int32_t R,
                const int32_t* idx_w, const double* w_w, const int32_t* idx_r, const double* w_r,
                const float* v, const float* alpha, const float* beta, const float* g,
                double eps, int32_t state_bf16, float* M, double* y, int32_t n_threads,
                int64_t* op_count) {
  return scan_impl<float, float>(B, T, H, N, d_v, W, R, idx_w, w_w, idx_r, w_r, v, alpha, beta, g, eps, state_bf16,
                          M, y, n_threads, op_count);
}

// The same recurrence with inputs and state in double and the state never
// rounded: the exact function whose derivatives oracle_scan_backward computes.
int oracle_scan_f64(int32_t B, int32_t T, int32_t H, int64_t N, int32_t d_v, int32_t W, int32_t R,
                    const int32_t* idx_w, const double* w_w, const int32_t* idx_r, const double* w_r,
                    const double* v, const double* alpha, const double* beta, double* M, double* y,
                    int32_t n_threads) {
  return scan_impl<double, double>(B, T, H, N, d_v, W, R, idx_w, w_w, idx_r, w_r, v, alpha, beta, nullptr, 0.0, 0, M,
                           y, n_threads, nullptr);
}

// Reverse-mode derivatives of the recurrence as oracle_scan_f64 computes it
// (no epilogue), for the loss L = sum_t <dy_t, y_t> + <dM_T, M_T>, by the chain
// rule through the pages' own two-step write ([explainer] 3.1 step 2):
//   m~ = alpha * m_old;   m_new = m~ + beta * k * (v - m~)
// and the read after the write ([explainer] 3.1 step 3): y_t = sum q_i M_t[i].
// The forward trajectory is recomputed first, keeping every overwritten value;
// the sweep then runs backwards over tokens (the read before the write, the
// write entries in reverse order), restoring the state as it goes.
//   M0   : [B,H,N,d_v] the state the forward started from (double)
//   dy   : [B,T,H,d_v] dL/dy;  dM: [B,H,N,d_v] in: dL/dM_T, out: dL/dM_0
//   dv   : [B,T,H,d_v] out;  dalpha, dbeta: [B,T,H] out
//   dw_w : [B,T,H,W] out, dL/dk_i;  dw_r: [B,T,H,R] out, dL/dq_i
// Returns 0, or -1 for invalid sizes, or -2 when an index is outside [0, N).
int oracle_scan_backward(int32_t B, int32_t T, int32_t H, int64_t N, int32_t d_v, int32_t W, int32_t R,
                         const int32_t* idx_w, const double* w_w, const int32_t* idx_r, const double* w_r,
                         const double* v, const double* alpha, const double* beta, const double* M0,
                         const double* dy, double* dM, double* dv, double* dalpha, double* dbeta,
                         double* dw_w, double* dw_r, int32_t n_threads) {
  if (B < 0 || T < 0 || H < 0 || N < 1 || d_v < 1 || W < 0 || R < 0) return -1;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * W; ++e)
    if (idx_w[e] < 0 || idx_w[e] >= N) return -2;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * R; ++e)
    if (idx_r[e] < 0 || idx_r[e] >= N) return -2;
  // Every (b, h) is independent; its scalar gradients sum over all columns,
  // so one (b, h) is one unit of work.
  parallel_for(static_cast<int64_t>(B) * H, std::max(1, n_threads), [&](int64_t u) {
    const int32_t h = static_cast<int32_t>(u % H);
    const int32_t b = static_cast<int32_t>(u / H);
    const int64_t state_off = (static_cast<int64_t>(b) * H + h) * N * d_v;
    std::vector<double> M(M0 + state_off, M0 + state_off + N * d_v);
    std::vector<double> old(static_cast<size_t>(T) * W * d_v);  // overwritten values, [t][j][c]
    // Forward: the recomputed trajectory.
    for (int32_t t = 0; t < T; ++t) {
      const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
      for (int32_t j = 0; j < W; ++j) {
        const int64_t i = idx_w[th * W + j];
        const double k_i = w_w[th * W + j];
        for (int32_t c = 0; c < d_v; ++c) {
          const double m_old = M[i * d_v + c];
          old[(static_cast<size_t>(t) * W + j) * d_v + c] = m_old;
          const double m_tilde = alpha[th] * m_old;
          M[i * d_v + c] = m_tilde + beta[th] * k_i * (v[th * d_v + c] - m_tilde);
        }
      }
    }
    // Backward: G = dL/dM_t, starting from dL/dM_T.
    std::vector<double> G(dM + state_off, dM + state_off + N * d_v);
    for (int32_t t = T - 1; t >= 0; --t) {
      const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
      const double a_t = alpha[th];
      const double b_t = beta[th];
      const double* dy_t = dy + th * d_v;
      const double* v_t = v + th * d_v;
      double* dv_t = dv + th * d_v;
      for (int32_t c = 0; c < d_v; ++c) dv_t[c] = 0.0;
      // Read: y_t = sum_r q_r M_t[i_r]  ->  dq_r = <dy_t, M_t[i_r]>, G[i_r] += q_r dy_t.
      for (int32_t r = 0; r < R; ++r) {
        const int64_t i = idx_r[th * R + r];
        double dq = 0.0;
        for (int32_t c = 0; c < d_v; ++c) {
#if ORACLE_MUTANT == 14
          // planted: the read gradient taken from the state before the write
          double m_c = M[i * d_v + c];
          for (int32_t j = 0; j < W; ++j)
            if (idx_w[th * W + j] == i) m_c = old[(static_cast<size_t>(t) * W + j) * d_v + c];
          dq += dy_t[c] * m_c;
#else
          dq += dy_t[c] * M[i * d_v + c];
#endif
        }
        dw_r[th * R + r] = dq;
        for (int32_t c = 0; c < d_v; ++c) G[i * d_v + c] += w_r[th * R + r] * dy_t[c];
      }
      // Write, entries in reverse order.
      double da_t = 0.0, db_t = 0.0;
      for (int32_t j = W - 1; j >= 0; --j) {
        const int64_t i = idx_w[th * W + j];
        const double k_i = w_w[th * W + j];
        double dk = 0.0;
        for (int32_t c = 0; c < d_v; ++c) {
          const double m_old = old[(static_cast<size_t>(t) * W + j) * d_v + c];
          const double m_tilde = a_t * m_old;
          const double g = G[i * d_v + c];                   // dL/dm_new
          const double d_tilde = g * (1.0 - b_t * k_i);      // dL/dm~
          dv_t[c] += g * b_t * k_i;
          db_t += g * k_i * (v_t[c] - m_tilde);
#if ORACLE_MUTANT == 15
          (void)d_tilde;  // planted: dk without its beta (v - m~) factor's m~ part
          dk += g * b_t * v_t[c];
#else
          dk += g * b_t * (v_t[c] - m_tilde);
#endif
#if ORACLE_MUTANT == 12
          da_t += g * m_old;  // planted: the (1 - beta k) factor dropped
#else
          da_t += d_tilde * m_old;
#endif
#if ORACLE_MUTANT == 13
          G[i * d_v + c] = g;  // planted: the adjoint passes the write undecayed
#else
          G[i * d_v + c] = d_tilde * a_t;
#endif
          M[i * d_v + c] = m_old;
        }
        dw_w[th * W + j] = dk;
      }
      dalpha[th] = da_t;
      dbeta[th] = db_t;
    }
    std::copy(G.begin(), G.end(), dM + state_off);
  });
  return 0;
}

// Derivative of the softmax selection weights with respect to the scores, for
// a fixed selection (the selected set and its order do not move under an
// infinitesimal change of distinct scores). With sigma_k = s1[a_k] + s2[b_k]
// and w = softmax(sigma): dL/dsigma_k = w_k (dw_k - sum_j w_j dw_j), and each
// sigma_k adds its derivative to s1[a_k] and to s2[b_k], slot = a*sqrt_n + b.
//   idx, w, dw : [n_units, K];  dscores: [n_units, 2*sqrt_n] out (zero where
//   no selected slot uses the entry). Returns 0, -1 for invalid sizes, -2 for
//   an index outside [0, N).
int oracle_pkm_topk_backward(int64_t n_units, int32_t sqrt_n, int32_t K, const int32_t* idx, const double* w,
                             const double* dw, double* dscores) {
  if (sqrt_n < 1 || K < 1 || n_units < 0) return -1;
  const int64_t N = static_cast<int64_t>(sqrt_n) * sqrt_n;
  for (int64_t u = 0; u < n_units; ++u) {
    const int32_t* id = idx + u * K;
    const double* wu = w + u * K;
    const double* du = dw + u * K;
    double* ds = dscores + u * 2 * sqrt_n;
    for (int32_t x = 0; x < 2 * sqrt_n; ++x) ds[x] = 0.0;
    double mean = 0.0;
    for (int32_t k = 0; k < K; ++k) mean += wu[k] * du[k];
    for (int32_t k = 0; k < K; ++k) {
      if (id[k] < 0 || id[k] >= N) return -2;
#if ORACLE_MUTANT == 16
      const double dsig = wu[k] * du[k];  // planted: the weighted mean not subtracted
#else
      const double dsig = wu[k] * (du[k] - mean);
#endif
#if ORACLE_MUTANT == 17
      ds[id[k] % sqrt_n] += dsig;  // planted: halves swapped
      ds[sqrt_n + id[k] / sqrt_n] += dsig;
#else
      ds[id[k] / sqrt_n] += dsig;
      ds[sqrt_n + id[k] % sqrt_n] += dsig;
#endif
    }
  }
  return 0;
}

// The epilogue alone on n_rows rows of d_v (double): y <- g * y / rms(y).
int oracle_rmsnorm_gate(int64_t n_rows, int32_t d_v, double* y, const double* g, double eps) {
  if (n_rows < 0 || d_v < 1) return -1;
  for (int64_t r = 0; r < n_rows; ++r) rmsnorm_gate_row(y + r * d_v, g + r * d_v, d_v, eps);
  return 0;
}

// Its derivatives for dL/dout: with x the row before the epilogue,
// r = sqrt(mean(x^2) + eps) and out = g * x / r,
//   dL/dx_j = g_j dout_j / r - x_j * sum_i(g_i dout_i x_i) / (d_v r^3)
//   dL/dg_i = dout_i x_i / r.
int oracle_rmsnorm_gate_backward(int64_t n_rows, int32_t d_v, const double* x, const double* g, const double* dout,
                                 double eps, double* dx, double* dg) {
  if (n_rows < 0 || d_v < 1) return -1;
  for (int64_t r = 0; r < n_rows; ++r) {
    const double* xr = x + r * d_v;
    const double* gr = g + r * d_v;
    const double* dr = dout + r * d_v;
    double ss = 0.0, dot = 0.0;
    for (int32_t c = 0; c < d_v; ++c) {
      ss += xr[c] * xr[c];
      dot += gr[c] * dr[c] * xr[c];
    }
    const double rms = std::sqrt(ss / d_v + eps);
    for (int32_t c = 0; c < d_v; ++c) {
#if ORACLE_MUTANT == 18
      dx[r * d_v + c] = gr[c] * dr[c] / rms;  // planted: the normaliser treated as a constant
#else
      dx[r * d_v + c] = gr[c] * dr[c] / rms - xr[c] * dot / (d_v * rms * rms * rms);
#endif
      dg[r * d_v + c] = dr[c] * xr[c] / rms;
    }
  }
  return 0;
}

uint8_t oracle_round_e4m3(double x) { return round_e4m3(x); }
double oracle_decode_e4m3(uint8_t c) { return decode_e4m3(c); }

// Quantises n_blocks blocks of 16 fp32 values: codes [n_blocks*16] uint8,
// exps [n_blocks] int8 (the block scale is 2^exp).
int oracle_quantize_fp8blk(const float* x, int64_t n_blocks, uint8_t* codes, int8_t* exps) {
  for (int64_t bI = 0; bI < n_blocks; ++bI) exps[bI] = static_cast<int8_t>(quantize_block(x + bI * 16, codes + bI * 16));
  return 0;
}

// The recurrence with the block-scaled fp8 state. The state is codes
// [B,H,N,d_v] uint8 and exps [B,H,N,d_v/16] int8 (in/out); d_v a multiple of
// 16. Each written row follows the pages' two-step write ([explainer] 3.1
// step 2) in double on the decoded row: m~ = alpha * M[i];
// M[i] = m~ + beta * k_i * (v - m~); the double row is then quantised block
// by block (the reduced-precision store). y (double) is the read of the
// decoded state after the write ([explainer] 3.1 step 3).
//   w_w, w_r: the selection weights (double, e.g. from oracle_pkm_topk).
int oracle_scan_fp8blk(int32_t B, int32_t T, int32_t H, int64_t N, int32_t d_v, int32_t W, int32_t R,
                       const int32_t* idx_w, const double* w_w, const int32_t* idx_r, const double* w_r,
                       const float* v, const float* alpha, const float* beta, uint8_t* codes, int8_t* exps,
                       double* y, int32_t n_threads) {
  if (B < 0 || T < 0 || H < 0 || N < 1 || d_v < 16 || d_v % 16 != 0 || W < 0 || R < 0) return -1;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * W; ++e)
    if (idx_w[e] < 0 || idx_w[e] >= N) return -2;
  for (int64_t e = 0; e < static_cast<int64_t>(B) * T * H * R; ++e)
    if (idx_r[e] < 0 || idx_r[e] >= N) return -2;
  const int32_t nb = d_v / 16;
  parallel_for(static_cast<int64_t>(B) * H, std::max(1, n_threads), [&](int64_t u) {
    const int32_t h = static_cast<int32_t>(u % H);
    const int32_t b = static_cast<int32_t>(u / H);
    uint8_t* C = codes + (static_cast<int64_t>(b) * H + h) * N * d_v;
    int8_t* X = exps + (static_cast<int64_t>(b) * H + h) * N * nb;
    std::vector<double> row(static_cast<size_t>(d_v));
    auto decoded = [&](int64_t i, int32_t c) { return decode_e4m3(C[i * d_v + c]) * std::ldexp(1.0, X[i * nb + c / 16]); };
    for (int32_t t = 0; t < T; ++t) {
      const int64_t th = (static_cast<int64_t>(b) * T + t) * H + h;
      const double a_t = alpha[th], b_t = beta[th];
      for (int32_t j = 0; j < W; ++j) {
        const int64_t i = idx_w[th * W + j];
        const double k_i = w_w[th * W + j];
        for (int32_t c = 0; c < d_v; ++c) {
          const double m_tilde = a_t * decoded(i, c);
          row[c] = m_tilde + b_t * k_i * (static_cast<double>(v[th * d_v + c]) - m_tilde);
        }
        for (int32_t q = 0; q < nb; ++q) X[i * nb + q] = static_cast<int8_t>(quantize_block(row.data() + 16 * q, C + i * d_v + 16 * q));
      }
      for (int32_t c = 0; c < d_v; ++c) {
        double acc = 0.0;
        for (int32_t r = 0; r < R; ++r) acc += w_r[th * R + r] * decoded(idx_r[th * R + r], c);
        y[th * d_v + c] = acc;
      }
    }
  });
  return 0;
}

}  // extern "C"
