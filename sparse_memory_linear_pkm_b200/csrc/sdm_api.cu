// C ABI of the SDM recurrent core: argument validation, workspace carving and
// kernel dispatch. See include/sdm.h for the contract of every entry point.
//
// The kernels live in the included headers; the launches of the kernels with
// many template instances sit in translation units of their own (sdm_tu_*.cu),
// declared in sdm_host.h, so that the library builds in parallel.

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>
#include <mutex>
#include <string>

#include "sdm.h"
#include "sdm_host.h"

namespace sdm_host {

using sdm::bf16;

// The per-device error word (one copy per device context). Every stream's
// calls on a device set bits in the same word, so a check on any stream
// reports (and clears) them all.
__device__ unsigned g_device_error;

thread_local std::string g_last_error;

sdm_status_t fail(sdm_status_t s, const std::string& msg) {
  g_last_error = msg;
  return s;
}
sdm_status_t ok() {
  g_last_error.clear();
  return SDM_OK;
}

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

sdm_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SDM_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(SDM_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
            cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) !=
            cudaSuccess ||
        (e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error)) != cudaSuccess)
      return fail(SDM_ERR_CUDA, std::string("device query: ") + cudaGetErrorString(e));
    d.ready = true;
  }
  *out = &d;
  return SDM_OK;
}

sdm_status_t launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SDM_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return SDM_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raises a kernel's dynamic shared-memory limit when a launch needs more than
// was set before on this device (one driver call per kernel and size instead
// of one per launch; keeps small, latency-bound calls cheap on the host).
std::mutex g_attr_mu;
std::vector<std::pair<std::pair<int, const void*>, size_t>> g_attr;
void set_smem(const void* kern, size_t smem) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (auto& e : g_attr) {
    if (e.first.first == dev && e.first.second == kern) {
      if (smem > e.second) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        e.second = smem;
      }
      return;
    }
  }
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  g_attr.push_back({{dev, kern}, smem});
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

int64_t slots_of(int32_t sqrt_n) { return static_cast<int64_t>(sqrt_n) * sqrt_n; }

sdm_status_t check_dtype(int32_t d, const char* name) {
  if (d != SDM_F32 && d != SDM_BF16) return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " is not SDM_F32 or SDM_BF16");
  return SDM_OK;
}

sdm_status_t check_k(int32_t K, int32_t sqrt_n, const char* name) {
  const int64_t lim = std::min<int64_t>(slots_of(sqrt_n), 256);
  if (K < 1 || K > lim)
    return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " must be in [1, min(N, 256)], got " + std::to_string(K));
  return SDM_OK;
}

sdm_status_t check_shape(const sdm_shape_t* s) {
  if (s == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, "shape is NULL");
  if (s->B < 0 || s->T < 0 || s->H < 0) return fail(SDM_ERR_INVALID_ARGUMENT, "B, T and H must be >= 0");
  if (s->sqrt_n < 1 || s->sqrt_n > 1024) return fail(SDM_ERR_INVALID_ARGUMENT, "sqrt_n must be in [1, 1024]");
  sdm_status_t st;
  if ((st = check_k(s->W, s->sqrt_n, "W")) != SDM_OK) return st;
  if ((st = check_k(s->R, s->sqrt_n, "R")) != SDM_OK) return st;
  if (s->d_v < 16 || s->d_v > 8192 || s->d_v % 16 != 0)
    return fail(SDM_ERR_INVALID_ARGUMENT, "d_v must be a multiple of 16 in [16, 8192]");
  if ((st = check_dtype(s->in_dtype, "in_dtype")) != SDM_OK) return st;
  if (s->state_dtype != SDM_FP8_B16 && (st = check_dtype(s->state_dtype, "state_dtype")) != SDM_OK) return st;
  if (s->state_dtype == SDM_FP8_B16 && s->d_v % 16 != 0)
    return fail(SDM_ERR_INVALID_ARGUMENT, "the fp8 state needs d_v a multiple of 16");
  if (!(s->rms_eps >= 0.0f) || s->rms_eps > 1e30f) return fail(SDM_ERR_INVALID_ARGUMENT, "rms_eps must be finite and >= 0");
  if (s->variant < SDM_VARIANT_AUTO || s->variant > SDM_VARIANT_PIPELINED)
    return fail(SDM_ERR_INVALID_ARGUMENT, "variant must be an sdm_variant_t value");
  if (s->tile < 0 || s->tile > 64) return fail(SDM_ERR_INVALID_ARGUMENT, "tile must be in [0, 64] (0: automatic)");
  if (static_cast<int64_t>(s->B) * s->H > 65535) return fail(SDM_ERR_UNSUPPORTED, "B*H above 65535");
  return SDM_OK;
}

sdm_status_t need_ptr(const void* p, const char* name, bool nonempty) {
  if (!nonempty) return SDM_OK;
  if (p == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " is NULL");
  if (!aligned16(p)) return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " is not 16-byte aligned");
  return SDM_OK;
}

size_t in_size(int32_t d) { return d == SDM_BF16 ? 2 : 4; }
size_t state_size(int32_t d) { return d == SDM_FP8_B16 ? 1 : in_size(d); }

// The per-token gates are read one element at a time: natural alignment
// suffices (a one-token slice of [B, T, H] is rarely 16-byte aligned).
sdm_status_t need_gate(const void* p, const char* name, bool nonempty, int32_t dtype) {
  if (!nonempty) return SDM_OK;
  if (p == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " is NULL");
  if (reinterpret_cast<uintptr_t>(p) % in_size(dtype) != 0)
    return fail(SDM_ERR_INVALID_ARGUMENT, std::string(name) + " is not aligned to its element size");
  return SDM_OK;
}

// ------------------------------------------------------------- selection --

sdm_status_t fast_topk_plan(int n, int K, FastTopkPlan* out) {
  FastTopkPlan P;
  sdm::FastTopkLayout& L = P.L;
  L.n = n;
  L.K = K;
  L.Kh = std::min(K, n);
  int C = 0;
  for (int ra = 0; ra < L.Kh; ++ra) C += std::min(L.Kh, K / (ra + 1));
  L.C = C;
  P.E = K <= 32 ? 1 : 2;                // winners sort width / 32
  P.EH = n <= 32 ? 1 : P.E;             // half sort width / 32
  P.CP = P.E == 1 ? 4 : (P.EH == 1 ? 7 : 9);
  if (C > 32 * P.CP) return fail(SDM_ERR_UNSUPPORTED, "selection candidate count above the register path");
  auto a16 = [](uint32_t x) { return (x + 15u) & ~15u; };
  L.table_bytes = a16(static_cast<uint32_t>(C) * 4u);
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) {
    const uint32_t o = off;
    off += a16(bytes);
    return o;
  };
  L.hist = take(256u * 4u);
  L.sel = take(64u * 8u);
  L.hv = take(2u * 64u * 4u);
  L.hx = take(2u * 64u * 4u);
  L.tie = take(2u * 4u * 32u * P.CP);
  L.warp_bytes = off;
  if (n > 32 * P.EH) {
    while (P.epl * 32 < n) P.epl *= 2;
  }
  *out = P;
  return SDM_OK;
}

// ------------------------------------------------------------ recurrence --

// Record layout; the hazard plan is only stored for the streaming kernel.
sdm::RecLayout rec_layout(int W, int R, bool plan = true) {
  sdm::RecLayout rl{};
  rl.Wp = (W + 3) / 4 * 4;
  rl.Rp = (R + 3) / 4 * 4;
  rl.Fp = plan ? (W + R + 7) / 8 * 8 : 0;
  rl.off_slot_w = 0;
  rl.off_k_w = rl.Wp;
  rl.off_slot_r = 2 * rl.Wp;
  rl.off_q_r = 2 * rl.Wp + rl.Rp;
  rl.off_fwd = 2 * rl.Wp + 2 * rl.Rp;
  rl.off_ab = rl.off_fwd + rl.Fp / 2;
  rl.words = rl.off_ab + 4;
  return rl;
}

// Instantiated streaming tiles: state bytes, columns per CTA, prefetch
// distance, staging chunk, warps.
struct StreamCfg {
  int state_bytes;
  int C, P, L, NW;
};
constexpr StreamCfg kStreamCfgs[] = {
    {4, 64, 3, 8, 16}, {4, 64, 2, 8, 16}, {4, 32, 4, 8, 16}, {4, 32, 4, 8, 8}, {4, 16, 8, 16, 16},
    {4, 16, 4, 8, 8},
    {2, 128, 3, 8, 16}, {2, 64, 4, 8, 16}, {2, 64, 6, 8, 16}, {2, 32, 8, 16, 16}, {2, 32, 8, 16, 8},
    {2, 16, 8, 16, 16}, {2, 16, 4, 8, 8},
};

// Instantiated pipelined tiles: state bytes, columns per CTA (128-byte row
// segments), stages, staging chunk, write warps, read warps, producer warps.
struct PipeCfg {
  int state_bytes;
  int C, P, L, NWW, NWR, NP, S;
};
constexpr PipeCfg kPipeCfgs[] = {
    {2, 64, 6, 16, 4, 3, 8, 1}, {2, 64, 6, 16, 4, 3, 4, 2}, {2, 64, 7, 8, 4, 3, 4, 2}, {2, 64, 6, 16, 4, 4, 8, 1},
    {2, 64, 6, 16, 4, 3, 4, 1}, {4, 32, 6, 16, 4, 3, 4, 1}, {4, 32, 4, 16, 4, 3, 4, 1}, {4, 32, 6, 16, 4, 3, 4, 2},
    // the block-scaled fp8 state: 64 codes (and 4 exponents) a row segment
    {1, 64, 6, 16, 4, 3, 8, 1}, {1, 64, 6, 16, 4, 3, 4, 1},
};

// Instantiated resident tiles: columns per warp, warps per CTA, staging
// chunk, entries per lane block.
struct ResidentCfg {
  int CW, NWARP, L, EB;
};
constexpr ResidentCfg kResidentCfgs[] = {
    {8, 1, 4, 4}, {8, 2, 4, 4}, {4, 2, 4, 2}, {16, 1, 4, 4}, {4, 4, 4, 2}, {8, 2, 8, 4}, {4, 4, 8, 2}, {8, 4, 8, 4},
};

size_t resident_smem(const sdm_shape_t& s, const ResidentCfg& k) {
  return sdm::resident_smem_bytes(static_cast<int>(slots_of(s.sqrt_n)), k.CW, k.NWARP, k.L,
                                  rec_layout(s.W, s.R, false).words, static_cast<int>(in_size(s.in_dtype)));
}
size_t streaming_smem(const sdm_shape_t& s, int C, int P, int L, int NW) {
  const sdm::RecLayout rl = rec_layout(s.W, s.R);
  return sdm::streaming_stage_bytes(P, s.W + s.R, s.W, C, static_cast<int>(in_size(s.state_dtype))) +
         2ull * L * rl.words * 4 + 2ull * L * C * in_size(s.in_dtype) + 2ull * NW * C * 4 + 2 * 8;
}
size_t pipelined_smem(const sdm_shape_t& s, const PipeCfg& k) {
  const sdm::PipeLayout pl = sdm::pipe_layout(s.W, s.R);
  return sdm::pipe_smem_bytes(k.P, k.L, pl.Wp, pl.Rp, pl.words, k.C, static_cast<int>(state_size(s.state_dtype)),
                              static_cast<int>(in_size(s.in_dtype)), k.NWR, k.S, s.state_dtype == SDM_FP8_B16);
}

// Whether every row of the pipelined kernel's stage space (gathered and
// written stages) has a 13-bit source code (the bits above are flags).
bool pipe_codes_fit(const sdm_shape_t& s, const PipeCfg& k) {
  const sdm::PipeLayout pl = sdm::pipe_layout(s.W, s.R);
  return static_cast<int64_t>(k.P) * (pl.Wp + pl.Rp) + static_cast<int64_t>(sdm::pipe_wstages(k.P, k.S)) * pl.Wp <=
         static_cast<int64_t>(sdm::kRowMask);
}

// Whether the automatic variant takes the pipelined kernel for few column
// tiles (on the long-context workload it measures 0.70 us per token against
// the streaming kernel's 0.86 us).
constexpr bool kPipelinedAuto = true;

// Picks the recurrence kernel and its tile. s.tile >= 1 forces entry s.tile
// (1-based) of the chosen kernel's table among the entries that fit the
// shape (for measurements); 0 takes the first that fits.
sdm_status_t choose_scan(const DeviceInfo& dev, const sdm_shape_t& s, ScanChoice* out) {
  // The fp8 state runs in the pipelined kernel (and in the single-launch
  // decode step, chosen before this).
  const bool fp8 = s.state_dtype == SDM_FP8_B16;
  if (fp8 && s.variant != SDM_VARIANT_AUTO && s.variant != SDM_VARIANT_PIPELINED)
    return fail(SDM_ERR_UNSUPPORTED, "the fp8 state (SDM_FP8_B16) runs in the pipelined variant only");
  if (fp8 && s.d_v % 256 != 0)
    return fail(SDM_ERR_UNSUPPORTED, "the fp8 state needs d_v a multiple of 256 (16-byte rows of block exponents)");
  const size_t lim = static_cast<size_t>(dev.max_smem_optin);
  auto pick = [&](size_t n_fit) -> int {  // index into the fitting entries, or -1
    if (s.tile == 0) return n_fit > 0 ? 0 : -1;
    return static_cast<size_t>(s.tile) <= n_fit ? s.tile - 1 : -1;
  };
  ScanChoice c;
  // A resident tile reads and writes all N rows once; below one touched row
  // per slot (T * (W + R) < N, e.g. a decode step) streaming only the
  // selected rows moves less.
  const bool few_tokens = static_cast<int64_t>(s.T) * (s.W + s.R) < slots_of(s.sqrt_n);
  if (!fp8 && (s.variant == SDM_VARIANT_RESIDENT || (s.variant == SDM_VARIANT_AUTO && !few_tokens))) {
    // Resident tiles in order of preference (measured on B200 at N = 1024,
    // d_v = 128: 8-column warp tiles, one warp per CTA, so up to five CTAs
    // share an SM); the first that divides d_v and fits is taken.
    std::vector<ResidentCfg> order;
    // (a CTA stages each token's v row of CW * NWARP columns with a 1-D bulk
    // copy: whole 16-byte units only)
    for (const ResidentCfg& k : kResidentCfgs)
      if (s.d_v % (k.CW * k.NWARP) == 0 && resident_smem(s, k) <= lim &&
          (k.CW * k.NWARP * in_size(s.in_dtype)) % 16 == 0)
        order.push_back(k);
    const int i = pick(order.size());
    if (i >= 0) {
      const ResidentCfg& k = order[i];
      c.kind = SDM_VARIANT_RESIDENT;
      c.resident = true;
      c.CW = k.CW;
      c.NWARP = k.NWARP;
      c.EB = k.EB;
      c.C = k.CW * k.NWARP;
      c.L = k.L;
      c.smem = resident_smem(s, k);
      *out = c;
      return SDM_OK;
    }
    if (s.variant == SDM_VARIANT_RESIDENT)
      return fail(SDM_ERR_UNSUPPORTED, s.tile == 0 ? "the state tile does not fit in shared memory (resident variant)"
                                                   : "no such resident tile for this shape");
  }
  const int s_state = static_cast<int>(state_size(s.state_dtype));
  const int64_t bh = static_cast<int64_t>(s.B) * s.H;
  // The pipelined kernel when 128-byte column tiles alone would leave SMs
  // idle: one SM moves about one random 128-byte row per 3 ns, so a grid
  // smaller than the SM count cannot approach the HBM bandwidth; splitting
  // each tile's slots over two CTAs doubles the SMs at work.
  const int c128 = 128 / s_state;
  const bool few_tiles = s.d_v % c128 == 0 && bh * (s.d_v / c128) < dev.sms;
  const bool rows_fit = bh * slots_of(s.sqrt_n) <= INT_MAX;  // TMA row coordinates are int32
  if ((s.variant == SDM_VARIANT_PIPELINED || fp8) && !rows_fit)
    return fail(SDM_ERR_UNSUPPORTED, "the pipelined variant needs B*H*N below 2^31 state rows");
  if (rows_fit && (s.variant == SDM_VARIANT_PIPELINED || fp8 ||
                   (s.variant == SDM_VARIANT_AUTO && kPipelinedAuto && few_tiles))) {
    std::vector<PipeCfg> order;
    for (const PipeCfg& k : kPipeCfgs)
      if (k.state_bytes == s_state && s.d_v % k.C == 0 && pipelined_smem(s, k) <= lim && pipe_codes_fit(s, k))
        order.push_back(k);
    const int i = pick(order.size());
    if (i >= 0) {
      const PipeCfg& k = order[i];
      c.kind = SDM_VARIANT_PIPELINED;
      c.C = k.C;
      c.P = k.P;
      c.L = k.L;
      c.NWW = k.NWW;
      c.NWR = k.NWR;
      c.NP = k.NP;
      c.S = k.S;
      c.parts = bh * (s.d_v / k.C) * 2 <= dev.sms ? 2 : 1;
      c.smem = pipelined_smem(s, k);
      *out = c;
      return SDM_OK;
    }
    if (s.variant == SDM_VARIANT_PIPELINED || fp8)
      return fail(SDM_ERR_UNSUPPORTED, s.tile == 0 ? "W + R too large for the pipelined stage rings"
                                                   : "no such pipelined tile for this shape");
  }
  // Streaming tiles, best first. Random row segments of >= 256 B run HBM near
  // its copy bandwidth, 128 B at ~75%, 64 B at ~40% (measured gathers on
  // B200), so wide segments win while the grid still fills the SMs.
  std::vector<StreamCfg> order;
  for (const StreamCfg& k : kStreamCfgs)
    if (k.state_bytes == s_state && s.d_v % k.C == 0 && k.C <= 32 * k.NW && streaming_smem(s, k.C, k.P, k.L, k.NW) <= lim)
      order.push_back(k);
  auto ctas = [&](const StreamCfg& k) { return bh * (s.d_v / k.C); };
  std::stable_sort(order.begin(), order.end(), [&](const StreamCfg& x, const StreamCfg& y) {
    const bool fx = ctas(x) >= dev.sms / 2, fy = ctas(y) >= dev.sms / 2;  // fills at least half the SMs
    if (fx != fy) return fx;
    const int rx = x.C * x.state_bytes, ry = y.C * y.state_bytes;
    if (rx != ry) return rx > ry;  // wider row segments first
    return x.P > y.P;
  });
  const int i = pick(order.size());
  if (i < 0)
    return fail(SDM_ERR_UNSUPPORTED, s.tile == 0 ? "W + R too large for the streaming stage ring"
                                                 : "no such streaming tile for this shape");
  const StreamCfg& k = order[i];
  c.kind = SDM_VARIANT_STREAMING;
  c.C = k.C;
  c.P = k.P;
  c.L = k.L;
  c.NWARP = k.NW;
  c.smem = streaming_smem(s, k.C, k.P, k.L, k.NW);
  *out = c;
  return SDM_OK;
}

// Bytes of the second slot part's read sums (pipelined kernel with two parts).
size_t y_other_bytes(const sdm_shape_t& s, const ScanChoice& c) {
  if (c.kind != SDM_VARIANT_PIPELINED || c.parts < 2) return 0;
  return align256(static_cast<size_t>(s.B) * s.T * s.H * s.d_v * 4u);
}
// Workspace of the chosen recurrence kernel: per-token records (and, for the
// pipelined kernel with two parts, the second part's read sums after them).
size_t records_bytes(const sdm_shape_t& s, const ScanChoice& c) {
  const int64_t n = static_cast<int64_t>(s.B) * s.H * s.T;
  if (c.kind == SDM_VARIANT_PIPELINED)
    return align256(static_cast<size_t>(n) * c.parts * sdm::pipe_layout(s.W, s.R).words * 4u) + y_other_bytes(s, c);
  return align256(static_cast<size_t>(n) * rec_layout(s.W, s.R).words * 4u);
}
// The same before a kernel is chosen (workspace queries): the chosen
// kernel's need on the current device, or the largest of all kernels' when
// no device can be queried.
size_t records_bytes(const sdm_shape_t& s) {
  const std::string saved = g_last_error;
  DeviceInfo* dev;
  ScanChoice c;
  if (device_info(&dev) == SDM_OK && choose_scan(*dev, s, &c) == SDM_OK) {
    g_last_error = saved;
    return records_bytes(s, c);
  }
  g_last_error = saved;
  ScanChoice pipe;
  pipe.kind = SDM_VARIANT_PIPELINED;
  pipe.parts = 2;
  return std::max(records_bytes(s, ScanChoice()), records_bytes(s, pipe));
}

template <typename Tin>
sdm_status_t launch_records(const sdm_shape_t& s, const int32_t* idx_w, const float* w_w, const int32_t* idx_r,
                            const float* w_r, const void* alpha, const void* beta, int P, uint32_t* rec,
                            unsigned* err, const DeviceInfo& dev, cudaStream_t st) {
  const sdm::RecLayout rl = rec_layout(s.W, s.R, P > 0);
  int log2_cells = 1;
  while ((1 << log2_cells) < 2 * s.W) ++log2_cells;
  const size_t smem =
      P > 0 ? static_cast<size_t>(sdm::kRecTokensPerBlock + P - 1) * (size_t{1} << log2_cells) * 4 : 0;
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return fail(SDM_ERR_UNSUPPORTED, "hazard tables exceed shared memory");
  auto kern = sdm::k_build_records<Tin>;
  set_smem(reinterpret_cast<const void*>(kern), smem);
  const int tblocks = (s.T + sdm::kRecTokensPerBlock - 1) / sdm::kRecTokensPerBlock;
  const dim3 grid(tblocks, s.B * s.H);
  kern<<<grid, 256, smem, st>>>(idx_w, w_w, idx_r, w_r, static_cast<const Tin*>(alpha), static_cast<const Tin*>(beta),
                                s.T, s.H, static_cast<int>(slots_of(s.sqrt_n)), s.W, s.R, P, log2_cells, rl, rec, err);
  return launch_status("record build launch");
}

// B copies of bytes_per_b bytes (a multiple of 16) of src into dst.
sdm_status_t copy_per_batch_row(const DeviceInfo& dev, int B, int64_t bytes_per_b, const void* src, void* dst,
                                cudaStream_t st) {
  const int64_t units = bytes_per_b / 16;
  if (units == 0 || B == 0) return SDM_OK;
  const int gx = static_cast<int>(std::min<int64_t>((units + 255) / 256, std::max(1, dev.sms * 8 / std::max(1, B))));
  for (int b0 = 0; b0 < B; b0 += 65535) {
    const int nb = std::min(65535, B - b0);
    sdm::k_state_init<<<dim3(gx, nb), 256, 0, st>>>(static_cast<const uint4*>(src),
                                                   static_cast<uint4*>(dst) + static_cast<int64_t>(b0) * units, units);
  }
  return launch_status("state init launch");
}

// M[b] <- M0 for every batch row. The fp8 state is the codes of all rows,
// then their exponents: two copies (M0's codes and exponents into M's).
sdm_status_t launch_state_init(const DeviceInfo& dev, const sdm_shape_t& s, const void* M0, void* M, cudaStream_t st) {
  const int64_t values = static_cast<int64_t>(s.H) * slots_of(s.sqrt_n) * s.d_v;  // one batch row's state values
  if (s.state_dtype != SDM_FP8_B16)
    return copy_per_batch_row(dev, s.B, values * static_cast<int64_t>(in_size(s.state_dtype)), M0, M, st);
  sdm_status_t r = copy_per_batch_row(dev, s.B, values, M0, M, st);
  if (r != SDM_OK) return r;
  return copy_per_batch_row(dev, s.B, values / 16, static_cast<const uint8_t*>(M0) + values,
                            static_cast<uint8_t*>(M) + static_cast<int64_t>(s.B) * values, st);
}

sdm_status_t launch_epilogue(const DeviceInfo& dev, const sdm_shape_t& s, float* y, const void* g, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(s.B) * s.T * s.H;
  if (rows == 0) return SDM_OK;
  const int grid = static_cast<int>(std::min<int64_t>((rows + 7) / 8, static_cast<int64_t>(dev.sms) * 16));
  if (s.in_dtype == SDM_BF16)
    sdm::k_rmsnorm_gate<bf16><<<grid, 256, 0, st>>>(y, static_cast<const bf16*>(g), rows, s.d_v, s.rms_eps);
  else
    sdm::k_rmsnorm_gate<float><<<grid, 256, 0, st>>>(y, static_cast<const float*>(g), rows, s.d_v, s.rms_eps);
  return launch_status("epilogue launch");
}

// Records + recurrence (+ epilogue). With M_in != M the resident kernel reads
// M_in (b-stride M_in_b_stride) and writes M; the streaming kernel works in
// place on M, which then must already hold the initial state.
// Records a caller event (no-op without events).
struct Trace {
  void* const* events = nullptr;
  void* const* chunk_events = nullptr;  // an overlapped call: two a chunk around its recurrence launch
  void mark(int i, cudaStream_t st) const {
    if (events != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st);
  }
  void mark_chunk(int64_t i, cudaStream_t st) const {
    if (chunk_events != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(chunk_events[i]), st);
  }
};

sdm_status_t run_scan(const DeviceInfo& dev, const sdm_shape_t& s, const ScanChoice& c, const int32_t* idx_w,
                      const float* w_w, const int32_t* idx_r, const float* w_r, const void* v, const void* alpha,
                      const void* beta, const void* g, const void* M_in, int64_t M_in_b_stride, void* M, float* y,
                      uint32_t* rec, cudaStream_t st, const Trace& tr = Trace(), bool init_before_scan = false,
                      const void* M0_for_init = nullptr, float* ckpt = nullptr, int ckpt_C = 0) {
  sdm_status_t r;
  if (c.kind == SDM_VARIANT_PIPELINED) {
    if ((r = launch_pipe_records(s, c, idx_w, w_w, idx_r, w_r, alpha, beta, rec, nullptr, dev, st)) != SDM_OK)
      return r;
    // the second part's read sums go after the records; a separate pass adds them into y
    const size_t y_other_off = records_bytes(s, c) - y_other_bytes(s, c);
    float* y_other = c.parts > 1 ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(rec) + y_other_off)
                                 : nullptr;
    tr.mark(2, st);
    if (init_before_scan && (r = launch_state_init(dev, s, M0_for_init, M, st)) != SDM_OK) return r;
    tr.mark(3, st);
    sdm::PipeArgs a{};
    a.B = s.B; a.T = s.T; a.H = s.H;
    a.N = static_cast<int>(slots_of(s.sqrt_n));
    a.d_v = s.d_v; a.W = s.W; a.R = s.R;
    a.parts = c.parts;
    a.pl = sdm::pipe_layout(s.W, s.R);
    a.rec = rec;
    a.v = v;
    a.M = M;
    a.y = y;
    a.y_other = y_other;
    a.err = dev.err;
    if ((r = launch_pipe(c, s, a, st)) != SDM_OK) return r;
    if (y_other != nullptr) {
      const int64_t n4 = static_cast<int64_t>(s.B) * s.T * s.H * s.d_v / 4;
      const int grid = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, static_cast<int64_t>(dev.sms) * 8));
      sdm::k_add_f4<<<grid, 256, 0, st>>>(reinterpret_cast<float4*>(y), reinterpret_cast<const float4*>(y_other), n4);
      if ((r = launch_status("part sum launch")) != SDM_OK) return r;
    }
    tr.mark(4, st);
    if (g != nullptr && (r = launch_epilogue(dev, s, y, g, st)) != SDM_OK) return r;
    tr.mark(5, st);
    return SDM_OK;
  }
  const int plan_p = c.resident ? 0 : c.P + 1;  // the streaming plan looks back P tokens
  if ((r = (s.in_dtype == SDM_BF16 ? launch_records<bf16>(s, idx_w, w_w, idx_r, w_r, alpha, beta, plan_p,
                                                          rec, dev.err, dev, st)
                                   : launch_records<float>(s, idx_w, w_w, idx_r, w_r, alpha, beta, plan_p,
                                                           rec, dev.err, dev, st))) != SDM_OK)
    return r;
  tr.mark(2, st);
  if (init_before_scan && (r = launch_state_init(dev, s, M0_for_init, M, st)) != SDM_OK) return r;
  tr.mark(3, st);
  sdm::ScanArgs a{};
  a.B = s.B; a.T = s.T; a.H = s.H;
  a.N = static_cast<int>(slots_of(s.sqrt_n));
  a.d_v = s.d_v; a.W = s.W; a.R = s.R;
  a.rl = rec_layout(s.W, s.R, !c.resident);
  a.rec = rec;
  a.v = v;
  a.M_in = M_in;
  a.M_in_b_stride = M_in_b_stride;
  a.M = M;
  a.y = y;
  a.err = dev.err;
  if ((r = launch_scan(c, s, a, st, ckpt, ckpt_C)) != SDM_OK) return r;
  tr.mark(4, st);
  if (g != nullptr && (r = launch_epilogue(dev, s, y, g, st)) != SDM_OK) return r;
  tr.mark(5, st);
  return SDM_OK;
}

// Scratch of sdm_layer_forward_noalloc. In host code this name only stands
// for the device array; its device address comes from cudaGetSymbolAddress,
// once per device (noalloc_scratch below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SDM_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up on
// first use with that device current.
sdm_status_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SDM_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(SDM_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(SDM_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SDM_OK;
}

}  // namespace

// ------------------------------------------------------------- backward --

namespace sdm_host {

sdm_status_t choose_bwd(const sdm_shape_t& s, BwdChoice* out) {
  if (s.state_dtype != SDM_F32)
    return fail(SDM_ERR_UNSUPPORTED, "sdm_scan_backward needs an fp32 state (state_dtype SDM_F32)");
  const int64_t N = slots_of(s.sqrt_n);
  const sdm::RecLayout rl = rec_layout(s.W, s.R, false);
  const int in_bytes = static_cast<int>(in_size(s.in_dtype));
  auto ring_bytes = [&](int U) {
    return static_cast<size_t>(sdm::kBwdStages) * sdm::bwd_stage(s.W, rl.words, U, in_bytes).words * 4;
  };
  BwdChoice c;
  const size_t on_chip = 2 * static_cast<size_t>(N) * 4 * 4 + ring_bytes(1);
  c.global = on_chip > kBwdSmemLimit;
  c.U = c.global ? (s.d_v % 32 == 0 ? 8 : 4) : 1;
  c.smem = c.global ? ring_bytes(c.U) : on_chip;
  c.nwb = s.tile == 1 ? 1 : 2;
  if (c.smem > kBwdSmemLimit) return fail(SDM_ERR_UNSUPPORTED, "backward staging exceeds shared memory (W, R too large)");
  if (c.global) {
    // Chunk length near sqrt(T N / W): checkpoints (T / C states) and the log
    // (C W rows) then take about the same memory.
    const double best = std::sqrt(static_cast<double>(std::max(1, s.T)) * static_cast<double>(N) / s.W);
    int C = kBwdChunk;
    while (C < best && C < (1 << 20)) C *= 2;
    c.C = std::max(1, std::min(C, s.T));
  } else {
    c.C = std::max(1, std::min<int>(kBwdChunk, s.T));
  }
  const int cols = 4 * c.U;
  c.ntile = s.d_v / cols;
  const int64_t tiles = static_cast<int64_t>(s.B) * s.H * c.ntile;
  const int64_t nC = (static_cast<int64_t>(s.T) + c.C - 1) / c.C;
  c.ckpt_bytes = align256(static_cast<size_t>(tiles) * std::max<int64_t>(0, nC - 1) * N * cols * 4);
  c.log_bytes = align256(static_cast<size_t>(tiles) * c.C * s.W * cols * 4);
  c.part_bytes = align256(static_cast<size_t>(s.B) * s.T * s.H * c.ntile * (s.W + s.R + 2) * 4);
  c.rec_bytes = align256(static_cast<size_t>(s.B) * s.H * s.T * rl.words * 4);
  c.work_bytes = c.global ? align256(static_cast<size_t>(s.B) * s.H * N * s.d_v * 4) : 0;
  *out = c;
  return SDM_OK;
}

}  // namespace

// ---------------------------------------------------------------- decode --

namespace sdm_host {

// The fused single-launch decode step (T = 1, W = R <= 64, automatic
// variant). Sets *used = false (and returns SDM_OK) when the shape is not one
// it covers, so the caller takes the general path.
sdm_status_t try_decode_step(const DeviceInfo& dev, const sdm_shape_t& s, const void* kp, const void* qp,
                             const void* v, const void* alpha, const void* beta, const void* g, void* M, float* y,
                             cudaStream_t st, bool* used) {
  *used = false;
  if (s.T != 1 || s.W != s.R || s.W > sdm::kFastTopkMaxK || s.variant != SDM_VARIANT_AUTO) return SDM_OK;
  if (static_cast<int64_t>(s.B) * s.H > 0x7FFFFFFFLL) return SDM_OK;
  FastTopkPlan P;
  if (fast_topk_plan(s.sqrt_n, s.W, &P) != SDM_OK) {
    g_last_error.clear();
    return SDM_OK;
  }
  const int VE = s.state_dtype == SDM_FP8_B16 ? 16 : 16 / static_cast<int>(in_size(s.state_dtype));
  const int UR = s.d_v / VE;
  const int groups = UR >= sdm::kDecodeThreads ? 1 : sdm::kDecodeThreads / UR;
  sdm::DecodeArgs a{};
  a.H = s.H;
  a.N = static_cast<int>(slots_of(s.sqrt_n));
  a.d_v = s.d_v;
  a.K = s.W;
  a.eps = s.rms_eps;
  a.L = P.L;
  a.kp = kp; a.qp = qp; a.v = v; a.alpha = alpha; a.beta = beta; a.g = g; a.M = M; a.y = y;
  a.exps = s.state_dtype == SDM_FP8_B16
               ? reinterpret_cast<int8_t*>(M) + static_cast<int64_t>(s.B) * s.H * slots_of(s.sqrt_n) * s.d_v
               : nullptr;
  a.sel_off = static_cast<uint32_t>(align16(P.L.table_bytes + 2ull * P.L.warp_bytes));
  a.part_off = static_cast<uint32_t>(a.sel_off + align16(16ull * s.W));
  a.err = dev.err;
  const size_t smem = a.part_off + static_cast<size_t>(groups) * s.d_v * 4;
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return SDM_OK;
  const int grid = s.B * s.H;
  const sdm_status_t r = launch_decode(P, s.in_dtype, s.state_dtype, a, smem, grid, st);
  if (r == SDM_OK) *used = true;
  return r;
}

}  // namespace

namespace sdm_host {
// sdm_scan_backward, optionally with the forward's checkpoints (ckpt_ext:
// [ceil(T / C) - 1][B,H,N,d_v] fp32 for this shape's backward chunk C), which
// replace the backward's own first pass.
sdm_status_t scan_backward_impl(const sdm_shape_t* shape, const int32_t* idx_w, const float* w_w,
                                const int32_t* idx_r, const float* w_r, const void* v, const void* alpha,
                                const void* beta, const float* M_in, int32_t m_in_shared, const float* dy, float* dM,
                                float* dv, float* dalpha, float* dbeta, float* dw_w, float* dw_r, void* workspace,
                                size_t workspace_bytes, void* stream, const float* ckpt_ext) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const sdm_shape_t& s = *shape;
  BwdChoice c;
  if ((r = choose_bwd(s, &c)) != SDM_OK) return r;
  const bool any = static_cast<int64_t>(s.B) * s.H > 0;
  const bool tok = static_cast<int64_t>(s.B) * s.T * s.H > 0;
  if ((r = need_ptr(idx_w, "idx_w", tok)) || (r = need_ptr(w_w, "w_w", tok)) || (r = need_ptr(idx_r, "idx_r", tok)) ||
      (r = need_ptr(w_r, "w_r", tok)) || (r = need_ptr(v, "v", tok)) || (r = need_gate(alpha, "alpha", tok, s.in_dtype)) ||
      (r = need_gate(beta, "beta", tok, s.in_dtype)) || (r = need_ptr(M_in, "M_in", any)) ||
      (r = need_ptr(dy, "dy", tok)) || (r = need_ptr(dM, "dM", any)) || (r = need_ptr(dv, "dv", tok)) ||
      (r = need_gate(dalpha, "dalpha", tok, SDM_F32)) || (r = need_gate(dbeta, "dbeta", tok, SDM_F32)) ||
      (r = need_ptr(dw_w, "dw_w", tok)) || (r = need_ptr(dw_r, "dw_r", tok)))
    return r;
  if (!any) return ok();
  const size_t need = c.total();
  if (workspace_bytes < need)
    return fail(SDM_ERR_INVALID_ARGUMENT,
                "workspace_bytes below sdm_scan_backward_workspace_bytes() = " + std::to_string(need));
  if ((r = need_ptr(workspace, "workspace", need > 0)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  if (static_cast<size_t>(dev->max_smem_optin) < c.smem)
    return fail(SDM_ERR_UNSUPPORTED, "the device's shared memory per block is below the backward tile's");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t N = slots_of(s.sqrt_n);
  if (s.T == 0) return ok();  // dL/dM_0 = dL/dM_T, already in dM
  sdm::BwdArgs a;
  a.B = s.B; a.T = s.T; a.H = s.H; a.N = static_cast<int>(N); a.d_v = s.d_v; a.W = s.W; a.R = s.R;
  a.C = c.C; a.ntile = c.ntile;
  a.rl = rec_layout(s.W, s.R, false);
  a.v = v;
  a.M_in = M_in;
  a.M_in_b_stride = m_in_shared ? 0 : static_cast<int64_t>(s.H) * N * s.d_v;
  a.dy = dy; a.dM = dM; a.dv = dv;
  char* ws = static_cast<char*>(workspace);
  a.part = reinterpret_cast<float*>(ws);
  a.ckpt = reinterpret_cast<float*>(ws + c.part_bytes);
  a.logbuf = reinterpret_cast<float*>(ws + c.part_bytes + c.ckpt_bytes);
  uint32_t* rec = reinterpret_cast<uint32_t*>(ws + c.part_bytes + c.ckpt_bytes + c.log_bytes);
  a.rec = rec;
  a.Mwork = c.global ? reinterpret_cast<float*>(ws + c.part_bytes + c.ckpt_bytes + c.log_bytes + c.rec_bytes) : nullptr;
  a.ckpt_ext = ckpt_ext;
  a.err = dev->err;
  if (s.in_dtype == SDM_BF16) {
    if ((r = launch_records<sdm::bf16>(s, idx_w, w_w, idx_r, w_r, alpha, beta, 0, rec, dev->err, *dev, st)) != SDM_OK)
      return r;
    r = launch_bwd(c, SDM_BF16, a, st);
  } else {
    if ((r = launch_records<float>(s, idx_w, w_w, idx_r, w_r, alpha, beta, 0, rec, dev->err, *dev, st)) != SDM_OK)
      return r;
    r = launch_bwd(c, SDM_F32, a, st);
  }
  if (r != SDM_OK) return r;
  const int64_t n_th = static_cast<int64_t>(s.B) * s.T * s.H;
  const int64_t total = n_th * (s.W + s.R + 2);
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 8LL * dev->sms));
  sdm::k_scan_backward_reduce<<<blocks, 256, 0, st>>>(a.part, n_th, s.W, s.R, c.ntile, dw_w, dw_r, dalpha, dbeta);
  if ((r = launch_status("backward reduce launch")) != SDM_OK) return r;
  return ok();
}

// The chunk and bytes of the checkpoints the forward stores for the
// backward of this shape: the resident recurrence with an fp32 state only.
sdm_status_t checkpoint_size(const DeviceInfo& dev, const sdm_shape_t& s, int32_t* chunk, size_t* bytes) {
  ScanChoice c;
  sdm_status_t r;
  if ((r = choose_scan(dev, s, &c)) != SDM_OK) return r;
  if (!c.resident || s.state_dtype != SDM_F32)
    return fail(SDM_ERR_UNSUPPORTED,
                "the forward stores backward checkpoints only with the resident recurrence and an fp32 state");
  BwdChoice b;
  if ((r = choose_bwd(s, &b)) != SDM_OK) return r;
  const int64_t n = (static_cast<int64_t>(s.T) + b.C - 1) / b.C;
  *chunk = b.C;
  *bytes = static_cast<size_t>(std::max<int64_t>(n - 1, 0)) * s.B * s.H * slots_of(s.sqrt_n) * s.d_v * 4;
  return SDM_OK;
}
}  // namespace sdm_host

namespace sdm_host {
// ------------------------------------------------- overlapped layer call --
//
// The pipelined recurrence runs few CTAs (one per SM, 2 x 2 x 32 = 128 on the
// long-context workload), so SMs are left over while it runs. A layer call
// with one batch row and at least two chunks of kOverlapChunk tokens runs as
// chunks: the selection of chunk k + 1 runs on a low-priority stream (on the
// spare SMs: its shared memory does not fit beside a recurrence CTA) while
// the recurrence of chunk k runs on a high-priority stream, continuing from
// the state in M_out; each chunk's records are built on the high-priority
// stream just before its recurrence (the spare SMs alone are too few for
// both selection and records in a chunk's recurrence time). The recurrence over chunks
// equals one recurrence bit for bit (the state is the checkpoint; the hazard
// plan only changes where a row is read from), and selection and records are
// per token, so the outputs are those of the one-pass call. Every dependency
// is a stream event on work enqueued earlier (no kernel waits on another).
constexpr int32_t kOverlapChunk = 65536;

bool overlapped(const sdm_shape_t& s, const ScanChoice& c) {
  return c.kind == SDM_VARIANT_PIPELINED && s.B == 1 && s.T >= 2 * kOverlapChunk;
}
int64_t overlap_chunks(const sdm_shape_t& s) { return (static_cast<int64_t>(s.T) + kOverlapChunk - 1) / kOverlapChunk; }

// Workspace of an overlapped call: two chunk buffers of selections, one of
// records, and the second slot part's read sums of the whole call.
size_t overlap_workspace(const sdm_shape_t& s, const ScanChoice& c) {
  const size_t tch = static_cast<size_t>(kOverlapChunk) * s.H;
  const size_t sel = 2 * align256(tch * s.W * 4) + 2 * align256(tch * s.R * 4);
  return 2 * sel + align256(tch * c.parts * sdm::pipe_layout(s.W, s.R).words * 4u) + y_other_bytes(s, c);
}

// The library's two streams on the current device, created on first use:
// the first at the greatest priority (the recurrence), the second at the
// least (selection and records), so that pending recurrence CTAs are placed
// first when SMs free up.
std::mutex g_lane_mu;
cudaStream_t g_lane[64][2] = {};
sdm_status_t lane_streams(cudaStream_t* hi, cudaStream_t* lo) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SDM_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(SDM_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_lane_mu);
  if (g_lane[dev][0] == nullptr) {
    int least = 0, greatest = 0;
    cudaStream_t a = nullptr, b = nullptr;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&a, cudaStreamNonBlocking, greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&b, cudaStreamNonBlocking, least)) != cudaSuccess) {
      if (a != nullptr) cudaStreamDestroy(a);
      return fail(SDM_ERR_CUDA, std::string("stream creation: ") + cudaGetErrorString(e));
    }
    g_lane[dev][0] = a;
    g_lane[dev][1] = b;
  }
  *hi = g_lane[dev][0];
  *lo = g_lane[dev][1];
  return SDM_OK;
}

// Events of one overlapped call, released once the call is enqueued (the
// driver keeps an event until the work recorded in it completes).
struct CallEvents {
  cudaEvent_t e[7] = {};
  ~CallEvents() {
    for (cudaEvent_t x : e)
      if (x != nullptr) cudaEventDestroy(x);
  }
  sdm_status_t create() {
    for (cudaEvent_t& x : e) {
      const cudaError_t err = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
      if (err != cudaSuccess) return fail(SDM_ERR_CUDA, std::string("cudaEventCreate: ") + cudaGetErrorString(err));
    }
    return SDM_OK;
  }
};

sdm_status_t layer_forward_overlapped(const DeviceInfo& dev, const sdm_shape_t& s, const ScanChoice& c,
                                      const void* kp, const void* qp, const void* v, const void* alpha,
                                      const void* beta, const void* g, const void* M0, void* M_out, float* y,
                                      unsigned char* ws, cudaStream_t caller, const Trace& tr) {
  sdm_status_t r;
  cudaStream_t hi = nullptr, lo = nullptr;
  if ((r = lane_streams(&hi, &lo)) != SDM_OK) return r;
  CallEvents ev;  // 0 fork; 1, 2 selection into buffer 0, 1; 3, 4 records from buffer 0, 1; 5, 6 join
  if ((r = ev.create()) != SDM_OK) return r;
  const int64_t tch = static_cast<int64_t>(kOverlapChunk) * s.H;
  const size_t rec_b = align256(static_cast<size_t>(tch) * c.parts * sdm::pipe_layout(s.W, s.R).words * 4u);
  int32_t* idx_w[2];
  float* w_w[2];
  int32_t* idx_r[2];
  float* w_r[2];
  for (int b = 0; b < 2; ++b) {
    idx_w[b] = reinterpret_cast<int32_t*>(ws);
    ws += align256(tch * s.W * 4);
    w_w[b] = reinterpret_cast<float*>(ws);
    ws += align256(tch * s.W * 4);
    idx_r[b] = reinterpret_cast<int32_t*>(ws);
    ws += align256(tch * s.R * 4);
    w_r[b] = reinterpret_cast<float*>(ws);
    ws += align256(tch * s.R * 4);
  }
  uint32_t* rec = reinterpret_cast<uint32_t*>(ws);
  ws += rec_b;
  float* y_other = c.parts > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  // Both lanes start after the caller's earlier work; the caller's stream
  // continues after both lanes' work, also when an enqueue fails part way.
  tr.mark(0, caller);
  cudaEventRecord(ev.e[0], caller);
  cudaStreamWaitEvent(hi, ev.e[0], 0);
  cudaStreamWaitEvent(lo, ev.e[0], 0);
  auto finish = [&](sdm_status_t status) {
    cudaEventRecord(ev.e[5], lo);
    cudaEventRecord(ev.e[6], hi);
    cudaStreamWaitEvent(caller, ev.e[5], 0);
    cudaStreamWaitEvent(caller, ev.e[6], 0);
    return status;
  };
  if ((r = launch_state_init(dev, s, M0, M_out, hi)) != SDM_OK) return finish(r);
  const size_t in_b = in_size(s.in_dtype);
  const auto* kpb = static_cast<const unsigned char*>(kp);
  const auto* qpb = static_cast<const unsigned char*>(qp);
  const auto* vb = static_cast<const unsigned char*>(v);
  const auto* ab = static_cast<const unsigned char*>(alpha);
  const auto* bb = static_cast<const unsigned char*>(beta);
  const int64_t key_row = 2LL * s.sqrt_n, n_chunks = overlap_chunks(s);
  for (int64_t k = 0; k < n_chunks; ++k) {
    const int b = static_cast<int>(k & 1);
    const int64_t t0 = k * kOverlapChunk;
    sdm_shape_t sk = s;
    sk.T = static_cast<int32_t>(std::min<int64_t>(kOverlapChunk, s.T - t0));
    const int64_t th = static_cast<int64_t>(sk.T) * s.H, h0 = t0 * s.H;  // the chunk's token-heads, its first one
    // chunk k's selection on the low-priority lane, once chunk k - 2's
    // records are through with buffer b
    if (k >= 2) cudaStreamWaitEvent(lo, ev.e[3 + b], 0);
    if ((r = topk_impl(dev, kpb + h0 * key_row * in_b, s.in_dtype, th, s.sqrt_n, s.W, idx_w[b], w_w[b], lo)) != SDM_OK ||
        (r = topk_impl(dev, qpb + h0 * key_row * in_b, s.in_dtype, th, s.sqrt_n, s.R, idx_r[b], w_r[b], lo)) != SDM_OK)
      return finish(r);
    if (k == 0) tr.mark(1, lo);
    cudaEventRecord(ev.e[1 + b], lo);
    // chunk k's records and recurrence on the high-priority lane
    cudaStreamWaitEvent(hi, ev.e[1 + b], 0);
    if ((r = launch_pipe_records(sk, c, idx_w[b], w_w[b], idx_r[b], w_r[b], ab + h0 * in_b, bb + h0 * in_b, rec,
                                 nullptr, dev, hi)) != SDM_OK)
      return finish(r);
    cudaEventRecord(ev.e[3 + b], hi);
    if (k == 0) {
      tr.mark(2, hi);
      tr.mark(3, hi);
    }
    sdm::PipeArgs a{};
    a.B = 1; a.T = sk.T; a.H = s.H;
    a.N = static_cast<int>(slots_of(s.sqrt_n));
    a.d_v = s.d_v; a.W = s.W; a.R = s.R;
    a.parts = c.parts;
    a.pl = sdm::pipe_layout(s.W, s.R);
    a.rec = rec;
    a.v = vb + h0 * s.d_v * in_b;
    a.M = M_out;
    a.y = y + h0 * s.d_v;
    a.y_other = y_other != nullptr ? y_other + h0 * s.d_v : nullptr;
    a.err = dev.err;
    tr.mark_chunk(2 * k, hi);
    if ((r = launch_pipe(c, sk, a, hi)) != SDM_OK) return finish(r);
    tr.mark_chunk(2 * k + 1, hi);
  }
  if (y_other != nullptr) {
    const int64_t n4 = static_cast<int64_t>(s.T) * s.H * s.d_v / 4;
    const int grid = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, static_cast<int64_t>(dev.sms) * 8));
    sdm::k_add_f4<<<grid, 256, 0, hi>>>(reinterpret_cast<float4*>(y), reinterpret_cast<const float4*>(y_other), n4);
    if ((r = launch_status("part sum launch")) != SDM_OK) return finish(r);
  }
  tr.mark(4, hi);
  if (g != nullptr && (r = launch_epilogue(dev, s, y, g, hi)) != SDM_OK) return finish(r);
  tr.mark(5, hi);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return finish(fail(SDM_ERR_CUDA, std::string("overlapped layer call: ") + cudaGetErrorString(e)));
  return finish(SDM_OK);
}

sdm_status_t layer_forward_impl(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                const void* alpha, const void* beta, const void* g, const void* M0, void* M_out,
                                float* y, void* workspace, size_t workspace_bytes, void* stream, void* const* events,
                                int32_t n_events, float* ckpt, size_t ckpt_bytes) {
  sdm_status_t r;
  if (!(n_events == 0 || (n_events >= 6 && n_events % 2 == 0 && events != nullptr)))
    return fail(SDM_ERR_INVALID_ARGUMENT,
                "n_events must be 0, or 6 (+ 2 a chunk of an overlapped call) with a non-NULL events array");
  Trace tr;
  if (n_events > 0) {
    for (int i = 0; i < n_events; ++i)
      if (events[i] == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, "events[] holds a NULL event");
    tr.events = events;
    if (n_events > 6) tr.chunk_events = events + 6;
  }
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const sdm_shape_t& s = *shape;
  const int64_t th = static_cast<int64_t>(s.B) * s.T * s.H;
  const bool any = th > 0;
  const bool any_state = static_cast<int64_t>(s.B) * s.H > 0;
  if ((r = need_ptr(kp, "kp", any)) || (r = need_ptr(qp, "qp", any)) || (r = need_ptr(v, "v", any)) ||
      (r = need_gate(alpha, "alpha", any, s.in_dtype)) || (r = need_gate(beta, "beta", any, s.in_dtype)) || (r = need_ptr(y, "y", any)) ||
      (r = need_ptr(M0, "M0", any_state)) || (r = need_ptr(M_out, "M_out", any_state)))
    return r;
  if (g != nullptr && (r = need_ptr(g, "g", any)) != SDM_OK) return r;
  if (!any_state) return ok();
  const size_t need = sdm_layer_forward_workspace_bytes(shape);
  if (any && workspace_bytes < need)
    return fail(SDM_ERR_INVALID_ARGUMENT,
                "workspace_bytes below sdm_layer_forward_workspace_bytes() = " + std::to_string(need));
  if (any && (r = need_ptr(workspace, "workspace", true)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!any) return launch_state_init(*dev, s, M0, M_out, st) == SDM_OK ? ok() : SDM_ERR_CUDA;
  ScanChoice c;
  if ((r = choose_scan(*dev, s, &c)) != SDM_OK) return r;
  const bool overlap = ckpt == nullptr && overlapped(s, c) && overlap_workspace(s, c) <= workspace_bytes;
  if (n_events > 6 && !(overlap && n_events == 6 + 2 * overlap_chunks(s)))
    return fail(SDM_ERR_INVALID_ARGUMENT, "n_events must be 6 + 2 * sdm_layer_forward_chunks() = " +
                                              std::to_string(6 + 2 * (overlap ? overlap_chunks(s) : 0)) +
                                              " for per-chunk events, or 6");
  int32_t ckpt_C = 0;
  if (ckpt != nullptr) {
    size_t need_ckpt = 0;
    if ((r = checkpoint_size(*dev, s, &ckpt_C, &need_ckpt)) != SDM_OK) return r;
    if (ckpt_bytes < need_ckpt)
      return fail(SDM_ERR_INVALID_ARGUMENT, "ckpt_bytes below sdm_layer_checkpoint_size() = " + std::to_string(need_ckpt));
    if (reinterpret_cast<uintptr_t>(ckpt) % 16 != 0) return fail(SDM_ERR_INVALID_ARGUMENT, "ckpt is not 16-byte aligned");
  }
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (overlap) {
    r = layer_forward_overlapped(*dev, s, c, kp, qp, v, alpha, beta, g, M0, M_out, y, ws, st, tr);
    return r == SDM_OK ? ok() : r;
  }
  int32_t* idx_w = reinterpret_cast<int32_t*>(ws);
  ws += align256(th * s.W * 4);
  float* w_w = reinterpret_cast<float*>(ws);
  ws += align256(th * s.W * 4);
  int32_t* idx_r = reinterpret_cast<int32_t*>(ws);
  ws += align256(th * s.R * 4);
  float* w_r = reinterpret_cast<float*>(ws);
  ws += align256(th * s.R * 4);
  uint32_t* rec = reinterpret_cast<uint32_t*>(ws);
  tr.mark(0, st);
  if ((r = topk_impl(*dev, kp, s.in_dtype, th, s.sqrt_n, s.W, idx_w, w_w, st)) != SDM_OK) return r;
  if ((r = topk_impl(*dev, qp, s.in_dtype, th, s.sqrt_n, s.R, idx_r, w_r, st)) != SDM_OK) return r;
  tr.mark(1, st);
  if (c.resident) {
    r = run_scan(*dev, s, c, idx_w, w_w, idx_r, w_r, v, alpha, beta, g, M0, 0, M_out, y, rec, st, tr, false, nullptr,
                 ckpt, ckpt_C);
  } else {
    r = run_scan(*dev, s, c, idx_w, w_w, idx_r, w_r, v, alpha, beta, g, M_out, 0, M_out, y, rec, st, tr,
                 /*init_before_scan=*/true, M0);
  }
  if (r != SDM_OK) return r;
  return ok();
}
}  // namespace sdm_host

using namespace sdm_host;

extern "C" {

int32_t sdm_abi_version(void) { return SDM_ABI_VERSION; }

const char* sdm_status_string(sdm_status_t status) {
  switch (status) {
    case SDM_OK: return "ok";
    case SDM_ERR_INVALID_ARGUMENT: return "invalid argument";
    case SDM_ERR_UNSUPPORTED: return "unsupported";
    case SDM_ERR_CUDA: return "CUDA error";
    case SDM_ERR_DEVICE_FAULT: return "device-side fault";
  }
  return "unknown status";
}

const char* sdm_last_error(void) { return g_last_error.c_str(); }

sdm_status_t sdm_pkm_topk(const void* scores, int32_t in_dtype, int32_t B, int32_t T, int32_t H, int32_t sqrt_n,
                          int32_t K, int32_t* idx_out, float* w_out, void* stream) {
  sdm_status_t r;
  if ((r = check_dtype(in_dtype, "in_dtype")) != SDM_OK) return r;
  if (B < 0 || T < 0 || H < 0) return fail(SDM_ERR_INVALID_ARGUMENT, "B, T and H must be >= 0");
  if (sqrt_n < 1 || sqrt_n > 1024) return fail(SDM_ERR_INVALID_ARGUMENT, "sqrt_n must be in [1, 1024]");
  if ((r = check_k(K, sqrt_n, "K")) != SDM_OK) return r;
  const int64_t units = static_cast<int64_t>(B) * T * H;
  if ((r = need_ptr(scores, "scores", units > 0)) != SDM_OK) return r;
  if ((r = need_ptr(idx_out, "idx_out", units > 0)) != SDM_OK) return r;
  if ((r = need_ptr(w_out, "w_out", units > 0)) != SDM_OK) return r;
  if (units == 0) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  if ((r = topk_impl(*dev, scores, in_dtype, units, sqrt_n, K, idx_out, w_out, static_cast<cudaStream_t>(stream))) != SDM_OK)
    return r;
  return ok();
}

sdm_status_t sdm_quantize_fp8blk(const float* x, int64_t n_blocks, uint8_t* codes, int8_t* exps, void* stream) {
  sdm_status_t r;
  if (n_blocks < 0) return fail(SDM_ERR_INVALID_ARGUMENT, "n_blocks must be >= 0");
  if ((r = need_ptr(x, "x", n_blocks > 0)) || (r = need_ptr(codes, "codes", n_blocks > 0))) return r;
  if (n_blocks > 0 && exps == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, "exps is NULL");
  if (n_blocks == 0) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int grid = static_cast<int>(std::min<int64_t>((n_blocks + 255) / 256, static_cast<int64_t>(dev->sms) * 16));
  sdm::k_quantize_fp8blk<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, n_blocks, codes, exps);
  if ((r = launch_status("fp8 quantize launch")) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_slot_counts(const int32_t* idx, int32_t B, int32_t T, int32_t H, int32_t K, int32_t N,
                             int32_t* counts, void* stream) {
  sdm_status_t r;
  if (B < 0 || T < 0 || H < 0) return fail(SDM_ERR_INVALID_ARGUMENT, "B, T and H must be >= 0");
  if (K < 1 || N < 1) return fail(SDM_ERR_INVALID_ARGUMENT, "K and N must be >= 1");
  if (static_cast<int64_t>(B) * H > 65535) return fail(SDM_ERR_UNSUPPORTED, "B*H above 65535");
  const int64_t entries = static_cast<int64_t>(B) * T * H * K;
  if ((r = need_ptr(idx, "idx", entries > 0)) != SDM_OK) return r;
  if ((r = need_ptr(counts, "counts", static_cast<int64_t>(B) * H > 0)) != SDM_OK) return r;
  if (entries == 0) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const bool local = N <= sdm::kCountSmemSlots;
  const bool vec = K % 4 == 0 && reinterpret_cast<uintptr_t>(idx) % 16 == 0;
  const size_t smem = local ? static_cast<size_t>(N) * 4 : 0;
  const void* kern = local ? (vec ? reinterpret_cast<const void*>(sdm::k_slot_counts<true, true>)
                                  : reinterpret_cast<const void*>(sdm::k_slot_counts<true, false>))
                           : (vec ? reinterpret_cast<const void*>(sdm::k_slot_counts<false, true>)
                                  : reinterpret_cast<const void*>(sdm::k_slot_counts<false, false>));
  set_smem(kern, smem);
  // About two waves of resident CTAs over all (b, h); at least 64 tokens a
  // CTA so that the shared-memory bins are worth their zeroing and flush.
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const int64_t want = 2LL * dev->sms * per_sm;
  const int64_t bh = static_cast<int64_t>(B) * H;
  const int64_t split = std::max<int64_t>(1, std::min<int64_t>((want + bh - 1) / bh, (T + 63) / 64));
  const int tokens_per_cta = static_cast<int>((T + split - 1) / split);
  const dim3 grid((T + tokens_per_cta - 1) / tokens_per_cta, static_cast<unsigned>(bh));
  void* args[] = {const_cast<int32_t**>(&idx), &T, &H, &K, &N, const_cast<int*>(&tokens_per_cta), &counts,
                  &dev->err};
  if (cudaLaunchKernel(kern, grid, dim3(256), args, smem, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(SDM_ERR_CUDA, std::string("slot count launch: ") + cudaGetErrorString(cudaGetLastError()));
  if ((r = launch_status("slot count launch")) != SDM_OK) return r;
  return ok();
}

size_t sdm_scan_workspace_bytes(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  if (check_shape(shape) != SDM_OK) return 0;
  g_last_error = saved;
  return records_bytes(*shape);
}

int32_t sdm_scan_variant(const sdm_shape_t* shape) {
  DeviceInfo* dev;
  ScanChoice c;
  if (check_shape(shape) != SDM_OK || device_info(&dev) != SDM_OK || choose_scan(*dev, *shape, &c) != SDM_OK)
    return -1;
  ok();
  return c.kind;
}


size_t sdm_scan_backward_workspace_bytes(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  BwdChoice c;
  if (check_shape(shape) != SDM_OK || choose_bwd(*shape, &c) != SDM_OK) return 0;
  g_last_error = saved;
  return c.total();
}


sdm_status_t sdm_scan_backward(const sdm_shape_t* shape, const int32_t* idx_w, const float* w_w,
                               const int32_t* idx_r, const float* w_r, const void* v, const void* alpha,
                               const void* beta, const float* M_in, int32_t m_in_shared, const float* dy, float* dM,
                               float* dv, float* dalpha, float* dbeta, float* dw_w, float* dw_r, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return scan_backward_impl(shape, idx_w, w_w, idx_r, w_r, v, alpha, beta, M_in, m_in_shared, dy, dM, dv, dalpha,
                            dbeta, dw_w, dw_r, workspace, workspace_bytes, stream, nullptr);
}

sdm_status_t sdm_layer_checkpoint_size(const sdm_shape_t* shape, int32_t* chunk_tokens, size_t* bytes) {
  sdm_status_t r;
  if (chunk_tokens == nullptr || bytes == nullptr) return fail(SDM_ERR_INVALID_ARGUMENT, "chunk_tokens or bytes is NULL");
  if ((r = check_shape(shape)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  if ((r = checkpoint_size(*dev, *shape, chunk_tokens, bytes)) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_rmsnorm_gate(float* y, const void* g, int32_t in_dtype, int64_t n_rows, int32_t d_v, float eps,
                              void* stream) {
  sdm_status_t r;
  if ((r = check_dtype(in_dtype, "in_dtype")) != SDM_OK) return r;
  if (n_rows < 0 || d_v < 1) return fail(SDM_ERR_INVALID_ARGUMENT, "n_rows must be >= 0 and d_v >= 1");
  if (!(eps >= 0.0f)) return fail(SDM_ERR_INVALID_ARGUMENT, "eps must be >= 0");
  if ((r = need_ptr(y, "y", n_rows > 0)) || (r = need_ptr(g, "g", n_rows > 0))) return r;
  if (n_rows == 0) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int grid = static_cast<int>(std::min<int64_t>((n_rows + 7) / 8, static_cast<int64_t>(dev->sms) * 16));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_dtype == SDM_BF16)
    sdm::k_rmsnorm_gate<bf16><<<grid, 256, 0, st>>>(y, static_cast<const bf16*>(g), n_rows, d_v, eps);
  else
    sdm::k_rmsnorm_gate<float><<<grid, 256, 0, st>>>(y, static_cast<const float*>(g), n_rows, d_v, eps);
  if ((r = launch_status("epilogue launch")) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_row_sumsq(const float* y, int64_t n_rows, int32_t d_v, float* ss, void* stream) {
  sdm_status_t r;
  if (n_rows < 0 || d_v < 1) return fail(SDM_ERR_INVALID_ARGUMENT, "n_rows must be >= 0 and d_v >= 1");
  if (n_rows == 0) return ok();
  if ((r = need_ptr(y, "y", true)) != SDM_OK || (r = need_gate(ss, "ss", true, SDM_F32)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int grid = static_cast<int>(std::min<int64_t>((n_rows + 7) / 8, static_cast<int64_t>(dev->sms) * 16));
  sdm::k_row_sumsq<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(y, n_rows, d_v, ss);
  if ((r = launch_status("row sum of squares launch")) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_rmsnorm_gate_rows(float* y, const void* g, int32_t in_dtype, const float* ss, int64_t n_rows,
                                   int32_t d_v, int32_t d_total, float eps, void* stream) {
  sdm_status_t r;
  if (n_rows < 0 || d_v < 1 || d_total < d_v)
    return fail(SDM_ERR_INVALID_ARGUMENT, "n_rows must be >= 0, d_v >= 1 and d_total >= d_v");
  if (!(eps >= 0.0f)) return fail(SDM_ERR_INVALID_ARGUMENT, "eps must be >= 0");
  if ((r = check_dtype(in_dtype, "in_dtype")) != SDM_OK) return r;
  if (n_rows == 0) return ok();
  if ((r = need_ptr(y, "y", true)) != SDM_OK || (r = need_gate(g, "g", true, in_dtype)) != SDM_OK ||
      (r = need_gate(ss, "ss", true, SDM_F32)) != SDM_OK)
    return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int grid = static_cast<int>(std::min<int64_t>((n_rows + 7) / 8, static_cast<int64_t>(dev->sms) * 16));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_dtype == SDM_BF16)
    sdm::k_rmsnorm_gate_rows<bf16><<<grid, 256, 0, st>>>(y, static_cast<const bf16*>(g), ss, n_rows, d_v, d_total, eps);
  else
    sdm::k_rmsnorm_gate_rows<float><<<grid, 256, 0, st>>>(y, static_cast<const float*>(g), ss, n_rows, d_v, d_total,
                                                          eps);
  if ((r = launch_status("column-slice epilogue launch")) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_rmsnorm_gate_backward(const float* y_pre, const void* g, int32_t in_dtype, const float* dout,
                                       int64_t n_rows, int32_t d_v, float eps, float* dy_pre, float* dg,
                                       void* stream) {
  sdm_status_t r;
  if ((r = check_dtype(in_dtype, "in_dtype")) != SDM_OK) return r;
  if (n_rows < 0 || d_v < 1) return fail(SDM_ERR_INVALID_ARGUMENT, "n_rows must be >= 0 and d_v >= 1");
  if (!(eps >= 0.0f)) return fail(SDM_ERR_INVALID_ARGUMENT, "eps must be >= 0");
  const bool any = n_rows > 0;
  if ((r = need_ptr(y_pre, "y_pre", any)) || (r = need_ptr(g, "g", any)) || (r = need_ptr(dout, "dout", any)) ||
      (r = need_ptr(dy_pre, "dy_pre", any)) || (r = need_ptr(dg, "dg", any)))
    return r;
  if (!any) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int grid = static_cast<int>(std::min<int64_t>((n_rows + 7) / 8, static_cast<int64_t>(dev->sms) * 16));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_dtype == SDM_BF16)
    sdm::k_rmsnorm_gate_backward<bf16><<<grid, 256, 0, st>>>(y_pre, static_cast<const bf16*>(g), dout, n_rows, d_v,
                                                             eps, dy_pre, dg);
  else
    sdm::k_rmsnorm_gate_backward<float><<<grid, 256, 0, st>>>(y_pre, static_cast<const float*>(g), dout, n_rows,
                                                              d_v, eps, dy_pre, dg);
  if ((r = launch_status("epilogue backward launch")) != SDM_OK) return r;
  return ok();
}

// Workspace of sdm_layer_backward: the two selections, their weight
// derivatives, dL/dy before the epilogue, then sdm_scan_backward's.
struct LayerBwdWs {
  size_t idx_w, w_w, idx_r, w_r, dw_w, dw_r, dy_pre, scan, total;
};
LayerBwdWs layer_bwd_ws(const sdm_shape_t& s, size_t scan_bytes) {
  const size_t th = static_cast<size_t>(s.B) * s.T * s.H;
  LayerBwdWs L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.idx_w = take(th * s.W * 4);
  L.w_w = take(th * s.W * 4);
  L.idx_r = take(th * s.R * 4);
  L.w_r = take(th * s.R * 4);
  L.dw_w = take(th * s.W * 4);
  L.dw_r = take(th * s.R * 4);
  L.dy_pre = take(th * s.d_v * 4);
  L.scan = take(scan_bytes);
  L.total = off;
  return L;
}

size_t sdm_layer_backward_workspace_bytes(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  BwdChoice c;
  if (check_shape(shape) != SDM_OK || choose_bwd(*shape, &c) != SDM_OK) return 0;
  g_last_error = saved;
  return layer_bwd_ws(*shape, c.total()).total;
}

sdm_status_t sdm_layer_backward(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                const void* alpha, const void* beta, const void* g, const float* M0,
                                const float* y_pre, const float* dy, float* dM, float* dkp, float* dqp, float* dv,
                                float* dalpha, float* dbeta, float* dg, void* workspace, size_t workspace_bytes,
                                void* stream) {
  return sdm_layer_backward_ckpt(shape, kp, qp, v, alpha, beta, g, M0, y_pre, dy, dM, dkp, dqp, dv, dalpha, dbeta, dg,
                                 nullptr, 0, workspace, workspace_bytes, stream);
}

sdm_status_t sdm_layer_backward_ckpt(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                     const void* alpha, const void* beta, const void* g, const float* M0,
                                     const float* y_pre, const float* dy, float* dM, float* dkp, float* dqp, float* dv,
                                     float* dalpha, float* dbeta, float* dg, const float* ckpt, size_t ckpt_bytes,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const sdm_shape_t& s = *shape;
  BwdChoice c;
  if ((r = choose_bwd(s, &c)) != SDM_OK) return r;
  if (ckpt != nullptr) {
    DeviceInfo* dev;
    if ((r = device_info(&dev)) != SDM_OK) return r;
    int32_t chunk = 0;
    size_t need_ckpt = 0;
    if ((r = checkpoint_size(*dev, s, &chunk, &need_ckpt)) != SDM_OK) return r;
    if (ckpt_bytes < need_ckpt)
      return fail(SDM_ERR_INVALID_ARGUMENT, "ckpt_bytes below sdm_layer_checkpoint_size() = " + std::to_string(need_ckpt));
    if (reinterpret_cast<uintptr_t>(ckpt) % 16 != 0) return fail(SDM_ERR_INVALID_ARGUMENT, "ckpt is not 16-byte aligned");
  }
  const bool tok = static_cast<int64_t>(s.B) * s.T * s.H > 0;
  if ((r = need_ptr(kp, "kp", tok)) || (r = need_ptr(qp, "qp", tok)) || (r = need_ptr(dkp, "dkp", tok)) ||
      (r = need_ptr(dqp, "dqp", tok)))
    return r;
  if (g != nullptr && ((r = need_ptr(y_pre, "y_pre", tok)) || (r = need_ptr(dg, "dg", tok)))) return r;
  const LayerBwdWs L = layer_bwd_ws(s, c.total());
  if (workspace_bytes < L.total)
    return fail(SDM_ERR_INVALID_ARGUMENT,
                "workspace_bytes below sdm_layer_backward_workspace_bytes() = " + std::to_string(L.total));
  if ((r = need_ptr(workspace, "workspace", true)) != SDM_OK) return r;
  if (!tok) return sdm_scan_backward(shape, nullptr, nullptr, nullptr, nullptr, v, alpha, beta, M0, 1, dy, dM, dv,
                                     dalpha, dbeta, nullptr, nullptr, nullptr, 0, stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* idx_w = reinterpret_cast<int32_t*>(ws + L.idx_w);
  float* w_w = reinterpret_cast<float*>(ws + L.w_w);
  int32_t* idx_r = reinterpret_cast<int32_t*>(ws + L.idx_r);
  float* w_r = reinterpret_cast<float*>(ws + L.w_r);
  float* dw_w = reinterpret_cast<float*>(ws + L.dw_w);
  float* dw_r = reinterpret_cast<float*>(ws + L.dw_r);
  float* dy_pre = reinterpret_cast<float*>(ws + L.dy_pre);
  if ((r = sdm_pkm_topk(kp, s.in_dtype, s.B, s.T, s.H, s.sqrt_n, s.W, idx_w, w_w, stream)) != SDM_OK) return r;
  if ((r = sdm_pkm_topk(qp, s.in_dtype, s.B, s.T, s.H, s.sqrt_n, s.R, idx_r, w_r, stream)) != SDM_OK) return r;
  const float* dy_scan = dy;
  if (g != nullptr) {
    if ((r = sdm_rmsnorm_gate_backward(y_pre, g, s.in_dtype, dy, static_cast<int64_t>(s.B) * s.T * s.H, s.d_v,
                                       s.rms_eps, dy_pre, dg, stream)) != SDM_OK)
      return r;
    dy_scan = dy_pre;
  }
  if ((r = scan_backward_impl(shape, idx_w, w_w, idx_r, w_r, v, alpha, beta, M0, 1, dy_scan, dM, dv, dalpha, dbeta,
                              dw_w, dw_r, ws + L.scan, c.total(), stream, ckpt)) != SDM_OK)
    return r;
  if ((r = sdm_pkm_topk_backward(idx_w, w_w, dw_w, s.B, s.T, s.H, s.sqrt_n, s.W, dkp, stream)) != SDM_OK) return r;
  if ((r = sdm_pkm_topk_backward(idx_r, w_r, dw_r, s.B, s.T, s.H, s.sqrt_n, s.R, dqp, stream)) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_pkm_topk_backward(const int32_t* idx, const float* w, const float* dw, int32_t B, int32_t T,
                                   int32_t H, int32_t sqrt_n, int32_t K, float* dscores, void* stream) {
  sdm_status_t r;
  if (B < 0 || T < 0 || H < 0) return fail(SDM_ERR_INVALID_ARGUMENT, "B, T and H must be >= 0");
  if (sqrt_n < 1 || sqrt_n > 1024) return fail(SDM_ERR_INVALID_ARGUMENT, "sqrt_n must be in [1, 1024]");
  if ((r = check_k(K, sqrt_n, "K")) != SDM_OK) return r;
  const int64_t units = static_cast<int64_t>(B) * T * H;
  if ((r = need_ptr(idx, "idx", units > 0)) || (r = need_ptr(w, "w", units > 0)) ||
      (r = need_ptr(dw, "dw", units > 0)) || (r = need_ptr(dscores, "dscores", units > 0)))
    return r;
  if (units == 0) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const int warps = 8;
  const size_t smem = static_cast<size_t>(warps) * 3 * K * 4;
  set_smem(reinterpret_cast<const void*>(sdm::k_pkm_topk_backward), smem);
  const int64_t blocks = (units + warps - 1) / warps;
  if (blocks > 0x7FFFFFFFLL) return fail(SDM_ERR_UNSUPPORTED, "too many token-heads for one launch");
  sdm::k_pkm_topk_backward<<<static_cast<unsigned>(blocks), warps * 32, smem, static_cast<cudaStream_t>(stream)>>>(
      idx, w, dw, units, sqrt_n, K, dscores, dev->err);
  if ((r = launch_status("selection backward launch")) != SDM_OK) return r;
  return ok();
}

sdm_status_t sdm_scan_describe(const sdm_shape_t* shape, char* out, size_t out_len) {
  sdm_status_t r;
  if (out == nullptr || out_len == 0) return fail(SDM_ERR_INVALID_ARGUMENT, "out is null or out_len is 0");
  out[0] = '\0';
  DeviceInfo* dev;
  ScanChoice c;
  if ((r = check_shape(shape)) != SDM_OK || (r = device_info(&dev)) != SDM_OK ||
      (r = choose_scan(*dev, *shape, &c)) != SDM_OK)
    return r;
  if (c.kind == SDM_VARIANT_RESIDENT)
    snprintf(out, out_len, "resident CW=%d NWARP=%d L=%d EB=%d smem=%zu", c.CW, c.NWARP, c.L, c.EB, c.smem);
  else if (c.kind == SDM_VARIANT_PIPELINED)
    snprintf(out, out_len, "pipelined C=%d P=%d L=%d NWW=%d NWR=%d NP=%d S=%d parts=%d smem=%zu", c.C, c.P, c.L, c.NWW,
             c.NWR, c.NP, c.S, c.parts, c.smem);
  else
    snprintf(out, out_len, "streaming C=%d P=%d L=%d NW=%d smem=%zu", c.C, c.P, c.L, c.NWARP, c.smem);
  return ok();
}

sdm_status_t sdm_scan(const sdm_shape_t* shape, const int32_t* idx_w, const float* w_w, const int32_t* idx_r,
                      const float* w_r, const void* v, const void* alpha, const void* beta, const void* g, void* M,
                      float* y, void* workspace, size_t workspace_bytes, void* stream) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const sdm_shape_t& s = *shape;
  const bool any = static_cast<int64_t>(s.B) * s.T * s.H > 0;
  if ((r = need_ptr(idx_w, "idx_w", any)) || (r = need_ptr(w_w, "w_w", any)) || (r = need_ptr(idx_r, "idx_r", any)) ||
      (r = need_ptr(w_r, "w_r", any)) || (r = need_ptr(v, "v", any)) || (r = need_gate(alpha, "alpha", any, s.in_dtype)) ||
      (r = need_gate(beta, "beta", any, s.in_dtype)) || (r = need_ptr(M, "M", any)) || (r = need_ptr(y, "y", any)))
    return r;
  if (g != nullptr && (r = need_ptr(g, "g", any)) != SDM_OK) return r;
  if (!any) return ok();
  const size_t need = records_bytes(s);
  if (workspace_bytes < need)
    return fail(SDM_ERR_INVALID_ARGUMENT, "workspace_bytes below sdm_scan_workspace_bytes() = " + std::to_string(need));
  if ((r = need_ptr(workspace, "workspace", true)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  ScanChoice c;
  if ((r = choose_scan(*dev, s, &c)) != SDM_OK) return r;
  const int64_t row_stride = static_cast<int64_t>(s.H) * slots_of(s.sqrt_n) * s.d_v;
  if ((r = run_scan(*dev, s, c, idx_w, w_w, idx_r, w_r, v, alpha, beta, g, M, row_stride, M, y,
                    static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream))) != SDM_OK)
    return r;
  return ok();
}

sdm_status_t sdm_state_init(const sdm_shape_t* shape, const void* M0, void* M, void* stream) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const bool any = static_cast<int64_t>(shape->B) * shape->H > 0;
  if ((r = need_ptr(M0, "M0", any)) != SDM_OK || (r = need_ptr(M, "M", any)) != SDM_OK) return r;
  if (!any) return ok();
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  if ((r = launch_state_init(*dev, *shape, M0, M, static_cast<cudaStream_t>(stream))) != SDM_OK) return r;
  return ok();
}

size_t sdm_layer_forward_workspace_bytes(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  if (check_shape(shape) != SDM_OK) return 0;
  g_last_error = saved;
  const sdm_shape_t& s = *shape;
  const size_t th = static_cast<size_t>(s.B) * s.T * s.H;
  return 2 * align256(th * s.W * 4) + 2 * align256(th * s.R * 4) + records_bytes(s);
}


sdm_status_t sdm_layer_forward_traced(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                      const void* alpha, const void* beta, const void* g, const void* M0,
                                      void* M_out, float* y, void* workspace, size_t workspace_bytes, void* stream,
                                      void* const* events, int32_t n_events) {
  return layer_forward_impl(shape, kp, qp, v, alpha, beta, g, M0, M_out, y, workspace, workspace_bytes, stream, events,
                            n_events, nullptr, 0);
}

sdm_status_t sdm_layer_forward_ckpt(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                    const void* alpha, const void* beta, const void* g, const void* M0, void* M_out,
                                    float* y, float* ckpt, size_t ckpt_bytes, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  sdm_status_t r;
  if ((r = need_ptr(ckpt, "ckpt", true)) != SDM_OK) return r;
  return layer_forward_impl(shape, kp, qp, v, alpha, beta, g, M0, M_out, y, workspace, workspace_bytes, stream,
                            nullptr, 0, ckpt, ckpt_bytes);
}

int32_t sdm_layer_forward_chunks(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  DeviceInfo* dev;
  ScanChoice c;
  if (check_shape(shape) != SDM_OK || device_info(&dev) != SDM_OK || choose_scan(*dev, *shape, &c) != SDM_OK)
    return -1;
  g_last_error = saved;
  return overlapped(*shape, c) ? static_cast<int32_t>(overlap_chunks(*shape)) : 1;
}

int32_t sdm_layer_forward_launches(const sdm_shape_t* shape, int32_t with_gate) {
  const std::string saved = g_last_error;
  DeviceInfo* dev;
  ScanChoice c;
  if (check_shape(shape) != SDM_OK || device_info(&dev) != SDM_OK || choose_scan(*dev, *shape, &c) != SDM_OK) {
    g_last_error = saved;
    return -1;
  }
  g_last_error = saved;
  // two selections, records, recurrence; the streaming and pipelined recurrences also copy M0
  // first; the pipelined one with two slot parts adds the second part's sums into y after
  const int parts_sum = c.kind == SDM_VARIANT_PIPELINED && c.parts > 1 ? 1 : 0;
  const int init = c.resident ? 0 : (shape->state_dtype == SDM_FP8_B16 ? 2 : 1);  // fp8: codes and exponents
  // an overlapped call: two selections, records and the recurrence per chunk
  const int64_t per_call = overlapped(*shape, c) ? 4 * overlap_chunks(*shape) : 4;
  return static_cast<int32_t>(per_call) + init + parts_sum + (with_gate ? 1 : 0);
}

sdm_status_t sdm_layer_forward(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                               const void* alpha, const void* beta, const void* g, const void* M0, void* M_out,
                               float* y, void* workspace, size_t workspace_bytes, void* stream) {
  return sdm_layer_forward_traced(shape, kp, qp, v, alpha, beta, g, M0, M_out, y, workspace, workspace_bytes,
                                  stream, nullptr, 0);
}

size_t sdm_layer_step_workspace_bytes(const sdm_shape_t* shape) { return sdm_layer_forward_workspace_bytes(shape); }

int32_t sdm_layer_step_launches(const sdm_shape_t* shape) {
  const std::string saved = g_last_error;
  if (check_shape(shape) != SDM_OK) return -1;
  const sdm_shape_t& s = *shape;
  FastTopkPlan P;
  const bool fused = s.T == 1 && s.W == s.R && s.W <= sdm::kFastTopkMaxK && s.variant == SDM_VARIANT_AUTO &&
                     fast_topk_plan(s.sqrt_n, s.W, &P) == SDM_OK;
  g_last_error = saved;
  return fused ? 1 : 4;  // else: two selections, records, recurrence
}

sdm_status_t sdm_layer_step(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                            const void* alpha, const void* beta, const void* g, void* M, float* y, void* workspace,
                            size_t workspace_bytes, void* stream) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const sdm_shape_t& s = *shape;
  const int64_t th = static_cast<int64_t>(s.B) * s.T * s.H;
  const bool any = th > 0;
  if ((r = need_ptr(kp, "kp", any)) || (r = need_ptr(qp, "qp", any)) || (r = need_ptr(v, "v", any)) ||
      (r = need_gate(alpha, "alpha", any, s.in_dtype)) || (r = need_gate(beta, "beta", any, s.in_dtype)) || (r = need_ptr(y, "y", any)) ||
      (r = need_ptr(M, "M", any)))
    return r;
  if (g != nullptr && (r = need_ptr(g, "g", any)) != SDM_OK) return r;
  if (!any) return ok();
  const size_t need = sdm_layer_step_workspace_bytes(shape);
  if (workspace_bytes < need)
    return fail(SDM_ERR_INVALID_ARGUMENT, "workspace_bytes below sdm_layer_step_workspace_bytes() = " + std::to_string(need));
  if ((r = need_ptr(workspace, "workspace", true)) != SDM_OK) return r;
  DeviceInfo* dev;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool fused = false;
  if ((r = try_decode_step(*dev, s, kp, qp, v, alpha, beta, g, M, y, st, &fused)) != SDM_OK) return r;
  if (fused) return ok();
  ScanChoice c;
  if ((r = choose_scan(*dev, s, &c)) != SDM_OK) return r;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* idx_w = reinterpret_cast<int32_t*>(ws);
  ws += align256(th * s.W * 4);
  float* w_w = reinterpret_cast<float*>(ws);
  ws += align256(th * s.W * 4);
  int32_t* idx_r = reinterpret_cast<int32_t*>(ws);
  ws += align256(th * s.R * 4);
  float* w_r = reinterpret_cast<float*>(ws);
  ws += align256(th * s.R * 4);
  uint32_t* rec = reinterpret_cast<uint32_t*>(ws);
  if ((r = topk_impl(*dev, kp, s.in_dtype, th, s.sqrt_n, s.W, idx_w, w_w, st)) != SDM_OK) return r;
  if ((r = topk_impl(*dev, qp, s.in_dtype, th, s.sqrt_n, s.R, idx_r, w_r, st)) != SDM_OK) return r;
  const int64_t row_stride = static_cast<int64_t>(s.H) * slots_of(s.sqrt_n) * s.d_v;
  if ((r = run_scan(*dev, s, c, idx_w, w_w, idx_r, w_r, v, alpha, beta, g, M, row_stride, M, y, rec, st)) != SDM_OK)
    return r;
  return ok();
}

sdm_status_t sdm_layer_forward_noalloc(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                       const void* alpha, const void* beta, const void* g, const void* M0,
                                       void* M_out, float* y, void* stream) {
  sdm_status_t r;
  if ((r = check_shape(shape)) != SDM_OK) return r;
  const size_t need = sdm_layer_forward_workspace_bytes(shape);
  if (need > SDM_NOALLOC_SCRATCH_BYTES)
    return fail(SDM_ERR_INVALID_ARGUMENT, "this shape needs " + std::to_string(need) +
                                              " bytes of scratch; the built-in scratch holds " +
                                              std::to_string(SDM_NOALLOC_SCRATCH_BYTES) + " bytes");
  void* ws = nullptr;
  if ((r = noalloc_scratch(&ws)) != SDM_OK) return r;
  return sdm_layer_forward(shape, kp, qp, v, alpha, beta, g, M0, M_out, y, ws, SDM_NOALLOC_SCRATCH_BYTES, stream);
}

sdm_status_t sdm_stream_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(SDM_ERR_CUDA, std::string("cudaStreamSynchronize: ") + cudaGetErrorString(e));
  DeviceInfo* dev;
  sdm_status_t r;
  if ((r = device_info(&dev)) != SDM_OK) return r;
  unsigned word = 0;
  if ((e = cudaMemcpy(&word, dev->err, sizeof(word), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return fail(SDM_ERR_CUDA, std::string("reading the device error word: ") + cudaGetErrorString(e));
  if (word != 0) {
    const unsigned zero = 0;
    cudaMemcpy(dev->err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    char hex[16];
    std::snprintf(hex, sizeof(hex), "0x%x", word);
    std::string msg = std::string("device error word ") + hex + ":";
    if (word & sdm::kErrIndexOutOfRange) msg += " slot index outside [0, N) skipped;";
    if (word & sdm::kErrWaitTimeout) msg += " bounded wait expired (the outputs of every call since the last check are undefined);";
    return fail(SDM_ERR_DEVICE_FAULT, msg);
  }
  return ok();
}

}  // extern "C"
