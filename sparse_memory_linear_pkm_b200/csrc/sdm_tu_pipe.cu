// Launches of the pipelined recurrence and of its record build.

#include <algorithm>

#include "sdm_host.h"

namespace sdm_host {

template <typename Tin>
sdm_status_t launch_pipe_records_typed(const sdm_shape_t& s, const ScanChoice& c, const int32_t* idx_w, const float* w_w,
                                 const int32_t* idx_r, const float* w_r, const void* alpha, const void* beta,
                                 uint32_t* rec, float* y_zero, const DeviceInfo& dev, cudaStream_t st) {
  int log2_cells = 1;
  while ((1 << log2_cells) < 2 * s.W) ++log2_cells;
  const size_t smem = sdm::pipe_records_smem(s.W, s.R, c.P, log2_cells, c.parts);
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return fail(SDM_ERR_UNSUPPORTED, "hazard tables exceed shared memory");
  auto kern = sdm::k_build_pipe_records<Tin>;
  set_smem(reinterpret_cast<const void*>(kern), smem);
  const int tblocks = (s.T + sdm::kPipeTokensPerBlock - 1) / sdm::kPipeTokensPerBlock;
  const dim3 grid(tblocks, s.B * s.H);
  kern<<<grid, 256, smem, st>>>(idx_w, w_w, idx_r, w_r, static_cast<const Tin*>(alpha), static_cast<const Tin*>(beta),
                                s.T, s.H, static_cast<int>(slots_of(s.sqrt_n)), s.W, s.R, c.P, c.parts, log2_cells,
                                sdm::pipe_layout(s.W, s.R), rec, y_zero, s.d_v, dev.err);
  return launch_status("pipelined record build launch");
}

template <typename Tin, typename Tst>
sdm_status_t launch_pipe_typed(const ScanChoice& c, const sdm::PipeArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H * a.parts, a.d_v / c.C);
  void (*kern)(sdm::PipeArgs) = nullptr;
#define SDM_PIPE(C_, P_, L_, NWW_, NWR_)                                                       \
  if (c.C == C_ && c.P == P_ && c.L == L_ && c.NWW == NWW_ && c.NWR == NWR_)                  \
    kern = sdm::k_scan_pipelined<Tin, Tst, C_, P_, L_, NWW_, NWR_>;
  if constexpr (sizeof(Tst) == 2) {
    SDM_PIPE(64, 6, 16, 4, 4) SDM_PIPE(64, 7, 16, 4, 4) SDM_PIPE(64, 6, 16, 8, 8) SDM_PIPE(64, 5, 16, 4, 4)
  } else {
    SDM_PIPE(32, 6, 16, 4, 4) SDM_PIPE(32, 4, 16, 4, 4)
  }
#undef SDM_PIPE
  if (kern == nullptr) return fail(SDM_ERR_UNSUPPORTED, "no pipelined kernel for the chosen tile");
  set_smem(reinterpret_cast<const void*>(kern), c.smem);
  kern<<<grid, (c.NWW + c.NWR) * 32, c.smem, st>>>(a);
  return launch_status("pipelined scan launch");
}

sdm_status_t launch_pipe(const ScanChoice& c, const sdm_shape_t& s, const sdm::PipeArgs& a, cudaStream_t st) {
  if (s.in_dtype == SDM_BF16)
    return s.state_dtype == SDM_BF16 ? launch_pipe_typed<bf16, bf16>(c, a, st) : launch_pipe_typed<bf16, float>(c, a, st);
  return s.state_dtype == SDM_BF16 ? launch_pipe_typed<float, bf16>(c, a, st) : launch_pipe_typed<float, float>(c, a, st);
}

sdm_status_t launch_pipe_records(const sdm_shape_t& s, const ScanChoice& c, const int32_t* idx_w, const float* w_w,
                                 const int32_t* idx_r, const float* w_r, const void* alpha, const void* beta,
                                 uint32_t* rec, float* y_zero, const DeviceInfo& dev, cudaStream_t st) {
  return s.in_dtype == SDM_BF16
             ? launch_pipe_records_typed<bf16>(s, c, idx_w, w_w, idx_r, w_r, alpha, beta, rec, y_zero, dev, st)
             : launch_pipe_records_typed<float>(s, c, idx_w, w_w, idx_r, w_r, alpha, beta, rec, y_zero, dev, st);
}

}  // namespace sdm_host
