// Launches of the resident and streaming recurrence kernels (template instances
// for each tile and dtype pair).

#include <algorithm>

#include "sdm_host.h"

namespace sdm_host {

template <typename Tin, typename Tst>
sdm_status_t launch_scan_typed(const ScanChoice& c, const sdm::ScanArgs& a, cudaStream_t st, float* ckpt,
                               int ckpt_C) {
  const dim3 grid(a.B * a.H, a.d_v / c.C);
  void (*kern)(sdm::ScanArgs) = nullptr;
  if (c.resident) {
    void (*rkern)(sdm::ScanArgs, float*, int) = nullptr;
    // the checkpoint-storing build (fp32 state only) when the call stores the backward's checkpoints
#define SDM_RES(CW_, NW_, L_, EB_)                                                                     \
    if (c.CW == CW_ && c.NWARP == NW_ && c.L == L_ && c.EB == EB_) {                                    \
      if constexpr (sizeof(Tst) == 4) {                                                                \
        rkern = ckpt != nullptr ? sdm::k_scan_resident<Tin, Tst, CW_, NW_, L_, EB_, true>              \
                                : sdm::k_scan_resident<Tin, Tst, CW_, NW_, L_, EB_, false>;             \
      } else {                                                                                         \
        rkern = sdm::k_scan_resident<Tin, Tst, CW_, NW_, L_, EB_, false>;                              \
      }                                                                                                \
    }
    SDM_RES(8, 2, 4, 4) SDM_RES(8, 1, 4, 4) SDM_RES(16, 1, 4, 4) SDM_RES(4, 4, 4, 2) SDM_RES(4, 2, 4, 2)
    SDM_RES(8, 2, 8, 4) SDM_RES(4, 4, 8, 2) SDM_RES(8, 4, 8, 4)
#undef SDM_RES
    if (rkern == nullptr) return fail(SDM_ERR_UNSUPPORTED, "no resident kernel for the chosen tile");
    set_smem(reinterpret_cast<const void*>(rkern), c.smem);
    rkern<<<grid, c.NWARP * 32, c.smem, st>>>(a, ckpt, ckpt_C);
    return launch_status("scan launch");
  } else {
#define SDM_STREAM(C_, P_, L_, NW_) \
    if (c.C == C_ && c.P == P_ && c.L == L_ && c.NWARP == NW_) kern = sdm::k_scan_streaming<Tin, Tst, C_, P_, L_, NW_>;
    if constexpr (sizeof(Tst) == 4) {
      SDM_STREAM(64, 3, 8, 16) SDM_STREAM(64, 2, 8, 16) SDM_STREAM(32, 4, 8, 16) SDM_STREAM(32, 4, 8, 8)
      SDM_STREAM(16, 8, 16, 16) SDM_STREAM(16, 4, 8, 8)
    } else {
      SDM_STREAM(128, 3, 8, 16) SDM_STREAM(64, 4, 8, 16) SDM_STREAM(64, 6, 8, 16) SDM_STREAM(32, 8, 16, 16)
      SDM_STREAM(32, 8, 16, 8) SDM_STREAM(16, 8, 16, 16) SDM_STREAM(16, 4, 8, 8)
    }
#undef SDM_STREAM
  }
  if (kern == nullptr) return fail(SDM_ERR_UNSUPPORTED, "no streaming kernel for the chosen tile");
  set_smem(reinterpret_cast<const void*>(kern), c.smem);
  kern<<<grid, c.NWARP * 32, c.smem, st>>>(a);
  return launch_status("scan launch");
}

sdm_status_t launch_scan(const ScanChoice& c, const sdm_shape_t& s, const sdm::ScanArgs& a, cudaStream_t st,
                         float* ckpt, int ckpt_C) {
  if (s.in_dtype == SDM_BF16)
    return s.state_dtype == SDM_BF16 ? launch_scan_typed<bf16, bf16>(c, a, st, ckpt, ckpt_C)
                                     : launch_scan_typed<bf16, float>(c, a, st, ckpt, ckpt_C);
  return s.state_dtype == SDM_BF16 ? launch_scan_typed<float, bf16>(c, a, st, ckpt, ckpt_C)
                                   : launch_scan_typed<float, float>(c, a, st, ckpt, ckpt_C);
}

}  // namespace sdm_host
