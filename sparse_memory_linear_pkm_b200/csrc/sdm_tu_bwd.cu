// Launches of the recurrence backward kernel.

#include <algorithm>

#include "sdm_host.h"

namespace sdm_host {

template <typename Tin, int U, bool G, int NWB>
sdm_status_t launch_bwd_inst(const BwdChoice& c, const sdm::BwdArgs& a, cudaStream_t st) {
  const void* kern = reinterpret_cast<const void*>(sdm::k_scan_backward<Tin, U, G, NWB>);
  set_smem(kern, c.smem);
  const int64_t grid = static_cast<int64_t>(a.B) * a.H * c.ntile;
  if (grid > 0x7FFFFFFFLL) return fail(SDM_ERR_UNSUPPORTED, "too many column tiles for one launch");
  sdm::k_scan_backward<Tin, U, G, NWB><<<static_cast<unsigned>(grid), NWB * 32, c.smem, st>>>(a);
  return launch_status("backward launch");
}

template <typename Tin>
sdm_status_t launch_bwd_typed(const BwdChoice& c, const sdm::BwdArgs& a, cudaStream_t st) {
  if (!c.global) {
    // Two warps share each shared-memory tile unless the shape's tile asks for one.
    if (c.nwb == 1) return launch_bwd_inst<Tin, 1, false, 1>(c, a, st);
    return launch_bwd_inst<Tin, 1, false, 2>(c, a, st);
  }
  return c.U == 8 ? launch_bwd_inst<Tin, 8, true, 1>(c, a, st) : launch_bwd_inst<Tin, 4, true, 1>(c, a, st);
}

sdm_status_t launch_bwd(const BwdChoice& c, int32_t in_dtype, const sdm::BwdArgs& a, cudaStream_t st) {
  return in_dtype == SDM_BF16 ? launch_bwd_typed<bf16>(c, a, st) : launch_bwd_typed<float>(c, a, st);
}

}  // namespace sdm_host
