// The decode step's template instances for one (input dtype, state dtype)
// pair: included by the sdm_tu_decode_*.cu units, which instantiate
// launch_decode_for for their pair (the instances compile in parallel).
#pragma once

#include "sdm_host.h"

namespace sdm_host {

template <typename Tin, typename Tst, int E, int EH, int EPL, int CP>
sdm_status_t launch_decode_inst(const sdm::DecodeArgs& a, size_t smem, int grid, cudaStream_t st) {
  auto kern = sdm::k_decode_step<Tin, Tst, E, EH, EPL, CP>;
  set_smem(reinterpret_cast<const void*>(kern), smem);
  kern<<<grid, sdm::kDecodeThreads, smem, st>>>(a);
  return launch_status("decode step launch");
}

template <typename Tin, typename Tst>
sdm_status_t launch_decode_for(const FastTopkPlan& P, const sdm::DecodeArgs& a, size_t smem, int grid,
                                 cudaStream_t st) {
#define SDM_DECODE(E_, EH_, EPL_, CP_)                                 \
  if (P.E == E_ && P.EH == EH_ && P.epl == EPL_ && P.CP == CP_) \
    return launch_decode_inst<Tin, Tst, E_, EH_, EPL_, CP_>(a, smem, grid, st);
  SDM_DECODE(1, 1, 1, 4) SDM_DECODE(1, 1, 2, 4) SDM_DECODE(1, 1, 4, 4) SDM_DECODE(1, 1, 8, 4)
  SDM_DECODE(1, 1, 16, 4) SDM_DECODE(1, 1, 32, 4)
  SDM_DECODE(2, 1, 1, 7)
  SDM_DECODE(2, 2, 1, 9) SDM_DECODE(2, 2, 4, 9) SDM_DECODE(2, 2, 8, 9)
  SDM_DECODE(2, 2, 16, 9) SDM_DECODE(2, 2, 32, 9)
#undef SDM_DECODE
  return fail(SDM_ERR_UNSUPPORTED, "no decode kernel for this sqrt_n and K");
}

}  // namespace sdm_host
