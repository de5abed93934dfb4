// Dispatch of the single-launch decode step to the instances of its
// (input dtype, state dtype) pair, compiled in sdm_tu_decode_*.cu.

#include <algorithm>

#include "sdm_host.h"

namespace sdm_host {

sdm_status_t launch_decode(const FastTopkPlan& P, int32_t in_dtype, int32_t state_dtype, const sdm::DecodeArgs& a,
                           size_t smem, int grid, cudaStream_t st) {
  if (in_dtype == SDM_BF16)
    return state_dtype == SDM_FP8_B16 ? launch_decode_for<bf16, sdm::Fp8Blk>(P, a, smem, grid, st)
           : state_dtype == SDM_BF16  ? launch_decode_for<bf16, bf16>(P, a, smem, grid, st)
                                      : launch_decode_for<bf16, float>(P, a, smem, grid, st);
  return state_dtype == SDM_FP8_B16 ? launch_decode_for<float, sdm::Fp8Blk>(P, a, smem, grid, st)
         : state_dtype == SDM_BF16  ? launch_decode_for<float, bf16>(P, a, smem, grid, st)
                                    : launch_decode_for<float, float>(P, a, smem, grid, st);
}

}  // namespace sdm_host
