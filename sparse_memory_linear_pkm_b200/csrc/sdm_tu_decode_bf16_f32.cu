// Decode-step instances for bf16 inputs and a fp32 state.

#include "sdm_decode_launch.h"

namespace sdm_host {

template sdm_status_t launch_decode_for<bf16, float>(const FastTopkPlan&, const sdm::DecodeArgs&, size_t, int,
                                                        cudaStream_t);

}  // namespace sdm_host
