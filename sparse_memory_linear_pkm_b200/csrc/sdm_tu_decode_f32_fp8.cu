// Decode-step instances for float inputs and a block-scaled fp8 state.

#include "sdm_decode_launch.h"

namespace sdm_host {

template sdm_status_t launch_decode_for<float, sdm::Fp8Blk>(const FastTopkPlan&, const sdm::DecodeArgs&, size_t, int,
                                                        cudaStream_t);

}  // namespace sdm_host
