// Host-side declarations shared by the translation units of libsdm_b200.so
// (internal: none of this is part of the C ABI in sdm.h). The entry points
// live in sdm_api.cu; the launches of kernels with many template instances
// live in sdm_tu_*.cu so that the library compiles in parallel.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <string>

#include "sdm.h"
#include "pkm_topk.cuh"
#include "pkm_topk_fast.cuh"
#include "sdm_misc.cuh"
#include "sdm_records.cuh"
#include "sdm_scan.cuh"
#include "sdm_backward.cuh"
#include "sdm_decode.cuh"
#include "sdm_pipelined.cuh"

namespace sdm_host {

using sdm::bf16;

// Per-device facts and the device address of the error word.
struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
  int smem_per_sm = 0;
  unsigned* err = nullptr;
  bool ready = false;
};

// Records msg as the calling thread's last error and returns s.
sdm_status_t fail(sdm_status_t s, const std::string& msg);
// SDM_ERR_CUDA (with the launch error named after `what`) if the last launch failed.
sdm_status_t launch_status(const char* what);
// Raises a kernel's dynamic shared-memory limit to at least smem on the current device.
void set_smem(const void* kern, size_t smem);
size_t in_size(int32_t dtype);
size_t state_size(int32_t dtype);  // bytes of one state value (fp8 state: the code byte)
int64_t slots_of(int32_t sqrt_n);

// The recurrence kernel picked for a shape and its tile.
struct ScanChoice {
  int kind = SDM_VARIANT_STREAMING;  // SDM_VARIANT_RESIDENT, _STREAMING or _PIPELINED
  bool resident = false;
  int C = 16;  // columns per CTA
  int P = 4;
  int L = 16;
  int CW = 8, NWARP = 2, EB = 4;  // resident: columns per warp, warps per CTA, entry block
  int NWW = 4, NWR = 4, NP = 4, parts = 1;  // pipelined: write, read and producer warps, slot parts per tile
  int S = 1;                                  // pipelined: tokens per barrier step
  size_t smem = 0;
};

constexpr size_t kBwdSmemLimit = 232448;  // sm_100 opt-in shared memory per block
constexpr int kBwdChunk = 128;            // tokens per checkpoint chunk

struct BwdChoice {
  bool global = false;  // state and adjoint tiles in global memory (large N)
  int U = 1;            // 16-byte units (4 columns) per lane and entry: tile width 4 U
  int C = kBwdChunk;
  int ntile = 0;
  int nwb = 2;          // shared-memory tiles: warps per tile (shape.tile 1: one, else two)
  size_t smem = 0;
  size_t rec_bytes = 0, ckpt_bytes = 0, log_bytes = 0, part_bytes = 0, work_bytes = 0;
  size_t total() const { return rec_bytes + ckpt_bytes + log_bytes + part_bytes + work_bytes; }
};

// Layout and template parameters of the register-path selection (K <= 64).
struct FastTopkPlan {
  sdm::FastTopkLayout L{};
  int E = 1, EH = 1, epl = 1, CP = 4;
};
sdm_status_t fast_topk_plan(int n, int K, FastTopkPlan* out);

// sdm_tu_topk.cu: the selection (register path for K <= 64, shared-memory path above).
sdm_status_t topk_impl(const DeviceInfo& dev, const void* scores, int32_t in_dtype, int64_t units, int n, int K,
                       int32_t* idx, float* w, cudaStream_t st);
// sdm_tu_scan.cu: the resident and streaming recurrence kernels.
// ckpt (resident kernel, fp32 state): also store the backward's checkpoints
// every ckpt_C tokens ([n-1][B,H,N,d_v] fp32).
sdm_status_t launch_scan(const ScanChoice& c, const sdm_shape_t& s, const sdm::ScanArgs& a, cudaStream_t st,
                         float* ckpt = nullptr, int ckpt_C = 0);
// sdm_tu_pipe.cu: the pipelined recurrence and its records (y_zero: rows the parts add into, or null).
sdm_status_t launch_pipe_records(const sdm_shape_t& s, const ScanChoice& c, const int32_t* idx_w, const float* w_w,
                                 const int32_t* idx_r, const float* w_r, const void* alpha, const void* beta,
                                 uint32_t* rec, float* y_zero, const DeviceInfo& dev, cudaStream_t st);
sdm_status_t launch_pipe(const ScanChoice& c, const sdm_shape_t& s, const sdm::PipeArgs& a, cudaStream_t st);
// sdm_tu_bwd.cu: the recurrence backward.
sdm_status_t launch_bwd(const BwdChoice& c, int32_t in_dtype, const sdm::BwdArgs& a, cudaStream_t st);
// sdm_tu_decode.cu: the single-launch decode step, dispatched to the instances
// of launch_decode_for that sdm_tu_decode_<in>_<state>.cu compile.
sdm_status_t launch_decode(const FastTopkPlan& P, int32_t in_dtype, int32_t state_dtype, const sdm::DecodeArgs& a,
                           size_t smem, int grid, cudaStream_t st);
template <typename Tin, typename Tst>
sdm_status_t launch_decode_for(const FastTopkPlan& P, const sdm::DecodeArgs& a, size_t smem, int grid,
                               cudaStream_t st);

}  // namespace sdm_host
