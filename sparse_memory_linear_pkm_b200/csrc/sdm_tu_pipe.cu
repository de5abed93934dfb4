// Launches of the pipelined recurrence and of its record build.

#include <algorithm>
#include <climits>
#include <mutex>
#include <type_traits>

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
                                s.T, s.H, static_cast<int>(slots_of(s.sqrt_n)), s.W, s.R, c.P, c.S, c.parts, log2_cells,
                                sdm::pipe_layout(s.W, s.R), rec, y_zero, s.d_v, dev.err);
  return launch_status("pipelined record build launch");
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (no link against libcuda).
EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <typename Tin, typename Tst>
sdm_status_t launch_pipe_typed(const ScanChoice& c, const sdm::PipeArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.H * a.parts, a.d_v / c.C);
  void (*kern)(sdm::PipeArgs) = nullptr;
#define SDM_PIPE(C_, P_, L_, NWW_, NWR_, NP_, S_)                                                          \
  if (c.C == C_ && c.P == P_ && c.L == L_ && c.NWW == NWW_ && c.NWR == NWR_ && c.NP == NP_ && c.S == S_)      \
    kern = sdm::k_scan_pipelined<Tin, Tst, C_, P_, L_, NWW_, NWR_, NP_, S_>;
  if constexpr (std::is_same<Tst, sdm::Fp8Blk>::value) {
    SDM_PIPE(64, 6, 16, 4, 3, 8, 1) SDM_PIPE(64, 6, 16, 4, 3, 4, 1)
  } else if constexpr (sizeof(Tst) == 2) {
    SDM_PIPE(64, 6, 16, 4, 3, 8, 1) SDM_PIPE(64, 6, 16, 4, 3, 4, 2) SDM_PIPE(64, 7, 8, 4, 3, 4, 2)
    SDM_PIPE(64, 6, 16, 4, 4, 8, 1) SDM_PIPE(64, 6, 16, 4, 3, 4, 1)
  } else {
    SDM_PIPE(32, 6, 16, 4, 3, 4, 1) SDM_PIPE(32, 4, 16, 4, 3, 4, 1) SDM_PIPE(32, 6, 16, 4, 3, 4, 2)
  }
#undef SDM_PIPE
  if (kern == nullptr) return fail(SDM_ERR_UNSUPPORTED, "no pipelined kernel for the chosen tile");
  set_smem(reinterpret_cast<const void*>(kern), c.smem);
  kern<<<grid, (c.NP + 1 + c.NWW + c.NWR) * 32, c.smem, st>>>(a);  // producers, the control warp, writers, readers
  return launch_status("pipelined scan launch");
}

sdm_status_t launch_pipe(const ScanChoice& c, const sdm_shape_t& s, const sdm::PipeArgs& args, cudaStream_t st) {
  // The state as a 2-D tensor of B*H*N rows of d_v values; one box is one
  // C-column segment of one row (the unit the TMA row gathers fetch).
  sdm::PipeArgs a = args;
  const uint64_t rows = static_cast<uint64_t>(a.B) * a.H * a.N;
  if (rows > static_cast<uint64_t>(INT_MAX)) return fail(SDM_ERR_UNSUPPORTED, "B*H*N above 2^31 - 1 state rows");
  const EncodeTiledFn encode = encode_tiled();
  if (encode == nullptr) return fail(SDM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const bool fp8 = s.state_dtype == SDM_FP8_B16;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(a.d_v), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(a.d_v) * state_size(s.state_dtype)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(c.C), 1u}, estride[2] = {1u, 1u};
  const CUtensorMapDataType dt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                     : (s.state_dtype == SDM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  CUresult e = encode(&a.state_map, dt, 2, a.M, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (e != CUDA_SUCCESS) return fail(SDM_ERR_CUDA, "cuTensorMapEncodeTiled failed with " + std::to_string(e));
  if (fp8) {
    // The block exponents after the codes: rows of d_v/16 bytes (a multiple
    // of 16: d_v % 256 == 0, checked by the chooser); one box is the 16
    // exponents of 256 columns, 16-byte aligned, that hold a tile's C/16.
    a.exps = reinterpret_cast<int8_t*>(static_cast<uint8_t*>(a.M) + rows * a.d_v);
    const cuuint64_t xdim[2] = {static_cast<cuuint64_t>(a.d_v / 16), static_cast<cuuint64_t>(rows)};
    const cuuint64_t xstride[1] = {static_cast<cuuint64_t>(a.d_v / 16)};
    const cuuint32_t xbox[2] = {16u, 1u};
    e = encode(&a.exps_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.exps, xdim, xstride, xbox, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (e != CUDA_SUCCESS) return fail(SDM_ERR_CUDA, "cuTensorMapEncodeTiled (exponents) failed with " + std::to_string(e));
    return s.in_dtype == SDM_BF16 ? launch_pipe_typed<bf16, sdm::Fp8Blk>(c, a, st)
                                  : launch_pipe_typed<float, sdm::Fp8Blk>(c, a, st);
  }
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
