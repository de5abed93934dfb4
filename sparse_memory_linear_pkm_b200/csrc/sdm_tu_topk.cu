// Launches of the product-key selection kernels (template instances for each
// sqrt_n / K class and input dtype).

#include <algorithm>

#include "sdm_host.h"

namespace sdm_host {

sdm::TopkLayout topk_layout(int n, int K) {
  sdm::TopkLayout L{};
  L.n = n;
  L.K = K;
  L.Kh = std::min(K, n);
  int C = 0;
  for (int ra = 0; ra < L.Kh; ++ra) C += std::min(L.Kh, K / (ra + 1));
  L.C = C;
  auto a16 = [](uint32_t x) { return (x + 15u) & ~15u; };
  L.table_bytes = a16(static_cast<uint32_t>(C) * 4u);
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) {
    const uint32_t o = off;
    off += a16(bytes);
    return o;
  };
  L.vals = take(2u * n * 4u);
  L.hist = take(256u * 4u);
  L.hkey = take(static_cast<uint32_t>(L.Kh) * 8u);
  L.hval = take(2u * L.Kh * 4u);
  L.hidx = take(2u * L.Kh * 4u);
  L.c_hi = take(C * 4u);
  L.c_lo = take(C * 4u);
  L.c_slot = take(C * 4u);
  L.tie = take(C * 2u);
  L.f_hi = take(K * 4u);
  L.f_lo = take(K * 4u);
  L.f_slot = take(K * 4u);
  L.warp_bytes = off;
  return L;
}

template <typename Tin, int E, int EH, int EPL, int CP>
sdm_status_t launch_topk_fast_inst(const DeviceInfo& dev, const Tin* scores, int64_t units,
                                   const sdm::FastTopkLayout& L, int32_t* idx, float* w, cudaStream_t st) {
  auto kern = sdm::k_pkm_topk_fast<Tin, E, EH, EPL, CP>;
  const size_t smem = L.table_bytes + static_cast<size_t>(sdm::kFastTopkWarps) * L.warp_bytes;
  set_smem(reinterpret_cast<const void*>(kern), smem);
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, sdm::kFastTopkWarps * 32, smem);
  const int64_t blocks_needed = (units + sdm::kFastTopkWarps - 1) / sdm::kFastTopkWarps;
  const int grid =
      static_cast<int>(std::min<int64_t>(blocks_needed, static_cast<int64_t>(dev.sms) * std::max(1, per_sm) * 4));
  kern<<<grid, sdm::kFastTopkWarps * 32, smem, st>>>(scores, units, L, idx, w);
  return launch_status("pkm_topk launch");
}

// Register path for K <= 64.
template <typename Tin>
sdm_status_t launch_topk_fast(const DeviceInfo& dev, const void* scores, int64_t units, int n, int K,
                              int32_t* idx, float* w, cudaStream_t st) {
  FastTopkPlan P;
  sdm_status_t r;
  if ((r = fast_topk_plan(n, K, &P)) != SDM_OK) return r;
  const sdm::FastTopkLayout& L = P.L;
  const int E = P.E, EH = P.EH, CP = P.CP;
  const Tin* x = static_cast<const Tin*>(scores);
  const int epl = P.epl;
#define SDM_FAST_TOPK(E_, EH_, EPL_, CP_)                      \
  if (E == E_ && EH == EH_ && epl == EPL_ && CP == CP_) \
    return launch_topk_fast_inst<Tin, E_, EH_, EPL_, CP_>(dev, x, units, L, idx, w, st);
  SDM_FAST_TOPK(1, 1, 1, 4) SDM_FAST_TOPK(1, 1, 2, 4) SDM_FAST_TOPK(1, 1, 4, 4) SDM_FAST_TOPK(1, 1, 8, 4)
  SDM_FAST_TOPK(1, 1, 16, 4) SDM_FAST_TOPK(1, 1, 32, 4)
  SDM_FAST_TOPK(2, 1, 1, 7)
  SDM_FAST_TOPK(2, 2, 1, 9) SDM_FAST_TOPK(2, 2, 4, 9) SDM_FAST_TOPK(2, 2, 8, 9)
  SDM_FAST_TOPK(2, 2, 16, 9) SDM_FAST_TOPK(2, 2, 32, 9)
#undef SDM_FAST_TOPK
  return fail(SDM_ERR_UNSUPPORTED, "no selection kernel for this sqrt_n and K");
}

template <typename Tin>
sdm_status_t launch_topk(const DeviceInfo& dev, const void* scores, int64_t units, int n, int K, int32_t* idx,
                         float* w, cudaStream_t st) {
  if (units == 0) return SDM_OK;
  if (K <= sdm::kFastTopkMaxK) return launch_topk_fast<Tin>(dev, scores, units, n, K, idx, w, st);
  const sdm::TopkLayout L = topk_layout(n, K);
  int warps = 4;
  while (warps > 1 && L.table_bytes + static_cast<size_t>(warps) * L.warp_bytes > static_cast<size_t>(dev.max_smem_optin))
    --warps;
  const size_t smem = L.table_bytes + static_cast<size_t>(warps) * L.warp_bytes;
  if (smem > static_cast<size_t>(dev.max_smem_optin)) return fail(SDM_ERR_UNSUPPORTED, "selection scratch exceeds shared memory");
  auto kern = sdm::k_pkm_topk_general<Tin>;
  set_smem(reinterpret_cast<const void*>(kern), smem);
  const int64_t blocks_needed = (units + warps - 1) / warps;
  const int grid = static_cast<int>(std::min<int64_t>(blocks_needed, static_cast<int64_t>(dev.sms) * 16));
  kern<<<grid, warps * 32, smem, st>>>(static_cast<const Tin*>(scores), units, L, idx, w);
  return launch_status("pkm_topk launch");
}

sdm_status_t topk_impl(const DeviceInfo& dev, const void* scores, int32_t in_dtype, int64_t units, int n, int K,
                       int32_t* idx, float* w, cudaStream_t st) {
  return in_dtype == SDM_BF16 ? launch_topk<bf16>(dev, scores, units, n, K, idx, w, st)
                              : launch_topk<float>(dev, scores, units, n, K, idx, w, st);
}

}  // namespace sdm_host
