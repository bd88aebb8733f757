// Instantiations of the MoE FFN kernel and their launch.
#include <algorithm>

#include "launch.cuh"
#include "moe.cuh"

namespace ocrdec {

namespace {

constexpr int kSmemPerCta = 227 * 1024;  // opt-in shared memory of one CTA (sm_100)

template <int RG>
int static_smem() {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, moe_kernel<RG>) != cudaSuccess) return -1;
  return (int)a.sharedSizeBytes;
}

template <int RG>
cudaError_t prepare_one() {
  const int st = static_smem<RG>();
  if (st < 0) return cudaErrorInvalidDeviceFunction;
  cudaError_t e = cudaFuncSetAttribute(moe_kernel<RG>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerCta - st);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(moe_kernel<RG>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int RG>
cudaError_t launch_rg(const MoeLaunch& g, const LaunchCfg& lc) {
  MoeParams p = g.p;
  const int st = static_smem<RG>();
  if (st < 0) return cudaErrorInvalidDeviceFunction;
  // the deepest weight ring that fits next to the rows and the item buffers
  int nst = kMoeMaxStages;
  while (nst > 2 && (int)moe_smem_bytes(p.d, p.f, RG, nst) + st > kSmemPerCta) --nst;
  if ((int)moe_smem_bytes(p.d, p.f, RG, nst) + st > kSmemPerCta) return cudaErrorInvalidValue;
  p.nst = nst;
  const size_t smem = moe_smem_bytes(p.d, p.f, RG, nst);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, moe_kernel<RG>, kMoeThreads, smem) != cudaSuccess ||
      per_sm < 1)
    return cudaErrorInvalidConfiguration;
  // one CTA per SM: every CTA of the grid is resident at once (the combine
  // waits until all CTAs have read the residual)
  const int grid = lc.num_sms;
  return launch_ex(moe_kernel<RG>, dim3(grid), dim3(kMoeThreads), smem, lc, g.tm_gu, g.tm_sgu, g.tm_dn, g.tm_sdn, p);
}

}  // namespace

cudaError_t moe_prepare() {
  cudaError_t e = prepare_one<1>();
  if (e == cudaSuccess) e = prepare_one<2>();
  if (e == cudaSuccess) e = prepare_one<4>();
  if (e == cudaSuccess) e = prepare_one<8>();
  return e;
}

cudaError_t launch_moe(const MoeLaunch& g, const int rows_bound, const LaunchCfg& lc) {
  const MoeParams& p = g.p;
  if (p.d % 128 || p.d > kGemvMaxK || p.f % kChunk || p.f > 1024 || p.f % kBoxRows) return cudaErrorInvalidValue;
  if (p.tiles_gu != p.f / kBoxRows || p.tiles_dn != p.d / kTile || p.tiles_dn > kMoeMaxTilesDn) return cudaErrorInvalidValue;
  if (p.E > kMaxExperts || p.S > kMaxShared || p.top_k > kMaxTopK || !p.ctr) return cudaErrorInvalidValue;
  if (rows_bound <= 1) return launch_rg<1>(g, lc);
  if (rows_bound <= 2) return launch_rg<2>(g, lc);
  if (rows_bound <= 4) return launch_rg<4>(g, lc);
  if (rows_bound <= kRmax) return launch_rg<8>(g, lc);
  return cudaErrorInvalidValue;
}

}  // namespace ocrdec
