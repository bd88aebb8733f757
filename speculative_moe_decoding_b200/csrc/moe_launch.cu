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
  // two CTAs per SM with a ring of at least four stages if they fit (two
  // in-order pipelines per SM stream faster than one with twice the ring),
  // else one CTA with the deepest ring that fits
  int nst = 0, per_sm = 0;
  for (int want = 2; want >= 1 && !nst; --want)
    for (int n = kMoeMaxStages; n >= (want == 2 ? 4 : 2); --n) {
      int occ = 0;
      const size_t smem = moe_smem_bytes(p.d, p.f, RG, n);
      if ((int)smem + st > kSmemPerCta) continue;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, moe_kernel<RG>, kMoeThreads, smem) != cudaSuccess)
        return cudaErrorInvalidConfiguration;
      if (occ >= want) {
        nst = n;
        per_sm = want;
        break;
      }
    }
  if (!nst) return cudaErrorInvalidValue;
  p.nst = nst;
  // every CTA of the grid is resident at once (the combines wait until all
  // CTAs have read the residual)
  const int grid = per_sm * lc.num_sms;
  return launch_ex(moe_kernel<RG>, dim3(grid), dim3(kMoeThreads), moe_smem_bytes(p.d, p.f, RG, nst), lc, g.tm_gu,
                   g.tm_sgu, g.tm_dn, g.tm_sdn, p);
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
