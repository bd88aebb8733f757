// Instantiations of the weight-streaming GEMV and their dispatch.
#include <algorithm>

#include "launch.cuh"

namespace ocrdec {

void gemv_plan(GemvShape& s) {
  const int nch = s.K / 8;
  const int max_cps = kStageBytes / (kTR * 16);
  s.ns = (nch + max_cps - 1) / max_cps;
  s.cps = (nch + s.ns - 1) / s.ns;
  s.tiles_per_mat = s.N / kTR;
}

template <class Src>
static size_t smem_max() {
  return (size_t)kStages * kStageBytes + (Src::kSmem ? (size_t)kRmax * kGemvMaxK * 2 : 0);
}

template <int RG, class Src, class Epi>
static cudaError_t configure_one() {
  return cudaFuncSetAttribute(gemv_kernel<kTR, RG, Src, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_max<Src>());
}

template <class Src, class Epi>
static cudaError_t configure_rg() {
  cudaError_t e = configure_one<1, Src, Epi>();
  if (e == cudaSuccess) e = configure_one<2, Src, Epi>();
  if (e == cudaSuccess) e = configure_one<4, Src, Epi>();
  return e;
}

cudaError_t gemv_prepare() {
  cudaError_t e = configure_rg<SrcNorm, EpiQKV>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiStore<false>>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiSwiGLU>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiArgmax>();
  if (e == cudaSuccess) e = configure_rg<SrcBf16, EpiStore<false>>();
  if (e == cudaSuccess) e = configure_rg<SrcBf16, EpiStore<true>>();
  return e;
}

template <int RG, class Src, class Epi>
static cudaError_t launch_one(const GemvLaunch& g, const typename Src::Params& sp, const typename Epi::Params& ep,
                              const LaunchCfg& lc) {
  auto kern = gemv_kernel<kTR, RG, Src, Epi>;
  if (Src::kSmem && g.s.K > kGemvMaxK) return cudaErrorInvalidValue;
  size_t smem = (size_t)kStages * kStageBytes + (Src::kSmem ? (size_t)kRmax * g.s.K * 2 : 0);
  int grid = g.grid;
  if (grid <= 0) grid = g.s.mats ? lc.num_sms : std::min(g.s.tiles_per_mat, lc.num_sms);
  return launch_ex(kern, dim3(grid), dim3(kGemvThreads), smem, lc, g.s, sp, ep);
}

template <class Src, class Epi>
static cudaError_t launch_rg(const GemvLaunch& g, const typename Src::Params& sp, const typename Epi::Params& ep,
                             const LaunchCfg& lc) {
  if (g.rows_bound <= 1) return launch_one<1, Src, Epi>(g, sp, ep, lc);
  if (g.rows_bound <= 2) return launch_one<2, Src, Epi>(g, sp, ep, lc);
  return launch_one<4, Src, Epi>(g, sp, ep, lc);
}

cudaError_t launch_gemv(const GemvLaunch& g, const LaunchCfg& lc) {
  if (g.s.N % kTR || g.s.K % 8 || (g.s.pair_half && g.s.pair_half % (kTR / 2))) return cudaErrorInvalidValue;
  if (g.s.ns > 1 && g.s.mats) return cudaErrorInvalidValue;
  if (g.src == SrcKind::Norm) {
    switch (g.epi) {
      case EpiKind::QKV: return launch_rg<SrcNorm, EpiQKV>(g, g.norm, g.qkv, lc);
      case EpiKind::Store: return launch_rg<SrcNorm, EpiStore<false>>(g, g.norm, g.store, lc);
      case EpiKind::SwiGLU: return launch_rg<SrcNorm, EpiSwiGLU>(g, g.norm, g.swiglu, lc);
      case EpiKind::Argmax: return launch_rg<SrcNorm, EpiArgmax>(g, g.norm, g.argmax, lc);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (g.epi) {
    case EpiKind::Store: return launch_rg<SrcBf16, EpiStore<false>>(g, g.bf, g.store, lc);
    case EpiKind::StoreAdd: {
      EpiStore<true>::Params ep{g.store.y, g.store.ld, g.store.nslot, g.store.row_dst};
      return launch_rg<SrcBf16, EpiStore<true>>(g, g.bf, ep, lc);
    }
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ocrdec
