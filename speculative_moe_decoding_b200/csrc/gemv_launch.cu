// Instantiations of the weight-streaming GEMV and their dispatch.
#include <algorithm>

#include "launch.cuh"

namespace ocrdec {

void gemv_plan(GemvShape& s) {
  s.ns = (s.K + kSlice - 1) / kSlice;
  s.tiles_per_mat = s.pair_half ? (s.N / (2 * s.pair_half)) * (s.pair_half / kBoxRows) : (s.N + kTile - 1) / kTile;
  s.kparts = 1;
}

int gemv_kparts(const GemvShape& s, int target_items) {
  // Split only long, short matrices: a part posts partial sums, fences and
  // counts, which costs about as much as streaming four slices, so parts are
  // at least four slices long and only matrices too short to give every SM a
  // tile are split.
  constexpr int kMinSlicesPerPart = 4;
  if (s.tiles_per_mat >= 64 || s.ns < 2 * kMinSlicesPerPart) return 1;
  int want = (target_items + s.tiles_per_mat - 1) / s.tiles_per_mat;
  want = std::min(want, (s.ns + kMinSlicesPerPart - 1) / kMinSlicesPerPart);
  const int spp = (s.ns + want - 1) / want;  // slices per part
  int kp = (s.ns + spp - 1) / spp;           // parts, all non-empty
  if ((long long)s.tiles_per_mat * kp * kNW * 32 > kSplitPartFloats || s.tiles_per_mat > kSplitMaxTiles) return 1;
  return kp;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t encode_weight_map(const void* base, int K, int N, int E, CUtensorMap* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  // 4-D view of the [E][N][K] bfloat16 array: (64-column chunk, row, chunk
  // index, matrix); a box is 4 chunks x 16 rows, stored with the 128-byte
  // swizzle that makes the consumers' ldmatrix reads conflict-free
  if ((reinterpret_cast<uintptr_t>(base) & 15) || K % kChunk || K <= 0 || N <= 0 || E <= 0)
    return cudaErrorInvalidValue;
  cuuint64_t dims[4] = {(cuuint64_t)kChunk, (cuuint64_t)N, (cuuint64_t)(K / kChunk), (cuuint64_t)E};
  cuuint64_t strides[3] = {(cuuint64_t)K * 2, (cuuint64_t)kChunk * 2, (cuuint64_t)K * 2 * N};
  cuuint32_t box[4] = {kChunk, kBoxRows, kSlice / kChunk, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 5-D view of a KV cache [planes][H][cap][Dh] (planes = slots x layers):
// (64-column chunk, position, chunk index, head, plane); a box is one
// 64-position chunk of one head, stored [chunk][position][128 B] with the
// 128-byte swizzle.
cudaError_t encode_kv_map(const void* base, int Dh, int cap, int H, int planes, CUtensorMap* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  if ((reinterpret_cast<uintptr_t>(base) & 15) || Dh % 64 || cap <= 0 || H <= 0 || planes <= 0)
    return cudaErrorInvalidValue;
  const cuuint64_t row = (cuuint64_t)Dh * 2;
  cuuint64_t dims[5] = {64, (cuuint64_t)cap, (cuuint64_t)(Dh / 64), (cuuint64_t)H, (cuuint64_t)planes};
  cuuint64_t strides[4] = {row, 128, row * cap, row * cap * H};
  cuuint32_t box[5] = {64, 64, (cuuint32_t)(Dh / 64), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D view of W_o [d][d] for the attention kernel's output projection:
// (64-column chunk, row, chunk index); a box is one CTA's block, d/8 rows x the
// head's Dh columns, stored [chunk][row][128 B] with the 128-byte swizzle.
cudaError_t encode_oproj_map(const void* base, int d, int Dh, CUtensorMap* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  if ((reinterpret_cast<uintptr_t>(base) & 15) || d % 64 || Dh % 64 || d / 8 > 256 || d % 8) return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {64, (cuuint64_t)d, (cuuint64_t)(d / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)(d / 8), (cuuint32_t)(Dh / 64)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int RG, class Src, class Epi>
static cudaError_t configure_one() {
  cudaError_t e = cudaFuncSetAttribute(gemv_kernel<RG, Src, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemv_smem_bytes<Src, RG>(kGemvMaxK));
  // every kernel of the library asks for the same (maximal) shared-memory
  // carveout, so consecutive kernels never wait for an SM reconfiguration
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemv_kernel<RG, Src, Epi>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <class Src, class Epi>
static cudaError_t configure_rg() {
  cudaError_t e = configure_one<1, Src, Epi>();
  if (e == cudaSuccess) e = configure_one<2, Src, Epi>();
  if (e == cudaSuccess) e = configure_one<4, Src, Epi>();
  if (e == cudaSuccess) e = configure_one<8, Src, Epi>();
  return e;
}

cudaError_t gemv_prepare() {
  cudaError_t e = configure_rg<SrcNorm, EpiQKV>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiStore<false>>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiSwiGLU>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiArgmax>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm, EpiArgmaxAccept>();
  if (e == cudaSuccess) e = configure_rg<SrcBf16, EpiStore<false>>();
  if (e == cudaSuccess) e = configure_rg<SrcBf16, EpiStore<true>>();
  if (e == cudaSuccess) e = configure_rg<SrcNorm8, EpiArgmax>();
  return e;
}

template <int RG, class Src, class Epi>
static cudaError_t launch_one(const GemvLaunch& g, const typename Src::Params& sp, const typename Epi::Params& ep,
                              const LaunchCfg& lc) {
  auto kern = gemv_kernel<RG, Src, Epi>;
  if (Src::kSmem && g.s.K > kGemvMaxK) return cudaErrorInvalidValue;
  const size_t smem = gemv_smem_bytes<Src, RG>(g.s.K);
  // as many CTAs per SM as fit (two for the common shapes: they hide each
  // other's latencies)
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int slots = std::min(per_sm, 2) * lc.num_sms;
  int grid = g.grid > 0 ? std::min(g.grid, slots) : slots;
  grid = std::min(grid, g.s.tiles_per_mat * g.s.kparts);
  return launch_ex(kern, dim3(grid), dim3(kGemvThreads), smem, lc, g.tm_w, g.s, sp, ep);
}

template <class Src, class Epi>
static cudaError_t launch_rg(const GemvLaunch& g, const typename Src::Params& sp, const typename Epi::Params& ep,
                             const LaunchCfg& lc) {
  if (g.rows_bound <= 1) return launch_one<1, Src, Epi>(g, sp, ep, lc);
  if (g.rows_bound <= 2) return launch_one<2, Src, Epi>(g, sp, ep, lc);
  if (g.rows_bound <= 4) return launch_one<4, Src, Epi>(g, sp, ep, lc);
  return launch_one<8, Src, Epi>(g, sp, ep, lc);
}

cudaError_t launch_gemv(const GemvLaunch& g, const LaunchCfg& lc) {
  if (g.s.K % kChunk || (g.s.pair_half && (g.s.pair_half % kBoxRows || g.s.N % (2 * g.s.pair_half))))
    return cudaErrorInvalidValue;
  if (g.rows_bound > kRmax) return cudaErrorInvalidValue;
  if (g.s.kparts > 1 && (!g.s.part || !g.s.tile_counter)) return cudaErrorInvalidValue;
  if (!g.s.work) return cudaErrorInvalidValue;
  if (g.src == SrcKind::Norm8) {
    if (g.epi != EpiKind::Argmax) return cudaErrorInvalidValue;
    return launch_rg<SrcNorm8, EpiArgmax>(g, g.norm, g.argmax, lc);
  }
  if (g.src == SrcKind::Norm) {
    switch (g.epi) {
      case EpiKind::QKV: return launch_rg<SrcNorm, EpiQKV>(g, g.norm, g.qkv, lc);
      case EpiKind::Store: return launch_rg<SrcNorm, EpiStore<false>>(g, g.norm, g.store, lc);
      case EpiKind::SwiGLU: return launch_rg<SrcNorm, EpiSwiGLU>(g, g.norm, g.swiglu, lc);
      case EpiKind::Argmax: return launch_rg<SrcNorm, EpiArgmax>(g, g.norm, g.argmax, lc);
      case EpiKind::ArgmaxAccept: {
        EpiArgmaxAccept::Params ep{g.argmax, g.accept};
        return launch_rg<SrcNorm, EpiArgmaxAccept>(g, g.norm, ep, lc);
      }
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
