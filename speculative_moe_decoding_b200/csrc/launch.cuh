// Host-side launch helpers shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "fused_epi.cuh"
#include "moe.cuh"

namespace ocrdec {

struct LaunchCfg {
  cudaStream_t stream;
  bool pdl;     // launch with programmatic stream serialization
  int num_sms;
};

// cudaLaunchKernelEx with optional programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, const LaunchCfg& lc,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = lc.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = lc.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same, with thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, const LaunchCfg& lc,
                      int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = lc.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = lc.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

enum class SrcKind { Norm, Bf16, Norm8 };  // Norm8: e4m3 weights and activation parts
enum class EpiKind { Store, StoreAdd, SwiGLU, QKV, Argmax, ArgmaxAccept };

// One GEMV launch: shape + the parameters of the chosen source and epilogue.
struct GemvLaunch {
  CUtensorMap tm_w;   // the matrix
  GemvShape s{};
  SrcKind src = SrcKind::Norm;
  EpiKind epi = EpiKind::Store;
  SrcNorm::Params norm{};
  SrcBf16::Params bf{};
  EpiStore<false>::Params store{};
  EpiSwiGLU::Params swiglu{};
  EpiQKV::Params qkv{};
  EpiArgmax::Params argmax{};
  AcceptParams accept{};  // EpiKind::ArgmaxAccept (with argmax)
  int rows_bound = kRmax;  // static bound on rows of one work item (selects the row-group width)
  int grid = 0;            // 0: derived from the work and the SM count
};

// Fills ns / tiles_per_mat from N, K and pair_half (and kparts = 1).
void gemv_plan(GemvShape& s);
// Split-K for a dense launch with few tiles: the number of K-parts (every part
// non-empty) that brings the item count near `target_items`.  Depends on the
// shape alone, so every launch of a matrix reduces in the same order.
int gemv_kparts(const GemvShape& s, int target_items);
constexpr int kSplitPartFloats = 1 << 19;  // partial-sum buffer (floats) shared by split launches
constexpr int kSplitMaxTiles = 4096;       // per-tile counters
// 3-D tensor map (columns K, rows N, matrices E) of a bfloat16 weight array with
// the GEMV's 256 x 16 box; base 16-byte aligned.
cudaError_t encode_oproj_map(const void* base, int d, int Dh, CUtensorMap* out);
cudaError_t encode_kv_map(const void* base, int Dh, int cap, int H, int planes, CUtensorMap* out);
cudaError_t encode_weight_map(const void* base, int K, int N, int E, CUtensorMap* out);
cudaError_t launch_gemv(const GemvLaunch& g, const LaunchCfg& lc);
// Raises the dynamic shared-memory limit of every GEMV instantiation to the
// largest size any launch uses (call outside stream capture, once per device).
cudaError_t gemv_prepare();
constexpr int kGemvMaxK = 2048;  // largest K of a normalised (shared-memory) source

// One launch of the MoE FFN kernel (moe.cuh): routed / shared gate-up and
// down tensor maps and the parameters.
struct MoeLaunch {
  CUtensorMap tm_gu, tm_sgu, tm_dn, tm_sdn;
  MoeParams p{};
};
cudaError_t launch_moe(const MoeLaunch& g, int rows_bound, const LaunchCfg& lc);
cudaError_t moe_prepare();
constexpr int kWorkSlots = 4;   // GEMV work-counter pairs cycled by a decoder context


}  // namespace ocrdec
