// Weight-streaming GEMV for a handful of rows (batch-1 speculative decoding).
//
// y[r][n] = sum_k W[n][k] * x[r][k] for the R <= kRmax rows of a pass.  The
// work is HBM-bound: every weight byte is read once per pass.  The kernel is
// built around the tensor-memory-access (TMA) unit and the tensor cores:
//   * one producer thread streams weight tiles of 32 rows x 256 columns
//     (16 KB, two 16-row boxes) into a kStages-deep shared-memory ring with
//     cp.async.bulk.tensor (4-D tensor map: 64-column chunk, row, chunk index,
//     expert; 128-byte swizzle; no multicast), each stage completing an
//     mbarrier by transaction bytes.  Columns past K and rows past N arrive
//     zero-filled, so ragged shapes need no special case.  The boxes carry
//     an L2 evict-first policy: weights are read once per pass, and the
//     pass's reused data (KV caches, activations, code) should stay in L2;
//   * each of the kNW consumer warps owns one 16-row box and one 64-column
//     quarter of every slice and multiplies it with the pass rows on the
//     tensor cores (mma m16n8k16, bfloat16 in, float32 accumulate; the up to
//     8 pass rows are the 8 columns of B, each as a bfloat16 high and low
//     part), so a 16 KB stage costs a warp eight MMAs instead of hundreds of
//     FMAs - at R = 4 the FMA version was issue-bound below the HBM roofline;
//   * after the item's last slice the four column-quarter partials of every
//     output are added in quarter order through shared memory and the warps
//     run the epilogue.
// Every output's reduction order is fixed by K alone (k16 steps, slices,
// quarters) - never by R or by which rows share the pass: each MMA output
// column depends on its own B column only.  That is what makes the
// speculative path bit-identical to k = 0.
//
// Work items are 32-row tiles (or K-parts of them) claimed by CTAs from a
// per-launch counter.  (The MoE experts have their own persistent kernel,
// moe.cuh, built from the same tiles.)
#pragma once

#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "route.cuh"

namespace ocrdec {

constexpr int kNW = 8;                          // consumer warps
constexpr int kConsumers = kNW * 32;            // consumer threads
constexpr int kGemvThreads = kConsumers + 32;   // + producer warp
constexpr int kWarpRows = 4;                    // output rows per warp in the epilogue
constexpr int kTile = kNW * kWarpRows;          // 32 rows per tile
constexpr int kSlice = 256;                     // columns per stage
constexpr int kChunk = 64;                      // columns per 128-byte swizzled row of a box
constexpr int kBoxRows = 16;                    // rows per TMA box (two boxes per stage)
constexpr int kBoxBytes = kBoxRows * kSlice * 2;  // 8 KB: [4 chunks][16 rows][128 B]
constexpr int kStageBytes = 2 * kBoxBytes;      // 16 KB of weights per stage
constexpr int kStages = 4;
constexpr int kXStride = kSlice * 2 + 16;       // staged activation row (512 B + 16 B pad, ldmatrix-conflict-free)
constexpr int kRedFloats = 2 * 4 * kTile * 8;   // quarter partials, double-buffered by item

// Barrier over the consumer warps only (the producer warp does not take part).
struct ConsumerBarrier {
  __device__ void operator()() const { named_sync(1, kConsumers); }
};

struct GemvShape {
  int N, K;
  int ns;               // 256-column slices
  int pair_half;        // 0: tile = 32 consecutive rows; else 16 rows + the 16 rows pair_half below
  int tiles_per_mat;
  // rows of the pass
  const int* nrows;     // device row count, or nullptr to use rows_static
  int rows_static;
  int* status;
  int* counter;         // last-block counter (argmax epilogues)
  // split-K: each tile's K-slices are cut into kparts contiguous
  // parts handled by separate work items; the last part of a tile to finish
  // adds the parts' partial sums in part order and runs the epilogue
  int kparts;           // 1 = no split
  float* part;          // [tiles][kparts][kNW * 32] partial sums
  int* tile_counter;    // [tiles], zero between launches
  int tag;              // timeline-trace tag of this launch
  // dynamic work distribution: work[0] = next item to claim, work[1] = CTAs
  // done claiming; the last CTA resets both (zero between launches)
  int* work;
};

// Rows of one item: entry q = pass row | (output slot << 8).
struct RowSet {
  int n;
  int e[kRmax];
  __device__ __forceinline__ int r(int q) const { return e[q] & 0xff; }
  __device__ __forceinline__ int slot(int q) const { return e[q] >> 8; }
  __device__ __forceinline__ int r_sel(int q) const;     // runtime q
  __device__ __forceinline__ int slot_sel(int q) const;
};

// a[i] for a runtime i without indexing the array (which would move it to
// local memory): a chain of selects over the unrolled entries.
template <int N>
__device__ __forceinline__ int sel(const int (&a)[N], int i) {
  int v = a[0];
#pragma unroll
  for (int k = 1; k < N; ++k) v = (i == k) ? a[k] : v;
  return v;
}
__device__ __forceinline__ int RowSet::r_sel(int q) const { return sel(e, q) & 0xff; }
__device__ __forceinline__ int RowSet::slot_sel(int q) const { return sel(e, q) >> 8; }

__device__ __forceinline__ int pass_rows(const GemvShape& s) {
  int R = s.nrows ? *(volatile const int*)s.nrows : s.rows_static;
  return R < 0 ? 0 : (R > kRmax ? kRmax : R);
}

// First matrix row of each of the two 16-row boxes of a tile.
__device__ __forceinline__ void tile_boxes(const GemvShape& s, int tile, int* r0, int* r1) {
  if (s.pair_half == 0) {
    *r0 = tile * kTile;
    *r1 = tile * kTile + kBoxRows;
    return;
  }
  const int per_blk = s.pair_half / kBoxRows;
  const int blk = tile / per_blk, j = tile - blk * per_blk;
  *r0 = blk * 2 * s.pair_half + j * kBoxRows;
  *r1 = *r0 + s.pair_half;
}

// Stage row of local row i (0..3) of warp w.  Plain tiles: 4 consecutive rows.
// Paired tiles: rows 0,1 from the first box and their partners 2,3 from the
// second box (local i and i + 2 form a pair).
__device__ __forceinline__ int stage_row(bool paired, int w, int i) {
  return paired ? (i < 2 ? 2 * w + i : kBoxRows + 2 * w + (i - 2)) : kWarpRows * w + i;
}

__device__ __forceinline__ int matrix_row(int r0, int r1, int srow) {
  return srow < kBoxRows ? r0 + srow : r1 + (srow - kBoxRows);
}

// 4-D tensor-map load of one box: 4 chunks of 64 columns x 16 rows of matrix
// `mat`, starting at column chunk c4 and row `row`; shared layout
// [chunk][row][128 B] with the 128-byte swizzle.
__device__ __forceinline__ void tma_load_box(void* dst, const CUtensorMap* map, int c4, int row, int mat,
                                             uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(c4), "r"(mat), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- tensor-core fragments ----------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&b)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(b[0]), "=r"(b[1]) : "r"(addr));
}
// d += A (16x16, row) * B (16x8, col); bfloat16 in, float32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// d += A (16x32, row) * B (32x8, col); e4m3 in, float32 accumulate.  The
// 32-byte k-step spans the same bytes as a bf16 m16n8k16 step, so the same
// swizzled tiles and ldmatrix addresses feed it.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// float <-> e4m3 (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t f2e4m3(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m32f(uint32_t b) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3)));
}

// Four floats as high and low e4m3 parts, bytes in k order.
__device__ __forceinline__ void split_e4m3x4(const float (&f)[4], uint32_t& hi, uint32_t& lo) {
  hi = lo = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h = f2e4m3(f[i]);
    hi |= h << (8 * i);
    lo |= f2e4m3(__fsub_rn(f[i], e4m32f(h))) << (8 * i);
  }
}

// Four floats as high and low bfloat16 parts (high = bf16(f), low = bf16(f - high)).
__device__ __forceinline__ void split_bf16x4(float f0, float f1, float f2, float f3, uint2& hi, uint2& lo) {
  const bf16 h0 = f2bf(f0), h1 = f2bf(f1), h2 = f2bf(f2), h3 = f2bf(f3);
  hi.x = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
  hi.y = (uint32_t)__bfloat16_as_ushort(h2) | ((uint32_t)__bfloat16_as_ushort(h3) << 16);
  lo.x = pack2(__fsub_rn(f0, bf2f(h0)), __fsub_rn(f1, bf2f(h1)));
  lo.y = pack2(__fsub_rn(f2, bf2f(h2)), __fsub_rn(f3, bf2f(h3)));
}

// ---------------------------------------------------------------------------
// activation sources: the B operand (row-set entry q = MMA column q)
// ---------------------------------------------------------------------------

// Activations enter the MMAs as two bfloat16 parts, high = bf16(v) and
// low = bf16(v - high), each multiplied with the weights and accumulated in
// float32: the products carry float32-level precision of v (the only bfloat16
// rounding left on the path is the weights' own).  Rows of a source: RG
// high rows, then RG low rows; MMA column q >= RG reads row q % RG (its result
// is never used).

// Rows of a float32 matrix, RMS-normalised and scaled by a gain vector, kept in
// shared memory for the whole kernel as high / low bfloat16 rows of K + 8
// elements (the pad makes the eight rows of an ldmatrix fall in distinct
// banks).
struct SrcNorm {
  struct Params {
    const float* x;
    int ldx;
    const int* row_src;  // pass row r reads x row row_src[r] (nullptr: r)
    const bf16* gain;
    float eps;
  };
  static constexpr bool kSmem = true;    // activations live in shared memory (prologue)
  static constexpr bool kStaged = false; // activations are not part of the weight stages
  static constexpr bool kFp8 = false;    // bf16 weights and activation parts
  static constexpr int kG = 2;           // float4 groups per thread per row: K <= 2048
  __host__ __device__ static constexpr size_t smem_bytes(int K, int RG) { return (size_t)2 * RG * (K + 8) * 2; }

  // Gains are weights: loaded before the dependency wait.
  struct Pre {
    float4 g[kG];
  };
  __device__ static void pre_wait(const Params& p, int K, int tid, Pre& pre) {
    const int ng = K / 4;
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      int m = tid + j * kConsumers;
      if (m < ng) {
        uint2 u = *reinterpret_cast<const uint2*>(p.gain + 4 * m);
        pre.g[j] = make_float4(bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y));
      }
    }
  }

  // All consumer threads, after the dependency wait.  Thread t owns the float4
  // groups t, t + 256 of each row, read straight from L2 (the rows were just
  // written by the previous kernel); rows go four at a time: sums of squares,
  // one barrier, then the scaled values as high and low parts.
  template <int RG>
  __device__ static void prologue(const Params& p, int K, int R, unsigned char* xsm, float* red, int tid,
                                  const Pre& pre) {
    bf16* xh = reinterpret_cast<bf16*>(xsm);
    const int ld = K + 8, ng = K / 4;
    bf16* xl = xh + RG * ld;
    const int lane = tid & 31, warp = tid >> 5;
    for (int rb = 0; rb < R; rb += 4) {
      float4 v[4][kG];
      float a[4];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = rb + rr;
        a[rr] = 0.f;
        const int src = r < R ? (p.row_src ? min(max(p.row_src[r], 0), kRmax - 1) : r) : 0;
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          int m = tid + j * kConsumers;
          v[rr][j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (r < R && m < ng) v[rr][j] = __ldcg(reinterpret_cast<const float4*>(p.x + (long long)src * p.ldx) + m);
        }
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          a[rr] = __fmaf_rn(v[rr][j].x, v[rr][j].x, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].y, v[rr][j].y, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].z, v[rr][j].z, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].w, v[rr][j].w, a[rr]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) a[rr] = __fadd_rn(a[rr], __shfl_xor_sync(0xffffffffu, a[rr], o));
      if (lane == 0)
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) red[(rb + rr) * kNW + warp] = a[rr];
      named_sync(1, kConsumers);
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = rb + rr;
        if (r >= R) break;
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) ss = __fadd_rn(ss, red[r * kNW + w]);
        const float sc = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)K), p.eps));
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          int m = tid + j * kConsumers;
          if (m < ng) {
            const float f0 = __fmul_rn(__fmul_rn(v[rr][j].x, sc), pre.g[j].x);
            const float f1 = __fmul_rn(__fmul_rn(v[rr][j].y, sc), pre.g[j].y);
            const float f2 = __fmul_rn(__fmul_rn(v[rr][j].z, sc), pre.g[j].z);
            const float f3 = __fmul_rn(__fmul_rn(v[rr][j].w, sc), pre.g[j].w);
            uint2 hi, lo;
            split_bf16x4(f0, f1, f2, f3, hi, lo);
            *reinterpret_cast<uint2*>(xh + r * ld + 4 * m) = hi;
            *reinterpret_cast<uint2*>(xl + r * ld + 4 * m) = lo;
          }
        }
      }
    }
    named_sync(1, kConsumers);
  }

  // Shared address of the high B-fragment row data for ldmatrix.x2: row `row`
  // of this lane (lane & 7), column k0 (+8 for lanes 8..15) of the slice start;
  // the low part is lo_offset bytes further.
  __device__ static uint32_t b_base(const unsigned char* xsm, const unsigned char* stage_x, int K, int row, int lane) {
    return smem_u32(xsm) + (uint32_t)(row * (K + 8) + ((lane >> 3) & 1) * 8) * 2;
  }
  template <int RG>
  __device__ static uint32_t lo_offset(int K) { return (uint32_t)(RG * (K + 8) * 2); }
  __device__ static uint32_t b_slice(int slc) { return (uint32_t)slc * kSlice * 2; }
};

// Rows of a bfloat16 matrix pair (high, low parts) in global memory: row
// (row_src[r] * nslot + slot).  The producer copies each slice of the item's
// rows into the stage next to the weight boxes (row-set entry q at slot q, its
// low part at slot RG + q, kXStride apart), so consumers read them from shared
// memory.
struct SrcBf16 {
  struct Params {
    const bf16* x;       // high parts
    const bf16* x_lo;    // low parts (same layout)
    long long ld;
    int nslot;
    const int* row_src;
  };
  static constexpr bool kSmem = false;
  static constexpr bool kStaged = true;
  static constexpr bool kFp8 = false;
  __host__ __device__ static constexpr size_t smem_bytes(int, int) { return 0; }
  struct Pre {};
  __device__ static void pre_wait(const Params&, int, int, Pre&) {}
  template <int RG>
  __device__ static void prologue(const Params&, int, int, unsigned char*, float*, int, const Pre&) {}
  __device__ static long long row_off(const Params& p, int r, int slot) {
    return (long long)((p.row_src ? p.row_src[r] : r) * p.nslot + slot) * p.ld;
  }
  __device__ static uint32_t b_base(const unsigned char*, const unsigned char* stage_x, int, int row, int lane) {
    return smem_u32(stage_x) + (uint32_t)(row * kXStride + ((lane >> 3) & 1) * 16);
  }
  template <int RG>
  __device__ static uint32_t lo_offset(int) { return (uint32_t)(RG * kXStride); }
  __device__ static uint32_t b_slice(int) { return 0; }
};

// The same normalised rows as e4m3 high and low parts, for e4m3 weights (the
// draft's quantised LM head).  Layout and addressing are those of SrcNorm with
// K counted in byte pairs: the kernel's K is half the number of columns, and
// a row of K pairs holds 2K e4m3 values in column order.
struct SrcNorm8 {
  typedef SrcNorm::Params Params;
  static constexpr bool kSmem = true;
  static constexpr bool kStaged = false;
  static constexpr bool kFp8 = true;
  static constexpr int kG = 2;  // float4 groups per thread per row: 2K <= 2048
  __host__ __device__ static constexpr size_t smem_bytes(int K, int RG) { return SrcNorm::smem_bytes(K, RG); }
  typedef SrcNorm::Pre Pre;
  __device__ static void pre_wait(const Params& p, int K, int tid, Pre& pre) { SrcNorm::pre_wait(p, 2 * K, tid, pre); }

  template <int RG>
  __device__ static void prologue(const Params& p, int K, int R, unsigned char* xsm, float* red, int tid,
                                  const Pre& pre) {
    const int Kc = 2 * K, ng = Kc / 4, ld = (K + 8) * 2;  // columns, float4 groups, row bytes
    unsigned char* xh = xsm;
    unsigned char* xl = xsm + (size_t)RG * ld;
    const int lane = tid & 31, warp = tid >> 5;
    for (int rb = 0; rb < R; rb += 4) {
      float4 v[4][kG];
      float a[4];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = rb + rr;
        a[rr] = 0.f;
        const int src = r < R ? (p.row_src ? min(max(p.row_src[r], 0), kRmax - 1) : r) : 0;
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          const int m = tid + j * kConsumers;
          v[rr][j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (r < R && m < ng) v[rr][j] = __ldcg(reinterpret_cast<const float4*>(p.x + (long long)src * p.ldx) + m);
        }
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          a[rr] = __fmaf_rn(v[rr][j].x, v[rr][j].x, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].y, v[rr][j].y, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].z, v[rr][j].z, a[rr]);
          a[rr] = __fmaf_rn(v[rr][j].w, v[rr][j].w, a[rr]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) a[rr] = __fadd_rn(a[rr], __shfl_xor_sync(0xffffffffu, a[rr], o));
      if (lane == 0)
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) red[(rb + rr) * kNW + warp] = a[rr];
      named_sync(1, kConsumers);
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = rb + rr;
        if (r >= R) break;
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) ss = __fadd_rn(ss, red[r * kNW + w]);
        const float sc = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)Kc), p.eps));
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          const int m = tid + j * kConsumers;
          if (m < ng) {
            const float f[4] = {__fmul_rn(__fmul_rn(v[rr][j].x, sc), pre.g[j].x),
                                __fmul_rn(__fmul_rn(v[rr][j].y, sc), pre.g[j].y),
                                __fmul_rn(__fmul_rn(v[rr][j].z, sc), pre.g[j].z),
                                __fmul_rn(__fmul_rn(v[rr][j].w, sc), pre.g[j].w)};
            uint32_t hi, lo;
            split_e4m3x4(f, hi, lo);
            *reinterpret_cast<uint32_t*>(xh + (size_t)r * ld + 4 * m) = hi;
            *reinterpret_cast<uint32_t*>(xl + (size_t)r * ld + 4 * m) = lo;
          }
        }
      }
    }
    named_sync(1, kConsumers);
  }
  __device__ static uint32_t b_base(const unsigned char* xsm, const unsigned char* sx, int K, int row, int lane) {
    return SrcNorm::b_base(xsm, sx, K, row, lane);
  }
  template <int RG>
  __device__ static uint32_t lo_offset(int K) { return SrcNorm::lo_offset<RG>(K); }
  __device__ static uint32_t b_slice(int slc) { return SrcNorm::b_slice(slc); }
};

// ---------------------------------------------------------------------------
// epilogues: run by one warp on its 4 reduced rows.  Lane L = 8 i + q holds
// (in v) the result of local row i for pass-row slot q of the item's row set.
// ---------------------------------------------------------------------------

struct WarpOut {
  float v;           // value for (local row i, row-set entry q) of this lane
  int i, q;          // i = lane >> 3, q = lane & 7
  int n;             // matrix row of local row i (may be >= N in a ragged tile)
};

// out[(row(r) * nslot + slot) * ld + n] = v   (or += v when kAdd)
template <bool kAdd>
struct EpiStore {
  struct Params {
    float* y;
    long long ld;
    int nslot;
    const int* row_dst;  // pass row r -> output row (nullptr: r)
  };
  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs,
                               int lane) {
    if (o.q >= rs.n) return;
    int nrow = o.n;
    if (nrow >= s.N) return;
    int r = rs.r_sel(o.q);
    long long row = (long long)(p.row_dst ? p.row_dst[r] : r) * p.nslot + rs.slot_sel(o.q);
    float* dst = p.y + row * p.ld + nrow;
    if (kAdd) *dst = __fadd_rn(*dst, o.v);
    else *dst = o.v;
  }
  __device__ static void finish(const Params&, const GemvShape&, int, int) {}
};

// SwiGLU on paired tiles (gate row n, up row n + pair_half):
// h[(r * nslot + slot) * ld + n] = silu(gate) * up, as high and low bfloat16 parts
struct EpiSwiGLU {
  struct Params {
    bf16* h;      // high parts
    bf16* h_lo;   // low parts (the next GEMV's second operand)
    long long ld;
    int nslot;
  };
  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs,
                               int lane) {
    float up = __shfl_down_sync(0xffffffffu, o.v, 16);
    if (o.i >= 2 || o.q >= rs.n) return;
    float gt = o.v;
    float act = __fdiv_rn(gt, __fadd_rn(1.f, expf(-gt)));
    long long row = (long long)rs.r_sel(o.q) * p.nslot + rs.slot_sel(o.q);
    const float hv = __fmul_rn(act, up);
    const bf16 hi = f2bf(hv);
    p.h[row * p.ld + o.n] = hi;
    p.h_lo[row * p.ld + o.n] = f2bf(__fsub_rn(hv, bf2f(hi)));
  }
  __device__ static void finish(const Params&, const GemvShape&, int, int) {}
};

// Q/K/V projection on paired tiles of one head (dims j and j + head_dim/2):
// RoPE (rotate-half) on q and k with the table cos/sin[pos][j]; q -> float32
// qbuf[r][H][Dh]; k, v -> bfloat16 KV cache at (slot, head, pos).
struct EpiQKV {
  struct Params {
    float* q;             // [R][H*Dh]
    bf16* kc;             // K cache of this layer for slot 0: [H][cap][Dh]
    bf16* vc;
    long long slot_stride;  // elements between slots in the cache arrays
    int cap, H, Dh;
    const float2* rope;   // [cap][Dh/2] (cos, sin)
    const int* row_slot;  // pass row -> slot
    const int* row_pos;   // pass row -> position
  };
  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs,
                               int lane) {
    float b = __shfl_down_sync(0xffffffffu, o.v, 16);
    if (o.i >= 2 || o.q >= rs.n) return;
    float a = o.v;
    int n = o.n;                  // row of the first half
    int blk = n / p.Dh;                // 0..3H-1 : q heads, k heads, v heads
    int dim = n - blk * p.Dh;          // < Dh/2
    int half = p.Dh / 2;
    int r = rs.r_sel(o.q);
    int pos = p.row_pos[r];
    if (blk < 2 * p.H) {
      float2 cs = p.rope[(long long)pos * half + dim];
      float a2 = __fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));
      float b2 = __fadd_rn(__fmul_rn(b, cs.x), __fmul_rn(a, cs.y));
      a = a2;
      b = b2;
    }
    if (blk < p.H) {
      float* q = p.q + (long long)r * p.H * p.Dh + blk * p.Dh;
      q[dim] = a;
      q[dim + half] = b;
    } else {
      int h = blk < 2 * p.H ? blk - p.H : blk - 2 * p.H;
      bf16* c = (blk < 2 * p.H ? p.kc : p.vc) + (long long)p.row_slot[r] * p.slot_stride +
                ((long long)h * p.cap + pos) * p.Dh;
      c[dim] = f2bf(a);
      c[dim + half] = f2bf(b);
    }
  }
  __device__ static void finish(const Params&, const GemvShape&, int, int) {}
};

// Greedy argmax over all rows of the matrix (LM head).  Each warp keeps a
// running (value, index) per pass row; at the end the warps merge in order,
// the CTA writes its partial, and the last CTA to finish merges the partials
// (larger value, then lower index) and writes the tokens.
struct EpiArgmax {
  struct Params {
    int* tok;           // token of pass row r at tok[row_dst(r) * tok_stride]
    int tok_stride;
    float* logits;      // optional [R][N]
    float2* partial;    // [gridDim][kRmax] (value, index as float bits)
    const int* row_dst; // pass row -> tok/logits row (nullptr: r)
    const float* row_scale;  // optional [N]: each logit times this (quantised heads' inverse row scales)
  };
  __device__ static float* best_v() { __shared__ float v[kNW * kRmax]; return v; }
  __device__ static int* best_i() { __shared__ int v[kNW * kRmax]; return v; }

  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs,
                               int lane) {
    int nrow = o.n;
    bool valid = o.q < rs.n && nrow < s.N;
    const float lv = p.row_scale && nrow < s.N ? __fmul_rn(o.v, __ldg(p.row_scale + nrow)) : o.v;
    if (p.logits && valid) {
      int r = rs.r_sel(o.q);
      p.logits[(long long)(p.row_dst ? p.row_dst[r] : r) * s.N + nrow] = lv;
    }
    float bv = valid ? lv : -INFINITY;
    int bi = valid ? nrow : 0x7fffffff;
#pragma unroll
    for (int m = 8; m <= 16; m <<= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, m);
      int oi = __shfl_xor_sync(0xffffffffu, bi, m);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane < kRmax && lane < rs.n) {
      const int w = threadIdx.x >> 5;
      const int r = rs.r_sel(lane);
      float cv = best_v()[w * kRmax + r];
      int ci = best_i()[w * kRmax + r];
      if (bv > cv || (bv == cv && bi < ci)) {
        best_v()[w * kRmax + r] = bv;
        best_i()[w * kRmax + r] = bi;
      }
    }
  }

  __device__ static void init(int tid) {
    if (tid < kNW * kRmax) { best_v()[tid] = -INFINITY; best_i()[tid] = 0x7fffffff; }
  }

  // Per-CTA partial, then the last CTA merges all partials; returns true in the
  // last CTA, where s_tok[r] holds the token of pass row r (r < R).
  __device__ static bool merge(const Params& p, const GemvShape& s, int R, int tid, int* s_tok) {
    __shared__ int last;
    if (tid < kRmax) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int w = 0; w < kNW; ++w) {
        float v = best_v()[w * kRmax + tid];
        int i = best_i()[w * kRmax + tid];
        if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
      }
      p.partial[blockIdx.x * kRmax + tid] = make_float2(bv, __int_as_float(bi));
    }
    __threadfence();
    named_sync(1, kConsumers);
    if (tid == 0) last = (atomicAdd(s.counter, 1) == (int)gridDim.x - 1);
    named_sync(1, kConsumers);
    if (!last) return false;
    __threadfence();
    // every consumer thread takes the partials b = tid, tid + 256, ... of each
    // row (all loads in flight together); then warps, then the 8 warp results.
    // (value, lower index) is a total order, so the grouping cannot change it.
    __shared__ float m_v[kNW][kRmax];
    __shared__ int m_i[kNW][kRmax];
    const int lane = tid & 31, warp = tid >> 5;
    float bv[kRmax];
    int bi[kRmax];
#pragma unroll
    for (int r = 0; r < kRmax; ++r) {
      bv[r] = -INFINITY;
      bi[r] = 0x7fffffff;
    }
    for (int b = tid; b < (int)gridDim.x; b += kConsumers) {
      float2 e[kRmax];
#pragma unroll
      for (int r = 0; r < kRmax; ++r)
        if (r < R) e[r] = __ldcg(p.partial + b * kRmax + r);
#pragma unroll
      for (int r = 0; r < kRmax; ++r)
        if (r < R) {
          const int ei = __float_as_int(e[r].y);
          if (e[r].x > bv[r] || (e[r].x == bv[r] && ei < bi[r])) { bv[r] = e[r].x; bi[r] = ei; }
        }
    }
#pragma unroll
    for (int r = 0; r < kRmax; ++r) {
      if (r >= R) break;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv[r], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi[r], o);
        if (ov > bv[r] || (ov == bv[r] && oi < bi[r])) { bv[r] = ov; bi[r] = oi; }
      }
      if (lane == 0) {
        m_v[warp][r] = bv[r];
        m_i[warp][r] = bi[r];
      }
    }
    named_sync(1, kConsumers);
    if (tid < R) {
      float v = m_v[0][tid];
      int i = m_i[0][tid];
      for (int w = 1; w < kNW; ++w)
        if (m_v[w][tid] > v || (m_v[w][tid] == v && m_i[w][tid] < i)) { v = m_v[w][tid]; i = m_i[w][tid]; }
      p.tok[(p.row_dst ? p.row_dst[tid] : tid) * p.tok_stride] = i;
      s_tok[tid] = i;
    }
    if (tid == 0) *s.counter = 0;
    return true;
  }

  __device__ static void finish(const Params& p, const GemvShape& s, int R, int tid) {
    __shared__ int s_tok[kRmax];
    merge(p, s, R, tid, s_tok);
  }
};

template <class Epi>
__device__ __forceinline__ void epi_init(int tid) {}
template <>
__device__ __forceinline__ void epi_init<EpiArgmax>(int tid) { EpiArgmax::init(tid); }

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

// Work item -> (matrix, tile, slice range).  Dense mode may split a tile's
// slices into s.kparts parts (items tile * kparts + part).
struct ItemPos {
  int m, t, kp, sl0, sl1;
};

__device__ __forceinline__ ItemPos item_pos(const GemvShape& s, int item) {
  ItemPos ip;
  if (s.kparts > 1) {
    ip.m = 0;
    ip.t = item / s.kparts;
    ip.kp = item - ip.t * s.kparts;
    const int spp = (s.ns + s.kparts - 1) / s.kparts;
    ip.sl0 = ip.kp * spp;
    ip.sl1 = min(s.ns, ip.sl0 + spp);
  } else {
    ip.m = item / s.tiles_per_mat;
    ip.t = item - ip.m * s.tiles_per_mat;
    ip.kp = 0;
    ip.sl0 = 0;
    ip.sl1 = s.ns;
  }
  return ip;
}


template <class Src, int RG>
constexpr int stage_stride() {
  // weights, then (staged sources) the slice rows, high and low; 1 KB-aligned
  // for the swizzle
  return Src::kStaged ? (kStageBytes + 2 * RG * kXStride + 1023) / 1024 * 1024 : kStageBytes;
}

// Dynamic shared memory of one CTA: 1 KB alignment slack, the ring, the
// source's rows and the quarter partials.
template <class Src, int RG>
constexpr size_t gemv_smem_bytes(int K) {
  return 1024 + (size_t)kStages * stage_stride<Src, RG>() + Src::smem_bytes(K, RG) + kRedFloats * 4;
}

template <int RG, class Src, class Epi>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvShape s, const typename Src::Params sp,
            const typename Epi::Params ep) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ int s_tag[kStages];  // item of the stage's slice (set with its first slice), -1 = end
  __shared__ float red_pro[kRmax * kNW];
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  TraceMarks tm;  // trace (consumer thread 0): wait returned, prologue done, main loop done
  constexpr int kStride = stage_stride<Src, RG>();
  // the 128-byte swizzle repeats every 1 KB: the ring starts on a 1 KB boundary
  unsigned char* stages = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char* xsm = stages + kStages * kStride;
  float* red = reinterpret_cast<float*>(xsm + Src::smem_bytes(s.K, RG));
  const bool paired = s.pair_half != 0;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], Src::kStaged ? 2 : 1);
      mbar_init(&empty_bar[i], kNW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kNW) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    uint32_t it = 0;
    int R = 0;
    const uint64_t wpol = l2_evict_first_policy();  // weights are read once per pass
    auto stage_wait = [&](int st) {
      // a wait that gives up records OCRDEC_ETIMEOUT and proceeds: control flow
      // stays uniform so the block always terminates
      if (it >= kStages) mbar_wait(&empty_bar[st], ((it / kStages) & 1) ^ 1, s.status);
    };
    // Stage = two weight boxes (one arrival with their transaction bytes) and,
    // for a staged bf16 source, the pass rows' slice (a second arrival,
    // declared only after the dependency wait).
    auto issue_w = [&](int item, int t, int slc, bool first) {
      int r0, r1;
      tile_boxes(s, t, &r0, &r1);
      const int st = it % kStages;
      stage_wait(st);
      s_tag[st] = first ? item : -2;
      mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
      unsigned char* dst = stages + st * kStride;
      tma_load_box(dst, &tm_w, slc * (kSlice / kChunk), r0, 0, &full_bar[st], wpol);
      tma_load_box(dst + kBoxBytes, &tm_w, slc * (kSlice / kChunk), r1, 0, &full_bar[st], wpol);
      ++it;
    };
    auto issue_x = [&](uint32_t j, int slc) {
      if (!Src::kStaged) return;
      const int st = j % kStages;
      unsigned char* dst = stages + st * kStride + kStageBytes;
      const int cols = min(kSlice, s.K - slc * kSlice);
      const int nq = min(R, RG);
      mbar_arrive_expect_tx(&full_bar[st], (uint32_t)(2 * nq * cols * 2));
      const SrcBf16::Params& bp = reinterpret_cast<const SrcBf16::Params&>(sp);
#pragma unroll
      for (int q = 0; q < RG; ++q)
        if (q < nq) {
          const long long off = SrcBf16::row_off(bp, q, 0) + slc * kSlice;
          bulk_g2s(dst + q * kXStride, bp.x + off, cols * 2, &full_bar[st]);
          bulk_g2s(dst + (RG + q) * kXStride, bp.x_lo + off, cols * 2, &full_bar[st]);
        }
    };
    // items are claimed from the launch's work counter, so faster SMs take more
    const int total = s.tiles_per_mat * s.kparts;
    int item = -1, sl = 0, sl_end = 0;
    auto claim = [&]() {
      item = atomicAdd(&s.work[0], 1);
      if (item < total) {
        const ItemPos ip = item_pos(s, item);
        sl = ip.sl0;
        sl_end = ip.sl1;
      }
    };
    // the weights do not depend on earlier kernels: the stages of the CTA's
    // first item are requested before the dependency wait (one item only, so
    // that CTAs resident early do not take the work of those still arriving)
    int pre_sl[kStages];
    int npre = 0;
    claim();
    bool claimed = false;  // item/sl hold a claimed item not yet fully issued
    if (item < total) {
      const ItemPos ip = item_pos(s, item);
      while (sl < sl_end && it < (uint32_t)kStages) {
        pre_sl[npre++] = sl;
        issue_w(item, ip.t, sl, sl == ip.sl0);
        ++sl;
      }
      claimed = sl < sl_end;
    }
    pdl_wait();
    const bool ok = !status_bad(s.status);
    if (ok) {
      R = min(pass_rows(s), RG);
      for (int j = 0; j < npre; ++j) issue_x((uint32_t)j, pre_sl[j]);
      if (!claimed) claim();
      while (item < total) {
        const ItemPos ip = item_pos(s, item);
        const uint32_t j = it;
        issue_w(item, ip.t, sl, sl == ip.sl0);
        issue_x(j, sl);
        if (++sl == sl_end) claim();
      }
    } else if (Src::kStaged) {
      // aborting: complete the second arrival of every prefetched stage
      for (int j = 0; j < npre; ++j) mbar_arrive(&full_bar[j]);
    }
    // end marker: a stage with no data
    {
      const int st = it % kStages;
      stage_wait(st);
      s_tag[st] = -1;
      mbar_arrive(&full_bar[st]);
      if (Src::kStaged) mbar_arrive(&full_bar[st]);
      ++it;
    }
    // the last CTA done claiming resets the launch's counters
    __threadfence();
    if (atomicAdd(&s.work[1], 1) == (int)gridDim.x - 1) {
      __threadfence();
      s.work[0] = 0;
      s.work[1] = 0;
    }
    // drain: every issued copy has landed before the block can exit
    for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
      mbar_wait(&full_bar[j % kStages], (j / kStages) & 1, s.status);
    return;
  }

  // ---------------- consumers ----------------
  typename Src::Pre pre;
  Src::pre_wait(sp, s.K, tid, pre);
  pdl_wait();
  if (tid == 0) {
    tm.t0 = gtimer();
    s_abort = status_bad(s.status);
  }
  named_sync(1, kConsumers);
  if (s_abort) {
    // consume the producer's stages up to its end marker so it can finish
    uint32_t it = 0;
    while (true) {
      const int st = it % kStages;
      mbar_wait(&full_bar[st], (it / kStages) & 1, s.status);
      const int tag = s_tag[st];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
      ++it;
      if (tag == -1) break;
    }
    return;
  }
  pdl_trigger();

  const int R = min(pass_rows(s), RG);
  __shared__ int s_last_part;
  epi_init<Epi>(tid);
  Src::template prologue<RG>(sp, s.K, R, xsm, red_pro, tid, pre);
  if (!Src::kSmem) named_sync(1, kConsumers);
  if (tid == 0) tm.t1 = gtimer();

  // this warp's share of every stage: box g (16 rows), column quarter kq
  const int g = warp & 1, kq = warp >> 1;
  const int nchunks = s.K / kChunk;
  // A fragments (ldmatrix.x4): lane -> row (lane & 7) + 8 * bit 3, chunk +1 for lanes 16..31
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const uint32_t a_off = (uint32_t)(g * kBoxBytes + kq * (kBoxRows * 128) + a_row * 128);
  const int a_sw = a_row & 7, a_hi = lane >> 4;
  // epilogue mapping: lane L = 8 i + q takes local row i, pass row q
  const int ep_i = lane >> 3, ep_q = lane & 7;
  const int ep_srow = stage_row(paired, warp, ep_i);
  // the pass rows: entry q = row q
  RowSet rs;
  rs.n = R;
#pragma unroll
  for (int q = 0; q < kRmax; ++q) rs.e[q] = q;
  // B rows of this lane: pass row (lane & 7); columns past RG reuse row q % RG
  const int bq = (lane & 7) % RG;
  const uint32_t b_lo = Src::template lo_offset<RG>(s.K);

  uint32_t it = 0;
  int nitem = 0;
  while (true) {
    const int st0 = it % kStages;
    mbar_wait(&full_bar[st0], (it / kStages) & 1, s.status);
    const int item = s_tag[st0];
    if (item < 0) {  // end marker
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st0]);
      ++it;
      break;
    }
    const ItemPos ip = item_pos(s, item);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sl = ip.sl0; sl < ip.sl1; ++sl, ++it) {
      const int st = it % kStages;
      mbar_wait(&full_bar[st], (it / kStages) & 1, s.status);
      if (sl * (kSlice / kChunk) + kq < nchunks) {
        const unsigned char* stg = stages + st * kStride;
        const uint32_t a_base = smem_u32(stg) + a_off;
        const uint32_t b_addr = Src::b_base(xsm, stg + kStageBytes, s.K, bq, lane) + Src::b_slice(sl) +
                                (uint32_t)kq * kChunk * 2;
#pragma unroll
        for (int k16 = 0; k16 < kChunk / 16; ++k16) {
          uint32_t a[4], bh[2], bl[2];
          ldsm_x4(a_base + (uint32_t)((((2 * k16 + a_hi) ^ a_sw)) << 4), a);
          ldsm_x2(b_addr + k16 * 32, bh);
          ldsm_x2(b_addr + b_lo + k16 * 32, bl);
          if constexpr (Src::kFp8) {
            mma_e4m3(d, a, bh);
            mma_e4m3(d, a, bl);
          } else {
            mma_bf16(d, a, bh);
            mma_bf16(d, a, bl);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
    // quarter partials -> shared, then every output adds its quarters in order
    float* rb = red + (nitem & 1) * (4 * kTile * 8);
    ++nitem;
    {
      const int r = g * kBoxRows + (lane >> 2), c = 2 * (lane & 3);
      *reinterpret_cast<float2*>(rb + (kq * kTile + r) * 8 + c) = make_float2(d[0], d[1]);
      *reinterpret_cast<float2*>(rb + (kq * kTile + r + 8) * 8 + c) = make_float2(d[2], d[3]);
    }
    named_sync(1, kConsumers);
    WarpOut o;
    o.v = __fadd_rn(__fadd_rn(__fadd_rn(rb[(0 * kTile + ep_srow) * 8 + ep_q], rb[(1 * kTile + ep_srow) * 8 + ep_q]),
                              rb[(2 * kTile + ep_srow) * 8 + ep_q]),
                    rb[(3 * kTile + ep_srow) * 8 + ep_q]);
    if (s.kparts > 1) {
      // post this part; the tile's last part adds all parts in part order
      float* pt = s.part + ((long long)ip.t * s.kparts) * (kNW * 32);
      pt[ip.kp * (kNW * 32) + warp * 32 + lane] = o.v;
      __threadfence();
      named_sync(1, kConsumers);
      if (tid == 0) s_last_part = (atomicAdd(&s.tile_counter[ip.t], 1) == s.kparts - 1);
      named_sync(1, kConsumers);
      if (!s_last_part) continue;
      __threadfence();
      float v = 0.f;
      for (int kp = 0; kp < s.kparts; ++kp) v = __fadd_rn(v, __ldcg(pt + kp * (kNW * 32) + warp * 32 + lane));
      o.v = v;
      if (tid == 0) s.tile_counter[ip.t] = 0;
    }
    o.i = ep_i;
    o.q = ep_q;
    int r0, r1;
    tile_boxes(s, ip.t, &r0, &r1);
    o.n = matrix_row(r0, r1, ep_srow);
    Epi::apply(ep, s, o, rs, lane);
  }
  named_sync(1, kConsumers);
  if (tid == 0) tm.t2 = gtimer();
  Epi::finish(ep, s, R, tid);
  if (tid == 0) trace_end(s.status, s.tag, tm);
}

}  // namespace ocrdec
