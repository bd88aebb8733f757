// Weight-streaming GEMV for a handful of rows (batch-1 speculative decoding).
//
// y[r][n] = sum_k W[n][k] * x[r][k] for the R <= kRmax rows of a pass.  The
// work is HBM-bound: every weight byte is read once per pass.  The kernel is
// built around the tensor-memory-access (TMA) unit:
//   * one producer thread streams weight boxes of 32 rows x 256 columns
//     (16 KB) into a kStages-deep shared-memory ring with
//     cp.async.bulk.tensor (3-D tensor map: column, row, expert; no multicast),
//     each stage completing an mbarrier by transaction bytes.  Columns past K
//     and rows past N arrive zero-filled, so ragged shapes need no special case;
//   * each of the kNW consumer warps owns 4 rows of every box: lane l handles
//     the 16-byte chunk l of the 256-column slice for all 4 rows, with the
//     matching activation chunk of every pass row loaded once per slice;
//   * after the last slice a warp reduces its rows across lanes with a fixed
//     transpose-reduce (xor 16, 8) and butterfly (xor 4, 2, 1), and runs the
//     epilogue itself - no block-wide barrier per tile.
// Every output's reduction order is fixed by K alone (slice order, lane, the
// shuffle tree) - never by R, the row-group width or which rows share the
// pass - which is what makes the speculative path bit-identical to k = 0.
//
// Work items are (matrix, 32-row tile) pairs handed to CTAs in contiguous
// ranges.  Dense mode has one matrix; expert mode walks a device-side list of
// touched experts (shared experts first) so only the experts routed in this
// pass are streamed.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace ocrdec {

constexpr int kNW = 8;                          // consumer warps
constexpr int kConsumers = kNW * 32;            // consumer threads
constexpr int kGemvThreads = kConsumers + 32;   // + producer warp
constexpr int kWarpRows = 4;                    // weight rows per warp per tile
constexpr int kTile = kNW * kWarpRows;          // 32 rows per tile
constexpr int kSlice = 256;                     // columns per stage
constexpr int kBoxRows = 16;                    // rows per TMA box (two boxes per stage)
constexpr int kStageBytes = kTile * kSlice * 2; // 16 KB of weights per stage
constexpr int kStages = 4;
constexpr int kRmax = 8;                        // rows per pass on the GEMV path
constexpr int kXSliceBytes = kSlice * 2;        // one activation row of a staged bf16 slice (512 B)

struct GemvShape {
  int N, K;
  int ns;               // 256-column slices
  int pair_half;        // 0: tile = 32 consecutive rows; else 16 rows + the 16 rows pair_half below
  int tiles_per_mat;
  // expert mode (mats != nullptr)
  const int* mats;      // mats[m] = routed expert id (< n_experts) or n_experts + shared index
  const int* n_mats;
  int n_experts, top_k;
  const int* counts;    // rows routed to each expert
  const int* offsets;   // start of each expert's entries in rowlist
  const int* rowlist;   // entries r | (slot << 8)
  // rows of the pass
  const int* nrows;     // device row count, or nullptr to use rows_static
  int rows_static;
  int* status;
  int* counter;         // last-block counter (argmax / routing epilogues)
  // split-K (dense mode): each tile's K-slices are cut into kparts contiguous
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

__device__ __forceinline__ void mat_info(const GemvShape& s, int m, int R, int* coord_e, bool* shared,
                                         RowSet* rs) {
  if (!s.mats) {
    *coord_e = 0;
    *shared = false;
    if (rs) {
      rs->n = R;
#pragma unroll
      for (int i = 0; i < kRmax; ++i) rs->e[i] = i;
    }
    return;
  }
  int e = s.mats[m];
  if (e < s.n_experts) {
    *coord_e = e;
    *shared = false;
    if (rs) {
      int n = s.counts[e], off = s.offsets[e];
      n = n > kRmax ? kRmax : n;
      rs->n = n;
#pragma unroll
      for (int i = 0; i < kRmax; ++i) rs->e[i] = i < n ? s.rowlist[off + i] : 0;
    }
  } else {
    int sh = e - s.n_experts;
    *coord_e = sh;
    *shared = true;
    if (rs) {
      rs->n = R;
#pragma unroll
      for (int i = 0; i < kRmax; ++i) rs->e[i] = i | ((s.top_k + sh) << 8);
    }
  }
}

// 3-D tensor-map load: box (256 columns, 16 rows, 1 matrix) at (c0, row, mat).
__device__ __forceinline__ void tma_load_box(void* dst, const CUtensorMap* map, int c0, int row, int mat,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(row), "r"(mat), "r"(smem_u32(bar))
      : "memory");
}

// ---- packed float pairs (Blackwell f32x2 FMA) -------------------------------
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t pk2(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 upk2(f2_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
// acc.{x,y} = fma(a.{x,y}, b.{x,y}, acc.{x,y}), each rounded like a scalar fma
__device__ __forceinline__ void ffma2(f2_t& acc, f2_t a, f2_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
// a bfloat16 pair (low half = element 0) as a float pair
__device__ __forceinline__ f2_t bf2_to_f2(uint32_t u) {
  return pk2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// The 8 elements of one 16-byte weight chunk, or of the matching activation
// chunk, as 4 float pairs (0,1), (2,3), (4,5), (6,7).
struct Pairs8 {
  f2_t p[4];
};

__device__ __forceinline__ Pairs8 pairs_from_bf16(const uint4& u) {
  Pairs8 r;
  r.p[0] = bf2_to_f2(u.x);
  r.p[1] = bf2_to_f2(u.y);
  r.p[2] = bf2_to_f2(u.z);
  r.p[3] = bf2_to_f2(u.w);
  return r;
}

// ---------------------------------------------------------------------------
// activation sources: 16-byte chunk c16 of pass row r (slot for expert outputs)
// ---------------------------------------------------------------------------

// Rows of a float32 matrix, RMS-normalised, scaled by a gain vector and rounded
// to bfloat16 (the GEMV input precision), kept as float32 in shared memory for
// the whole kernel (K = model width).  The raw rows arrive by bulk copy; each
// is then normalised in place into two planes: plane 0 holds elements
// 8c..8c+3 of every 16-byte chunk c, plane 1 elements 8c+4..8c+7, so a lane's
// two 16-byte loads are consecutive across the warp.
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
  static constexpr int kBytesPerElem = 4;
  static constexpr int kMaxPer = 16;     // elements per thread per row: K <= 16 * 256

  static constexpr int kG = kMaxPer / 4;  // float4 groups per thread per row (K <= 4096)
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
  // One thread, right after the dependency wait: copy Rc raw rows into xs.
  // Rc is a bound known at launch (the pass's row count is read in parallel),
  // so the copies wait on no other load; source rows are clamped to the
  // kRmax-row buffers they index.
  __device__ static void issue(const Params& p, int K, int Rc, float* xs, uint64_t* xbar) {
    if (Rc <= 0) return;
    mbar_arrive_expect_tx(xbar, (uint32_t)(Rc * K * 4));
    for (int r = 0; r < Rc; ++r) {
      const int src = p.row_src ? min(max(p.row_src[r], 0), kRmax - 1) : r;
      bulk_g2s(xs + r * K, p.x + (long long)src * p.ldx, K * 4, xbar);
    }
  }

  // All consumer threads.  Thread t owns the float4 groups t, t + 256, ... of
  // each row; a group of raw elements [4m, 4m + 4) is plane (m & 1) at offset
  // (m >> 1) * 4 - contiguous in both layouts - so each group is read, scaled
  // and written back as one float4.  The sums of squares of all rows are formed
  // together (one barrier); a row is rewritten in place only once every thread
  // has read it, which the barrier after each row's reads guarantees.
  __device__ static void prologue(const Params& p, int K, int R, int Rc, float* xs, float* red, uint64_t* xbar,
                                  int* status, int tid, const Pre& pre) {
    const int ng = K / 4;
    if (Rc > 0) mbar_wait(xbar, 0, status);
    const int lane = tid & 31, warp = tid >> 5;
    const int half = K / 2;
    float a[kRmax];
    float4 v[kG];
#pragma unroll
    for (int r = 0; r < kRmax; ++r) {
      a[r] = 0.f;
      if (r < R) {
        const float4* row = reinterpret_cast<const float4*>(xs + r * K);
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          int m = tid + j * kConsumers;
          if (m < ng) {
            float4 t = row[m];
            if (r == 0) v[j] = t;
            a[r] = __fmaf_rn(t.x, t.x, a[r]);
            a[r] = __fmaf_rn(t.y, t.y, a[r]);
            a[r] = __fmaf_rn(t.z, t.z, a[r]);
            a[r] = __fmaf_rn(t.w, t.w, a[r]);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < kRmax; ++r) a[r] = __fadd_rn(a[r], __shfl_xor_sync(0xffffffffu, a[r], o));
    if (lane == 0)
#pragma unroll
      for (int r = 0; r < kRmax; ++r)
        if (r < R) red[r * kNW + warp] = a[r];
    named_sync(1, kConsumers);  // sums posted; row 0 read by every thread
    for (int r = 0; r < R; ++r) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < kNW; ++w) ss = __fadd_rn(ss, red[r * kNW + w]);
      const float sc = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)K), p.eps));
      float* row = xs + r * K;
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        int m = tid + j * kConsumers;
        if (m < ng) {
          float4 o;
          o.x = round_bf(__fmul_rn(__fmul_rn(v[j].x, sc), pre.g[j].x));
          o.y = round_bf(__fmul_rn(__fmul_rn(v[j].y, sc), pre.g[j].y));
          o.z = round_bf(__fmul_rn(__fmul_rn(v[j].z, sc), pre.g[j].z));
          o.w = round_bf(__fmul_rn(__fmul_rn(v[j].w, sc), pre.g[j].w));
          *reinterpret_cast<float4*>(row + (m & 1) * half + (m >> 1) * 4) = o;
        }
      }
      if (r + 1 < R) {
        const float4* nrow = reinterpret_cast<const float4*>(xs + (r + 1) * K);
#pragma unroll
        for (int j = 0; j < kG; ++j) {
          int m = tid + j * kConsumers;
          if (m < ng) v[j] = nrow[m];
        }
      }
      named_sync(1, kConsumers);  // row r written; row r + 1 read by every thread
    }
    if (R == 0) named_sync(1, kConsumers);
  }

  __device__ static Pairs8 chunk(const Params& p, const float* xs, const unsigned char* xstage, int K, int q, int r,
                                 int slot, int c16, int lane) {
    const float* base = xs + r * K + c16 * 4;
    float4 lo = *reinterpret_cast<const float4*>(base);
    float4 hi = *reinterpret_cast<const float4*>(base + K / 2);
    Pairs8 o;
    o.p[0] = pk2(lo.x, lo.y);
    o.p[1] = pk2(lo.z, lo.w);
    o.p[2] = pk2(hi.x, hi.y);
    o.p[3] = pk2(hi.z, hi.w);
    return o;
  }
};

// Rows of a bfloat16 matrix in global memory: row (row_src[r] * nslot + slot).
// The producer copies each slice of the item's rows into the stage next to the
// weight box (row-set entry q at offset q * 512 B), so consumers read them from
// shared memory.
struct SrcBf16 {
  struct Params {
    const bf16* x;
    long long ld;
    int nslot;
    const int* row_src;
  };
  static constexpr bool kSmem = false;
  static constexpr bool kStaged = true;
  static constexpr int kBytesPerElem = 0;
  struct Pre {};
  __device__ static void pre_wait(const Params&, int, int, Pre&) {}
  __device__ static void issue(const Params&, int, int, float*, uint64_t*) {}
  __device__ static void prologue(const Params&, int, int, int, float*, float*, uint64_t*, int*, int, const Pre&) {}
  __device__ static const bf16* row_ptr(const Params& p, int r, int slot) {
    return p.x + (long long)((p.row_src ? p.row_src[r] : r) * p.nslot + slot) * p.ld;
  }
  __device__ static Pairs8 chunk(const Params& p, const float*, const unsigned char* xstage, int K, int q, int r,
                                 int slot, int c16, int lane) {
    return pairs_from_bf16(*reinterpret_cast<const uint4*>(xstage + q * kXSliceBytes + lane * 16));
  }
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
// h[(r * nslot + slot) * ld + n] = bf16(silu(gate) * up)
struct EpiSwiGLU {
  struct Params {
    bf16* h;
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
    p.h[row * p.ld + o.n] = f2bf(__fmul_rn(act, up));
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
  };
  __device__ static float* best_v() { __shared__ float v[kNW * kRmax]; return v; }
  __device__ static int* best_i() { __shared__ int v[kNW * kRmax]; return v; }

  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs,
                               int lane) {
    int nrow = o.n;
    bool valid = o.q < rs.n && nrow < s.N;
    if (p.logits && valid) {
      int r = rs.r_sel(o.q);
      p.logits[(long long)(p.row_dst ? p.row_dst[r] : r) * s.N + nrow] = o.v;
    }
    float bv = valid ? o.v : -INFINITY;
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
    if (tid < R) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      const volatile float2* part = p.partial;
      for (int b = 0; b < (int)gridDim.x; ++b) {
        float ev = part[b * kRmax + tid].x;
        int ei = __float_as_int(part[b * kRmax + tid].y);
        if (ev > bv || (ev == bv && ei < bi)) { bv = ev; bi = ei; }
      }
      p.tok[(p.row_dst ? p.row_dst[tid] : tid) * p.tok_stride] = bi;
      s_tok[tid] = bi;
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

// Streams the tiles of one work item through the ring and returns the warp's
// reduced values: lane L = 8 i + q gets local row i (0..3) for row-set entry q.
// NR = live rows of the item (row-set entries 0..NR-1); the arithmetic of a
// row does not depend on NR.
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

template <class Src>
constexpr int stage_stride() {
  return kStageBytes + (Src::kStaged ? kRmax * kXSliceBytes : 0);
}

template <int NR, class Src>
__device__ __forceinline__ float consume_item(const GemvShape& s, const typename Src::Params& sp, const float* xs,
                                              const unsigned char* stages, uint64_t* full_bar, uint64_t* empty_bar,
                                              uint32_t& it, const RowSet& rs, const int (&srow)[kWarpRows],
                                              int nch, int lane, int sl0, int sl1) {
  f2_t acc[kWarpRows][NR > 0 ? NR : 1];
#pragma unroll
  for (int i = 0; i < kWarpRows; ++i)
#pragma unroll
    for (int q = 0; q < (NR > 0 ? NR : 1); ++q) acc[i][q] = 0ull;

  for (int sl = sl0; sl < sl1; ++sl, ++it) {
    const int st = it % kStages;
    mbar_wait(&full_bar[st], (it / kStages) & 1, s.status);
    const int c = sl * 32 + lane;  // this lane's 16-byte chunk of the row
    if (NR > 0 && c < nch) {
      const unsigned char* stg = stages + st * stage_stride<Src>();
      Pairs8 xv[NR > 0 ? NR : 1];
#pragma unroll
      for (int q = 0; q < NR; ++q) xv[q] = Src::chunk(sp, xs, stg + kStageBytes, s.K, q, rs.r(q), rs.slot(q), c, lane);
      const unsigned char* w_st = stg + lane * 16;
#pragma unroll
      for (int i = 0; i < kWarpRows; ++i) {
        Pairs8 wv = pairs_from_bf16(*reinterpret_cast<const uint4*>(w_st + srow[i] * (kSlice * 2)));
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int q = 0; q < NR; ++q) ffma2(acc[i][q], wv.p[e], xv[q].p[e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[st]);
  }

  // per lane: even + odd partial; then transpose over lane bits 4, 3 and a
  // butterfly over bits 2..0, after which lane L holds local row L >> 3
  float out = 0.f;
#pragma unroll
  for (int q = 0; q < NR; ++q) {
    float r4[kWarpRows];
#pragma unroll
    for (int i = 0; i < kWarpRows; ++i) {
      float2 t = upk2(acc[i][q]);
      r4[i] = __fadd_rn(t.x, t.y);
    }
    const bool up16 = lane & 16;
    float a0 = __fadd_rn(up16 ? r4[2] : r4[0], __shfl_xor_sync(0xffffffffu, up16 ? r4[0] : r4[2], 16));
    float a1 = __fadd_rn(up16 ? r4[3] : r4[1], __shfl_xor_sync(0xffffffffu, up16 ? r4[1] : r4[3], 16));
    const bool up8 = lane & 8;
    float b = __fadd_rn(up8 ? a1 : a0, __shfl_xor_sync(0xffffffffu, up8 ? a0 : a1, 8));
    b = __fadd_rn(b, __shfl_xor_sync(0xffffffffu, b, 4));
    b = __fadd_rn(b, __shfl_xor_sync(0xffffffffu, b, 2));
    b = __fadd_rn(b, __shfl_xor_sync(0xffffffffu, b, 1));
    if ((lane & 7) == q) out = b;
  }
  return out;
}

template <int RG, class Src>
__device__ __forceinline__ float consume_dispatch(int n, const GemvShape& s, const typename Src::Params& sp,
                                                  const float* xs, const unsigned char* stages, uint64_t* full_bar,
                                                  uint64_t* empty_bar, uint32_t& it, const RowSet& rs,
                                                  const int (&srow)[kWarpRows], int nch, int lane, int sl0,
                                                  int sl1) {
#define OCRDEC_CONSUME(NRV) \
  consume_item<NRV, Src>(s, sp, xs, stages, full_bar, empty_bar, it, rs, srow, nch, lane, sl0, sl1)
  if (n <= 0) return OCRDEC_CONSUME(0);
  if (n == 1 || RG == 1) return OCRDEC_CONSUME(1);
  if (n == 2 || RG == 2) return OCRDEC_CONSUME((RG >= 2 ? 2 : 1));
  if (n == 3) return OCRDEC_CONSUME((RG >= 3 ? 3 : 1));
  if (n == 4 || RG == 4) return OCRDEC_CONSUME((RG >= 4 ? 4 : 1));
  if (n == 5) return OCRDEC_CONSUME((RG >= 5 ? 5 : 1));
  if (n == 6) return OCRDEC_CONSUME((RG >= 6 ? 6 : 1));
  if (n == 7) return OCRDEC_CONSUME((RG >= 7 ? 7 : 1));
  return OCRDEC_CONSUME((RG >= 8 ? 8 : 1));
#undef OCRDEC_CONSUME
}

template <int RG, class Src, class Epi>
__global__ void __launch_bounds__(kGemvThreads, RG >= 8 ? 1 : 2)
gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_sh,
            const GemvShape s, const typename Src::Params sp, const typename Epi::Params ep) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], xbar;
  __shared__ int s_tag[kStages];  // item of the stage's slice (set with its first slice), -1 = end
  __shared__ float red_pro[kRmax * kNW];
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  TraceMarks tm;  // trace (consumer thread 0): wait returned, prologue done, main loop done
  constexpr int kStride = stage_stride<Src>();
  unsigned char* stages = smem;
  float* xs = reinterpret_cast<float*>(smem + kStages * kStride);
  const bool paired = s.pair_half != 0;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], Src::kStaged ? 2 : 1);
      mbar_init(&empty_bar[i], kNW);
    }
    mbar_init(&xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kNW) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    uint32_t it = 0;
    int R = 0;
    RowSet prs;  // rows of the current item (bf16 sources staged with the weights)
    int prs_m = -1;
    auto stage_wait = [&](int st) {
      // a wait that gives up records OCRDEC_ETIMEOUT and proceeds: control flow
      // stays uniform so the block always terminates
      if (it >= kStages) mbar_wait(&empty_bar[st], ((it / kStages) & 1) ^ 1, s.status);
    };
    // Stage = weight box (one arrival with its transaction bytes) and, for a
    // staged bf16 source, the item's activation slice rows (a second arrival,
    // declared only after the dependency wait).
    auto issue_w = [&](int item, int m, int t, int slc, bool first) {
      int ce;
      bool sh;
      mat_info(s, m, 0, &ce, &sh, nullptr);
      const CUtensorMap* map = sh ? &tm_sh : &tm_w;
      int r0, r1;
      tile_boxes(s, t, &r0, &r1);
      const int st = it % kStages;
      stage_wait(st);
      s_tag[st] = first ? item : -2;
      mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
      unsigned char* dst = stages + st * kStride;
      tma_load_box(dst, map, slc * kSlice, r0, ce, &full_bar[st]);
      tma_load_box(dst + kStageBytes / 2, map, slc * kSlice, r1, ce, &full_bar[st]);
      ++it;
    };
    auto issue_x = [&](uint32_t j, int m, int slc) {
      if (!Src::kStaged) return;
      if (m != prs_m) {
        int ce;
        bool sh;
        mat_info(s, m, R, &ce, &sh, &prs);
        prs_m = m;
      }
      const int st = j % kStages;
      unsigned char* dst = stages + st * kStride + kStageBytes;
      const int cols = min(kSlice, s.K - slc * kSlice);
      mbar_arrive_expect_tx(&full_bar[st], (uint32_t)(prs.n * cols * 2));
#pragma unroll
      for (int q = 0; q < kRmax; ++q)
        if (q < prs.n)
          bulk_g2s(dst + q * kXSliceBytes,
                   SrcBf16::row_ptr(reinterpret_cast<const SrcBf16::Params&>(sp), prs.r(q), prs.slot(q)) + slc * kSlice,
                   cols * 2, &full_bar[st]);
    };
    // items are claimed from the launch's work counter, so faster SMs take more
    int total = s.mats ? 0 : s.tiles_per_mat * s.kparts;
    // dense weights do not depend on earlier kernels: the stages of the CTA's
    // first item are requested before the dependency wait (one item only, so
    // that CTAs resident early do not take the work of those still arriving)
    int pre_sl[kStages];
    int npre = 0;
    int item = -1, sl = 0, sl_end = 0;
    auto claim = [&]() {
      item = atomicAdd(&s.work[0], 1);
      if (item < total) {
        ItemPos ip = item_pos(s, item);
        sl = ip.sl0;
        sl_end = ip.sl1;
      }
    };
    bool claimed = false;  // item/sl hold a claimed item not yet fully issued
    if (!s.mats) {
      claim();
      if (item < total) {
        const ItemPos ip = item_pos(s, item);
        while (sl < sl_end && it < (uint32_t)kStages) {
          pre_sl[npre++] = sl;
          issue_w(item, 0, ip.t, sl, sl == ip.sl0);
          ++sl;
        }
        claimed = sl < sl_end;
      }
    }
    pdl_wait();
    const bool ok = !status_bad(s.status);
    if (ok) {
      R = min(pass_rows(s), RG);
      for (int j = 0; j < npre; ++j) issue_x((uint32_t)j, 0, pre_sl[j]);
      if (s.mats) total = *s.n_mats * s.tiles_per_mat;
      if (!claimed) claim();
      while (item < total) {
        const ItemPos ip = item_pos(s, item);
        const uint32_t j = it;
        issue_w(item, ip.m, ip.t, sl, sl == ip.sl0);
        issue_x(j, ip.m, sl);
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
  // rows copied for a normalised source: the pass bound of this variant (the
  // engine's row buffers hold kRmax rows) or the exact static count
  const int Rc = s.nrows ? min(RG, kRmax) : min(s.rows_static, kRmax);
  if (tid == 0) {
    tm.t0 = gtimer();
    Src::issue(sp, s.K, Rc, xs, &xbar);
    s_abort = status_bad(s.status);
  }
  named_sync(1, kConsumers);
  if (s_abort) {
    if (Src::kSmem && tid == 0 && Rc > 0) mbar_wait(&xbar, 0, s.status);  // the row copies land first
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
  const int nch = s.K / 8;  // 16-byte chunks per row
  __shared__ int s_last_part;

  epi_init<Epi>(tid);
  if (Src::kSmem) Src::prologue(sp, s.K, R, Rc, xs, red_pro, &xbar, s.status, tid, pre);
  else named_sync(1, kConsumers);
  if (tid == 0) tm.t1 = gtimer();

  uint32_t it = 0;
  int cur_m = -1;
  RowSet rs;
  int ce = 0;
  bool sh = false;
  int srow[kWarpRows];
#pragma unroll
  for (int i = 0; i < kWarpRows; ++i) srow[i] = stage_row(paired, warp, i);

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
    if (ip.m != cur_m) {
      mat_info(s, ip.m, R, &ce, &sh, &rs);
      cur_m = ip.m;
    }
    WarpOut o;
    o.v = consume_dispatch<RG, Src>(rs.n, s, sp, xs, stages, full_bar, empty_bar, it, rs, srow, nch, lane, ip.sl0,
                                    ip.sl1);
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
    o.i = lane >> 3;
    o.q = lane & 7;
    int r0, r1;
    tile_boxes(s, ip.t, &r0, &r1);
    o.n = matrix_row(r0, r1, sel(srow, o.i));
    Epi::apply(ep, s, o, rs, lane);
  }
  named_sync(1, kConsumers);
  if (tid == 0) tm.t2 = gtimer();
  Epi::finish(ep, s, R, tid);
  if (tid == 0) trace_end(s.status, s.tag, tm);
}

}  // namespace ocrdec
