// Weight-streaming GEMV for a handful of rows (batch-1 speculative decoding).
//
// y[r][n] = sum_k W[n][k] * x[r][k] for the R <= kRmax rows of a pass.  The
// work is HBM-bound: every weight byte is read once per pass, so the kernel is
// built around the bulk-copy (TMA) unit:
//   * one producer thread streams weight tiles (TR rows x one K-slice) into a
//     kStages-deep ring of shared-memory stages with cp.async.bulk, each stage
//     completing an mbarrier by transaction bytes;
//   * kNW consumer warps own 16-byte K-chunks of the stage (thread t owns chunks
//     t, t+256, ...), load the matching activation chunk of up to RG rows once
//     and apply it to all TR weight rows of the tile;
//   * each output is then reduced across the warp by a transpose-reduce whose
//     shape depends on TR only, and across warps in warp order.
// Every output's reduction order is therefore fixed by (K, TR) alone - never by
// R, RG or which other rows share the pass - which is what makes the
// speculative path bit-identical to k = 0.
//
// Work items are (matrix, tile) pairs handed to CTAs in contiguous ranges.
// Dense mode has one matrix; expert mode walks a device-side list of touched
// experts (shared experts first) so only the experts routed in this pass are
// streamed.
#pragma once

#include "common.cuh"

namespace ocrdec {

constexpr int kNW = 8;                      // consumer warps
constexpr int kConsumers = kNW * 32;        // consumer threads
constexpr int kGemvThreads = kConsumers + 32;  // + producer warp
constexpr int kStages = 3;
constexpr int kStageBytes = 24 * 1024;
constexpr int kRmax = 8;                    // rows per pass on the GEMV path

struct GemvShape {
  const bf16* W;        // dense matrix, or expert 0 of the routed experts
  const bf16* W_sh;     // expert mode: shared expert 0
  long long mat_stride; // elements between consecutive expert matrices
  int N, K;
  int cps;              // 16-byte chunks per K-slice
  int ns;               // K-slices (> 1 only in dense mode)
  int pair_half;        // 0: tile = TR consecutive rows; else TR/2 rows + the TR/2 rows pair_half below
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
  int* counter;         // last-block counter (argmax epilogue)
};

struct RowSet {
  int n;
  int r[kRmax];
  int slot[kRmax];
};

__device__ __forceinline__ int pass_rows(const GemvShape& s) {
  int R = s.nrows ? *(volatile const int*)s.nrows : s.rows_static;
  return R < 0 ? 0 : (R > kRmax ? kRmax : R);
}

// Matrix row of tile-row i.
template <int TR>
__device__ __forceinline__ int tile_row(const GemvShape& s, int tile, int i) {
  if (s.pair_half == 0) return tile * TR + i;
  constexpr int H2 = TR / 2;
  int per_blk = s.pair_half / H2;
  int blk = tile / per_blk, j = tile - blk * per_blk;
  int base = blk * 2 * s.pair_half + j * H2;
  return i < H2 ? base + i : base + s.pair_half + (i - H2);
}

__device__ __forceinline__ void mat_info(const GemvShape& s, int m, int R, const bf16** Wm, int* expert,
                                         RowSet* rs) {
  if (!s.mats) {
    *Wm = s.W;
    *expert = 0;
    if (rs) {
      rs->n = R;
      for (int i = 0; i < kRmax; ++i) { rs->r[i] = i; rs->slot[i] = 0; }
    }
    return;
  }
  int e = s.mats[m];
  *expert = e;
  if (e < s.n_experts) {
    *Wm = s.W + (long long)e * s.mat_stride;
    if (rs) {
      int n = s.counts[e], off = s.offsets[e];
      n = n > kRmax ? kRmax : n;
      rs->n = n;
      for (int i = 0; i < kRmax; ++i) {
        int v = i < n ? s.rowlist[off + i] : 0;
        rs->r[i] = v & 0xff;
        rs->slot[i] = v >> 8;
      }
    }
  } else {
    int sh = e - s.n_experts;
    *Wm = s.W_sh + (long long)sh * s.mat_stride;
    if (rs) {
      rs->n = R;
      for (int i = 0; i < kRmax; ++i) { rs->r[i] = i; rs->slot[i] = s.top_k + sh; }
    }
  }
}

// ---------------------------------------------------------------------------
// activation sources
// ---------------------------------------------------------------------------

// Rows of a float32 matrix, RMS-normalised, scaled by a gain vector and rounded
// to bfloat16 into shared memory once per kernel (K = model width).
struct SrcNorm {
  struct Params {
    const float* x;
    int ldx;
    const int* row_src;  // pass row r reads x row row_src[r] (nullptr: r)
    const bf16* gain;
    float eps;
  };
  static constexpr bool kSmem = true;

  __device__ static void prologue(const Params& p, int K, int R, bf16* xs, float* red, int tid) {
    // per-row sum of squares: thread-strided partials, warp butterfly, warps in order
    __shared__ float scale[kRmax];
    int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int r = 0; r < kRmax; ++r) {
      float a = 0.f;
      if (r < R) {
        const float* xr = p.x + (long long)(p.row_src ? p.row_src[r] : r) * p.ldx;
        for (int k = tid; k < K; k += kConsumers) a = __fmaf_rn(xr[k], xr[k], a);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0) red[warp * kRmax + r] = a;
    }
    named_sync(1, kConsumers);
    if (tid < kRmax) {
      float a = 0.f;
      for (int w = 0; w < kNW; ++w) a = __fadd_rn(a, red[w * kRmax + tid]);
      scale[tid] = rsqrtf(__fadd_rn(__fdiv_rn(a, (float)K), p.eps));
    }
    named_sync(1, kConsumers);
    for (int r = 0; r < R; ++r) {
      const float* xr = p.x + (long long)(p.row_src ? p.row_src[r] : r) * p.ldx;
      float sc = scale[r];
      for (int k = tid; k < K; k += kConsumers)
        xs[r * K + k] = f2bf(__fmul_rn(__fmul_rn(xr[k], sc), bf2f(p.gain[k])));
    }
    named_sync(1, kConsumers);
  }

  __device__ static uint4 chunk(const Params& p, const bf16* xs, int K, int r, int slot, int c16) {
    return *reinterpret_cast<const uint4*>(xs + r * K + c16 * 8);
  }
};

// Rows of a bfloat16 matrix in global memory: row (row_src[r] * nslot + slot).
struct SrcBf16 {
  struct Params {
    const bf16* x;
    long long ld;
    int nslot;
    const int* row_src;
  };
  static constexpr bool kSmem = false;
  __device__ static void prologue(const Params&, int, int, bf16*, float*, int) {}
  __device__ static uint4 chunk(const Params& p, const bf16*, int K, int r, int slot, int c16) {
    int row = (p.row_src ? p.row_src[r] : r) * p.nslot + slot;
    return ld_v4(p.x + (long long)row * p.ld + c16 * 8);
  }
};

// ---------------------------------------------------------------------------
// epilogues: called by all consumer threads with red[w][i][rg] complete
// ---------------------------------------------------------------------------

template <int TR, int RG>
__device__ __forceinline__ float red_sum(const float* red, int i, int rg) {
  float a = 0.f;
#pragma unroll
  for (int w = 0; w < kNW; ++w) a = __fadd_rn(a, red[(w * TR + i) * RG + rg]);
  return a;
}

// out[(row(r) * nslot + slot) * ld + n] = v   (or += v when kAdd)
template <bool kAdd>
struct EpiStore {
  struct Params {
    float* y;
    long long ld;
    int nslot;
    const int* row_dst;  // pass row r -> output row (nullptr: r)
  };
  template <int TR, int RG>
  __device__ static void apply(const Params& p, const GemvShape& s, int expert, int tile, const float* red,
                               const RowSet& rs, int g, int tid) {
    if (tid >= TR * RG) return;
    int i = tid / RG, rg = tid % RG, j = g * RG + rg;
    if (j >= rs.n) return;
    float v = red_sum<TR, RG>(red, i, rg);
    int r = rs.r[j];
    long long row = (long long)(p.row_dst ? p.row_dst[r] : r) * p.nslot + rs.slot[j];
    float* dst = p.y + row * p.ld + tile_row<TR>(s, tile, i);
    if (kAdd) *dst = __fadd_rn(*dst, v);
    else *dst = v;
  }
  __device__ static void finish(const Params&, const GemvShape&, int, int) {}
};

// SwiGLU on paired tiles (gate rows i, up rows i + pair_half):
// h[(r * nslot + slot) * ld + n] = bf16(silu(gate) * up)
struct EpiSwiGLU {
  struct Params {
    bf16* h;
    long long ld;
    int nslot;
  };
  template <int TR, int RG>
  __device__ static void apply(const Params& p, const GemvShape& s, int expert, int tile, const float* red,
                               const RowSet& rs, int g, int tid) {
    constexpr int H2 = TR / 2;
    if (tid >= H2 * RG) return;
    int i = tid / RG, rg = tid % RG, j = g * RG + rg;
    if (j >= rs.n) return;
    float gt = red_sum<TR, RG>(red, i, rg);
    float up = red_sum<TR, RG>(red, i + H2, rg);
    float act = __fdiv_rn(gt, __fadd_rn(1.f, expf(-gt)));
    int n = tile_row<TR>(s, tile, i);  // gate row index = position in the hidden vector
    long long row = (long long)rs.r[j] * p.nslot + rs.slot[j];
    p.h[row * p.ld + n] = f2bf(__fmul_rn(act, up));
  }
  __device__ static void finish(const Params&, const GemvShape&, int, int) {}
};

// Q/K/V projection on paired tiles of one head (dims i and i + head_dim/2):
// RoPE (rotate-half) on q and k with the table cos/sin[pos][i]; q -> float32
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
  template <int TR, int RG>
  __device__ static void apply(const Params& p, const GemvShape& s, int expert, int tile, const float* red,
                               const RowSet& rs, int g, int tid) {
    constexpr int H2 = TR / 2;
    if (tid >= H2 * RG) return;
    int i = tid / RG, rg = tid % RG, j = g * RG + rg;
    if (j >= rs.n) return;
    float a = red_sum<TR, RG>(red, i, rg);
    float b = red_sum<TR, RG>(red, i + H2, rg);
    int n = tile_row<TR>(s, tile, i);  // row of the first half
    int blk = n / p.Dh;                // 0..3H-1 : q heads, k heads, v heads
    int dim = n - blk * p.Dh;          // < Dh/2
    int half = p.Dh / 2;
    int r = rs.r[j];
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

// Greedy argmax over all rows of the matrix (LM head): per-CTA running maximum
// (first index wins ties), then the last CTA to finish merges the per-CTA
// partials (larger value, then lower index) and writes tok[r].
struct EpiArgmax {
  struct Params {
    int* tok;           // token of pass row r at tok[row_dst(r) * tok_stride]
    int tok_stride;
    float* logits;      // optional [R][N]
    float2* partial;    // [gridDim][kRmax] (value, index as float bits)
    const int* row_dst; // pass row -> tok/logits row (nullptr: r)
  };
  __device__ static float* best_v() { __shared__ float v[kRmax]; return v; }
  __device__ static int* best_i() { __shared__ int v[kRmax]; return v; }

  template <int TR, int RG>
  __device__ static void apply(const Params& p, const GemvShape& s, int expert, int tile, const float* red,
                               const RowSet& rs, int g, int tid) {
    if (p.logits && tid < TR * RG) {
      int i = tid / RG, rg = tid % RG, j = g * RG + rg;
      if (j < rs.n) {
        int r = rs.r[j];
        int orow = p.row_dst ? p.row_dst[r] : r;
        p.logits[(long long)orow * s.N + tile_row<TR>(s, tile, i)] = red_sum<TR, RG>(red, i, rg);
      }
    }
    if (tid >= RG) return;
    int j = g * RG + tid;
    if (j >= rs.n) return;
    int r = rs.r[j];
    float bv = best_v()[r];
    int bi = best_i()[r];
    for (int i = 0; i < TR; ++i) {
      float v = red_sum<TR, RG>(red, i, tid);
      int n = tile_row<TR>(s, tile, i);
      if (v > bv || (v == bv && n < bi)) { bv = v; bi = n; }
    }
    best_v()[r] = bv;
    best_i()[r] = bi;
  }

  __device__ static void init(int tid) {
    if (tid < kRmax) { best_v()[tid] = -INFINITY; best_i()[tid] = 0x7fffffff; }
  }

  __device__ static void finish(const Params& p, const GemvShape& s, int R, int tid) {
    __shared__ int last;
    if (tid < kRmax)
      p.partial[blockIdx.x * kRmax + tid] = make_float2(best_v()[tid], __int_as_float(best_i()[tid]));
    __threadfence();
    named_sync(1, kConsumers);
    if (tid == 0) last = (atomicAdd(s.counter, 1) == (int)gridDim.x - 1);
    named_sync(1, kConsumers);
    if (!last) return;
    __threadfence();
    if (tid < R) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      const volatile float2* part = p.partial;
      for (int b = 0; b < (int)gridDim.x; ++b) {
        float2 e = const_cast<const float2&>(part[b * kRmax + tid]);
        int ei = __float_as_int(e.y);
        if (e.x > bv || (e.x == bv && ei < bi)) { bv = e.x; bi = ei; }
      }
      p.tok[(p.row_dst ? p.row_dst[tid] : tid) * p.tok_stride] = bi;
    }
    if (tid == 0) *s.counter = 0;
  }
};

template <class Epi>
__device__ __forceinline__ void epi_init(int tid) {}
template <>
__device__ __forceinline__ void epi_init<EpiArgmax>(int tid) { EpiArgmax::init(tid); }

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

// After log2(TR) halving stages (xor 16, 8, ...) every lane holds one
// partially reduced value whose tile row is decoded from its lane bits; a
// butterfly over the remaining lane bits finishes the sum.
template <int N, int M>
__device__ __forceinline__ void transpose_stage(float* v, int lane) {
  if constexpr (N > 1) {
    constexpr int H = N / 2;
    const bool upper = (lane & M) != 0;
#pragma unroll
    for (int j = 0; j < H; ++j) {
      float send = upper ? v[j] : v[j + H];
      float keep = upper ? v[j + H] : v[j];
      v[j] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, M));
    }
    transpose_stage<H, M / 2>(v, lane);
  }
}

template <int TR>
__device__ __forceinline__ void warp_transpose_reduce(float* v, int lane) {
  transpose_stage<TR, 16>(v, lane);
}

template <int TR>
__device__ __forceinline__ int transpose_row(int lane) {
  int i = 0, n = TR;
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) {
    if (n <= 1) break;
    n >>= 1;
    if (lane & m) i += n;
  }
  return i;
}

template <int TR>
constexpr int transpose_stages() { return TR >= 16 ? 4 : TR >= 8 ? 3 : TR >= 4 ? 2 : TR >= 2 ? 1 : 0; }

template <int TR, int RG, class Src, class Epi>
__global__ void __launch_bounds__(kGemvThreads, 1)
gemv_kernel(const GemvShape s, const typename Src::Params sp, const typename Epi::Params ep) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ float red[2][kNW * TR * RG];
  __shared__ float red_pro[kNW * kRmax];

  __shared__ int s_abort;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  unsigned char* stages = smem;
  bf16* xs = reinterpret_cast<bf16*>(smem + kStages * kStageBytes);
  const int stage_stride_row = s.cps * 16;  // bytes per tile row in a stage

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kNW);
    }
    fence_mbar_init();
  }
  pdl_wait();
  if (tid == 0) s_abort = status_bad(s.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();
  const int R = pass_rows(s);
  const int n_mats = s.mats ? *s.n_mats : 1;
  const int total = n_mats * s.tiles_per_mat;
  const int start = (int)(((long long)blockIdx.x * total) / gridDim.x);
  const int end = (int)(((long long)(blockIdx.x + 1) * total) / gridDim.x);
  const int ngroups_dense = (R + RG - 1) / RG;
  const int nch = s.K / 8;  // 16-byte chunks per row

  if (warp == kNW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int item = start; item < end && ok; ++item) {
        int m = item / s.tiles_per_mat, t = item - m * s.tiles_per_mat;
        const bf16* Wm;
        int e;
        mat_info(s, m, R, &Wm, &e, nullptr);
        int passes = s.ns == 1 ? 1 : ngroups_dense;
        for (int ps = 0; ps < passes && ok; ++ps) {
          for (int sl = 0; sl < s.ns && ok; ++sl, ++it) {
            int st = it % kStages;
            // a wait that gives up records OCRDEC_ETIMEOUT and proceeds: control flow
            // stays uniform so the block always terminates
            if (it >= kStages) mbar_wait(&empty_bar[st], ((it / kStages) & 1) ^ 1, s.status);
            int c0 = sl * s.cps;
            int cn = min(s.cps, nch - c0);
            uint32_t seg = cn * 16;
            mbar_arrive_expect_tx(&full_bar[st], seg * TR);
            unsigned char* dst = stages + st * kStageBytes;
            if (s.ns == 1 && s.pair_half == 0) {
              bulk_g2s(dst, Wm + (long long)t * TR * s.K, seg * TR, &full_bar[st]);
            } else if (s.ns == 1) {
              constexpr int H2 = TR / 2;
              bulk_g2s(dst, Wm + (long long)tile_row<TR>(s, t, 0) * s.K, seg * H2, &full_bar[st]);
              bulk_g2s(dst + H2 * stage_stride_row, Wm + (long long)tile_row<TR>(s, t, H2) * s.K, seg * H2,
                       &full_bar[st]);
            } else {
              for (int i = 0; i < TR; ++i)
                bulk_g2s(dst + i * stage_stride_row, Wm + (long long)tile_row<TR>(s, t, i) * s.K + c0 * 8, seg,
                         &full_bar[st]);
            }
          }
        }
      }
      // drain: every issued copy has landed before the block can exit
      for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait(&full_bar[j % kStages], (j / kStages) & 1, s.status);
    }
    return;
  }

  // ---------------- consumers ----------------
  epi_init<Epi>(tid);
  if (Src::kSmem) Src::prologue(sp, s.K, R, xs, red_pro, tid);
  else named_sync(1, kConsumers);

  uint32_t it = 0;
  int red_buf = 0;
  int cur_m = -1;
  RowSet rs;
  const bf16* Wm = nullptr;
  int expert = 0;
  bool ok = true;
  for (int item = start; item < end && ok; ++item) {
    int m = item / s.tiles_per_mat, t = item - m * s.tiles_per_mat;
    if (m != cur_m) {
      mat_info(s, m, R, &Wm, &expert, &rs);
      cur_m = m;
    }
    const int ngroups = (rs.n + RG - 1) / RG;
    const int passes = s.ns == 1 ? 1 : ngroups;
    for (int ps = 0; ps < passes && ok; ++ps) {
      const int g_lo = s.ns == 1 ? 0 : ps;
      const int g_hi = s.ns == 1 ? ngroups : ps + 1;
      float acc[TR][RG];
      for (int sl = 0; sl < s.ns; ++sl, ++it) {
        int st = it % kStages;
        mbar_wait(&full_bar[st], (it / kStages) & 1, s.status);
        const unsigned char* w_st = stages + st * kStageBytes;
        int c0 = sl * s.cps;
        int cn = min(s.cps, nch - c0);
        for (int g = g_lo; g < g_hi; ++g) {
          if (s.ns == 1 || sl == 0) {
#pragma unroll
            for (int i = 0; i < TR; ++i)
#pragma unroll
              for (int q = 0; q < RG; ++q) acc[i][q] = 0.f;
          }
          for (int c = tid; c < cn; c += kConsumers) {
            float xv[RG][8];
#pragma unroll
            for (int q = 0; q < RG; ++q) {
              int j = g * RG + q;
              if (j < rs.n) {
                uint4 u = Src::chunk(sp, xs, s.K, rs.r[j], rs.slot[j], c0 + c);
                unpack8(u, xv[q]);
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) xv[q][e] = 0.f;
              }
            }
#pragma unroll
            for (int i = 0; i < TR; ++i) {
              uint4 u = *reinterpret_cast<const uint4*>(w_st + i * stage_stride_row + c * 16);
              float wv[8];
              unpack8(u, wv);
#pragma unroll
              for (int e = 0; e < 8; ++e)
#pragma unroll
                for (int q = 0; q < RG; ++q) acc[i][q] = __fmaf_rn(wv[e], xv[q][e], acc[i][q]);
            }
          }
          if (sl == s.ns - 1) {
            // reduce: warp transpose-reduce per row of the group, then warps in order
            float* rb = red[red_buf];
#pragma unroll
            for (int q = 0; q < RG; ++q) {
              float v[TR];
#pragma unroll
              for (int i = 0; i < TR; ++i) v[i] = acc[i][q];
              warp_transpose_reduce<TR>(v, lane);
#pragma unroll
              for (int m2 = (32 >> transpose_stages<TR>()) / 2; m2 > 0; m2 >>= 1)
                v[0] = __fadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], m2));
              if ((lane & ((32 >> transpose_stages<TR>()) - 1)) == 0)
                rb[(warp * TR + transpose_row<TR>(lane)) * RG + q] = v[0];
            }
            named_sync(1, kConsumers);
            Epi::template apply<TR, RG>(ep, s, expert, t, rb, rs, g, tid);
            red_buf ^= 1;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
      }
    }
  }
  named_sync(1, kConsumers);
  Epi::finish(ep, s, R, tid);
}

}  // namespace ocrdec
