// The MoE FFN sub-layer of one decoder layer as one persistent kernel:
// routing, the shared and routed experts' gate/up and down projections, and
// the combine
//   x[r] += sum_s gate[r][s] * down_s(silu(gate_s(xn[r])) * up_s(xn[r]))   (routed, ascending id)
//         + sum_sh down_sh(silu(gate_sh(xn[r])) * up_sh(xn[r]))            (shared)
// with xn = RMSNorm(x) * g, softmax routing over all experts and top-k.
//
// Work items, claimed in this order (the first one of a CTA statically, the
// rest from a counter):
//   gate/up items (matrix m, 16 + 16 paired rows), m over the matrices to
//   stream - shared experts first, then the touched routed experts in
//   ascending id - then down items (matrix m, 32 output rows).
// Every CTA routes the pass itself (same inputs, same order: the same
// tables), so the only data that crosses CTAs is:
//   * SwiGLU outputs h of matrix m, written by its gate/up items; a down item
//     of m copies its rows (TMA bulk copy) only after all gate/up tiles of m
//     have signalled (per-matrix counter, bounded wait);
//   * expert outputs y of one 32-row output tile; the last of the matrices'
//     down items of that tile adds them, in a fixed order, to the residual.
// The weights of the shared experts' gate/up do not depend on the routing,
// so a CTA whose first item is one of them requests its stages before the
// dependency wait.  The residual's RMSNorm scale comes from the attention
// kernel's per-block sums of squares (the same ones the router logits use),
// so the whole prologue is one round of loads (router partials, residual
// rows) followed by on-chip work.
//
// Reductions are fixed by the shapes alone (MMA k-steps, slices, quarters;
// the combine's slot order), never by the number of rows in the pass: the
// speculative path stays bit-identical to k = 0.
#pragma once

#include "gemv.cuh"

namespace ocrdec {

constexpr int kMoeMaxStages = 8;
constexpr int kMoeMaxTilesDn = 64;                   // d / 32 for d <= 2048
constexpr int kTagMoe = 11;
// counter block of the MoE kernel (ints, zero between launches)
constexpr int kMoeCtrClaim = 0, kMoeCtrRead = 1, kMoeCtrExit = 2;
constexpr int kMoeCtrGu = 8;                                   // [kMaxShared + kMaxExperts]
constexpr int kMoeCtrDn = kMoeCtrGu + kMaxShared + kMaxExperts;  // [kMoeMaxTilesDn]
constexpr int kMoeCtrInts = kMoeCtrDn + kMoeMaxTilesDn;

struct MoeParams {
  int d, f;             // model width, expert (and shared) ffn width
  int E, S, top_k;
  int tiles_gu;         // f / 16 paired tiles (16 gate + 16 up rows) per gate/up matrix
  int tiles_dn;         // d / 32 output tiles per down matrix
  int nst;              // stages in the weight ring
  float eps;
  float* x;             // residual rows [R][d]: read at the start, += the FFN output per tile
  const int* nrows;     // rows of the pass
  const bf16* gain;     // FFN RMSNorm gains [d]
  const float* rpart;   // router partials [R][kRouteParts][kRouteLd] (dot products, sums of squares)
  bf16* h;              // SwiGLU outputs [R][nslot][f], high parts
  bf16* h_lo;           // low parts
  float* y;             // expert outputs [R][nslot][d]
  int* ctr;             // kMoeCtrInts counters, zero between launches
  int* touched;         // optional: [0] += routed experts touched, [1] += 1
  int* status;
};

__host__ __device__ constexpr size_t moe_xn_bytes(int d, int RG) { return (size_t)2 * RG * (d + 8) * 2; }
__host__ __device__ constexpr size_t moe_xb_bytes(int f, int RG) { return (size_t)2 * RG * (f + 8) * 2; }
__host__ __device__ constexpr size_t moe_smem_bytes(int d, int f, int RG, int nst) {
  return 1024 + (size_t)nst * kStageBytes + moe_xn_bytes(d, RG) + 2 * moe_xb_bytes(f, RG) + kRedFloats * 4;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Waits until *p >= target (another CTA's release).  Gives up - recording
// OCRDEC_ETIMEOUT - after about a second, and at once if the status word is
// already set (a failed launch leaves counters that never fill).
__device__ __forceinline__ bool spin_geq(const int* p, int target, int* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (ld_acquire(p) >= target) return true;
    if ((i & 255) == 255) {
      if (status_bad(status)) return false;
      __nanosleep(64);
    }
  }
  set_status(status, OCRDEC_ETIMEOUT);
  return false;
}

// Orders this thread's later async-proxy (TMA) reads of global memory after
// the generic-proxy writes it has acquired.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

struct MoeItem {
  bool down;
  int m, t;
};

__device__ __forceinline__ MoeItem moe_item(const MoeParams& p, int n_mats, int i) {
  MoeItem it;
  const int G = n_mats * p.tiles_gu;
  it.down = i >= G;
  if (!it.down) {
    it.m = i / p.tiles_gu;
    it.t = i - it.m * p.tiles_gu;
  } else {
    i -= G;
    it.m = i / p.tiles_dn;
    it.t = i - it.m * p.tiles_dn;
  }
  return it;
}

// Matrix m of the pass: tensor-map coordinate, shared or routed, and its rows.
__device__ __forceinline__ void moe_mat(const MoeParams& p, const RouteTables& rt, int m, int R, int* coord,
                                        bool* shared, RowSet* rs) {
  const int e = m < p.S ? p.E + m : rt.mats[m];
  if (e < p.E) {
    *coord = e;
    *shared = false;
    if (rs) {
      const int n = min(rt.counts[e], kRmax), off = rt.offsets[e];
      rs->n = n;
#pragma unroll
      for (int i = 0; i < kRmax; ++i) rs->e[i] = i < n ? rt.rowlist[off + i] : 0;
    }
  } else {
    const int sh = e - p.E;
    *coord = sh;
    *shared = true;
    if (rs) {
      rs->n = R;
#pragma unroll
      for (int i = 0; i < kRmax; ++i) rs->e[i] = i | ((p.top_k + sh) << 8);
    }
  }
}

// The consumer warps' item loop of moe_kernel.
template <int RG>
__device__ __forceinline__ void moe_items(const MoeParams& p, unsigned char* stages, unsigned char* xn,
                                          unsigned char* xb, float* red, const int* s_tag,
                                          const int (*s_rs)[kRmax + 1], uint64_t* full_bar, uint64_t* empty_bar,
                                          uint64_t* x_empty, int n_mats, const float* s_gates, int R, int tid,
                                          int* s_last) {
  const int warp = tid >> 5, lane = tid & 31;
  const int nst = p.nst, nslot = p.top_k + p.S;
  // ---- the items ----
  const int g = warp & 1, kq = warp >> 1;
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const uint32_t a_off = (uint32_t)(g * kBoxBytes + kq * (kBoxRows * 128) + a_row * 128);
  const int a_sw = a_row & 7, a_hi = lane >> 4;
  const int ep_i = lane >> 3, ep_q = lane & 7;
  const int ns_gu = (p.d + kSlice - 1) / kSlice, ns_dn = (p.f + kSlice - 1) / kSlice;
  const int nch_gu = p.d / kChunk, nch_dn = p.f / kChunk;
  int st = 0;
  uint32_t ph = 0;
  int nitem = 0, ndown = 0;
  RowSet rs;
  while (true) {
    mbar_wait(&full_bar[st], ph, p.status);
    const int item = s_tag[st];
    if (item < 0) {  // end marker
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
      break;
    }
    const MoeItem mi = moe_item(p, n_mats, item);
    rs.n = s_rs[st][0];
#pragma unroll
    for (int q = 0; q < kRmax; ++q) rs.e[q] = s_rs[st][1 + q];
    const int bq = (lane & 7) % RG;
    const int ns = mi.down ? ns_dn : ns_gu, nch = mi.down ? nch_dn : nch_gu;
    const int xbuf = ndown & 1;
    // B operand rows: a gate/up item reads the normalised pass row of its
    // row-set entry; a down item the entry's copied row
    uint32_t b_base, b_lo;
    if (!mi.down) {
      b_base = smem_u32(xn) + (uint32_t)(rs.r_sel(bq) * (p.d + 8) + ((lane >> 3) & 1) * 8) * 2;
      b_lo = (uint32_t)(RG * (p.d + 8) * 2);
    } else {
      b_base = smem_u32(xb + (size_t)xbuf * moe_xb_bytes(p.f, RG)) + (uint32_t)(bq * (p.f + 8) + ((lane >> 3) & 1) * 8) * 2;
      b_lo = (uint32_t)(RG * (p.f + 8) * 2);
    }
    b_base += (uint32_t)kq * kChunk * 2;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sl = 0; sl < ns; ++sl) {
      if (sl > 0) mbar_wait(&full_bar[st], ph, p.status);
      if (sl * (kSlice / kChunk) + kq < nch) {
        const uint32_t a_base = smem_u32(stages + (size_t)st * kStageBytes) + a_off;
        const uint32_t b_addr = b_base + (uint32_t)sl * kSlice * 2;
#pragma unroll
        for (int k16 = 0; k16 < kChunk / 16; ++k16) {
          uint32_t a[4], bh[2], bl[2];
          ldsm_x4(a_base + (uint32_t)(((2 * k16 + a_hi) ^ a_sw) << 4), a);
          ldsm_x2(b_addr + k16 * 32, bh);
          ldsm_x2(b_addr + b_lo + k16 * 32, bl);
          mma_bf16(d, a, bh);
          mma_bf16(d, a, bl);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
      if (++st == nst) { st = 0; ph ^= 1u; }
    }
    if (mi.down) {
      if (lane == 0) mbar_arrive(&x_empty[xbuf]);  // the item's rows are no longer read
      ++ndown;
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
    const int srow = stage_row(!mi.down, warp, ep_i);
    const float v = __fadd_rn(__fadd_rn(__fadd_rn(rb[(0 * kTile + srow) * 8 + ep_q], rb[(1 * kTile + srow) * 8 + ep_q]),
                                        rb[(2 * kTile + srow) * 8 + ep_q]),
                              rb[(3 * kTile + srow) * 8 + ep_q]);
    if (!mi.down) {
      // SwiGLU: lanes of local rows 0, 1 hold gate rows, rows 2, 3 their up rows
      const float up = __shfl_down_sync(0xffffffffu, v, 16);
      if (ep_i < 2 && ep_q < rs.n) {
        const int n = mi.t * kBoxRows + srow;  // feature (gate row) index
        const float act = __fdiv_rn(v, __fadd_rn(1.f, expf(-v)));
        const float hv = __fmul_rn(act, up);
        const bf16 hi = f2bf(hv);
        const long long row = (long long)rs.r_sel(ep_q) * nslot + rs.slot_sel(ep_q);
        p.h[row * p.f + n] = hi;
        p.h_lo[row * p.f + n] = f2bf(__fsub_rn(hv, bf2f(hi)));
        __threadfence();
      }
      named_sync(1, kConsumers);
      if (tid == 0) atomicAdd(p.ctr + kMoeCtrGu + mi.m, 1);  // after every thread's fence: release
    } else {
      const int n = mi.t * kTile + srow;  // the tile's 32 consecutive output rows
      if (ep_q < rs.n && n < p.d) {
        const long long row = (long long)rs.r_sel(ep_q) * nslot + rs.slot_sel(ep_q);
        p.y[row * p.d + n] = v;
        __threadfence();
      }
      named_sync(1, kConsumers);
      if (tid == 0) *s_last = atomicAdd(p.ctr + kMoeCtrDn + mi.t, 1) == n_mats - 1;
      named_sync(1, kConsumers);
      if (*s_last) {
        // the tile's last matrix: every expert output of its rows is in.
        // x[r][n] += sum gate * y (routed slots in order) + sum y (shared)
        if (tid == 0) spin_geq(p.ctr + kMoeCtrRead, (int)gridDim.x, p.status);  // all CTAs read x
        named_sync(1, kConsumers);
        __threadfence();
        for (int idx = tid; idx < R * kTile; idx += kConsumers) {
          const int r = idx / kTile, nn = mi.t * kTile + (idx - r * kTile);
          if (nn >= p.d) continue;
          constexpr int kSlots = kMaxTopK + kMaxShared;
          float yv[kSlots];
#pragma unroll
          for (int s = 0; s < kSlots; ++s) yv[s] = s < nslot ? __ldcg(p.y + ((size_t)r * nslot + s) * p.d + nn) : 0.f;
          const float xo = __ldcg(p.x + (size_t)r * p.d + nn);
          float t = 0.f;
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
            if (s < p.top_k) t = __fmaf_rn(s_gates[r * p.top_k + (s < kMaxTopK ? s : 0)], yv[s], t);
            else if (s < nslot) t = __fadd_rn(t, yv[s]);
          }
          p.x[(size_t)r * p.d + nn] = __fadd_rn(xo, t);
        }
      }
    }
  }
}


template <int RG>
__global__ void __launch_bounds__(kGemvThreads, 1)
moe_kernel(const __grid_constant__ CUtensorMap tm_gu, const __grid_constant__ CUtensorMap tm_sgu,
           const __grid_constant__ CUtensorMap tm_dn, const __grid_constant__ CUtensorMap tm_sdn,
           const MoeParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kMoeMaxStages], empty_bar[kMoeMaxStages], x_empty[2], tab_bar;
  __shared__ int s_tag[kMoeMaxStages];            // item of the stage's first slice, -2 other slices, -1 end
  __shared__ int s_rs[kMoeMaxStages][kRmax + 1];  // the item's row set (n, entries), with its first slice
  __shared__ RouteTables s_rt;
  __shared__ float s_lg[kRmax * kMaxExperts];
  __shared__ int s_ids[kRmax * kMaxTopK];
  __shared__ float s_gates[kRmax * kMaxTopK];
  __shared__ float s_ss[kRmax * kRouteParts];
  __shared__ int s_abort, s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nst = p.nst;
  unsigned char* stages = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char* xn = stages + (size_t)nst * kStageBytes;
  unsigned char* xb = xn + moe_xn_bytes(p.d, RG);
  float* red = reinterpret_cast<float*>(xb + 2 * moe_xb_bytes(p.f, RG));
  const int nslot = p.top_k + p.S;

  if (tid == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full_bar[i], 2);  // weights (transaction bytes) + activations (copy or plain arrival)
      mbar_init(&empty_bar[i], kNW);
    }
    mbar_init(&x_empty[0], kNW);
    mbar_init(&x_empty[1], kNW);
    mbar_init(&tab_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kNW) {
    // ================= producer (one thread) =================
    if (lane != 0) return;
    const uint64_t wpol = l2_evict_first_policy();
    int st = 0;
    uint32_t ph = 0, it = 0;   // ring slot, its phase parity, stages issued
    uint32_t xitems = 0;        // down items whose rows were copied
    int R = 0, n_mats = 0;
    auto next_slot = [&]() {
      ++it;
      if (++st == nst) { st = 0; ph ^= 1u; }
    };
    // one stage: two 16-row weight boxes of one 256-column slice, then the
    // activations' arrival (a down item's first stage: the rows' bulk copy)
    auto issue = [&](int item, const MoeItem& mi, int slc, bool first) {
      int coord;
      bool sh;
      RowSet rs;
      moe_mat(p, s_rt, mi.m, R, &coord, &sh, first ? &rs : nullptr);
      const CUtensorMap* map = mi.down ? (sh ? &tm_sdn : &tm_dn) : (sh ? &tm_sgu : &tm_gu);
      int r0, r1;
      if (mi.down) { r0 = mi.t * kTile; r1 = r0 + kBoxRows; }
      else { r0 = mi.t * kBoxRows; r1 = r0 + p.f; }  // gate rows, then their up rows f below
      if (it >= (uint32_t)nst) mbar_wait(&empty_bar[st], ph ^ 1u, p.status);
      s_tag[st] = first ? item : -2;
      if (first) {
        s_rs[st][0] = rs.n;
#pragma unroll
        for (int q = 0; q < kRmax; ++q) s_rs[st][1 + q] = rs.e[q];
      }
      mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
      unsigned char* dst = stages + (size_t)st * kStageBytes;
      tma_load_box(dst, map, slc * (kSlice / kChunk), r0, coord, &full_bar[st], wpol);
      tma_load_box(dst + kBoxBytes, map, slc * (kSlice / kChunk), r1, coord, &full_bar[st], wpol);
      if (!(mi.down && first)) {
        mbar_arrive(&full_bar[st]);
      } else {
        // the item's rows of h: wait until every gate/up tile of the matrix is in
        const int xbuf = xitems & 1;
        const uint32_t use = xitems >> 1;
        ++xitems;
        spin_geq(p.ctr + kMoeCtrGu + mi.m, p.tiles_gu, p.status);
        fence_proxy_async_global();
        if (use > 0) mbar_wait(&x_empty[xbuf], (use - 1) & 1, p.status);
        const int nq = min(rs.n, RG);
        unsigned char* xdst = xb + (size_t)xbuf * moe_xb_bytes(p.f, RG);
        mbar_arrive_expect_tx(&full_bar[st], (uint32_t)(2 * nq * p.f * 2));
#pragma unroll
        for (int q = 0; q < RG; ++q)
          if (q < nq) {
            const long long off = (long long)((rs.e[q] & 0xff) * nslot + (rs.e[q] >> 8)) * p.f;
            bulk_g2s(xdst + (size_t)q * (p.f + 8) * 2, p.h + off, p.f * 2, &full_bar[st]);
            bulk_g2s(xdst + (size_t)(RG + q) * (p.f + 8) * 2, p.h_lo + off, p.f * 2, &full_bar[st]);
          }
      }
      next_slot();
    };
    const int ns_gu = (p.d + kSlice - 1) / kSlice, ns_dn = (p.f + kSlice - 1) / kSlice;
    auto issue_item = [&](int item) {
      const MoeItem mi = moe_item(p, n_mats, item);
      const int ns = mi.down ? ns_dn : ns_gu;
      for (int s = 0; s < ns; ++s) issue(item, mi, s, s == 0);
    };
    // the shared experts' gate/up weights do not depend on the routing: a CTA
    // whose first item is one of them requests it before the dependency wait
    // (the pass's row count was written by the pass setup, kernels earlier)
    const int first = blockIdx.x;
    bool pre = false;
    if (first < p.S * p.tiles_gu) {
      R = min(max(__ldcg(p.nrows), 0), RG);
      n_mats = p.S;  // enough to name the item: shared matrices come first
      issue_item(first);
      pre = true;
    }
    pdl_wait();
    // the tables (and so the item count) once the consumers have routed the pass
    int total = 0;
    if (mbar_wait(&tab_bar, 0, p.status)) {
      R = min(max(__ldcg(p.nrows), 0), RG);
      n_mats = s_rt.n_mats;
      total = n_mats * (p.tiles_gu + p.tiles_dn);
    }
    if (!pre && first < total) issue_item(first);
    while (true) {
      const int item = (int)gridDim.x + atomicAdd(p.ctr + kMoeCtrClaim, 1);
      if (item >= total) break;
      issue_item(item);
    }
    // end marker: a stage with no data
    if (it >= (uint32_t)nst) mbar_wait(&empty_bar[st], ph ^ 1u, p.status);
    s_tag[st] = -1;
    mbar_arrive(&full_bar[st]);
    mbar_arrive(&full_bar[st]);
    next_slot();
    // drain: every issued copy has landed before the thread exits
    {
      int s = st;
      uint32_t q = ph;
      for (uint32_t j = 0; j < it && j < (uint32_t)nst; ++j) {
        if (--s < 0) { s = nst - 1; q ^= 1u; }
        mbar_wait(&full_bar[s], q, p.status);
      }
    }
    return;
  }

  // ================= consumers (8 warps) =================
  TraceMarks tm;
  // gains are weights: before the dependency wait
  float4 gv[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int mq = tid + j * kConsumers;
    gv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mq < p.d / 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p.gain + 4 * mq);
      gv[j] = make_float4(bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y));
    }
  }
  pdl_wait();
  if (tid == 0) {
    tm.t0 = gtimer();
    s_abort = status_bad(p.status);
  }
  const int R = min(max(__ldcg(p.nrows), 0), RG);
  const int E = p.E;
  // ---- one round of loads: residual rows, router dot products, sums of squares ----
  float4 xv[RG][2];
#pragma unroll
  for (int r = 0; r < RG; ++r)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int mq = tid + j * kConsumers;
      xv[r][j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < R && mq < p.d / 4) xv[r][j] = __ldcg(reinterpret_cast<const float4*>(p.x + (size_t)r * p.d) + mq);
    }
  constexpr int kLgPer = kRmax * kMaxExperts / kConsumers;  // logits per thread (2)
  float dk[kLgPer][kRouteParts];
#pragma unroll
  for (int i = 0; i < kLgPer; ++i) {
    const int idx = tid + i * kConsumers;
    const int r = idx / max(E, 1), e = idx - r * E;
#pragma unroll
    for (int k = 0; k < kRouteParts; ++k)
      dk[i][k] = idx < R * E ? __ldcg(p.rpart + ((size_t)r * kRouteParts + k) * kRouteLd + e) : 0.f;
  }
  if (tid < R * kRouteParts)
    s_ss[tid] = __ldcg(p.rpart + (size_t)tid * kRouteLd + kMaxExperts);  // row tid / 8, block tid % 8
  named_sync(1, kConsumers);
  // the RMSNorm scale of each row from the blocks' sums of squares (block order)
  float sc[RG];
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kRouteParts; ++k) ss = __fadd_rn(ss, r < R ? s_ss[r * kRouteParts + k] : 0.f);
    sc[r] = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)p.d), p.eps));
  }
  // router logits: block-ordered dot products times the row's scale
#pragma unroll
  for (int i = 0; i < kLgPer; ++i) {
    const int idx = tid + i * kConsumers;
    if (idx < R * E) {
      const int r = idx / E;
      float dot = 0.f;
#pragma unroll
      for (int k = 0; k < kRouteParts; ++k) dot = __fadd_rn(dot, dk[i][k]);
      float s = sc[0];
#pragma unroll
      for (int q = 1; q < RG; ++q) s = r == q ? sc[q] : s;
      s_lg[idx] = __fmul_rn(dot, s);
    }
  }
  // normalised rows as bfloat16 high / low parts (rows R..RG-1 zero)
  {
    bf16* xh = reinterpret_cast<bf16*>(xn);
    bf16* xl = xh + RG * (p.d + 8);
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int mq = tid + j * kConsumers;
        if (mq < p.d / 4) {
          const float4 v = xv[r][j];
          const float4 g = gv[j];
          uint2 hi, lo;
          split_bf16x4(__fmul_rn(__fmul_rn(v.x, sc[r]), g.x), __fmul_rn(__fmul_rn(v.y, sc[r]), g.y),
                       __fmul_rn(__fmul_rn(v.z, sc[r]), g.z), __fmul_rn(__fmul_rn(v.w, sc[r]), g.w), hi, lo);
          if (r >= R) hi = lo = make_uint2(0u, 0u);
          *reinterpret_cast<uint2*>(xh + r * (p.d + 8) + 4 * mq) = hi;
          *reinterpret_cast<uint2*>(xl + r * (p.d + 8) + 4 * mq) = lo;
        }
      }
  }
  named_sync(1, kConsumers);
  if (tid == 0) {
    // this CTA has read the residual: the combines may now overwrite it
    __threadfence();
    atomicAdd(p.ctr + kMoeCtrRead, 1);
  }
  // ---- routing: softmax over all experts, top-k, bucketing ----
  if (!s_abort) {
    RouteParams rp{};
    rp.logits = s_lg;
    rp.E = E;
    rp.top_k = p.top_k;
    rp.S = p.S;
    rp.ids = s_ids;
    rp.gates = s_gates;
    rp.counts = s_rt.counts;
    rp.offsets = s_rt.offsets;
    rp.rowlist = s_rt.rowlist;
    rp.mats = s_rt.mats;
    rp.n_mats = &s_rt.n_mats;
    route_rows(rp, R, tid, kConsumers, ConsumerBarrier{});
  } else if (tid == 0) {
    s_rt.n_mats = 0;
  }
  named_sync(1, kConsumers);
  if (tid == 0) {
    mbar_arrive(&tab_bar);  // releases the tables to the producer
    if (blockIdx.x == 0 && p.touched && !s_abort) {
      atomicAdd(&p.touched[0], s_rt.n_mats - p.S);
      atomicAdd(&p.touched[1], 1);
    }
    tm.t1 = gtimer();
  }
  if (s_abort) {
    // consume the producer's stages (a prefetched item, the end marker) so it can finish
    int st = 0;
    uint32_t ph = 0;
    while (true) {
      mbar_wait(&full_bar[st], ph, p.status);
      const int tag = s_tag[st];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
      if (++st == nst) { st = 0; ph ^= 1u; }
      if (tag == -1) break;
    }
  } else {
    pdl_trigger();
    moe_items<RG>(p, stages, xn, xb, red, s_tag, s_rs, full_bar, empty_bar, x_empty, s_rt.n_mats, s_gates, R,
                  tid, &s_last);
  }
  named_sync(1, kConsumers);
  if (tid == 0) {
    tm.t2 = gtimer();
    trace_end(p.status, kTagMoe, tm);
    // the last CTA to finish clears the counters for the next launch (every
    // claim, signal and wait of this launch is behind it)
    __threadfence();
    if (atomicAdd(p.ctr + kMoeCtrExit, 1) == (int)gridDim.x - 1) {
      __threadfence();
      for (int i = 0; i < kMoeCtrInts; ++i) p.ctr[i] = 0;
    }
  }
}

}  // namespace ocrdec
