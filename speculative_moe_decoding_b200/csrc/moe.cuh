// The MoE FFN sub-layer of one decoder layer as one persistent kernel:
// routing, the shared and routed experts' gate/up and down projections, and
// the combine
//   x[r] += sum_s gate[r][s] * down_s(silu(gate_s(xn[r])) * up_s(xn[r]))   (routed, ascending id)
//         + sum_sh down_sh(silu(gate_sh(xn[r])) * up_sh(xn[r]))            (shared)
// with xn = RMSNorm(x) * g, softmax routing over all experts and top-k.
//
// Work items, in this order:
//   the shared experts' gate/up tiles (16 gate + 16 up rows), the routed
//   experts' gate/up tiles (the experts touched by the pass, ascending id),
//   then the down tiles (32 output rows) of the same matrices in the same
//   order.
// CTA c takes item c first, then claims items from a counter, each once the
// previous item's stages are requested: the TMA stream of some SMs runs slower
// than others from launch to launch, and claiming lets the fast ones take
// more.  The shared items do not depend on the routing: every CTA whose
// first item is one of them requests its weights before the dependency wait.
//
// Warp roles:
//   * the producer thread streams weight tiles (TMA, 4-D tensor maps,
//     128-byte swizzle, L2 evict-first, no multicast) into a ring of 16 KB
//     stages and never waits for anything but free stages and the routing
//     tables: the TMA unit's throughput per SM, not the ring depth, bounds
//     the stream, so the SM must keep issuing;
//   * the rows thread copies each down item's rows of the SwiGLU output h into
//     a row buffer once all gate/up tiles of its matrix are published (an
//     acquire on the matrix's counter); the producer hands it the CTA's down
//     items through a shared-memory queue;
//   * eight MMA warps route the pass first (softmax over all experts, top-k,
//     bucketing), then compute each tile (mma m16n8k16, bf16 weights times the
//     activations' bf16 high and low parts, fp32 accumulation) and post their
//     column-quarter partials to a small queue; they do no global round trips;
//   * the epilogue warp adds the quarter partials in order, applies SwiGLU /
//     stores and publishes each tile with a GPU-scope release; the last of
//     the matrices to finish an output tile (an acq_rel count per tile) adds
//     all the experts' outputs of that tile to the residual in a fixed order,
//     so no CTA waits for another's down tile.
// The residual's RMSNorm scale comes from the attention kernel's per-block
// sums of squares (the same ones the router logits use), so the prologue is
// one round of loads (router partials, residual rows).
//
// Reductions are fixed by the shapes alone (MMA k-steps, slices, quarters;
// the combine's slot order), never by the number of rows in the pass: the
// speculative path stays bit-identical to k = 0.
#pragma once

#include "gemv.cuh"

namespace ocrdec {

constexpr int kMoeMaxStages = 8;
constexpr int kMoeMaxTilesDn = 64;  // d / 32 for d <= 2048
constexpr int kTagMoe = 11;
// counter block of the MoE kernel (ints, zero between launches)
constexpr int kMoeCtrRead = 0;   // CTAs that have read the residual
constexpr int kMoeCtrExit = 1;   // CTAs done
constexpr int kMoeCtrClaim = 3;  // next item to claim (minus gridDim)
constexpr int kMoeCtrGu = 8;                                    // [kMaxShared + kMaxExperts] gate/up tiles published per matrix
constexpr int kMoeCtrDn = kMoeCtrGu + kMaxShared + kMaxExperts;  // [kMoeMaxTilesDn] matrices done per down tile
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

constexpr int kMoeThreads = kConsumers + 96;  // 8 MMA warps, the producer, epilogue and rows warps
constexpr int kMoeProducerWarp = kNW, kMoeEpilogueWarp = kNW + 1, kMoeRowsWarp = kNW + 2;
constexpr int kMoeRedSlots = 2;  // partial slots between the MMA warps and the epilogue warp
constexpr int kMoeQueue = 16;    // down items handed from the producer to the rows thread
constexpr int kMoeRedSlotFloats = 4 * kTile * 8;

__host__ __device__ constexpr size_t moe_xn_bytes(int d, int RG) { return (size_t)2 * RG * (d + 8) * 2; }
__host__ __device__ constexpr size_t moe_xb_bytes(int f, int RG) { return (size_t)2 * RG * (f + 8) * 2; }
// Dynamic shared memory: 1 KB alignment slack, the weight ring, the normalised
// rows, the down items' row buffer and the partial slots (which hold the
// routing's logits and scratch before the first item).  Small enough for two
// CTAs per SM at four stages and up to four rows: one SM's two CTAs stream
// faster than one CTA with twice the ring (each CTA consumes its stages in
// order, so the other covers its stalls).
__host__ __device__ constexpr size_t moe_smem_bytes(int d, int f, int RG, int nst) {
  return 1024 + (size_t)nst * kStageBytes + moe_xn_bytes(d, RG) + moe_xb_bytes(f, RG) +
         (size_t)kMoeRedSlots * kMoeRedSlotFloats * 4;
}
static_assert(kMoeRedSlots * kMoeRedSlotFloats * 4 >= kRmax * kMaxExperts * 4 + kRouteScratchBytes,
              "the routing's logits and scratch fit in the partial slots");

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

// GPU-scope release / acquire-release additions.  A warp publishes its stores
// with __syncwarp() and one lane's release addition (the barrier orders the
// other lanes' stores before it); a release addition returns nothing.
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_add(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Orders this thread's later async-proxy (TMA) reads of global memory after
// the generic-proxy writes it has acquired.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Item i of the pass: kind, matrix (shared experts are matrices 0..S-1, the
// touched routed experts follow), tile.  All gate/up tiles come first, then
// all down tiles; the first S * tiles_gu items (the shared experts' gate/up)
// do not depend on the routing, and n_mats only matters past them.
struct MoeItem {
  bool down;
  int m, t;
};

__device__ __forceinline__ MoeItem moe_item(const MoeParams& p, int n_mats, int i) {
  MoeItem it;
  const int n_gu = n_mats * p.tiles_gu;
  it.down = i >= n_gu;
  if (!it.down) {
    it.m = i / p.tiles_gu;
    it.t = i - it.m * p.tiles_gu;
  } else {
    i -= n_gu;
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

// Shared state of one CTA.
struct MoeShared {
  uint64_t full_bar[kMoeMaxStages], empty_bar[kMoeMaxStages];  // weight ring
  uint64_t x_full, x_empty;                                    // the down items' row buffer
  uint64_t red_full[kMoeRedSlots], red_empty[kMoeRedSlots];    // MMA warps -> epilogue warp
  uint64_t tab_bar;                                            // routing tables ready (MMA warps -> others)
  uint64_t xin_bar;                                            // the residual rows' copy landed
  int s_tag[kMoeMaxStages];            // per stage: item (first slice), -2 (other slices), -1 (end)
  int s_meta[kMoeMaxStages];           // per first stage: down << 31 | m << 16 | t
  int s_rs[kMoeMaxStages][kRmax + 1];  // the item's row set (n, entries), with its first slice
  int s_item[kMoeRedSlots];            // item meta of a partial slot (-1: no more items)
  int q_meta[kMoeQueue];               // down items for the rows thread, in claim order
  volatile int q_n;                    // entries pushed
  volatile int q_taken;                // entries the rows thread has taken
  volatile int q_done;                 // the producer claims no more
  int s_irs[kMoeRedSlots][kRmax + 1];
  RouteTables rt;
  int ids[kRmax * kMaxTopK];
  float gates[kRmax * kMaxTopK];
  float ss[kRmax * kRouteParts];
  int abort_flag;
};

// Item descriptors passed through shared memory (never -1: t < 2^16, m < 2^15).
__device__ __forceinline__ int moe_meta(const MoeItem& mi) {
  return (mi.down ? (int)0x80000000u : 0) | (mi.m << 16) | mi.t;
}
__device__ __forceinline__ MoeItem moe_unmeta(int v) {
  MoeItem mi;
  mi.down = v < 0;
  mi.m = (v >> 16) & 0x7fff;
  mi.t = v & 0xffff;
  return mi;
}

template <int RG>
__global__ void __launch_bounds__(kMoeThreads, RG <= 4 ? 2 : 1)
moe_kernel(const __grid_constant__ CUtensorMap tm_gu, const __grid_constant__ CUtensorMap tm_sgu,
           const __grid_constant__ CUtensorMap tm_dn, const __grid_constant__ CUtensorMap tm_sdn,
           const MoeParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(16) MoeShared sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nst = p.nst;
  unsigned char* stages = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char* xn = stages + (size_t)nst * kStageBytes;
  unsigned char* xb = xn + moe_xn_bytes(p.d, RG);
  float* red = reinterpret_cast<float*>(xb + moe_xb_bytes(p.f, RG));
  // routing scratch in the partial slots (free until the first item): logits
  // [kRmax][kMaxExperts], probabilities, selected slots
  float* lg = red;
  float (*rt_p)[kMaxExperts] = reinterpret_cast<float (*)[kMaxExperts]>(red + kRmax * kMaxExperts);
  unsigned char (*rt_slot)[kMaxExperts] =
      reinterpret_cast<unsigned char (*)[kMaxExperts]>(red + 2 * kRmax * kMaxExperts);
  const int nslot = p.top_k + p.S;
  const int n_shared_items = p.S * p.tiles_gu;  // the items that do not depend on the routing

  if (tid == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&sh.full_bar[i], 1);  // the weights' transaction bytes
      mbar_init(&sh.empty_bar[i], kNW);
    }
    mbar_init(&sh.x_full, 1);
    mbar_init(&sh.x_empty, kNW);
    for (int i = 0; i < kMoeRedSlots; ++i) {
      mbar_init(&sh.red_full[i], kNW);
      mbar_init(&sh.red_empty[i], 1);
    }
    mbar_init(&sh.tab_bar, 1);
    mbar_init(&sh.xin_bar, 1);
    sh.q_n = 0;
    sh.q_taken = 0;
    sh.q_done = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kMoeProducerWarp) {
    // ================= producer (one thread): weights and row copies =================
    if (lane != 0) return;
    // the four tensor maps' descriptors into the TMA unit's cache up front (the
    // items alternate between them)
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_gu)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_sgu)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_dn)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_sdn)) : "memory");
    const uint64_t wpol = l2_evict_first_policy();
    int st = 0;
    uint32_t ph = 0, it = 0;  // ring slot, its phase parity, stages issued
    int R = 0, n_mats = p.S;
    auto next_slot = [&]() {
      ++it;
      if (++st == nst) { st = 0; ph ^= 1u; }
    };
    // one stage: two 16-row weight boxes of one 256-column slice
    auto issue = [&](int item, const MoeItem& mi, int slc, bool first) {
      int coord;
      bool shm;
      RowSet rs;
      moe_mat(p, sh.rt, mi.m, R, &coord, &shm, first ? &rs : nullptr);
      const CUtensorMap* map = mi.down ? (shm ? &tm_sdn : &tm_dn) : (shm ? &tm_sgu : &tm_gu);
      int r0, r1;
      if (mi.down) { r0 = mi.t * kTile; r1 = r0 + kBoxRows; }
      else { r0 = mi.t * kBoxRows; r1 = r0 + p.f; }  // gate rows, then their up rows f below
      if (it >= (uint32_t)nst) mbar_wait(&sh.empty_bar[st], ph ^ 1u, p.status);
      sh.s_tag[st] = first ? item : -2;
      if (first) {
        sh.s_meta[st] = moe_meta(mi);
        sh.s_rs[st][0] = rs.n;
#pragma unroll
        for (int q = 0; q < kRmax; ++q) sh.s_rs[st][1 + q] = rs.e[q];
      }
      mbar_arrive_expect_tx(&sh.full_bar[st], kStageBytes);
      unsigned char* dst = stages + (size_t)st * kStageBytes;
      tma_load_box(dst, map, slc * (kSlice / kChunk), r0, coord, &sh.full_bar[st], wpol);
      tma_load_box(dst + kBoxBytes, map, slc * (kSlice / kChunk), r1, coord, &sh.full_bar[st], wpol);
      next_slot();
    };
    const int ns_gu = (p.d + kSlice - 1) / kSlice, ns_dn = (p.f + kSlice - 1) / kSlice;
    // a down item goes to the rows thread's queue first (its rows' copy can
    // then start while its weights are requested)
    auto issue_item = [&](int item, const MoeItem& mi) {
      const int ns = mi.down ? ns_dn : ns_gu;
      if (mi.down) {
        for (uint32_t w = 0; sh.q_n - sh.q_taken >= kMoeQueue && w < kSpinLimit; ++w) __nanosleep(64);
        sh.q_meta[sh.q_n % kMoeQueue] = moe_meta(mi);
        __threadfence_block();
        sh.q_n = sh.q_n + 1;
      }
      for (int s = 0; s < ns; ++s) issue(item, mi, s, s == 0);
    };
    // the first item, if it does not depend on the routing, before the
    // dependency wait (the pass's row count was written by the pass setup,
    // kernels earlier); a shared down item's rows after it
    const int first = blockIdx.x;
    const bool pre = first < n_shared_items;
    if (pre) {
      R = min(max(__ldcg(p.nrows), 0), RG);
      issue_item(first, moe_item(p, p.S, first));
    }
    pdl_wait();
    R = min(max(__ldcg(p.nrows), 0), RG);
    // a failed earlier launch: request nothing more
    const bool abort_p = status_bad(p.status);
    int total = -1;  // known once the routing is
    auto need_total = [&]() {
      if (total >= 0) return;
      total = n_shared_items;
      if (mbar_wait(&sh.tab_bar, 0, p.status)) {
        n_mats = sh.rt.n_mats;
        total = n_mats * (p.tiles_gu + p.tiles_dn);
      }
    };
    if (!abort_p) {
      // items: the first one (unless already issued), then claims.  The next
      // item is claimed once the current one's stages are all requested: the
      // ring still holds them while the claim returns, and a CTA never holds
      // an item it has not started when the items run out (the kernel ends
      // with the slowest CTA)
      if (!pre) {
        need_total();
        if (first < total) issue_item(first, moe_item(p, n_mats, first));
      }
      while (true) {
        const int cur = (int)gridDim.x + atomicAdd(p.ctr + kMoeCtrClaim, 1);
        if (cur >= n_shared_items) need_total();
        if (total >= 0 && cur >= total) break;
        issue_item(cur, moe_item(p, n_mats, cur));
      }
    }
    __threadfence_block();
    sh.q_done = 1;
    // end marker: a stage with no data
    if (it >= (uint32_t)nst) mbar_wait(&sh.empty_bar[st], ph ^ 1u, p.status);
    sh.s_tag[st] = -1;
    mbar_arrive(&sh.full_bar[st]);
    next_slot();
    // drain: every issued copy has landed before the thread exits
    {
      int s = st;
      uint32_t q = ph;
      for (uint32_t j = 0; j < it && j < (uint32_t)nst; ++j) {
        if (--s < 0) { s = nst - 1; q ^= 1u; }
        mbar_wait(&sh.full_bar[s], q, p.status);
      }
    }
    return;
  }

  if (warp == kMoeRowsWarp) {
    // ================= rows thread: the down items' activation rows =================
    // Takes the CTA's down items from the producer's queue, in claim order,
    // and copies each one's rows of h into the next row buffer once all
    // gate/up tiles of its matrix are published and the buffer's previous
    // item is done.
    if (lane != 0) return;
    pdl_wait();
    const int R = min(max(__ldcg(p.nrows), 0), RG);
    if (status_bad(p.status)) return;  // the MMA warps skip the items of a failed launch
    uint32_t xitems = 0;
    bool tables = false;
    for (int k = 0;; ++k) {
      // the next down item from the producer's queue, or the end
      uint32_t w = 0;
      while (sh.q_n <= k && !sh.q_done && w++ < kSpinLimit) __nanosleep(32);
      __threadfence_block();   // the entries pushed before the end flag are seen
      if (sh.q_n <= k) break;  // done (or the producer gave up)
      const MoeItem mi = moe_unmeta(sh.q_meta[k % kMoeQueue]);
      sh.q_taken = k + 1;
      if (mi.m >= p.S && !tables) tables = mbar_wait(&sh.tab_bar, 0, p.status);
      int coord;
      bool shm;
      RowSet rs;
      moe_mat(p, sh.rt, mi.m, R, &coord, &shm, &rs);
      const uint32_t xuse = xitems++;
      spin_geq(p.ctr + kMoeCtrGu + mi.m, p.tiles_gu, p.status);       // every gate/up tile of the matrix
      fence_proxy_async_global();  // the rows were written through the generic proxy
      if (xuse > 0) mbar_wait(&sh.x_empty, (xuse - 1) & 1, p.status);  // the previous down item is done
      const int nq = min(rs.n, RG);
      unsigned char* xdst = xb;
      mbar_arrive_expect_tx(&sh.x_full, (uint32_t)(2 * nq * p.f * 2));
#pragma unroll
      for (int q = 0; q < RG; ++q)
        if (q < nq) {
          const long long off = (long long)((rs.e[q] & 0xff) * nslot + (rs.e[q] >> 8)) * p.f;
          bulk_g2s(xdst + (size_t)q * (p.f + 8) * 2, p.h + off, p.f * 2, &sh.x_full);
          bulk_g2s(xdst + (size_t)(RG + q) * (p.f + 8) * 2, p.h_lo + off, p.f * 2, &sh.x_full);
        }
    }
    return;
  }

  if (warp == kMoeEpilogueWarp) {
    // ================= epilogue warp: every tile's epilogue =================
    TraceMarks tm;
    pdl_wait();
    if (lane == 0) tm.t0 = gtimer();
    const int R = min(max(__ldcg(p.nrows), 0), RG);
    int n_mats = -1;  // from the routing, needed at the first down tile
    for (int j = 0;; ++j) {
      const int slot = j % kMoeRedSlots;
      mbar_wait(&sh.red_full[slot], (j / kMoeRedSlots) & 1, p.status);
      const int meta = sh.s_item[slot];
      if (meta == -1) break;
      const MoeItem mi = moe_unmeta(meta);
      RowSet rs;
      rs.n = sh.s_irs[slot][0];
#pragma unroll
      for (int q = 0; q < kRmax; ++q) rs.e[q] = sh.s_irs[slot][1 + q];
      const float* rb = red + slot * kMoeRedSlotFloats;
      // each output adds its four column-quarter partials in quarter order
      auto qsum = [&](int row, int c0) {
        float4 a[4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) a[kq] = *reinterpret_cast<const float4*>(rb + (kq * kTile + row) * 8 + c0);
        float4 o;
        o.x = __fadd_rn(__fadd_rn(__fadd_rn(a[0].x, a[1].x), a[2].x), a[3].x);
        o.y = __fadd_rn(__fadd_rn(__fadd_rn(a[0].y, a[1].y), a[2].y), a[3].y);
        o.z = __fadd_rn(__fadd_rn(__fadd_rn(a[0].z, a[1].z), a[2].z), a[3].z);
        o.w = __fadd_rn(__fadd_rn(__fadd_rn(a[0].w, a[1].w), a[2].w), a[3].w);
        return o;
      };
      if (!mi.down) {
        // lane: feature (gate row) lane / 2 of the tile, row-set entries c0..c0+3
        const int fl = lane >> 1, c0 = (lane & 1) * 4;
        const float4 gt = qsum(fl, c0), up = qsum(kBoxRows + fl, c0);
        const float gv[4] = {gt.x, gt.y, gt.z, gt.w}, uv[4] = {up.x, up.y, up.z, up.w};
        const int n = mi.t * kBoxRows + fl;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int q = c0 + c;
          if (q < rs.n) {
            const float act = __fdiv_rn(gv[c], __fadd_rn(1.f, expf(-gv[c])));
            const float hv = __fmul_rn(act, uv[c]);
            const bf16 hi = f2bf(hv);
            const long long row = (long long)rs.r_sel(q) * nslot + rs.slot_sel(q);
            p.h[row * p.f + n] = hi;
            p.h_lo[row * p.f + n] = f2bf(__fsub_rn(hv, bf2f(hi)));
          }
        }
      } else {
        // lane: output row lane of the tile, all row-set entries
        const float4 v0 = qsum(lane, 0), v1 = qsum(lane, 4);
        const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const int n = mi.t * kTile + lane;
#pragma unroll
        for (int q = 0; q < kRmax; ++q)
          if (q < rs.n) {
            const long long row = (long long)rs.r_sel(q) * nslot + rs.slot_sel(q);
            p.y[row * p.d + n] = vv[q];
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.red_empty[slot]);  // the partials are read
      if (!mi.down) {
        if (lane == 0) red_release_add(p.ctr + kMoeCtrGu + mi.m, 1);  // publish the tile
        continue;
      }
      if (n_mats < 0) {
        mbar_wait(&sh.tab_bar, 0, p.status);
        n_mats = sh.rt.n_mats;
        if (lane == 0) tm.t1 = gtimer();
      }
      // publish the tile's outputs; the last of the matrices to finish this
      // output tile adds x[r][n] += sum gate * y (routed slots in order) +
      // sum y (shared).  Every CTA must have read x first (it normalises it).
      // All loads are issued together, this tile's own outputs included.
      int last = 0;
      if (lane == 0) {
        last = atom_acq_rel_add(p.ctr + kMoeCtrDn + mi.t, 1) == n_mats - 1;
        if (last) spin_geq(p.ctr + kMoeCtrRead, (int)gridDim.x, p.status);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      __syncwarp();
      if (!last) continue;
      // lane: column lane of rows k (k < RG); four rows x eight slots per
      // round of loads (one round for up to eight slots), the sum carried
      // across rounds in slot order
#pragma unroll
      for (int k0 = 0; k0 < RG; k0 += 4) {
        float t[4] = {0.f, 0.f, 0.f, 0.f}, xo[4];
        const int nn = mi.t * kTile + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = k0 + k;
          xo[k] = k0 + k < RG && r < R ? __ldcg(p.x + (size_t)r * p.d + nn) : 0.f;
        }
        for (int s0 = 0; s0 < nslot; s0 += 8) {
          float yv[4][8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = k0 + k;
            const bool ok = k0 + k < RG && r < R;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              yv[k][j] = ok && s0 + j < nslot ? __ldcg(p.y + ((size_t)r * nslot + s0 + j) * p.d + nn) : 0.f;
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = k0 + k;
            if (k0 + k >= RG || r >= R) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int sl = s0 + j;
              if (sl < p.top_k) t[k] = __fmaf_rn(sh.gates[r * p.top_k + sl], yv[k][j], t[k]);
              else if (sl < nslot) t[k] = __fadd_rn(t[k], yv[k][j]);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = k0 + k;
          if (k0 + k < RG && r < R) p.x[(size_t)r * p.d + nn] = __fadd_rn(xo[k], t[k]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      tm.t2 = gtimer();
      trace_end(p.status, kTagMoe, tm);
      // the last CTA to finish clears the counters for the next launch: every
      // signal and wait of this launch is behind it
      __threadfence();
      if (atomicAdd(p.ctr + kMoeCtrExit, 1) == (int)gridDim.x - 1) {
        __threadfence();
        for (int k = 0; k < kMoeCtrInts; ++k) p.ctr[k] = 0;
      }
    }
    return;
  }

  // ================= MMA warps =================
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
  if (tid == 0) sh.abort_flag = status_bad(p.status);
  const int R = min(max(__ldcg(p.nrows), 0), RG);
  const int E = p.E;
  // ---- one round of loads: the residual rows (bulk copies into the
  // normalised-row buffer, as float32, until they are normalised), router dot
  // products, sums of squares ----
  float* xin = reinterpret_cast<float*>(xn);  // [R][d] float32 (fits: 4 RG d <= 4 RG (d + 8))
  if (tid == 0) {
    mbar_arrive_expect_tx(&sh.xin_bar, (uint32_t)(R * p.d * 4));
    for (int r = 0; r < R; ++r) bulk_g2s(xin + (size_t)r * p.d, p.x + (size_t)r * p.d, p.d * 4, &sh.xin_bar);
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
    sh.ss[tid] = __ldcg(p.rpart + (size_t)tid * kRouteLd + kMaxExperts);  // row tid / 8, block tid % 8
  named_sync(1, kConsumers);
  // the RMSNorm scale of each row from the blocks' sums of squares (block order)
  float sc[RG];
#pragma unroll
  for (int r = 0; r < RG; ++r) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kRouteParts; ++k) ss = __fadd_rn(ss, r < R ? sh.ss[r * kRouteParts + k] : 0.f);
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
      lg[idx] = __fmul_rn(dot, s);
    }
  }
  named_sync(1, kConsumers);
  const bool abort_now = sh.abort_flag != 0;
  // ---- routing: softmax over all experts, top-k, bucketing (the producer
  // waits for the tables before its first routed item) ----
  if (!abort_now) {
    RouteParams rp{};
    rp.logits = lg;
    rp.s_p = rt_p;
    rp.s_slot = rt_slot;
    rp.E = E;
    rp.top_k = p.top_k;
    rp.S = p.S;
    rp.ids = sh.ids;
    rp.gates = sh.gates;
    rp.counts = sh.rt.counts;
    rp.offsets = sh.rt.offsets;
    rp.rowlist = sh.rt.rowlist;
    rp.mats = sh.rt.mats;
    rp.n_mats = &sh.rt.n_mats;
    route_rows(rp, R, tid, kConsumers, ConsumerBarrier{});
  } else if (tid == 0) {
    sh.rt.n_mats = p.S;
  }
  named_sync(1, kConsumers);
  if (tid == 0) {
    mbar_arrive(&sh.tab_bar);  // releases the tables to the producer, the rows thread and the epilogue warp
    if (blockIdx.x == 0 && p.touched && !abort_now) {
      atomicAdd(&p.touched[0], sh.rt.n_mats - p.S);
      atomicAdd(&p.touched[1], 1);
    }
  }
  // normalised rows as bfloat16 high / low parts (rows R..RG-1 zero), in
  // place of the float32 rows: every thread reads its values, then writes
  {
    mbar_wait(&sh.xin_bar, 0, p.status);
    float4 xv[RG][2];
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int mq = tid + j * kConsumers;
        xv[r][j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < R && mq < p.d / 4) xv[r][j] = reinterpret_cast<const float4*>(xin + (size_t)r * p.d)[mq];
      }
    named_sync(1, kConsumers);
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
  if (tid == 0) red_release_add(p.ctr + kMoeCtrRead, 1);  // x read: the combines may overwrite it
  if (!abort_now) pdl_trigger();

  // ---- the items: MMAs only; partials go to the epilogue warp ----
  const int g = warp & 1, kq = warp >> 1;
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const uint32_t a_off = (uint32_t)(g * kBoxBytes + kq * (kBoxRows * 128) + a_row * 128);
  const int a_sw = a_row & 7, a_hi = lane >> 4;
  const int ns_gu = (p.d + kSlice - 1) / kSlice, ns_dn = (p.f + kSlice - 1) / kSlice;
  const int nch_gu = p.d / kChunk, nch_dn = p.f / kChunk;
  int st = 0;
  uint32_t ph = 0;
  int j = 0, ndown = 0;
  RowSet rs;
  while (true) {
    mbar_wait(&sh.full_bar[st], ph, p.status);
    const int item = sh.s_tag[st];
    if (item < 0) {  // end marker
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty_bar[st]);
      break;
    }
    const int meta = sh.s_meta[st];
    const MoeItem mi = moe_unmeta(meta);
    rs.n = sh.s_rs[st][0];
#pragma unroll
    for (int q = 0; q < kRmax; ++q) rs.e[q] = sh.s_rs[st][1 + q];
    const int ns = mi.down ? ns_dn : ns_gu, nch = mi.down ? nch_dn : nch_gu;
    // four independent accumulators (even / odd k16 steps x high / low parts)
    // keep the tensor pipe busy: one warp's MMAs no longer form one chain
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    float dh0[4] = {0.f, 0.f, 0.f, 0.f}, dl0[4] = {0.f, 0.f, 0.f, 0.f};
    float dh1[4] = {0.f, 0.f, 0.f, 0.f}, dl1[4] = {0.f, 0.f, 0.f, 0.f};
    if (!abort_now) {
      // B operand rows: a gate/up item reads the normalised pass row of its
      // row-set entry; a down item the entry's copied row
      const int bq = (lane & 7) % RG;
      uint32_t b_base, b_lo;
      if (!mi.down) {
        b_base = smem_u32(xn) + (uint32_t)(rs.r_sel(bq) * (p.d + 8) + ((lane >> 3) & 1) * 8) * 2;
        b_lo = (uint32_t)(RG * (p.d + 8) * 2);
      } else {
        mbar_wait(&sh.x_full, ndown & 1, p.status);  // the item's rows are in
        b_base = smem_u32(xb) + (uint32_t)(bq * (p.f + 8) + ((lane >> 3) & 1) * 8) * 2;
        b_lo = (uint32_t)(RG * (p.f + 8) * 2);
      }
      b_base += (uint32_t)kq * kChunk * 2;
      for (int sl = 0; sl < ns; ++sl) {
        if (sl > 0) mbar_wait(&sh.full_bar[st], ph, p.status);
        if (sl * (kSlice / kChunk) + kq < nch) {
          const uint32_t a_base = smem_u32(stages + (size_t)st * kStageBytes) + a_off;
          const uint32_t b_addr = b_base + (uint32_t)sl * kSlice * 2;
#pragma unroll
          for (int k16 = 0; k16 < kChunk / 16; k16 += 2) {
            uint32_t a0[4], a1[4], bh0[2], bl0[2], bh1[2], bl1[2];
            ldsm_x4(a_base + (uint32_t)(((2 * k16 + a_hi) ^ a_sw) << 4), a0);
            ldsm_x4(a_base + (uint32_t)(((2 * (k16 + 1) + a_hi) ^ a_sw) << 4), a1);
            ldsm_x2(b_addr + k16 * 32, bh0);
            ldsm_x2(b_addr + b_lo + k16 * 32, bl0);
            ldsm_x2(b_addr + (k16 + 1) * 32, bh1);
            ldsm_x2(b_addr + b_lo + (k16 + 1) * 32, bl1);
            mma_bf16(dh0, a0, bh0);
            mma_bf16(dl0, a0, bl0);
            mma_bf16(dh1, a1, bh1);
            mma_bf16(dl1, a1, bl1);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty_bar[st]);
        if (++st == nst) { st = 0; ph ^= 1u; }
      }
      // the four accumulators in a fixed order
#pragma unroll
      for (int e = 0; e < 4; ++e) d[e] = __fadd_rn(__fadd_rn(dh0[e], dh1[e]), __fadd_rn(dl0[e], dl1[e]));
    } else {
      for (int sl = 0; sl < ns; ++sl) {  // aborting: consume the stages without computing
        if (sl > 0) mbar_wait(&sh.full_bar[st], ph, p.status);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty_bar[st]);
        if (++st == nst) { st = 0; ph ^= 1u; }
      }
    }
    if (mi.down) {
      if (lane == 0) mbar_arrive(&sh.x_empty);  // the item's rows are no longer read
      ++ndown;
    }
    if (abort_now) continue;  // nothing to post
    // this warp's quarter partials -> a free slot of the epilogue queue
    const int slot = j % kMoeRedSlots;
    if (j >= kMoeRedSlots) mbar_wait(&sh.red_empty[slot], ((j / kMoeRedSlots) - 1) & 1, p.status);
    float* rb = red + slot * kMoeRedSlotFloats;
    {
      const int r = g * kBoxRows + (lane >> 2), c = 2 * (lane & 3);
      *reinterpret_cast<float2*>(rb + (kq * kTile + r) * 8 + c) = make_float2(d[0], d[1]);
      *reinterpret_cast<float2*>(rb + (kq * kTile + r + 8) * 8 + c) = make_float2(d[2], d[3]);
    }
    if (warp == 0 && lane == 0) {
      sh.s_item[slot] = meta;
      sh.s_irs[slot][0] = rs.n;
#pragma unroll
      for (int q = 0; q < kRmax; ++q) sh.s_irs[slot][1 + q] = rs.e[q];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.red_full[slot]);
    ++j;
  }
  // no more items: an end entry for the epilogue warp
  {
    const int slot = j % kMoeRedSlots;
    if (j >= kMoeRedSlots) mbar_wait(&sh.red_empty[slot], ((j / kMoeRedSlots) - 1) & 1, p.status);
    if (warp == 0 && lane == 0) sh.s_item[slot] = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.red_full[slot]);
  }
}

}  // namespace ocrdec
