// The attention block of one layer for the pass rows, split over a
// thread-block cluster per (slot, head), with every contraction on the tensor
// cores: RMSNorm -> QKV projection -> RoPE -> causal attention over the slot's
// KV cache -> output projection -> residual add (-> router partials).
//
// QKV projection.  CTA k of the cluster of head h holds 3 * Dh/8 rows of
// W_qkv: for each of q, k, v, the head's dims k*Dh/16 + j and their rotation
// partners Dh/2 + k*Dh/16 + j (j < Dh/16; RoPE rotates dim i with dim
// i + Dh/2), copied into shared memory before the dependency wait.  Each warp
// loads its eighth of the reduction width of the pass rows straight into MMA
// B fragments, the rows' RMSNorm scale comes from the warps' sums of squares,
// and the scaled rows (bfloat16 high and low parts) multiply the W_qkv rows;
// the warps' partial sums are added in warp order.  Rotated q goes to every
// CTA of the cluster through distributed shared memory; the new K and V rows
// go to the cache and, the same way, to every CTA.
//
// Attention.  For pass row r (position pos_r) and head h:
//   out[r][h] = softmax_j(q_r . k_j / sqrt(Dh)) v_j over positions j = 0..pos_r.
// The position axis is cut into fixed kAttnChunk-position chunks; CTA k takes
// chunks k, k + kAttnSplit, ... in increasing order, kAttnBufs at a time (a
// group; two buffers are the kernel's own, the third reuses the space the
// W_qkv rows held):
//   * TMA brings each chunk's K and V rows into shared memory (5-D tensor map
//     over the cache, 128-byte swizzle, no multicast); the pass's own rows are
//     then written over their positions from the broadcast K and V rows, so
//     every chunk can be requested before the dependency wait;
//   * scores S[j][r] = K[j] . q_r as m16n8k16 MMAs (positions x rows, the up
//     to 8 pass rows are the 8 MMA columns); q is split into bfloat16 high and
//     low parts, so the products carry float32-level precision;
//   * an online softmax per row (running max M, sum L) over the group;
//   * O[d][r] += V[j][d] P[r][j] as MMAs on V transposed (ldmatrix .trans),
//     P again split into bfloat16 high and low parts; each warp owns 16 dims.
// Each CTA then stores its (M, L) and the O of dims [k, k+1) * Dh/kAttnSplit
// into CTA k (distributed shared memory); CTA k merges the eight states of its
// dims in rank order and stores them (bf16 high and low parts) into the head
// output of every CTA of the cluster.
//
// Output projection.  CTA k multiplies the head's output by its block of W_o
// (rows [k, k+1) * d/kAttnSplit, the head's Dh columns; brought by TMA into
// the space the W_qkv rows held) and writes the partial sums per head; the
// last of the H heads to finish a row block adds the partials in head order
// to the residual stream.  In MoE layers that last arriver also writes the
// block's router partials (route.cuh): the dot products of its columns of W_r
// with g * x (g the FFN RMSNorm gains, x the new residual, as bf16 high and
// low parts, on the tensor cores) and the block's sum of squares of x; the MoE
// kernel finishes the router logits from them.
//
// Which CTA takes a chunk and the order of every sum depend only on the model
// width and positions (an MMA column depends on its own row's data only;
// positions a row does not see carry p = 0 exactly), so a row's result does
// not depend on the other rows of the pass.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "route.cuh"

namespace ocrdec {

constexpr int kAttnChunk = 64;
constexpr int kAttnSplit = 8;    // CTAs per (slot, head): one cluster
constexpr int kAttnBufs = 3;     // K/V chunks per group
constexpr int kAttnRingBufs = 2; // of them in the dedicated ring; the third in region B once the W_qkv rows are read
constexpr int kTagAttention = 40;
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kAttnRows = 8;     // rows of one slot in a pass (MMA columns)
constexpr int kAttnMaxDh = 128;
constexpr int kAttnMaxHeads = 16;  // heads summed by the fused output projection
constexpr int kAttnMaxD = 1280;    // model width: the CTA's W_qkv rows stay in shared memory
constexpr int kAttnMaxKs = kAttnMaxD / 16 / kAttnWarps;  // k16 steps of the QKV projection per warp
constexpr int kAttnQTiles = 3;   // 16-row MMA tiles of a CTA's W_qkv rows (Dh 128: 3, Dh 64: 2)
constexpr int kAttnQLd = kAttnMaxDh + 8;                // bf16 q row (+16 B: conflict-free ldmatrix)
constexpr int kAttnPLd = kAttnBufs * kAttnChunk + 8;    // bf16 P row
constexpr int kAttnChunkBytes = kAttnChunk * kAttnMaxDh * 2;  // K (or V) of one chunk: [half][pos][128 B]
static_assert(kAttnSplit == kRouteParts, "router partials: one per attention row block");

// Dynamic shared memory: 1 KB alignment slack (the 128-byte swizzle repeats
// every 1 KB), two K/V chunk buffers, region B, and the router block.  Region
// B first holds the CTA's W_qkv rows (16-row tiles, rows padded by 16 bytes),
// then the W_o block (d / kAttnSplit rows x Dh, swizzled), the scores, P,
// either the QKV projection's per-warp partial sums or (later) the merge's
// receive buffer, and the third K/V chunk buffer.
constexpr int attn_qkv_tiles(int Dh) { return (3 * (Dh / 16) + 7) / 8; }
constexpr size_t attn_qkv_bytes(int d, int Dh) { return (size_t)attn_qkv_tiles(Dh) * 16 * (d + 8) * 2; }
constexpr size_t attn_sc_bytes() { return (size_t)kAttnRows * kAttnBufs * kAttnChunk * 4; }
constexpr size_t attn_p_bytes() { return (size_t)2 * kAttnRows * kAttnPLd * 2; }
constexpr size_t attn_red_bytes() { return (size_t)kAttnWarps * kAttnQTiles * 32 * 4 * 4; }
constexpr size_t attn_wo_bytes(int d, int Dh) { return (size_t)(d / kAttnSplit) * Dh * 2; }
// the merge's receive buffer: every CTA's (M, L) of every row and O of the
// receiving CTA's Dh / kAttnSplit dims
constexpr size_t attn_recv_bytes(int Dh) { return (size_t)kAttnSplit * kAttnRows * (2 + Dh / kAttnSplit) * 4; }
constexpr size_t attn_tail_bytes(int Dh) {
  return attn_red_bytes() > attn_recv_bytes(Dh) ? attn_red_bytes() : attn_recv_bytes(Dh);
}
// offset in region B of the third K/V chunk buffer (1 KB aligned: the swizzle)
constexpr size_t attn_buf2_off(int d, int Dh) {
  return (attn_wo_bytes(d, Dh) + attn_sc_bytes() + attn_p_bytes() + attn_tail_bytes(Dh) + 1023) / 1024 * 1024;
}
constexpr size_t attn_regionb_bytes(int d, int Dh) {
  return attn_qkv_bytes(d, Dh) > attn_buf2_off(d, Dh) + 2 * kAttnChunkBytes ? attn_qkv_bytes(d, Dh)
                                                                           : attn_buf2_off(d, Dh) + 2 * kAttnChunkBytes;
}

// Router block of a CTA (MoE layers): W_r rows (E rounded up to 16, zero
// padded) x the CTA's d / kAttnSplit columns, rows padded by 16 bytes, then the
// FFN RMSNorm gains of those columns.
constexpr size_t attn_router_bytes(int d, int E) {
  return E > 0 ? ((size_t)(E + 15) / 16 * 16 * (d / kAttnSplit + 8) + d / kAttnSplit) * 2 : 0;
}

constexpr size_t attn_smem_bytes(int d, int Dh, int E) {
  return 1024 + (size_t)kAttnRingBufs * 2 * kAttnChunkBytes + attn_regionb_bytes(d, Dh) + attn_router_bytes(d, E);
}

struct AttnParams {
  int layer;               // cache layer index (map coordinate slot * n_layers + layer)
  int n_layers;            // layers in the cache (1 for the draft cache)
  int cap, H, Dh;          // Dh 64 or 128
  float scale;             // 1/sqrt(Dh)
  const int* slot_row0;    // [B] first pass row of each slot
  const int* slot_nrows;   // [B] rows of each slot in this pass
  const int* row_pos;      // [R]
  int rows_pre_wait;       // 1: the pass rows were written two or more kernels back (read before the wait)
  float* x;                // residual rows [R][d] (+= the projected attention output)
  float* yp;               // [H][kRmax][d] per-head partial projections
  int* cnt;                // [B][kAttnSplit] arrivals per row block, zero between launches
  int d;                   // model width (= H * Dh), a multiple of 16 * kAttnSplit
  // QKV projection
  const bf16* wqkv;        // [3d][d]: q rows, k rows, v rows (head-major within each)
  const bf16* g_attn;      // attention RMSNorm gains [d]
  float eps;
  const float2* rope;      // [cap][Dh/2] (cos, sin) of position * theta^(-2i/Dh)
  bf16* kc;                // K cache of this layer, slot 0: [H][cap][Dh] per slot
  bf16* vc;
  long long slot_stride;   // elements between slots in the cache arrays
  // MoE layers: the router partials of the updated residual rows (see route.cuh)
  const bf16* wr;          // W_r [E][d], or nullptr (dense FFN layer)
  const bf16* g_ffn;       // FFN RMSNorm gains [d]
  float* rpart;            // [rows][kRouteParts][kRouteLd]
  int E;
  int* status;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Split cluster barrier: every thread arrives early (no ordering) and waits
// right before its first access to another CTA's shared memory, which is then
// guaranteed to have started.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Arrival count with acquire-release semantics at GPU scope: after a CTA
// barrier it publishes the CTA's earlier writes, and the CTA that sees the
// final count (followed by a CTA barrier) observes every arriver's writes.
__device__ __forceinline__ int attn_arrive_acq_rel(int* p) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Orders this thread's generic shared-memory writes before later TMA
// (async-proxy) writes to the same addresses.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bulk copy of weights (read once per pass): evict-first in L2.
__device__ __forceinline__ void bulk_g2s_weights(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// Generic address of `p` in the shared memory of the cluster's CTA `rank`;
// plain loads through it read that CTA's shared memory.
template <class T>
__device__ __forceinline__ const T* cluster_map(const T* p, uint32_t rank) {
  uint64_t r;
  asm("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(p), "r"(rank));
  return reinterpret_cast<const T*>(r);
}

// 5-D tensor-map load of one chunk of K or V: 64 columns x 64 positions x
// Dh/64 halves at (position p0, head h, cache plane pl) -> [half][pos][128 B].
__device__ __forceinline__ void tma_load_kv(void* dst, const CUtensorMap* map, int p0, int h, int pl, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(p0), "r"(0), "r"(h), "r"(pl), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tensor-map load of a W_o block: 64 columns x nb rows x Dh/64 chunks at
// (row r0, column chunk c0) -> [chunk][row][128 B].
// The weights are read once per pass: evict-first in L2.
__device__ __forceinline__ void tma_load_wo(void* dst, const CUtensorMap* map, int r0, int c0, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(r0), "r"(c0), "r"(smem_u32(bar)),
      "l"(l2_evict_first_policy())
      : "memory");
}

__device__ __forceinline__ void attn_ldsm_x4(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void attn_ldsm_x4_t(uint32_t addr, uint32_t (&a)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(addr));
}
__device__ __forceinline__ void attn_ldsm_x2(uint32_t addr, uint32_t (&b)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(b[0]), "=r"(b[1]) : "r"(addr));
}
__device__ __forceinline__ void attn_mma(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Shared address of the 16-byte unit `u` (0..7) of position `pos`, half `hf`
// of a swizzled chunk tile.
__device__ __forceinline__ uint32_t kv_addr(uint32_t base, int hf, int pos, int u) {
  return base + (uint32_t)(hf * kAttnChunk * 128 + pos * 128 + ((u ^ (pos & 7)) << 4));
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_wo, const AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t bar[kAttnBufs], qkv_bar, wo_bar, r_bar;
  __shared__ __align__(16) bf16 s_head[2][kAttnRows][kAttnQLd];  // the head's merged output, high / low parts
  __shared__ __align__(16) bf16 s_q[2][kAttnRows][kAttnQLd];     // rotated q, high / low parts
  __shared__ __align__(16) bf16 s_kn[2][kAttnRows][kAttnMaxDh];  // the pass rows' new K (0) and V (1)
  __shared__ __align__(16) bf16 s_stage[4][kAttnRows][16];        // this CTA's q high, q low, K, V dims
  __shared__ float s_ss[kAttnWarps][kAttnRows];                   // per-warp sums of squares of the rows
  __shared__ int s_last;
  __shared__ int s_abort;
  __shared__ int s_pos[kAttnRows];
  __shared__ float s_M[kAttnRows], s_L[kAttnRows], s_corr[kAttnRows];

  const int k = (int)cluster_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Dh = p.Dh, d = p.d;
  unsigned char* ring = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t ring_s = smem_u32(ring);
  unsigned char* regb = ring + (size_t)kAttnRingBufs * 2 * kAttnChunkBytes;
  // K/V chunk buffer b (K then V): two in the ring, the third in region B
  auto kvbuf = [&](int b) {
    return b < kAttnRingBufs ? ring + (size_t)b * 2 * kAttnChunkBytes : regb + attn_buf2_off(d, Dh);
  };
  // region B while projecting: the CTA's W_qkv rows [tile][16][d + 8]
  bf16* s_w = reinterpret_cast<bf16*>(regb);
  const int ldq = d + 8;
  // region B afterwards: the W_o block [Dh/64][nb rows][128 B], scores, P, the projection's partial sums
  unsigned char* wo_s = regb;
  const size_t wob = attn_wo_bytes(d, Dh);
  float(*sc)[kAttnBufs * kAttnChunk] = reinterpret_cast<float(*)[kAttnBufs * kAttnChunk]>(regb + wob);
  bf16(*s_p)[kAttnRows][kAttnPLd] = reinterpret_cast<bf16(*)[kAttnRows][kAttnPLd]>(regb + wob + attn_sc_bytes());
  float* red = reinterpret_cast<float*>(regb + wob + attn_sc_bytes() + attn_p_bytes());
  // merge receive buffer (same place as red, used after every CTA's projection):
  // [source CTA][row] (M, L), then [source CTA][row][Dh / kAttnSplit] O of this CTA's dims
  float* rcv_ml = red;
  float* rcv_o = red + kAttnSplit * kAttnRows * 2;
  const int dpr = Dh / kAttnSplit;  // merged dims per CTA
  const int nb = d / kAttnSplit;  // W_o rows of this CTA
  const int E16 = p.wr ? (p.E + 15) / 16 * 16 : 0;
  const int ldw = nb + 8;
  bf16* s_wr = reinterpret_cast<bf16*>(regb + attn_regionb_bytes(d, Dh));  // [E16][ldw]
  bf16* s_gr = s_wr + (size_t)E16 * ldw;                                    // [nb]
  const int P = Dh / 16;                  // dims of each of q, k, v per CTA and half
  const int nt = attn_qkv_tiles(Dh);      // 16-row tiles of W_qkv rows
  const int ks = d / 16 / kAttnWarps;     // k16 steps of the projection per warp

  if (tid == 0) {
    for (int i = 0; i < kAttnBufs; ++i) mbar_init(&bar[i], 1);
    mbar_init(&qkv_bar, 1);
    mbar_init(&wo_bar, 1);
    mbar_init(&r_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t wpol = l2_evict_first_policy();
  // Weights first.  Tile t, row i of the W_qkv block is list entry
  // li = 8t + (i & 7): matrix m = li / P (q, k, v), j = li % P, head dim
  // (i >> 3) * Dh/2 + k*P + j; rows i and i + 8 of a tile are a RoPE pair.
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(&qkv_bar, (uint32_t)(6 * P * d * 2));
    __syncwarp();
    for (int row = lane; row < nt * 16; row += 32) {
      const int t = row >> 4, i = row & 15, li = t * 8 + (i & 7);
      if (li < 3 * P) {
        const int m = li / P, j = li - m * P;
        const int dim = (i >> 3) * (Dh / 2) + k * P + j;
        bulk_g2s_weights(s_w + (size_t)row * ldq, p.wqkv + ((size_t)m * d + h * Dh + dim) * d, (uint32_t)(d * 2),
                         &qkv_bar, wpol);
      }
    }
  }
  for (int i = p.E * ldw + tid; i < E16 * ldw; i += kAttnThreads) s_wr[i] = f2bf(0.f);  // padding rows
  for (int row = 3 * P + (tid >> 6); row < nt * 8; row += kAttnThreads / 64)          // padding entries (Dh 64)
    for (int c = tid & 63; c < d; c += 64) {
      s_w[(size_t)((row >> 3) * 16 + (row & 7)) * ldq + c] = f2bf(0.f);
      s_w[(size_t)((row >> 3) * 16 + (row & 7) + 8) * ldq + c] = f2bf(0.f);
    }
  // the attention RMSNorm gains of this lane's B-fragment columns (see below)
  uint32_t gq[kAttnMaxKs][2];
#pragma unroll
  for (int s = 0; s < kAttnMaxKs; ++s)
    if (s < ks) {
      const int kk = (warp * ks + s) * 16 + (lane & 3) * 2;
      gq[s][0] = __ldg(reinterpret_cast<const unsigned int*>(p.g_attn + kk));
      gq[s][1] = __ldg(reinterpret_cast<const unsigned int*>(p.g_attn + kk + 8));
    }
  cluster_arrive_relaxed();

  // pass rows: the slot's rows r0 .. r0 + nr - 1 at positions s_pos
  int r0 = 0, nr = 0, maxpos = -1, n_my = 0;
  const int plane = b * p.n_layers + p.layer;
  auto setup_rows = [&]() {
    r0 = p.slot_row0[b];
    nr = max(0, min(p.slot_nrows[b], kAttnRows));
    if (tid < kAttnRows) {
      s_pos[tid] = tid < nr ? p.row_pos[r0 + tid] : -1;  // -1: sees nothing
      s_M[tid] = -INFINITY;
      s_L[tid] = 0.f;
    }
    __syncthreads();
    maxpos = -1;
    for (int i = 0; i < nr; ++i) maxpos = max(maxpos, s_pos[i]);
    maxpos = min(maxpos, p.cap - 1);
    const int nch = maxpos >= 0 ? maxpos / kAttnChunk + 1 : 0;  // chunks of the slot
    n_my = nch > k ? (nch - 1 - k) / kAttnSplit + 1 : 0;        // this CTA's chunks
  };
  // chunk i of this CTA: position p0, valid positions npos, ring buffer i % kAttnBufs
  auto chunk_p0 = [&](int i) { return (k + i * kAttnSplit) * kAttnChunk; };
  auto chunk_npos = [&](int i) { return min(kAttnChunk, maxpos + 1 - chunk_p0(i)); };
  auto issue = [&](int i) {
    const int buf = i % kAttnBufs;
    unsigned char* kd = kvbuf(buf);
    mbar_arrive_expect_tx(&bar[buf], (uint32_t)(2 * kAttnChunk * Dh * 2));
    tma_load_kv(kd, &tm_k, chunk_p0(i), h, plane, &bar[buf]);
    tma_load_kv(kd + kAttnChunkBytes, &tm_v, chunk_p0(i), h, plane, &bar[buf]);
  };
  // The cache rows this pass writes are written over in shared memory once
  // their chunk lands, so every chunk may be requested before the wait.
  // the RoPE (cos, sin) of this thread's projection output (see below)
  float2 rcs = make_float2(1.f, 0.f);
  auto load_rope = [&]() {
    if (tid < nt * 64) {
      const int t = tid >> 6, L = (tid >> 1) & 31, r = (L & 3) * 2 + (tid & 1), li = t * 8 + (L >> 2);
      const int pos = s_pos[r];
      if (li < 2 * P && r < nr && pos >= 0 && pos < p.cap) rcs = p.rope[(long long)pos * (Dh / 2) + k * P + li % P];
    }
  };
  // The first group's chunks are requested once the W_qkv rows have landed
  // (they are needed only after the projection, and the two would share the
  // SM's bandwidth while the kernel before this one still streams).
  int n_issued = 0;
  if (p.rows_pre_wait) {
    setup_rows();
    load_rope();
  }
  // the router block is needed last: requested after everything else
  if (warp == 0 && p.wr) {
    if (lane == 0) mbar_arrive_expect_tx(&r_bar, (uint32_t)((p.E + 1) * nb * 2));
    __syncwarp();
    for (int e = lane; e < p.E; e += 32)
      bulk_g2s_weights(s_wr + (size_t)e * ldw, p.wr + (size_t)e * d + k * nb, (uint32_t)(nb * 2), &r_bar, wpol);
    if (lane == 0) bulk_g2s(s_gr, p.g_ffn + k * nb, (uint32_t)(nb * 2), &r_bar);
  }

  pdl_wait();
  TraceMarks tm;  // trace: wait returned, q/k/v broadcast, first group's softmax done
  if (tid == 0) {
    tm.t0 = gtimer();
    s_abort = status_bad(p.status);
  }
  __syncthreads();
  const bool abort = s_abort != 0;
  if (!p.rows_pre_wait) {
    setup_rows();
    load_rope();
  }
  const bool work = !abort && nr > 0;
  if (work) n_issued = min(n_my, kAttnBufs);
  pdl_trigger();

  // fragment lane roles
  const int fr_row = (lane & 7) + ((lane >> 3) & 1) * 8;   // ldmatrix.x4 row within a 16-row tile
  const int fr_hi = lane >> 4;                             // second 16-byte unit for lanes 16..31
  const int b_n = lane & 7, b_k8 = ((lane >> 3) & 1) * 8;  // ldmatrix.x2: MMA column and k offset

  // ---- QKV projection: warp w takes k16 steps [w*ks, (w+1)*ks) of the rows ----
  if (work) {
    // B fragments straight from the residual rows: lane -> pass row lane / 4,
    // columns (lane % 4) * 2 + {0, 1, 8, 9} of each k16 step
    const int n = lane >> 2;
    float xv[kAttnMaxKs][4];
    const float* xr = p.x + (long long)(r0 + n) * d;
#pragma unroll
    for (int s = 0; s < kAttnMaxKs; ++s) {
      xv[s][0] = xv[s][1] = xv[s][2] = xv[s][3] = 0.f;
      if (s < ks && n < nr) {
        const int kk = (warp * ks + s) * 16 + (lane & 3) * 2;
        const float2 u = __ldcg(reinterpret_cast<const float2*>(xr + kk));
        const float2 v = __ldcg(reinterpret_cast<const float2*>(xr + kk + 8));
        xv[s][0] = u.x;
        xv[s][1] = u.y;
        xv[s][2] = v.x;
        xv[s][3] = v.y;
      }
    }
    // the row's sum of squares: lane order, then its 4 lanes, then warps in order
    float a = 0.f;
#pragma unroll
    for (int s = 0; s < kAttnMaxKs; ++s)
#pragma unroll
      for (int e = 0; e < 4; ++e) a = __fmaf_rn(xv[s][e], xv[s][e], a);
    a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 2));
    if ((lane & 3) == 0) s_ss[warp][n] = a;
    __syncthreads();
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) ss = __fadd_rn(ss, s_ss[w][n]);
    const float rs = rsqrtf(__fadd_rn(__fdiv_rn(ss, (float)d), p.eps));
    uint32_t bh[kAttnMaxKs][2], bl[kAttnMaxKs][2];
#pragma unroll
    for (int s = 0; s < kAttnMaxKs; ++s) {
      float f[4];
      f[0] = __fmul_rn(__fmul_rn(xv[s][0], rs), bf_lo(gq[s][0]));
      f[1] = __fmul_rn(__fmul_rn(xv[s][1], rs), bf_hi(gq[s][0]));
      f[2] = __fmul_rn(__fmul_rn(xv[s][2], rs), bf_lo(gq[s][1]));
      f[3] = __fmul_rn(__fmul_rn(xv[s][3], rs), bf_hi(gq[s][1]));
      bh[s][0] = pack2(f[0], f[1]);
      bh[s][1] = pack2(f[2], f[3]);
      bl[s][0] = pack2(__fsub_rn(f[0], bf_lo(bh[s][0])), __fsub_rn(f[1], bf_hi(bh[s][0])));
      bl[s][1] = pack2(__fsub_rn(f[2], bf_lo(bh[s][1])), __fsub_rn(f[3], bf_hi(bh[s][1])));
    }
    mbar_wait(&qkv_bar, 0, p.status);
    if (tid == 0)  // the ring's chunks now; the third (region B) once the W_qkv rows are read
      for (int i = 0; i < n_issued && i < kAttnRingBufs; ++i) issue(i);
    float acc[kAttnQTiles][4];
#pragma unroll
    for (int t = 0; t < kAttnQTiles; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
    for (int s = 0; s < kAttnMaxKs; ++s)
      if (s < ks) {
        const int k0 = (warp * ks + s) * 16;
#pragma unroll
        for (int t = 0; t < kAttnQTiles; ++t)
          if (t < nt) {
            uint32_t af[4];
            attn_ldsm_x4(smem_u32(s_w + (size_t)(t * 16 + fr_row) * ldq + k0 + fr_hi * 8), af);
            attn_mma(acc[t], af, bh[s]);
            attn_mma(acc[t], af, bl[s]);
          }
      }
    __syncthreads();  // region B: the W_qkv rows are read
    if (tid == 0) {
      // the W_o block is a weight: requested as soon as its space is free
      mbar_arrive_expect_tx(&wo_bar, (uint32_t)(nb * Dh * 2));
      tma_load_wo(wo_s, &tm_wo, k * nb, h * (Dh / 64), &wo_bar);
      for (int i = kAttnRingBufs; i < n_issued; ++i) issue(i);
    }
#pragma unroll
    for (int t = 0; t < kAttnQTiles; ++t)
      if (t < nt)
        *reinterpret_cast<float4*>(red + ((warp * kAttnQTiles + t) * 32 + lane) * 4) =
            make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster runs: remote stores may start
  if (work && tid < nt * 64) {
    // output pair (tile t, rows i and i + 8, pass row r): warps' partials in order
    const int t = tid >> 6, L = (tid >> 1) & 31, par = tid & 1;
    float va = 0.f, vb = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      va = __fadd_rn(va, red[((w * kAttnQTiles + t) * 32 + L) * 4 + par]);
      vb = __fadd_rn(vb, red[((w * kAttnQTiles + t) * 32 + L) * 4 + 2 + par]);
    }
    const int i = L >> 2, r = (L & 3) * 2 + par, li = t * 8 + i;
    if (li < 3 * P) {
      const int m = li / P, j = li - m * P;  // dims k*P + j and Dh/2 + k*P + j
      const int pos = s_pos[r];
      const bool real = r < nr && pos >= 0 && pos < p.cap;
      if (m < 2 && real) {  // RoPE: the pair turns by pos * theta^(-2 (k*P + j) / Dh); rcs was loaded early
        const float a2 = __fsub_rn(__fmul_rn(va, rcs.x), __fmul_rn(vb, rcs.y));
        const float b2 = __fadd_rn(__fmul_rn(vb, rcs.x), __fmul_rn(va, rcs.y));
        va = a2;
        vb = b2;
      }
      // staged as runs of P contiguous dims (low dims, then their partners)
      if (m == 0) {
        const bf16 ha = f2bf(va), hb = f2bf(vb);
        s_stage[0][r][j] = ha;
        s_stage[0][r][P + j] = hb;
        s_stage[1][r][j] = f2bf(__fsub_rn(va, bf2f(ha)));
        s_stage[1][r][P + j] = f2bf(__fsub_rn(vb, bf2f(hb)));
      } else {
        s_stage[1 + m][r][j] = f2bf(va);
        s_stage[1 + m][r][P + j] = f2bf(vb);
      }
    }
  }
  __syncthreads();
  if (work) {
    // q (high, low), K and V runs to every CTA of the cluster, one P-dim run
    // per store: [destination][part][row][run]
    for (int w = tid; w < kAttnSplit * 4 * kAttnRows * 2; w += kAttnThreads) {
      const int q = w >> 6, part = (w >> 4) & 3, r = (w >> 1) & 7, run = w & 1;
      const int col = run * (Dh / 2) + k * P;
      bf16* dst = part < 2 ? &s_q[part][r][col] : &s_kn[part - 2][r][col];
      const bf16* src = &s_stage[part][r][run * P];
      if (P == 8)
        *reinterpret_cast<uint4*>(const_cast<bf16*>(cluster_map(dst, q))) = *reinterpret_cast<const uint4*>(src);
      else
        *reinterpret_cast<uint2*>(const_cast<bf16*>(cluster_map(dst, q))) = *reinterpret_cast<const uint2*>(src);
    }
    // the new K and V rows of the real pass rows to the cache
    if (tid < kAttnRows * 4) {
      const int r = tid >> 2, kv = (tid >> 1) & 1, run = tid & 1;
      const int pos = s_pos[r];
      if (r < nr && pos >= 0 && pos < p.cap) {
        bf16* c = (kv ? p.vc : p.kc) + (long long)b * p.slot_stride + ((long long)h * p.cap + pos) * Dh +
                  run * (Dh / 2) + k * P;
        const bf16* src = &s_stage[2 + kv][r][run * P];
        if (P == 8)
          *reinterpret_cast<uint4*>(c) = *reinterpret_cast<const uint4*>(src);
        else
          *reinterpret_cast<uint2*>(c) = *reinterpret_cast<const uint2*>(src);
      }
    }
  }
  cluster_sync_all();  // q and the new K / V rows are in every CTA
  if (tid == 0) tm.t1 = gtimer();

  // PV accumulators: warp w owns dims [16w, 16w + 16) (MMA m) for all 8 rows
  // (MMA n): o0 (dim 16w + lane/4, row 2(lane%4)), o1 (row + 1), o2/o3 (dim + 8)
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  const bool pv_warp = warp * 16 < Dh;

  for (int i0 = 0, grp = 0; work && i0 < n_my; i0 += kAttnBufs, ++grp) {
    const int ni = min(kAttnBufs, n_my - i0);
    for (int ii = 0; ii < ni; ++ii)
      mbar_wait(&bar[ii], grp & 1, p.status);  // gives up with OCRDEC_ETIMEOUT; control flow stays uniform

    // ---- the pass's own rows over their positions in the landed chunks ----
    auto local_chunk = [&](int pr) {  // group buffer of position pr, or -1
      if (pr < 0 || pr > maxpos) return -1;
      const int c = pr / kAttnChunk;
      if (c % kAttnSplit != k) return -1;
      const int ii = c / kAttnSplit - i0;
      return ii >= 0 && ii < ni ? ii : -1;
    };
    bool patch = false;
    for (int r = 0; r < nr; ++r) patch |= local_chunk(s_pos[r]) >= 0;
    if (patch) {
      for (int idx = tid; idx < nr * Dh; idx += kAttnThreads) {
        const int r = idx / Dh, dd = idx - r * Dh;
        const int pr = s_pos[r], ii = local_chunk(pr);
        if (ii < 0) continue;
        const int pp = pr % kAttnChunk;
        const size_t off = (dd >> 6) * kAttnChunk * 128 + pp * 128 + ((((dd & 63) >> 3) ^ (pp & 7)) << 4) +
                           (dd & 7) * 2;
        *reinterpret_cast<bf16*>(kvbuf(ii) + off) = s_kn[0][r][dd];
        *reinterpret_cast<bf16*>(kvbuf(ii) + off + kAttnChunkBytes) = s_kn[1][r][dd];
      }
      fence_proxy_async_smem();  // the buffer is refilled by TMA later
      __syncthreads();
    }

    // ---- scores: 16-position tiles t = warp, warp + 8, ... of the group ----
    for (int t = warp; t < ni * (kAttnChunk / 16); t += kAttnWarps) {
      const int ii = t / (kAttnChunk / 16), pt = (t % (kAttnChunk / 16)) * 16;
      const uint32_t kb = smem_u32(kvbuf(ii));
      float dacc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < Dh / 16; ++s) {
        uint32_t af[4], bh[2], bl[2];
        attn_ldsm_x4(kv_addr(kb, s >> 2, pt + fr_row, (s & 3) * 2 + fr_hi), af);
        attn_ldsm_x2(smem_u32(&s_q[0][b_n][s * 16 + b_k8]), bh);
        attn_ldsm_x2(smem_u32(&s_q[1][b_n][s * 16 + b_k8]), bl);
        attn_mma(dacc, af, bh);
        attn_mma(dacc, af, bl);
      }
      const int p0 = chunk_p0(i0 + ii), npos = chunk_npos(i0 + ii);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = pt + (lane >> 2) + (e >> 1) * 8;  // position in the chunk
        const int r = 2 * (lane & 3) + (e & 1);         // row
        const bool valid = j < npos && p0 + j <= s_pos[r];
        sc[r][ii * kAttnChunk + j] = valid ? __fmul_rn(dacc[e], p.scale) : -INFINITY;
      }
    }
    __syncthreads();

    // ---- online softmax update of each row over the group (warp w: row w).
    // Invisible positions hold -inf and give exp(-inf) = 0 exactly. ----
    const int nu = ni * kAttnChunk;
    for (int r = warp; r < nr; r += kAttnWarps) {
      float m = -INFINITY;
      for (int u = lane; u < nu; u += 32) m = fmaxf(m, sc[r][u]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (m == -INFINITY) {  // nothing visible to this row in the group
        for (int u = lane; u < nu; u += 32) {
          s_p[0][r][u] = f2bf(0.f);
          s_p[1][r][u] = f2bf(0.f);
        }
        if (lane == 0) s_corr[r] = 1.f;
        continue;
      }
      const float Mold = s_M[r];
      const float Mn = fmaxf(Mold, m);
      float l = 0.f;
      for (int u = lane; u < nu; u += 32) {
        const float e = expf(__fsub_rn(sc[r][u], Mn));
        const bf16 hi = f2bf(e);
        s_p[0][r][u] = hi;
        s_p[1][r][u] = f2bf(__fsub_rn(e, bf2f(hi)));
        l = __fadd_rn(l, e);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, off));
      __syncwarp();
      if (lane == 0) {
        const float corr = Mold == -INFINITY ? 0.f : expf(__fsub_rn(Mold, Mn));
        s_corr[r] = corr;
        s_L[r] = __fmaf_rn(s_L[r], corr, l);
        s_M[r] = Mn;
      }
    }
    __syncthreads();
    if (tid == 0 && grp == 0) tm.t2 = gtimer();

    // ---- O = O * corr + V^T P^T over the group's positions ----
    if (pv_warp) {
      const int c0 = 2 * (lane & 3);
      const float cr0 = c0 < nr ? s_corr[c0] : 1.f, cr1 = c0 + 1 < nr ? s_corr[c0 + 1] : 1.f;
      o[0] = __fmul_rn(o[0], cr0);
      o[1] = __fmul_rn(o[1], cr1);
      o[2] = __fmul_rn(o[2], cr0);
      o[3] = __fmul_rn(o[3], cr1);
      const int hf = (warp * 16) / 64, u0 = ((warp * 16) % 64) / 8;
      for (int ii = 0; ii < ni; ++ii) {
        const uint32_t vb = smem_u32(kvbuf(ii)) + (uint32_t)kAttnChunkBytes;
#pragma unroll
        for (int s = 0; s < kAttnChunk / 16; ++s) {
          // A = V^T (16 dims x 16 positions) from the stored [pos][dim] tile:
          // lanes 0-7 pos 0-7 dims 0-7, 8-15 pos 0-7 dims 8-15, 16-23 pos 8-15
          // dims 0-7, 24-31 pos 8-15 dims 8-15
          const int pos = s * 16 + (lane & 7) + (lane >> 4) * 8;
          const int u = u0 + ((lane >> 3) & 1);
          uint32_t af[4], bh[2], bl[2];
          attn_ldsm_x4_t(kv_addr(vb, hf, pos, u), af);
          const int pc = ii * kAttnChunk + s * 16 + b_k8;
          attn_ldsm_x2(smem_u32(&s_p[0][b_n][pc]), bh);
          attn_ldsm_x2(smem_u32(&s_p[1][b_n][pc]), bl);
          attn_mma(o, af, bh);
          attn_mma(o, af, bl);
        }
      }
    }
    __syncthreads();  // ring buffers, scores and probabilities are free again
    if (tid == 0)
      for (int ii = 0; ii < kAttnBufs && i0 + kAttnBufs + ii < n_my; ++ii) issue(i0 + kAttnBufs + ii);
  }

  // ---- this CTA's state: (M, L) to every CTA, the O of dims
  // [q*dpr, (q+1)*dpr) to CTA q (warp w holds dims [16w, 16w + 16)) ----
  if (work) {
    if (pv_warp) {
      const int c0 = 2 * (lane & 3);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int dm = warp * 16 + (lane >> 2) + (e >> 1) * 8, r = c0 + (e & 1);
        const int q = dm / dpr;
        if (r < nr)
          *const_cast<float*>(cluster_map(rcv_o + ((size_t)k * kAttnRows + r) * dpr + (dm - q * dpr), q)) = o[e];
      }
    }
    if (tid < kAttnRows * kAttnSplit) {
      const int r = tid & (kAttnRows - 1), q = tid / kAttnRows;
      float* dst = const_cast<float*>(cluster_map(rcv_ml + (k * kAttnRows + r) * 2, q));
      dst[0] = s_M[r];
      dst[1] = s_L[r];
    }
  } else if (tid == 0) {
    mbar_wait(&qkv_bar, 0, p.status);  // the W_qkv copies land before the CTA exits
  }
  cluster_sync_all();  // CTA k holds every CTA's state of its dims

  // ---- merge: CTA k forms dims [k*dpr, (k+1)*dpr) of every row, combining
  // the CTAs' states in rank order, and stores them (bf16) into the head
  // output of every CTA of the cluster ----
  if (work && tid < kAttnRows * dpr) {
    const int r = tid / dpr, dl = tid - r * dpr, dm = k * dpr + dl;
    bf16 hi = f2bf(0.f), lo = f2bf(0.f);  // rows past nr: zeros (MMA columns stay finite)
    if (r < nr) {
      float Mg = -INFINITY;
#pragma unroll
      for (int q = 0; q < kAttnSplit; ++q) Mg = fmaxf(Mg, rcv_ml[(q * kAttnRows + r) * 2]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int q = 0; q < kAttnSplit; ++q) {
        const float Mq = rcv_ml[(q * kAttnRows + r) * 2];
        const float f = Mq == -INFINITY ? 0.f : expf(__fsub_rn(Mq, Mg));
        L = __fmaf_rn(rcv_ml[(q * kAttnRows + r) * 2 + 1], f, L);
        O = __fmaf_rn(rcv_o[((size_t)q * kAttnRows + r) * dpr + dl], f, O);
      }
      const float ov = __fdiv_rn(O, L);
      hi = f2bf(ov);
      lo = f2bf(__fsub_rn(ov, bf2f(hi)));
    }
#pragma unroll
    for (int q = 0; q < kAttnSplit; ++q) {
      *const_cast<bf16*>(cluster_map(&s_head[0][r][dm], q)) = hi;
      *const_cast<bf16*>(cluster_map(&s_head[1][r][dm], q)) = lo;
    }
  }
  cluster_sync_all();  // every CTA holds the whole head output; no remote access follows

  // ---- output projection of this head, rows [k*nb, (k+1)*nb) of W_o:
  // yp[h][row][n] = sum_d W_o[n][h*Dh + d] * head[row][d] (MMAs: n x rows) ----
  if (work) {
    mbar_wait(&wo_bar, 0, p.status);
    const uint32_t wb = smem_u32(wo_s);
    for (int t = warp; t < nb / 16; t += kAttnWarps) {
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < Dh / 16; ++s) {
        uint32_t af[4], bh[2], bl[2];
        const int row = t * 16 + fr_row, u = (s & 3) * 2 + fr_hi;
        attn_ldsm_x4(wb + (uint32_t)((s >> 2) * nb * 128 + row * 128 + ((u ^ (row & 7)) << 4)), af);
        attn_ldsm_x2(smem_u32(&s_head[0][b_n][s * 16 + b_k8]), bh);
        attn_ldsm_x2(smem_u32(&s_head[1][b_n][s * 16 + b_k8]), bl);
        attn_mma(d4, af, bh);
        attn_mma(d4, af, bl);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int nn = k * nb + t * 16 + (lane >> 2) + (e >> 1) * 8;
        const int r = 2 * (lane & 3) + (e & 1);
        if (r < nr) p.yp[((long long)h * kAttnRows + r0 + r) * d + nn] = d4[e];
      }
    }
    // the last head to finish this row block adds the heads' partials in
    // head order to the residual stream.  The block's residual values are
    // read first (no kernel writes them meanwhile), so the tail after the
    // arrival count is one round of loads.
    // Float4 groups of the block: row r, columns k*nb + 4c .. 4c+3 (nb / 4
    // groups per row; at most 4 rows fit one pass of the CTA's threads).
    constexpr int kG4 = (kAttnRows * (kAttnMaxD / kAttnSplit) / 4 + kAttnThreads - 1) / kAttnThreads;
    const int n4 = nb / 4;
    float4 xv[kG4];
#pragma unroll
    for (int i = 0; i < kG4; ++i) {
      const int g = tid + i * kAttnThreads;
      xv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (g < nr * n4) {
        const int r = g / n4, c = (g - r * n4) * 4;
        xv[i] = __ldcg(reinterpret_cast<const float4*>(p.x + (long long)(r0 + r) * d + k * nb + c));
      }
    }
    __syncthreads();
    if (tid == 0) s_last = attn_arrive_acq_rel(&p.cnt[b * kAttnSplit + k]) == p.H - 1;
    __syncthreads();
    if (s_last) {
      // MoE layers: u = g * x (new residual) as bf16 high and low parts and
      // x itself go to the (now free) K/V ring for the router partials
      bf16* su = reinterpret_cast<bf16*>(ring);                                    // [2][kAttnRows][ldw]
      float* sx = reinterpret_cast<float*>(ring + (size_t)2 * kAttnRows * ldw * 2);  // [kAttnRows][nb]
#pragma unroll
      for (int i = 0; i < kG4; ++i) {
        const int g = tid + i * kAttnThreads;
        if (g >= kAttnRows * n4) break;
        const int r = g / n4, c = (g - r * n4) * 4;
        float4 xn = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < nr) {
          // the heads' partials of the group (all loads in flight), added in head order
          const float* yr = p.yp + (long long)(r0 + r) * d + k * nb + c;
          float4 y[kAttnMaxHeads];
#pragma unroll
          for (int hh = 0; hh < kAttnMaxHeads; ++hh)
            if (hh < p.H) y[hh] = __ldcg(reinterpret_cast<const float4*>(yr + (long long)hh * kAttnRows * d));
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int hh = 0; hh < kAttnMaxHeads; ++hh)
            if (hh < p.H) {
              v.x = __fadd_rn(v.x, y[hh].x);
              v.y = __fadd_rn(v.y, y[hh].y);
              v.z = __fadd_rn(v.z, y[hh].z);
              v.w = __fadd_rn(v.w, y[hh].w);
            }
          xn = make_float4(__fadd_rn(xv[i].x, v.x), __fadd_rn(xv[i].y, v.y), __fadd_rn(xv[i].z, v.z),
                           __fadd_rn(xv[i].w, v.w));
          *reinterpret_cast<float4*>(p.x + (long long)(r0 + r) * d + k * nb + c) = xn;
        }
        if (p.wr) {
          const float xe[4] = {xn.x, xn.y, xn.z, xn.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int nl = c + e;
            const float u = __fmul_rn(xe[e], bf2f(s_gr[nl]));
            const bf16 hi = f2bf(u);
            su[r * ldw + nl] = hi;
            su[(kAttnRows + r) * ldw + nl] = f2bf(__fsub_rn(u, bf2f(hi)));
            sx[r * nb + nl] = xe[e];
          }
        }
      }
      if (tid == 0) p.cnt[b * kAttnSplit + k] = 0;
      if (p.wr) {
        mbar_wait(&r_bar, 0, p.status);
        __syncthreads();
        float* rp = p.rpart + (size_t)r0 * kRouteParts * kRouteLd + k * kRouteLd;
        // each row's sum of squares over the block (warp w: row w, fixed order)
        if (warp < nr) {
          float s2 = 0.f;
          for (int nl = lane; nl < nb; nl += 32) s2 = __fmaf_rn(sx[warp * nb + nl], sx[warp * nb + nl], s2);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) s2 = __fadd_rn(s2, __shfl_xor_sync(0xffffffffu, s2, off));
          if (lane == 0) rp[(size_t)warp * kRouteParts * kRouteLd + kMaxExperts] = s2;
        }
        // dot products of the block's W_r columns with u (experts x rows MMAs)
        for (int t = warp; t < E16 / 16; t += kAttnWarps) {
          float d4[4] = {0.f, 0.f, 0.f, 0.f};
          for (int s = 0; s < nb / 16; ++s) {
            uint32_t af[4], bh[2], bl[2];
            attn_ldsm_x4(smem_u32(s_wr + (size_t)(t * 16 + fr_row) * ldw + s * 16 + fr_hi * 8), af);
            attn_ldsm_x2(smem_u32(su + b_n * ldw + s * 16 + b_k8), bh);
            attn_ldsm_x2(smem_u32(su + (kAttnRows + b_n) * ldw + s * 16 + b_k8), bl);
            attn_mma(d4, af, bh);
            attn_mma(d4, af, bl);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = t * 16 + (lane >> 2) + (q >> 1) * 8;
            const int r = 2 * (lane & 3) + (q & 1);
            if (e < p.E && r < nr) rp[(size_t)r * kRouteParts * kRouteLd + e] = d4[q];
          }
        }
      }
    }
  }
  // the router block's copy lands before the CTA exits
  if (tid == 0 && p.wr) mbar_wait(&r_bar, 0, p.status);
  if (tid == 0 && work && n_my > 0) trace_end(p.status, k == 0 ? kTagAttention + 1 : kTagAttention, tm);
}

}  // namespace ocrdec
