// Decode attention over a contiguous per-slot KV cache, split over a
// thread-block cluster.
//
// For pass row r (slot b, position pos_r) and head h:
//   out[r][h] = softmax_j(q_r . k_j / sqrt(Dh)) v_j over positions j = 0..pos_r
// (causal: rows of one pass see each other's keys up to their own position).
//
// The position axis is cut into fixed kAttnChunk-position chunks.  The
// kAttnSplit CTAs of one cluster serve one (slot, head); CTA k takes chunks
// k, k + kAttnSplit, ... in increasing order, kAttnBufs at a time: it streams
// their K and V rows into shared memory with bulk copies, scores them all,
// and keeps an online-softmax state per row (running max M, sum L,
// unnormalised output O) that is rescaled between such groups.  The CTAs then
// merge their states through distributed shared memory, rank by rank, each CTA
// producing Dh / kAttnSplit output dims.  Which CTA takes a chunk and the order
// of every sum depend only on positions, so a row's result does not depend on
// the other rows of the pass.
//
// Chunks that lie wholly below the pass's first new position are not written
// by the kernel before this one (which writes the pass rows' keys and values),
// so their copies are issued before the dependency wait.
#pragma once

#include "common.cuh"

namespace ocrdec {

constexpr int kAttnChunk = 64;
constexpr int kAttnSplit = 8;    // CTAs per (slot, head): one cluster
constexpr int kAttnBufs = 3;     // K/V chunk ring per CTA
constexpr int kTagAttention = 40;
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kAttnWarpPos = kAttnChunk / kAttnWarps;  // positions of a chunk per warp
constexpr int kAttnRows = 8;     // rows of one slot in a pass
constexpr int kAttnMaxDh = 128;

constexpr size_t attn_smem_bytes(int Dh) { return (size_t)kAttnBufs * 2 * kAttnChunk * Dh * 2; }

struct AttnParams {
  const float* q;          // [R][H*Dh]
  const bf16* kc;          // this layer, slot 0: [H][cap][Dh]
  const bf16* vc;
  long long slot_stride;   // elements between slots
  int cap, H, Dh;          // Dh 64 or 128
  float scale;             // 1/sqrt(Dh)
  const int* slot_row0;    // [B] first pass row of each slot
  const int* slot_nrows;   // [B] rows of each slot in this pass
  const int* row_pos;      // [R]
  bf16* out;               // [R][H*Dh]
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

// Generic address of `p` in the shared memory of the cluster's CTA `rank`;
// plain loads through it read that CTA's shared memory.
template <class T>
__device__ __forceinline__ const T* cluster_map(const T* p, uint32_t rank) {
  uint64_t r;
  asm("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(p), "r"(rank));
  return reinterpret_cast<const T*>(r);
}

__global__ void __launch_bounds__(kAttnThreads)
attention_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar[kAttnBufs];
  __shared__ int s_abort;
  __shared__ int s_pos[kAttnRows];
  __shared__ float qs[kAttnRows][kAttnMaxDh];
  __shared__ float sc[kAttnRows][kAttnBufs * kAttnChunk];
  __shared__ float ored[kAttnWarps][kAttnRows][kAttnMaxDh];
  __shared__ float s_M[kAttnRows], s_L[kAttnRows], s_corr[kAttnRows];
  __shared__ float s_O[kAttnRows][kAttnMaxDh];

  const int k = (int)cluster_rank();
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Dh = p.Dh;
  bf16* ring = reinterpret_cast<bf16*>(smem);

  if (tid == 0) {
    for (int i = 0; i < kAttnBufs; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
  }
  // pass rows and positions are written by the pass's setup kernel, which
  // finished before the kernel this one follows
  const int r0 = p.slot_row0[b];
  const int nr = max(0, min(p.slot_nrows[b], kAttnRows));
  if (tid < kAttnRows) s_pos[tid] = tid < nr ? p.row_pos[r0 + tid] : -1;  // -1: sees nothing
  if (tid < kAttnRows) {
    s_M[tid] = -INFINITY;
    s_L[tid] = 0.f;
  }
  __syncthreads();
  int minpos = 0x7fffffff, maxpos = -1;
  for (int i = 0; i < nr; ++i) {
    minpos = min(minpos, s_pos[i]);
    maxpos = max(maxpos, s_pos[i]);
  }
  maxpos = min(maxpos, p.cap - 1);
  const int nch = maxpos >= 0 ? maxpos / kAttnChunk + 1 : 0;  // chunks of the slot
  const int n_my = nch > k ? (nch - 1 - k) / kAttnSplit + 1 : 0;  // this CTA's chunks
  const long long head_base = (long long)b * p.slot_stride + (long long)h * p.cap * Dh;

  // chunk i of this CTA: position p0, valid positions npos, ring buffer i % kAttnBufs
  auto chunk_p0 = [&](int i) { return (k + i * kAttnSplit) * kAttnChunk; };
  auto chunk_npos = [&](int i) { return min(kAttnChunk, maxpos + 1 - chunk_p0(i)); };
  auto issue = [&](int i) {
    const int p0 = chunk_p0(i);
    const int buf = i % kAttnBufs;
    bf16* Ks = ring + (size_t)buf * 2 * kAttnChunk * Dh;
    const uint32_t bytes = chunk_npos(i) * Dh * 2;
    mbar_arrive_expect_tx(&bar[buf], 2 * bytes);
    bulk_g2s(Ks, p.kc + head_base + (long long)p0 * Dh, bytes, &bar[buf]);
    bulk_g2s(Ks + kAttnChunk * Dh, p.vc + head_base + (long long)p0 * Dh, bytes, &bar[buf]);
  };
  auto old_chunk = [&](int i) { return chunk_p0(i) + kAttnChunk <= minpos; };
  const int n_first = min(n_my, kAttnBufs);
  if (tid == 0)
    for (int i = 0; i < n_first; ++i)
      if (old_chunk(i)) issue(i);

  pdl_wait();
  TraceMarks tm;  // trace: wait returned, first group landed, its softmax done
  float qv[kAttnRows];
#pragma unroll
  for (int i = 0; i < kAttnRows; ++i)
    qv[i] = (i < nr && tid < Dh) ? p.q[(long long)(r0 + i) * p.H * Dh + h * Dh + tid] : 0.f;
  if (tid == 0) {
    tm.t0 = gtimer();
    const int ab = status_bad(p.status);
    s_abort = ab;
    if (!ab)
      for (int i = 0; i < n_first; ++i)
        if (!old_chunk(i)) issue(i);
  }
  if (tid < kAttnMaxDh)
#pragma unroll
    for (int i = 0; i < kAttnRows; ++i) qs[i][tid] = tid < Dh ? qv[i] : 0.f;
  __syncthreads();
  const bool work = !s_abort && nr > 0;
  pdl_trigger();

  // per-warp output accumulators: warp w owns offsets [w, w + 1) * kAttnWarpPos
  // of every chunk, lane l dims [l*dpl, (l+1)*dpl)
  const int dpl = Dh / 32;  // 4 (Dh 128) or 2 (Dh 64)
  float o[kAttnRows][4];
#pragma unroll
  for (int r = 0; r < kAttnRows; ++r)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[r][e] = 0.f;

  const int g4 = lane >> 3, l8 = lane & 7;
  const int ndc = Dh / 8;  // 16-byte chunks per key row (8 or 16)
  // Chunks are taken kAttnBufs at a time (a group); the online-softmax state
  // is rescaled between groups.
  for (int i0 = 0, grp = 0; work && i0 < n_my; i0 += kAttnBufs, ++grp) {
    const int ni = min(kAttnBufs, n_my - i0);
    for (int ii = 0; ii < ni; ++ii)
      mbar_wait(&bar[ii], grp & 1, p.status);  // gives up with OCRDEC_ETIMEOUT; control flow stays uniform
    if (tid == 0 && grp == 0) tm.t1 = gtimer();

    // ---- scores: 4 groups of 8 lanes per warp, one position per lane group;
    // lane l8 owns the 16-byte dim-chunks l8 and l8 + 8 of a key row
    for (int rb = 0; rb < nr; rb += 4) {
      float qr[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int d = (e < 8 ? l8 * 8 + e : (l8 + 8) * 8 + (e - 8));
          qr[q][e] = qs[rb + q][d];  // rows past nr and dims past Dh hold zeros
        }
      for (int ii = 0; ii < ni; ++ii) {
        const int p0 = chunk_p0(i0 + ii), npos = chunk_npos(i0 + ii);
        const bf16* Ks = ring + (size_t)ii * 2 * kAttnChunk * Dh;
#pragma unroll
        for (int j0 = 0; j0 < kAttnWarpPos; j0 += 4) {
          const int j = warp * kAttnWarpPos + j0 + g4;
          float kv[16];
          if (j < npos) {
            float t[8];
            unpack8(*reinterpret_cast<const uint4*>(Ks + j * Dh + l8 * 8), t);
#pragma unroll
            for (int e = 0; e < 8; ++e) kv[e] = t[e];
            if (l8 + 8 < ndc) {
              unpack8(*reinterpret_cast<const uint4*>(Ks + j * Dh + (l8 + 8) * 8), t);
#pragma unroll
              for (int e = 0; e < 8; ++e) kv[8 + e] = t[e];
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) kv[8 + e] = 0.f;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) kv[e] = 0.f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) a = __fmaf_rn(qr[q][e], kv[e], a);
            a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 4));
            a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 2));
            a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 1));
            const int r = rb + q;  // < kAttnRows; rows past nr have position -1
            const bool valid = j < npos && p0 + j <= s_pos[r];
            if (l8 == 0) sc[r][ii * kAttnChunk + j] = valid ? __fmul_rn(a, p.scale) : -INFINITY;
          }
        }
      }
    }
    __syncthreads();

    // ---- online softmax update of each row over the group (warp w: row w).
    // Invisible positions hold -inf and give exp(-inf) = 0 exactly, so a row's
    // sums do not depend on how many chunks the group has. ----
    const int nu = ni * kAttnChunk;
    for (int r = warp; r < nr; r += kAttnWarps) {
      float m = -INFINITY;
      for (int u = lane; u < nu; u += 32) m = fmaxf(m, sc[r][u]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (m == -INFINITY) {  // nothing visible to this row in the group
        for (int u = lane; u < nu; u += 32) sc[r][u] = 0.f;
        if (lane == 0) s_corr[r] = 1.f;
        continue;
      }
      const float Mold = s_M[r];
      const float Mn = fmaxf(Mold, m);
      float l = 0.f;
      for (int u = lane; u < nu; u += 32) {
        const float e = expf(__fsub_rn(sc[r][u], Mn));
        sc[r][u] = e;
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

    // ---- o = o * corr + sum p_j v_j over the warp's offsets, chunk by chunk ----
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r)
      if (r < nr) {
        const float cr = s_corr[r];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[r][e] = __fmul_rn(o[r][e], cr);
      }
    for (int ii = 0; ii < ni; ++ii) {
      const int npos = chunk_npos(i0 + ii);
      const bf16* Vs = ring + (size_t)ii * 2 * kAttnChunk * Dh + kAttnChunk * Dh;
#pragma unroll
      for (int jj = 0; jj < kAttnWarpPos; ++jj) {
        const int j = warp * kAttnWarpPos + jj;
        if (j >= npos) break;
        float vv[4];
        if (dpl == 4) {
          uint2 u = *reinterpret_cast<const uint2*>(Vs + j * Dh + lane * 4);
          vv[0] = bf_lo(u.x); vv[1] = bf_hi(u.x); vv[2] = bf_lo(u.y); vv[3] = bf_hi(u.y);
        } else {
          uint32_t u = *reinterpret_cast<const uint32_t*>(Vs + j * Dh + lane * 2);
          vv[0] = bf_lo(u); vv[1] = bf_hi(u); vv[2] = 0.f; vv[3] = 0.f;
        }
        // positions a row does not see have p = 0 exactly and add nothing;
        // the loads are unconditional so they issue together
        float pj[kAttnRows];
#pragma unroll
        for (int r = 0; r < kAttnRows; ++r) pj[r] = sc[r][ii * kAttnChunk + j];
#pragma unroll
        for (int r = 0; r < kAttnRows; ++r)
          if (r < nr)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[r][e] = __fmaf_rn(pj[r], vv[e], o[r][e]);
      }
    }
    __syncthreads();  // ring buffers and scores are free again
    if (tid == 0)
      for (int ii = 0; ii < kAttnBufs && i0 + kAttnBufs + ii < n_my; ++ii) issue(i0 + kAttnBufs + ii);
  }

  // ---- this CTA's state: O = sum of the warp partials in warp order ----
  if (work) {
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r)
      if (r < nr)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < dpl) ored[warp][r][lane * dpl + e] = o[r][e];
    __syncthreads();
    for (int idx = tid; idx < nr * Dh; idx += kAttnThreads) {
      const int r = idx / Dh, d = idx - r * Dh;
      float v = ored[0][r][d];
#pragma unroll
      for (int w = 1; w < kAttnWarps; ++w) v = __fadd_rn(v, ored[w][r][d]);
      s_O[r][d] = v;
    }
  } else if (s_abort && tid == 0) {
    // copies issued before the dependency wait land before the CTA exits
    for (int i = 0; i < n_first; ++i)
      if (old_chunk(i)) mbar_wait(&bar[i], 0, p.status);
  }
  cluster_sync_all();  // every CTA's state is visible to the cluster

  // ---- merge: CTA k writes dims [k*dpr, (k+1)*dpr) of every row, combining
  // the CTAs' states in rank order ----
  if (work) {
    const int dpr = Dh / kAttnSplit;
    if (tid < nr * dpr) {
      const int r = tid / dpr, d = k * dpr + (tid - r * dpr);
      // all remote loads are issued before any is used
      float Mk[kAttnSplit], Lk[kAttnSplit], Ok[kAttnSplit];
#pragma unroll
      for (int q = 0; q < kAttnSplit; ++q) {
        Mk[q] = *cluster_map(&s_M[r], q);
        Lk[q] = *cluster_map(&s_L[r], q);
        Ok[q] = *cluster_map(&s_O[r][d], q);
      }
      float Mg = -INFINITY;
#pragma unroll
      for (int q = 0; q < kAttnSplit; ++q) Mg = fmaxf(Mg, Mk[q]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int q = 0; q < kAttnSplit; ++q) {
        const float f = Mk[q] == -INFINITY ? 0.f : expf(__fsub_rn(Mk[q], Mg));
        L = __fmaf_rn(Lk[q], f, L);
        O = __fmaf_rn(Ok[q], f, O);
      }
      p.out[(long long)(r0 + r) * p.H * Dh + h * Dh + d] = f2bf(__fdiv_rn(O, L));
    }
  }
  cluster_sync_all();  // no CTA leaves while another may still read its state
  if (tid == 0 && work && n_my > 0) trace_end(p.status, k == 0 ? kTagAttention + 1 : kTagAttention, tm);
}

}  // namespace ocrdec
