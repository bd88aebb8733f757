// Split-K flash-decoding attention over a contiguous per-slot KV cache.
//
// For pass row r (slot b, position pos_r) and head h:
//   out[r][h] = softmax_j(q_r . k_j / sqrt(Dh)) v_j over positions j = 0..pos_r
// (causal: rows of one pass see each other's keys up to their own position).
// The position axis is cut into fixed kAttnChunk-position chunks; CTA (c, h, b)
// loads chunk c of head h for slot b into shared memory with two bulk copies,
// computes every row's partial (max m, sum l, unnormalised o) over the
// positions that row may see, and the last CTA of (b, h) merges the partials
// of each row in chunk order.  Chunk boundaries depend only on positions, so a
// row's result does not depend on the other rows of the pass.
#pragma once

#include "common.cuh"

namespace ocrdec {

constexpr int kAttnChunk = 64;
constexpr int kTagAttention = 40;
constexpr int kAttnThreads = 128;
constexpr int kAttnRows = 8;  // rows of one slot in a pass
constexpr int kAttnMaxChunks = 128;  // chunks per sequence: kv_capacity <= 8192

struct AttnParams {
  const float* q;          // [R][H*Dh]
  const bf16* kc;          // this layer, slot 0: [H][cap][Dh]
  const bf16* vc;
  long long slot_stride;   // elements between slots
  int cap, H, Dh;
  float scale;             // 1/sqrt(Dh)
  const int* slot_row0;    // [B] first pass row of each slot
  const int* slot_nrows;   // [B] rows of each slot in this pass
  const int* row_pos;      // [R]
  float* part;             // [R][H][max_chunks][Dh + 2]: o[Dh], m, l
  int max_chunks;
  int* counters;           // [B][H], zero between launches
  bf16* out;               // [R][H*Dh]
  int* status;
};

__global__ void __launch_bounds__(kAttnThreads)
attention_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  __shared__ float qs[kAttnRows][128];
  __shared__ float sc[kAttnRows][kAttnChunk];
  __shared__ float ored[4][kAttnRows][128];
  __shared__ float s_m[kAttnRows], s_l[kAttnRows];
  __shared__ int s_last;

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Dh = p.Dh;

  pdl_wait();
  TraceMarks tm;  // trace: wait returned, K/V landed, partials written
  if (tid == 0) tm.t0 = gtimer();
  if (tid == 0) s_abort = status_bad(p.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();

  __shared__ int s_pos[kAttnRows];
  const int r0 = p.slot_row0[b];
  const int nr = min(p.slot_nrows[b], kAttnRows);
  if (nr <= 0) return;
  if (tid < nr) s_pos[tid] = p.row_pos[r0 + tid];
  __syncthreads();
  int maxpos = 0;
  for (int i = 0; i < nr; ++i) maxpos = max(maxpos, s_pos[i]);
  const int nchunks = maxpos / kAttnChunk + 1;
  if (c >= nchunks) return;
  const int p0 = c * kAttnChunk;
  const int npos = min(kAttnChunk, maxpos + 1 - p0);

  bf16* Ks = reinterpret_cast<bf16*>(smem);
  bf16* Vs = Ks + kAttnChunk * Dh;
  const long long base = (long long)b * p.slot_stride + ((long long)h * p.cap + p0) * Dh;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    uint32_t bytes = npos * Dh * 2;
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_g2s(Ks, p.kc + base, bytes, &bar);
    bulk_g2s(Vs, p.vc + base, bytes, &bar);
  }
  // queries of this slot's rows (all loads in flight together)
#pragma unroll
  for (int i = 0; i < kAttnRows; ++i)
    if (i < nr && tid < Dh) qs[i][tid] = p.q[(long long)(r0 + i) * p.H * Dh + h * Dh + tid];
  __syncthreads();
  mbar_wait(&bar, 0, p.status);  // gives up with OCRDEC_ETIMEOUT recorded; control flow stays uniform
  if (tid == 0) tm.t1 = gtimer();

  // ---- scores: 4 lanes-groups of 8 per warp, one position per group ----
  // lane l8 of a group owns the 16-byte dim-chunks l8 and l8 + 8 of a key row
  const int g = lane >> 3, l8 = lane & 7;
  const int ndc = Dh / 8;  // 16-byte chunks per key row (8 or 16)
  for (int rb = 0; rb < nr; rb += 4) {
    float qr[4][16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        int d = (e < 8 ? l8 * 8 + e : (l8 + 8) * 8 + (e - 8));
        qr[i][e] = (rb + i < nr && (e < 8 || l8 + 8 < ndc)) ? qs[rb + i][d] : 0.f;
      }
    for (int j0 = warp * 16; j0 < warp * 16 + 16; j0 += 4) {
      int j = j0 + g;
      float kv[16];
      if (j < npos) {
        uint4 u0 = *reinterpret_cast<const uint4*>(Ks + j * Dh + l8 * 8);
        float t[8];
        unpack8(u0, t);
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[e] = t[e];
        if (l8 + 8 < ndc) {
          uint4 u1 = *reinterpret_cast<const uint4*>(Ks + j * Dh + (l8 + 8) * 8);
          unpack8(u1, t);
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
      for (int i = 0; i < 4; ++i) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) a = __fmaf_rn(qr[i][e], kv[e], a);
        a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 4));
        a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 2));
        a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 1));
        int r = rb + i;
        if (l8 == 0 && r < nr && j < kAttnChunk) {
          bool valid = j < npos && p0 + j <= s_pos[r];
          sc[r][j] = valid ? __fmul_rn(a, p.scale) : -INFINITY;
        }
      }
    }
  }
  __syncthreads();

  // ---- per-row chunk max and exp-sum (warp w takes rows w, w+4) ----
  for (int r = warp; r < nr; r += 4) {
    int lim = s_pos[r] - p0 + 1;  // visible positions of this row in the chunk
    lim = min(lim, npos);
    float m = -INFINITY;
    for (int j = lane; j < lim; j += 32) m = fmaxf(m, sc[r][j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int j = lane; j < kAttnChunk; j += 32) {
      float e = 0.f;
      if (j < lim) e = expf(__fsub_rn(sc[r][j], m));
      sc[r][j] = e;
      l = __fadd_rn(l, e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, o));
    if (lane == 0) { s_m[r] = m; s_l[r] = l; }
  }
  __syncthreads();

  if (tid == 0) tm.t2 = gtimer();  // trace: scores and softmax done
  // ---- o = sum_j p_j v_j: warp w takes positions 16w..16w+15 in order, lane l
  // dims [l*dpl, (l+1)*dpl); the 4 warp partials are then added in warp order ----
  const int ld = Dh + 2;
  const int dpl = Dh / 32;  // dims per lane: 4 (Dh 128) or 2 (Dh 64)
  {
    float o[kAttnRows][4];
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[r][e] = 0.f;
    int lim[kAttnRows];
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r) lim[r] = r < nr ? min(s_pos[r] - p0 + 1, npos) : 0;
    const int jb = warp * 16;
    for (int jj = 0; jj < 16; ++jj) {
      const int j = jb + jj;
      if (j >= npos) break;
      float vv[4];
      if (dpl == 4) {
        uint2 u = *reinterpret_cast<const uint2*>(Vs + j * Dh + lane * 4);
        vv[0] = bf_lo(u.x); vv[1] = bf_hi(u.x); vv[2] = bf_lo(u.y); vv[3] = bf_hi(u.y);
      } else {
        uint32_t u = *reinterpret_cast<const uint32_t*>(Vs + j * Dh + lane * 2);
        vv[0] = bf_lo(u); vv[1] = bf_hi(u); vv[2] = 0.f; vv[3] = 0.f;
      }
#pragma unroll
      for (int r = 0; r < kAttnRows; ++r) {
        if (j < lim[r]) {
          const float pj = sc[r][j];
#pragma unroll
          for (int e = 0; e < 4; ++e) o[r][e] = __fmaf_rn(pj, vv[e], o[r][e]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r)
      if (r < nr)
        for (int e = 0; e < dpl; ++e) ored[warp][r][lane * dpl + e] = o[r][e];
  }
  __syncthreads();
  for (int r = 0; r < nr; ++r) {
    int lim = min(s_pos[r] - p0 + 1, npos);
    if (lim <= 0) continue;
    float* dst = p.part + (((long long)(r0 + r) * p.H + h) * p.max_chunks + c) * ld;
    for (int d = tid; d < Dh; d += kAttnThreads)
      dst[d] = __fadd_rn(__fadd_rn(__fadd_rn(ored[0][r][d], ored[1][r][d]), ored[2][r][d]), ored[3][r][d]);
    if (tid == 0) { dst[Dh] = s_m[r]; dst[Dh + 1] = s_l[r]; }
  }

  // ---- last CTA of (slot, head) merges the chunks of every row ----
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[b * p.H + h], 1) == nchunks - 1);
  __syncthreads();
  if (!s_last) {
    if (tid == 0) trace_end(p.status, kTagAttention, tm);
    return;
  }
  __threadfence();
  // stage every (row, chunk) max and sum, then the per-chunk rescale factors
  __shared__ float s_m2[kAttnRows][kAttnMaxChunks];
  __shared__ float s_f[kAttnRows][kAttnMaxChunks];
  __shared__ float s_L[kAttnRows];
  const int maxc = min(nchunks, kAttnMaxChunks);
  for (int idx = tid; idx < nr * maxc; idx += kAttnThreads) {
    int r = idx / maxc, cc = idx - r * maxc;
    const float* pr = p.part + (((long long)(r0 + r) * p.H + h) * p.max_chunks + cc) * ld;
    int nc = s_pos[r] / kAttnChunk + 1;
    s_m2[r][cc] = cc < nc ? __ldcg(pr + Dh) : -INFINITY;     // m
    s_f[r][cc] = cc < nc ? __ldcg(pr + Dh + 1) : 0.f;       // l
  }
  __syncthreads();
  if (tid < nr) {
    const int r = tid;
    int nc = s_pos[r] / kAttnChunk + 1;
    float M = -INFINITY;
    for (int cc = 0; cc < nc; ++cc) M = fmaxf(M, s_m2[r][cc]);
    float L = 0.f;
    for (int cc = 0; cc < nc; ++cc) {
      float f = expf(__fsub_rn(s_m2[r][cc], M));
      L = __fmaf_rn(s_f[r][cc], f, L);
      s_m2[r][cc] = f;
    }
    s_L[r] = L;
  }
  __syncthreads();
  // O[r][d] = sum_c o_c[r][d] f[r][c]: the partials of 4 chunks x all rows are
  // requested before any is used, so the loads overlap
  int ncr[kAttnRows];
#pragma unroll
  for (int r = 0; r < kAttnRows; ++r) ncr[r] = r < nr ? s_pos[r] / kAttnChunk + 1 : 0;
  constexpr int kCB = 4;
  for (int d = tid; d < Dh; d += kAttnThreads) {
    float O[kAttnRows];
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r) O[r] = 0.f;
    for (int c0 = 0; c0 < maxc; c0 += kCB) {
      float v[kCB][kAttnRows];
#pragma unroll
      for (int j = 0; j < kCB; ++j)
#pragma unroll
        for (int r = 0; r < kAttnRows; ++r)
          v[j][r] = (c0 + j < ncr[r])
                        ? __ldcg(p.part + (((long long)(r0 + r) * p.H + h) * p.max_chunks + c0 + j) * ld + d)
                        : 0.f;
#pragma unroll
      for (int j = 0; j < kCB; ++j)
#pragma unroll
        for (int r = 0; r < kAttnRows; ++r)
          if (c0 + j < ncr[r]) O[r] = __fmaf_rn(v[j][r], s_m2[r][c0 + j], O[r]);
    }
#pragma unroll
    for (int r = 0; r < kAttnRows; ++r)
      if (r < nr) p.out[(long long)(r0 + r) * p.H * Dh + h * Dh + d] = f2bf(__fdiv_rn(O[r], s_L[r]));
  }
  if (tid == 0) {
    p.counters[b * p.H + h] = 0;
    trace_end(p.status, kTagAttention + 1, tm);  // the merging CTA
  }
}

}  // namespace ocrdec
