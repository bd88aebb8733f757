// Routing of the pass rows: softmax over all experts, top-k (ties to the
// lower id), gates = the softmax values; then bucketing: per-expert row lists
// and the list of matrices to stream (shared experts first, then the touched
// experts in ascending id).  The expert gate/up GEMV runs it in every CTA on
// logits it assembles from the attention kernel's router partials.
#pragma once

#include "common.cuh"

namespace ocrdec {

constexpr int kMaxExperts = 64;   // routed experts per layer
constexpr int kMaxShared = 8;     // shared experts per layer
constexpr int kMaxTopK = 8;
// Router partials written by the attention kernel: for every pass row and
// each of its kRouteParts output-row blocks, the E partial dot products of
// W_r with (g * x) over the block's columns, and at [kMaxExperts] the block's
// partial sum of squares of x.
constexpr int kRouteParts = 8;
constexpr int kRouteLd = kMaxExperts + 4;

// Routing tables of one pass (expert mode of the GEMV keeps them in shared memory).
struct RouteTables {
  int n_mats;
  int mats[kMaxShared + kMaxExperts];
  int counts[kMaxExperts];
  int offsets[kMaxExperts];
  int rowlist[kRmax * kMaxTopK];
};


struct RouteParams {
  const float* logits;  // [R][E]
  const int* nrows;
  int E, top_k, S;
  int* ids;             // [R][top_k], ascending expert id
  float* gates;         // [R][top_k]
  int* counts;          // [E]
  int* offsets;         // [E]
  int* rowlist;         // [R*top_k] entries r | (slot << 8)
  int* mats;            // [S + E]
  int* n_mats;
  int* touched;         // optional: [0] += routed experts touched, [1] += 1
  int* status;
  // shared-memory scratch: [kRmax][kMaxExperts] probabilities (16-byte
  // aligned) and [kRmax][kMaxExperts] selected slots
  float (*s_p)[kMaxExperts];
  unsigned char (*s_slot)[kMaxExperts];
};
// Bytes of the scratch route_rows needs.
constexpr int kRouteScratchBytes = kRmax * kMaxExperts * (4 + 1);

// Routing of the R rows by nthreads (>= 32 * R) cooperating threads; sync()
// is a barrier over exactly those threads.
template <class Sync>
__device__ void route_rows(const RouteParams& p, int R, int tid, int nthreads, Sync sync) {
  float (*s_p)[kMaxExperts] = p.s_p;                // softmax probabilities, -1 past E
  unsigned char (*s_slot)[kMaxExperts] = p.s_slot;  // slot of a selected expert, 0xff otherwise
  const int lane = tid & 31, warp = tid >> 5;
  const int E = p.E, K = p.top_k;
  // warp r: softmax of row r (fixed-order sums), top-k by rank and the slots
  if (warp < R) {
    const int r = warp;
    const float* lg = p.logits + r * E;
    constexpr int kPer = kMaxExperts / 32;
    float pe[kPer];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      int e = lane + 32 * i;
      pe[i] = e < E ? lg[e] : -INFINITY;
      m = fmaxf(m, pe[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      int e = lane + 32 * i;
      pe[i] = e < E ? expf(__fsub_rn(pe[i], m)) : 0.f;
      sum = __fadd_rn(sum, pe[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      int e = lane + 32 * i;
      pe[i] = e < E ? __fdiv_rn(pe[i], sum) : -1.f;
      s_p[r][e] = pe[i];
    }
    __syncwarp();
    // expert e is selected when fewer than K experts beat it (larger
    // probability, or equal probability and lower id)
    const float4* row4 = reinterpret_cast<const float4*>(s_p[r]);
    const int E4 = (E + 3) >> 2;
    int base = 0;
#pragma unroll 1
    for (int i = 0; 32 * i < E; ++i) {
      const int e = lane + 32 * i;
      const float pv = s_p[r][e];
      int beat = 0;
#pragma unroll 4
      for (int j = 0; j < E4; ++j) {
        const float4 q = row4[j];
        const int f = 4 * j;
        beat += (q.x > pv) || (q.x == pv && f < e);
        beat += (q.y > pv) || (q.y == pv && f + 1 < e);
        beat += (q.z > pv) || (q.z == pv && f + 2 < e);
        beat += (q.w > pv) || (q.w == pv && f + 3 < e);
      }
      // slots: the selected experts in ascending id
      const bool sel = e < E && beat < K;
      const unsigned msk = __ballot_sync(0xffffffffu, sel);
      const int slot = base + __popc(msk & ((1u << lane) - 1u));
      const bool ok = sel && slot < K;  // slot >= K only with NaN probabilities
      if (ok) {
        p.ids[r * K + slot] = e;
        p.gates[r * K + slot] = pv;
      }
      if (e < E) s_slot[r][e] = ok ? (unsigned char)slot : (unsigned char)0xff;
      base += __popc(msk);
    }
  }
  sync();
  // bucketing by one warp: per-expert row counts, their exclusive prefix, the
  // touched experts in ascending id after the shared ones, and each expert's
  // (row, slot) entries in row order
  if (warp == 0) {
    int base_c = 0, base_t = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int c = 0;
      if (e < E)
        for (int r = 0; r < R; ++r) c += s_slot[r][e] != 0xff;
      const int t = c > 0;
      int ic = c, it = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int vc = __shfl_up_sync(0xffffffffu, ic, o);
        int vt = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) { ic += vc; it += vt; }
      }
      if (e < E) {
        int off = base_c + ic - c;
        p.counts[e] = c;
        p.offsets[e] = off;
        if (t) p.mats[p.S + base_t + it - 1] = e;
        for (int r = 0; r < R; ++r) {
          const int sl = s_slot[r][e];
          if (sl != 0xff) p.rowlist[off++] = r | (sl << 8);
        }
      }
      base_c += __shfl_sync(0xffffffffu, ic, 31);
      base_t += __shfl_sync(0xffffffffu, it, 31);
    }
    if (lane < p.S) p.mats[lane] = E + lane;
    if (lane == 0) {
      *p.n_mats = p.S + base_t;
      if (p.touched) {
        atomicAdd(&p.touched[0], base_t);
        atomicAdd(&p.touched[1], 1);
      }
    }
  }
}

}  // namespace ocrdec
