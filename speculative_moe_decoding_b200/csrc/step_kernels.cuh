// Small kernels of the decode step: router softmax/top-k with expert
// bucketing, the MoE combine, pass setup (embedding gather, row metadata,
// draft inputs), greedy acceptance with commit and rollback, the benchmark's
// forced-acceptance override, and the RoPE table.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace ocrdec {

// Per-slot device state.  The first ten fields mirror ocrdec_slot_stats.
struct SlotState {
  int kv_len, n_context, n_generated, bonus, steps, tau_sum, hist[4];
  int pending;   // pairs (verifier hidden, next token) the draft has not consumed
  int pend_pos;  // position of the first pending pair
  int pad[2];
};

// Row metadata of one pass.
struct PassRows {
  int n;                 // rows in the pass
  int slot[kRmax];
  int pos[kRmax];
  int tok[kRmax];
  int slot_row0[kRmax];  // per slot: first row (slots < max_batch <= kRmax)
  int slot_nrows[kRmax];
  int last_row[kRmax];   // per slot: its last row (draft LM head rows)
  int n_last;            // number of slots with rows (draft LM head pass size)
};

// ---------------------------------------------------------------------------
// router: softmax over all experts, top-k (ties to the lower id), gates =
// softmax values; then bucketing: per-expert row lists and the list of matrices
// to stream (shared experts first, then touched experts in ascending id).
// One CTA, one warp per row.
// ---------------------------------------------------------------------------
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
};

__global__ void __launch_bounds__(256) route_kernel(const RouteParams p) {
  __shared__ int s_ids[kRmax][8];
  __shared__ int s_cnt[256];
  __shared__ int s_off[256];
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  if (tid == 0) s_abort = status_bad(p.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();
  const int R = min(*p.nrows, kRmax);
  const int E = p.E, K = p.top_k;
  if (warp < R) {
    const float* lg = p.logits + warp * E;
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, lg[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float pe[8];  // E <= 256
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int e = lane + 32 * i;
      pe[i] = e < E ? expf(__fsub_rn(lg[e], m)) : 0.f;
      sum = __fadd_rn(sum, pe[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
#pragma unroll
    for (int i = 0; i < 8; ++i) pe[i] = __fdiv_rn(pe[i], sum);
    int sel[8];
    float selg[8];
    for (int s = 0; s < K; ++s) {
      float bv = -1.f;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int e = lane + 32 * i;
        if (e < E && (pe[i] > bv || (pe[i] == bv && e < bi))) { bv = pe[i]; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      sel[s] = bi;
      selg[s] = bv;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i == bi) pe[i] = -2.f;  // taken
    }
    if (lane == 0) {
      // slot order = ascending expert id
      for (int a = 1; a < K; ++a)
        for (int b2 = a; b2 > 0 && sel[b2 - 1] > sel[b2]; --b2) {
          int ti = sel[b2]; sel[b2] = sel[b2 - 1]; sel[b2 - 1] = ti;
          float tg = selg[b2]; selg[b2] = selg[b2 - 1]; selg[b2 - 1] = tg;
        }
      for (int s = 0; s < K; ++s) {
        p.ids[warp * K + s] = sel[s];
        p.gates[warp * K + s] = selg[s];
        s_ids[warp][s] = sel[s];
      }
    }
  }
  __syncthreads();
  // bucketing: thread e counts its rows in (row, slot) order
  for (int e = tid; e < E; e += 256) {
    int n = 0;
    for (int r = 0; r < R; ++r)
      for (int s = 0; s < K; ++s) n += (s_ids[r][s] == e);
    s_cnt[e] = n;
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, u = 0;
    for (int sh = 0; sh < p.S; ++sh) p.mats[u++] = E + sh;
    for (int e = 0; e < E; ++e) {
      s_off[e] = off;
      off += s_cnt[e];
      if (s_cnt[e] > 0) p.mats[u++] = e;
    }
    *p.n_mats = u;
    if (p.touched) {
      p.touched[0] += u - p.S;
      p.touched[1] += 1;
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += 256) {
    int o = s_off[e];
    p.counts[e] = s_cnt[e];
    p.offsets[e] = o;
    for (int r = 0; r < R; ++r)
      for (int s = 0; s < K; ++s)
        if (s_ids[r][s] == e) p.rowlist[o++] = r | (s << 8);
  }
}

// x[r][n] += sum_s gate[r][s] * y[r][s][n] (routed, ascending expert id)
//            + sum_sh y[r][top_k + sh][n]   (shared)
struct CombineParams {
  float* x;
  const float* y;
  const float* gates;
  const int* nrows;
  int d, top_k, S;
  int* status;
};

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  pdl_wait();
  if (status_bad(p.status)) return;
  pdl_trigger();
  const int R = min(*p.nrows, kRmax);
  const int nslot = p.top_k + p.S;
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= R * p.d) return;
  int r = idx / p.d, n = idx - r * p.d;
  const float* yr = p.y + (long long)r * nslot * p.d + n;
  float t = 0.f;
  for (int s = 0; s < p.top_k; ++s) t = __fmaf_rn(p.gates[r * p.top_k + s], yr[(long long)s * p.d], t);
  for (int s = 0; s < p.S; ++s) t = __fadd_rn(t, yr[(long long)(p.top_k + s) * p.d]);
  p.x[idx] = __fadd_rn(p.x[idx], t);
}

// ---------------------------------------------------------------------------
// RoPE table: cos/sin of pos * theta^(-2i/Dh), float64 math, float32 values
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* tab, int cap, int Dh, double theta) {
  int half = Dh / 2;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)cap * half) return;
  int pos = (int)(idx / half), i = (int)(idx % half);
  double inv = pow(theta, -2.0 * (double)i / (double)Dh);
  double a = (double)pos * inv;
  tab[idx] = make_float2((float)cos(a), (float)sin(a));
}

// ---------------------------------------------------------------------------
// pass setup
// ---------------------------------------------------------------------------

// Verify pass: rows b*(k+1)+i = [bonus, proposals[b][0..k-1]] at kv_len+i;
// x rows = token embeddings.
struct VerifySetupParams {
  SlotState* slots;
  const int* proposals;  // [B][k]
  int B, k, cap, d, vocab;
  const bf16* embed;
  float* x;
  PassRows* rows;
  int* status;
};

__global__ void __launch_bounds__(256) verify_setup_kernel(const VerifySetupParams p) {
  __shared__ int s_tok[kRmax];
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) {
    s_bad = status_bad(p.status);
    if (!s_bad) {
      int R = p.B * (p.k + 1);
      for (int b = 0; b < p.B; ++b)
        if (p.slots[b].kv_len + p.k + 1 > p.cap) s_bad = 1;
      if (s_bad) set_status(p.status, OCRDEC_ECAPACITY);
      else {
        p.rows->n = R;
        p.rows->n_last = p.B;
        for (int b = 0; b < kRmax; ++b) {
          p.rows->slot_row0[b] = b < p.B ? b * (p.k + 1) : 0;
          p.rows->slot_nrows[b] = b < p.B ? p.k + 1 : 0;
          p.rows->last_row[b] = b < p.B ? b * (p.k + 1) + p.k : 0;
        }
        for (int b = 0; b < p.B; ++b)
          for (int i = 0; i <= p.k; ++i) {
            int r = b * (p.k + 1) + i;
            int t = i == 0 ? p.slots[b].bonus : p.proposals[b * p.k + i - 1];
            if (t < 0 || t >= p.vocab) {  // caller-supplied proposal out of range
              set_status(p.status, OCRDEC_EINVAL);
              s_bad = 1;
              t = 0;
            }
            p.rows->slot[r] = b;
            p.rows->pos[r] = p.slots[b].kv_len + i;
            p.rows->tok[r] = t;
            s_tok[r] = t;
          }
      }
    }
  }
  __syncthreads();
  if (s_bad) return;
  pdl_trigger();
  const int R = p.B * (p.k + 1);
  for (int idx = tid; idx < R * p.d; idx += blockDim.x) {
    int r = idx / p.d, n = idx - r * p.d;
    p.x[idx] = bf2f(p.embed[(long long)s_tok[r] * p.d + n]);
  }
}

// Prefill chunk: rows r = positions p0 + r of the context (visual rows, then
// prompt token embeddings).
struct PrefillSetupParams {
  int slot, p0, n, n_visual, vocab, n_prompt;
  const float* visual;  // [n_visual][d]
  const int* prompt;
  const bf16* embed;
  int d;
  float* x;
  PassRows* rows;
  int* status;
};

__global__ void __launch_bounds__(256) prefill_setup_kernel(const PrefillSetupParams p) {
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) {
    s_bad = status_bad(p.status);
    // prompt tokens of this chunk and of the next row (read by the draft pairs) must be in range
    for (int r = 0; r <= p.n && !s_bad; ++r) {
      int pos = p.p0 + r;
      if (pos >= p.n_visual && pos - p.n_visual < p.n_prompt) {
        int t = p.prompt[pos - p.n_visual];
        if (t < 0 || t >= p.vocab) {
          set_status(p.status, OCRDEC_EINVAL);
          s_bad = 1;
        }
      }
    }
  }
  __syncthreads();
  if (s_bad) return;
  pdl_trigger();
  if (tid == 0) {
    p.rows->n = p.n;
    p.rows->n_last = 1;
    for (int b = 0; b < kRmax; ++b) {
      p.rows->slot_row0[b] = 0;
      p.rows->slot_nrows[b] = b == p.slot ? p.n : 0;
      p.rows->last_row[b] = p.n - 1;
    }
    for (int r = 0; r < p.n; ++r) {
      int pos = p.p0 + r;
      p.rows->slot[r] = p.slot;
      p.rows->pos[r] = pos;
      p.rows->tok[r] = pos < p.n_visual ? -1 : p.prompt[pos - p.n_visual];
    }
  }
  for (int idx = tid; idx < p.n * p.d; idx += blockDim.x) {
    int r = idx / p.d, n = idx - r * p.d;
    int pos = p.p0 + r;
    p.x[idx] = pos < p.n_visual ? p.visual[(long long)pos * p.d + n]
                                : bf2f(p.embed[(long long)p.prompt[pos - p.n_visual] * p.d + n]);
  }
}

// Draft input rows: fcin[r] = [bf16(RMSNorm(h_r) * g_h) ; bf16(RMSNorm(e_r) * g_e)]
// where (h_r, e_r, pos_r) come from one of three row sources:
//   mode 0 (recursion 1): the pending pairs of each slot - verifier hidden
//          hpend[b][i] and the embedding of the committed token at pos+1;
//   mode 1 (recursion j >= 2): the draft's own output hidden xd[last_row[b]] and
//          the embedding of draft token dtok[b], at kv_len + j - 2;
//   mode 2 (prefill): verifier hidden x[p - p0] and the next context input
//          (visual vector or prompt embedding) for pairs p in [p0, p0 + n).
struct DraftSetupParams {
  int mode, B, j, d, max_k;
  float eps;
  SlotState* slots;
  const int* hist;       // [B][hist_ld] token history by position
  int hist_ld;
  const float* hpend;    // [B][max_k+1][d]
  const float* xd;       // draft residual of the previous recursion
  const int* dtok;       // previous draft token of slot b at dtok[b * dtok_stride]
  int dtok_stride;
  // prefill
  int slot, p0, n, n_visual;
  const float* xv;       // verifier residual of the prefill chunk
  const float* visual;
  const int* prompt;
  // common
  const bf16* embed;
  const bf16* g_h;
  const bf16* g_e;
  bf16* fcin;            // [R][2d]
  PassRows* rows;        // written
  const PassRows* rows_prev;  // mode 1: rows of the previous recursion (last_row)
  int* status;
};

__device__ __forceinline__ float block_sum_256(float v, float* red, int tid) {
  // fixed order: warp butterfly then warps 0..7 in order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  float a = 0.f;
  for (int w = 0; w < 8; ++w) a = __fadd_rn(a, red[w]);
  return a;
}

__global__ void __launch_bounds__(256) draft_setup_kernel(const DraftSetupParams p) {
  __shared__ int s_n, s_bad;
  __shared__ float red[8];
  __shared__ PassRows pr;
  __shared__ int s_prev_last[kRmax];
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) {
    s_bad = status_bad(p.status);
    if (p.mode == 1)
      for (int b = 0; b < kRmax; ++b) s_prev_last[b] = p.rows_prev->last_row[b];
    int n = 0;
    if (!s_bad) {
      for (int b = 0; b < kRmax; ++b) { pr.slot_row0[b] = 0; pr.slot_nrows[b] = 0; pr.last_row[b] = 0; }
      if (p.mode == 0) {
        for (int b = 0; b < p.B; ++b) {
          int np = min(p.slots[b].pending, p.max_k + 1);
          pr.slot_row0[b] = n;
          pr.slot_nrows[b] = np;
          for (int i = 0; i < np; ++i, ++n) {
            pr.slot[n] = b;
            pr.pos[n] = p.slots[b].pend_pos + i;
            pr.tok[n] = p.hist[b * p.hist_ld + p.slots[b].pend_pos + i + 1];
          }
          pr.last_row[b] = n - 1;
        }
        pr.n_last = p.B;
      } else if (p.mode == 1) {
        for (int b = 0; b < p.B; ++b) {
          pr.slot_row0[b] = b;
          pr.slot_nrows[b] = 1;
          pr.last_row[b] = b;
          pr.slot[b] = b;
          pr.pos[b] = p.slots[b].kv_len + p.j - 2;
          pr.tok[b] = p.dtok[b * p.dtok_stride];
        }
        n = p.B;
        pr.n_last = p.B;
      } else {
        pr.slot_row0[p.slot] = 0;
        pr.slot_nrows[p.slot] = p.n;
        pr.last_row[p.slot] = p.n - 1;
        for (int r = 0; r < p.n; ++r) {
          int pos = p.p0 + r;
          pr.slot[r] = p.slot;
          pr.pos[r] = pos;
          pr.tok[r] = pos + 1 < p.n_visual ? -1 : p.prompt[pos + 1 - p.n_visual];
        }
        n = p.n;
        pr.n_last = 1;
      }
      pr.n = n;
    }
    s_n = n;
  }
  __syncthreads();
  if (s_bad) return;
  pdl_trigger();
  const int d = p.d;
  for (int r = 0; r < s_n; ++r) {
    const int b = pr.slot[r];
    const float* h;
    if (p.mode == 0) h = p.hpend + ((long long)b * (p.max_k + 1) + (r - pr.slot_row0[b])) * d;
    else if (p.mode == 1) h = p.xd + (long long)s_prev_last[b] * d;
    else h = p.xv + (long long)r * d;
    const int tok = pr.tok[r];
    const float* ev = (p.mode == 2 && tok < 0) ? p.visual + (long long)(pr.pos[r] + 1) * d : nullptr;
    float sh = 0.f, se = 0.f;
    for (int n = tid; n < d; n += 256) {
      float hv = h[n];
      float e = ev ? ev[n] : bf2f(p.embed[(long long)tok * d + n]);
      sh = __fmaf_rn(hv, hv, sh);
      se = __fmaf_rn(e, e, se);
    }
    sh = block_sum_256(sh, red, tid);
    se = block_sum_256(se, red, tid);
    float ch = rsqrtf(__fadd_rn(__fdiv_rn(sh, (float)d), p.eps));
    float ce = rsqrtf(__fadd_rn(__fdiv_rn(se, (float)d), p.eps));
    for (int n = tid; n < d; n += 256) {
      float e = ev ? ev[n] : bf2f(p.embed[(long long)tok * d + n]);
      p.fcin[(long long)r * 2 * d + n] = f2bf(__fmul_rn(__fmul_rn(h[n], ch), bf2f(p.g_h[n])));
      p.fcin[(long long)r * 2 * d + d + n] = f2bf(__fmul_rn(__fmul_rn(e, ce), bf2f(p.g_e[n])));
    }
  }
  // publish the row metadata
  int* dst = reinterpret_cast<int*>(p.rows);
  const int* src = reinterpret_cast<const int*>(&pr);
  for (int i = tid; i < (int)(sizeof(PassRows) / sizeof(int)); i += 256) dst[i] = src[i];
}

// ---------------------------------------------------------------------------
// greedy acceptance, commit and rollback
// ---------------------------------------------------------------------------
struct AcceptParams {
  SlotState* slots;
  const int* g;          // [B*(k+1)] verifier argmax per row
  const int* proposals;  // [B][k]
  int B, k, d, max_k;
  int* hist;             // [B][hist_ld]
  int hist_ld;
  const float* x;        // verifier residual rows (pre final norm)
  float* hpend;          // [B][max_k+1][d]
  int* committed;        // [B][k+1], -1 past the commit
  int* n_committed;      // [B]
  int* status;
};

__global__ void __launch_bounds__(256) accept_kernel(const AcceptParams p) {
  __shared__ int s_a[kRmax];
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) s_abort = status_bad(p.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();
  if (tid < p.B) {
    const int b = tid, K1 = p.k + 1;
    const int* g = p.g + b * K1;
    int a = 0;
    while (a < p.k && p.proposals[b * p.k + a] == g[a]) ++a;
    SlotState& st = p.slots[b];
    const int n = st.kv_len;
    for (int i = 0; i <= p.k; ++i) p.committed[b * K1 + i] = i <= a ? g[i] : -1;
    for (int i = 0; i <= a; ++i) p.hist[b * p.hist_ld + n + 1 + i] = g[i];
    p.n_committed[b] = a + 1;
    st.kv_len = n + a + 1;
    st.n_generated += a + 1;
    st.bonus = g[a];
    st.steps += 1;
    st.tau_sum += a + 1;
    st.hist[a] += 1;
    st.pending = a + 1;
    st.pend_pos = n;
    s_a[b] = a;
  }
  __syncthreads();
  const int K1 = p.k + 1;
  for (int b = 0; b < p.B; ++b)
    for (int idx = tid; idx < (s_a[b] + 1) * p.d; idx += blockDim.x) {
      int i = idx / p.d, n = idx - i * p.d;
      p.hpend[((long long)b * (p.max_k + 1) + i) * p.d + n] = p.x[(long long)(b * K1 + i) * p.d + n];
    }
}

// Forced acceptance (benchmark harness): proposal for target t = kv_len + j.
struct ForceParams {
  const SlotState* slots;
  int* proposals;
  int B, k, max_k;
  const int* ref;
  const float* u;
  const int* alt;
  int n_pos;
  float p0, p1, p2;
  int* status;
};

__global__ void force_kernel(const ForceParams p) {
  pdl_wait();
  if (status_bad(p.status)) return;
  pdl_trigger();
  int idx = threadIdx.x;
  if (idx >= p.B * p.k) return;
  int b = idx / p.k, j = idx % p.k + 1;
  int t = p.slots[b].kv_len + j;
  if (t >= p.n_pos) { set_status(p.status, OCRDEC_EINVAL); return; }
  float pj = j == 1 ? p.p0 : (j == 2 ? p.p1 : p.p2);
  int want = p.ref[t];
  int a = p.alt[t * p.max_k + j - 1];
  p.proposals[idx] = p.u[t * p.max_k + j - 1] < pj ? want : (a < want ? a : a + 1);
}

// Prefill finish: first token, slot counters, the pending pair (h_{C-1}, t_C).
struct PrefillFinishParams {
  SlotState* slots;
  int slot, C, x_row, d, max_k;
  const int* tok;       // LM-head argmax of the last context row (tok[0])
  const float* x;       // verifier residual of the last chunk
  float* hpend;
  int* hist;
  int hist_ld;
  int* first_token;
  int* status;
};

__global__ void __launch_bounds__(256) prefill_finish_kernel(const PrefillFinishParams p) {
  pdl_wait();
  if (status_bad(p.status)) return;
  pdl_trigger();
  const int tid = threadIdx.x;
  const int t0 = p.tok[0];
  if (tid == 0) {
    SlotState& st = p.slots[p.slot];
    st.kv_len = p.C;
    st.n_context = p.C;
    st.n_generated = 1;
    st.bonus = t0;
    st.steps = 0;
    st.tau_sum = 0;
    for (int i = 0; i < 4; ++i) st.hist[i] = 0;
    st.pending = 1;
    st.pend_pos = p.C - 1;
    p.hist[p.slot * p.hist_ld + p.C] = t0;
    if (p.first_token) *p.first_token = t0;
  }
  for (int n = tid; n < p.d; n += blockDim.x)
    p.hpend[(long long)p.slot * (p.max_k + 1) * p.d + n] = p.x[(long long)p.x_row * p.d + n];
}

}  // namespace ocrdec
