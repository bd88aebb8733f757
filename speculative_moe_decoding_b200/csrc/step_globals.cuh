// The stand-alone kernels of the decode step (launched by the engine only):
// pass setup, routing, combine, acceptance, forced proposals, RoPE table.
#pragma once

#include "step_kernels.cuh"

namespace ocrdec {

__global__ void __launch_bounds__(256) route_kernel(const RouteParams p) {
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) s_abort = status_bad(p.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();
  route_rows(p, min(*p.nrows, kRmax), tid, 256, BlockSync{});
}

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  pdl_wait();
  if (status_bad(p.status)) return;
  pdl_trigger();
  TraceMarks tm;
  if (threadIdx.x == 0) tm.t0 = gtimer();  // trace: after the dependency wait
  const int R = min(*p.nrows, kRmax);
  const int nslot = p.top_k + p.S;
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < R * p.d) {
    int r = idx / p.d, n = idx - r * p.d;
    const float* yr = p.y + (long long)r * nslot * p.d + n;
    float t = 0.f;
    for (int s = 0; s < p.top_k; ++s) t = __fmaf_rn(p.gates[r * p.top_k + s], yr[(long long)s * p.d], t);
    for (int s = 0; s < p.S; ++s) t = __fadd_rn(t, yr[(long long)(p.top_k + s) * p.d]);
    p.x[idx] = __fadd_rn(p.x[idx], t);
  }
  if (threadIdx.x == 0) trace_end(p.status, 44, tm);
}

__global__ void rope_table_kernel(float2* tab, int cap, int Dh, double theta) {
  int half = Dh / 2;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)cap * half) return;
  int pos = (int)(idx / half), i = (int)(idx % half);
  double inv = pow(theta, -2.0 * (double)i / (double)Dh);
  double a = (double)pos * inv;
  tab[idx] = make_float2((float)cos(a), (float)sin(a));
}

__global__ void __launch_bounds__(256) verify_setup_kernel(const VerifySetupParams p) {
  __shared__ int s_tok[kRmax];
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  const int K1 = p.k + 1, R = p.B * K1;
  pdl_wait();
  TraceMarks tm;
  if (tid == 0) tm.t0 = gtimer();
  if (tid == 0) s_bad = status_bad(p.status);
  __syncthreads();
  if (s_bad) return;
  if (tid < R) {
    const int b = tid / K1, i = tid - b * K1;
    const int kv = p.slots[b].kv_len;
    int t = i == 0 ? p.slots[b].bonus : p.proposals[b * p.k + i - 1];
    if (kv + K1 > p.cap) {
      set_status(p.status, OCRDEC_ECAPACITY);
      s_bad = 1;
    }
    if (t < 0 || t >= p.vocab) {  // caller-supplied proposal out of range
      set_status(p.status, OCRDEC_EINVAL);
      s_bad = 1;
      t = 0;
    }
    p.rows->slot[tid] = b;
    p.rows->pos[tid] = kv + i;
    p.rows->tok[tid] = t;
    s_tok[tid] = t;
  }
  if (tid < kRmax) {
    const bool live = tid < p.B;
    p.rows->slot_row0[tid] = live ? tid * K1 : 0;
    p.rows->slot_nrows[tid] = live ? K1 : 0;
    p.rows->last_row[tid] = live ? tid * K1 + p.k : 0;
  }
  if (tid == 0) {
    p.rows->n = R;
    p.rows->n_last = p.B;
  }
  __syncthreads();
  if (s_bad) return;
  pdl_trigger();
  // embedding gather: every row's loads are issued before any is consumed
#pragma unroll
  for (int r = 0; r < kRmax; ++r) {
    if (r >= R) break;
    const bf16* e = p.embed + (long long)s_tok[r] * p.d;
    float* xr = p.x + (long long)r * p.d;
#pragma unroll 8
    for (int n = tid; n < p.d; n += 256) xr[n] = bf2f(e[n]);
  }
  if (tid == 0) trace_end(p.status, 42, tm);
}

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

__global__ void __launch_bounds__(256) draft_setup_kernel(const DraftSetupParams p) {
  __shared__ int s_bad;
  __shared__ PassRows pr;
  __shared__ int s_pend[kRmax], s_ppos[kRmax], s_kv[kRmax], s_prev_last[kRmax];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  TraceMarks tm;
  if (tid == 0) tm.t0 = gtimer();
  if (tid == 0) s_bad = status_bad(p.status);
  if (tid < kRmax) {
    const bool live = tid < p.B;
    s_pend[tid] = live && p.mode == 0 ? min(p.slots[tid].pending, p.max_k + 1) : 0;
    s_ppos[tid] = live && p.mode == 0 ? p.slots[tid].pend_pos : 0;
    s_kv[tid] = live && p.mode == 1 ? p.slots[tid].kv_len : 0;
    s_prev_last[tid] = p.mode == 1 ? p.rows_prev->last_row[tid] : 0;
  }
  __syncthreads();
  if (s_bad) return;
  pdl_trigger();
  // row metadata: thread r < kRmax fills row r; thread kRmax + b the per-slot fields
  if (tid < kRmax) {
    const int r = tid;
    int n = 0, slot = -1, pos = 0, tok = 0;
    if (p.mode == 0) {
      int acc = 0;
      for (int b = 0; b < p.B; ++b) {
        if (r >= acc && r < acc + s_pend[b]) { slot = b; pos = s_ppos[b] + (r - acc); }
        acc += s_pend[b];
      }
      n = acc;
      if (slot >= 0) tok = p.hist[slot * p.hist_ld + pos + 1];
    } else if (p.mode == 1) {
      n = p.B;
      if (r < p.B) { slot = r; pos = s_kv[r] + p.j - 2; tok = p.dtok[r * p.dtok_stride]; }
    } else {
      n = p.n;
      if (r < p.n) {
        slot = p.slot;
        pos = p.p0 + r;
        tok = pos + 1 < p.n_visual ? -1 : p.prompt[pos + 1 - p.n_visual];
      }
    }
    pr.slot[r] = slot < 0 ? 0 : slot;
    pr.pos[r] = pos;
    pr.tok[r] = tok;
    if (r == 0) {
      pr.n = n;
      pr.n_last = p.mode == 2 ? 1 : p.B;
    }
  } else if (tid < 2 * kRmax) {
    const int b = tid - kRmax;
    int row0 = 0, nrows = 0;
    if (p.mode == 0) {
      for (int q = 0; q < b && q < p.B; ++q) row0 += s_pend[q];
      nrows = b < p.B ? s_pend[b] : 0;
    } else if (p.mode == 1) {
      row0 = b;
      nrows = b < p.B ? 1 : 0;
    } else {
      nrows = b == p.slot ? p.n : 0;
    }
    pr.slot_row0[b] = row0;
    pr.slot_nrows[b] = nrows;
    pr.last_row[b] = p.mode == 2 ? p.n - 1 : (nrows > 0 ? row0 + nrows - 1 : 0);
  }
  __syncthreads();
  // fcin[r] = [RMSNorm(h_r) * g_h ; RMSNorm(e_r) * g_e] as high / low bf16 parts: all 256
  // threads per row, the sums of every row reduced in one round
  const int d = p.d;
  const int nrow = pr.n;
  __shared__ float red[8][kRmax][2];
  __shared__ const float* s_h[kRmax];
  __shared__ const float* s_ev[kRmax];
  __shared__ const bf16* s_eb[kRmax];
  if (tid < nrow) {
    const int r = tid, b = pr.slot[r];
    const float* h;
    if (p.mode == 0) h = p.hpend + ((long long)b * (p.max_k + 1) + (r - pr.slot_row0[b])) * d;
    else if (p.mode == 1) h = p.xd + (long long)s_prev_last[b] * d;
    else h = p.xv + (long long)r * d;
    const int tok = pr.tok[r];
    s_h[r] = h;
    s_ev[r] = (p.mode == 2 && tok < 0) ? p.visual + (long long)(pr.pos[r] + 1) * d : nullptr;
    s_eb[r] = p.embed + (long long)(tok < 0 ? 0 : tok) * d;
  }
  __syncthreads();
  float sh[kRmax], se[kRmax];
#pragma unroll
  for (int r = 0; r < kRmax; ++r) {
    sh[r] = 0.f;
    se[r] = 0.f;
    if (r < nrow) {
      const float* h = s_h[r];
      const float* ev = s_ev[r];
      const bf16* eb = s_eb[r];
#pragma unroll 4
      for (int n = tid; n < d; n += 256) {
        float hv = h[n];
        float e = ev ? ev[n] : bf2f(eb[n]);
        sh[r] = __fmaf_rn(hv, hv, sh[r]);
        se[r] = __fmaf_rn(e, e, se[r]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sh[r] = __fadd_rn(sh[r], __shfl_xor_sync(0xffffffffu, sh[r], o));
      se[r] = __fadd_rn(se[r], __shfl_xor_sync(0xffffffffu, se[r], o));
    }
    if (lane == 0) { red[warp][r][0] = sh[r]; red[warp][r][1] = se[r]; }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRmax; ++r) {
    if (r >= nrow) break;
    float a = 0.f, c = 0.f;
    for (int w = 0; w < 8; ++w) { a = __fadd_rn(a, red[w][r][0]); c = __fadd_rn(c, red[w][r][1]); }
    const float ch = rsqrtf(__fadd_rn(__fdiv_rn(a, (float)d), p.eps));
    const float ce = rsqrtf(__fadd_rn(__fdiv_rn(c, (float)d), p.eps));
    const float* h = s_h[r];
    const float* ev = s_ev[r];
    const bf16* eb = s_eb[r];
#pragma unroll 4
    for (int n = tid; n < d; n += 256) {
      float e = ev ? ev[n] : bf2f(eb[n]);
      const float zh = __fmul_rn(__fmul_rn(h[n], ch), bf2f(p.g_h[n]));
      const float ze = __fmul_rn(__fmul_rn(e, ce), bf2f(p.g_e[n]));
      const bf16 hh = f2bf(zh), he = f2bf(ze);
      p.fcin[(long long)r * 2 * d + n] = hh;
      p.fcin[(long long)r * 2 * d + d + n] = he;
      p.fcin_lo[(long long)r * 2 * d + n] = f2bf(__fsub_rn(zh, bf2f(hh)));
      p.fcin_lo[(long long)r * 2 * d + d + n] = f2bf(__fsub_rn(ze, bf2f(he)));
    }
  }
  // publish the row metadata
  int* dst = reinterpret_cast<int*>(p.rows);
  const int* src = reinterpret_cast<const int*>(&pr);
  for (int i = tid; i < (int)(sizeof(PassRows) / sizeof(int)); i += 256) dst[i] = src[i];
  if (tid == 0) trace_end(p.status, 43, tm);
}

__global__ void __launch_bounds__(256) accept_kernel(const AcceptParams p) {
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  pdl_wait();
  if (tid == 0) s_abort = status_bad(p.status);
  __syncthreads();
  if (s_abort) return;
  pdl_trigger();
  accept_rows(p, p.g, tid, 256, BlockSync{}, true);
}

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
