// The stand-alone kernels of the decode step (launched by the engine only):
// pass setup, acceptance, forced proposals, RoPE table.
#pragma once

#include "step_kernels.cuh"

namespace ocrdec {

// Row-wise e4m3 quantisation of a bfloat16 matrix [N][K] (the draft's copy of
// the LM head): row n is scaled so that its largest magnitude maps to 448
// (e4m3's largest finite value), rounded to nearest even, and inv[n] gets the
// scale's inverse (all-zero rows: scale 1).  One warp per row.
__global__ void __launch_bounds__(256) quantize_rows_e4m3_kernel(const bf16* W, int N, int K, unsigned char* W8,
                                                                float* inv) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (n >= N) return;
  const bf16* w = W + (size_t)n * K;
  float amax = 0.f;
  for (int k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(bf2f(w[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  for (int k = lane; k < K; k += 32) W8[(size_t)n * K + k] = (unsigned char)f2e4m3(__fmul_rn(bf2f(w[k]), scale));
  if (lane == 0) inv[n] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
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
  if (tid == 0) s_bad = 0;
  __syncthreads();
  pdl_wait();
  TraceMarks tm;
  if (tid == 0) tm.t0 = gtimer();
  // the status, slot state and proposals are read together
  int kv = 0, t = 0;
  if (tid < R) {
    const int b = tid / K1, i = tid - b * K1;
    kv = p.slots[b].kv_len;
    t = i == 0 ? p.slots[b].bonus : p.proposals[b * p.k + i - 1];
  }
  if (tid == 0 && status_bad(p.status)) s_bad = 1;
  if (tid < R) {
    const int b = tid / K1, i = tid - b * K1;
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
  // embedding gather, 8 columns per load: every load is issued before any
  // store (R * d / 8 <= 8 * 256)
  const int per_row = p.d / 8, total = R * per_row;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = tid + 256 * i;
    if (idx < total) {
      const int r = idx / per_row, c = idx - r * per_row;
      v[i] = ld_nc_v4(p.embed + (long long)s_tok[r] * p.d + c * 8);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = tid + 256 * i;
    if (idx < total) {
      const int r = idx / per_row, c = idx - r * per_row;
      const bf16* b = reinterpret_cast<const bf16*>(&v[i]);
      float4* xr = reinterpret_cast<float4*>(p.x + (long long)r * p.d + c * 8);
      xr[0] = make_float4(bf2f(b[0]), bf2f(b[1]), bf2f(b[2]), bf2f(b[3]));
      xr[1] = make_float4(bf2f(b[4]), bf2f(b[5]), bf2f(b[6]), bf2f(b[7]));
    }
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

// The draft's input rows (DraftSetupParams).  The gains, each row's hidden
// state and its token embedding arrive in shared memory by bulk copies (the
// gains before the grid dependency wait); the whole block then normalises
// each row.
__global__ void __launch_bounds__(256) draft_setup_kernel(const DraftSetupParams p) {
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ int s_bad;
  __shared__ PassRows pr;
  __shared__ int s_pend[kRmax], s_ppos[kRmax], s_kv[kRmax], s_prev_last[kRmax], s_dtok[kRmax];
  __shared__ uint64_t bars[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d;
  bf16* sg = reinterpret_cast<bf16*>(dsm);                  // [2][d] g_h, g_e
  float* sh_rows = reinterpret_cast<float*>(dsm + 4 * d);  // [kRmax][d] hidden rows
  bf16* se_rows = reinterpret_cast<bf16*>(sh_rows + kRmax * d);  // [kRmax][d] embedding rows
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bars[0], 4 * d);
    bulk_g2s(sg, p.g_h, 2 * d, &bars[0]);
    bulk_g2s(sg + d, p.g_e, 2 * d, &bars[0]);
  }
  pdl_wait();
  TraceMarks tm;
  if (tid == 0) tm.t0 = gtimer();
  // status, slot state, previous draft tokens and rows: one round of loads
  if (tid == 0) s_bad = status_bad(p.status);
  if (tid < kRmax) {
    const bool live = tid < p.B;
    s_pend[tid] = live && p.mode == 0 ? min(p.slots[tid].pending, p.max_k + 1) : 0;
    s_ppos[tid] = live && p.mode == 0 ? p.slots[tid].pend_pos : 0;
    s_kv[tid] = live && p.mode == 1 ? p.slots[tid].kv_len : 0;
    s_prev_last[tid] = p.mode == 1 ? p.rows_prev->last_row[tid] : 0;
    s_dtok[tid] = live && p.mode == 1 ? p.dtok[tid * p.dtok_stride] : 0;
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) mbar_wait(&bars[0], 0, p.status);  // the gains' copy lands before exit
    return;
  }
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
      if (r < p.B) { slot = r; pos = s_kv[r] + p.j - 2; tok = s_dtok[r]; }
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
  const int nrow = min(pr.n, kRmax);
  // one thread requests every row: the hidden state (float) and the token
  // embedding (bf16); a visual vector (prefill) is read in place
  if (tid == 0) {
    uint32_t bytes = 0;
    for (int r = 0; r < nrow; ++r) bytes += 4 * d + (pr.tok[r] < 0 ? 0 : 2 * d);
    mbar_arrive_expect_tx(&bars[1], bytes);
    for (int r = 0; r < nrow; ++r) {
      const int b = pr.slot[r], tok = pr.tok[r];
      const float* h;
      if (p.mode == 0) h = p.hpend + ((long long)b * (p.max_k + 1) + (r - pr.slot_row0[b])) * d;
      else if (p.mode == 1) h = p.xd + (long long)s_prev_last[b] * d;
      else h = p.xv + (long long)r * d;
      bulk_g2s(sh_rows + r * d, h, 4 * d, &bars[1]);
      if (tok >= 0) bulk_g2s(se_rows + r * d, p.embed + (long long)tok * d, 2 * d, &bars[1]);
    }
  }
  mbar_wait(&bars[0], 0, p.status);
  mbar_wait(&bars[1], 0, p.status);
  if (tid == 0) tm.t1 = gtimer();
  // fcin[r] as high / low bf16 parts, all 256 threads on every row: sums of
  // squares (thread, then warp, then the 8 warps in order), then the outputs
  __shared__ float red[kRmax][8][2];
  __shared__ float s_scale[kRmax][2];
  for (int r = 0; r < nrow; ++r) {
    const float* hr = sh_rows + r * d;
    const bf16* er = se_rows + r * d;
    const float* ev = pr.tok[r] < 0 ? p.visual + (long long)(pr.pos[r] + 1) * d : nullptr;
    float a = 0.f, c = 0.f;
    for (int n = tid; n < d; n += 256) {
      const float hv = hr[n];
      const float e = ev ? ev[n] : bf2f(er[n]);
      a = __fmaf_rn(hv, hv, a);
      c = __fmaf_rn(e, e, c);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
      c = __fadd_rn(c, __shfl_xor_sync(0xffffffffu, c, o));
    }
    if (lane == 0) {
      red[r][warp][0] = a;
      red[r][warp][1] = c;
    }
  }
  __syncthreads();
  if (tid < 2 * nrow) {
    const int r = tid >> 1, w = tid & 1;
    float v = 0.f;
    for (int q = 0; q < 8; ++q) v = __fadd_rn(v, red[r][q][w]);
    s_scale[r][w] = rsqrtf(__fadd_rn(__fdiv_rn(v, (float)d), p.eps));
  }
  __syncthreads();
  for (int idx = tid; idx < nrow * d; idx += 256) {  // column pairs of [h ; e]
    const int r = idx / d, n = 2 * (idx - r * d);
    const float* hr = sh_rows + r * d;
    const bf16* er = se_rows + r * d;
    const float* ev = pr.tok[r] < 0 ? p.visual + (long long)(pr.pos[r] + 1) * d : nullptr;
    float z[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int cidx = n + t;
      z[t] = cidx < d ? __fmul_rn(__fmul_rn(hr[cidx], s_scale[r][0]), bf2f(sg[cidx]))
                      : __fmul_rn(__fmul_rn(ev ? ev[cidx - d] : bf2f(er[cidx - d]), s_scale[r][1]), bf2f(sg[cidx]));
    }
    const __nv_bfloat162 zh = __floats2bfloat162_rn(z[0], z[1]);
    const __nv_bfloat162 zl = __floats2bfloat162_rn(__fsub_rn(z[0], __low2float(zh)),
                                                     __fsub_rn(z[1], __high2float(zh)));
    *reinterpret_cast<__nv_bfloat162*>(p.fcin + (long long)r * 2 * d + n) = zh;
    *reinterpret_cast<__nv_bfloat162*>(p.fcin_lo + (long long)r * 2 * d + n) = zl;
  }
  if (tid == 0) tm.t2 = gtimer();
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
