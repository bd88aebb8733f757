// Small kernels of the decode step: pass setup (embedding gather, row
// metadata, draft inputs), greedy acceptance with commit and rollback, the
// benchmark's forced-acceptance override, and the RoPE table.  (Routing is in
// route.cuh, the MoE FFN in moe.cuh.)
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "route.cuh"

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

constexpr int kMaxK = 3;  // draft tokens per step

struct BlockSync {
  __device__ void operator()() const { __syncthreads(); }
};



// ---------------------------------------------------------------------------
// RoPE table: cos/sin of pos * theta^(-2i/Dh), float64 math, float32 values
// ---------------------------------------------------------------------------


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



// Draft input rows: fcin[r] = [RMSNorm(h_r) * g_h ; RMSNorm(e_r) * g_e] as high and
// low bf16 parts (fcin, fcin_lo), at most kRmax rows,
// where (h_r, e_r, pos_r) come from one of three row sources:
//   mode 0 (recursion 1): the pending pairs of each slot - verifier hidden
//          hpend[b][i] and the embedding of the committed token at pos+1;
//   mode 1 (recursion j >= 2): the draft's own output hidden xd[last_row[b]] and
//          the embedding of draft token dtok[b], at kv_len + j - 2;
//   mode 2 (prefill): verifier hidden x[p - p0] and the next context input
//          (visual vector or prompt embedding) for pairs p in [p0, p0 + n).
// Dynamic shared memory of draft_setup_kernel: gains, hidden rows, embedding rows.
constexpr size_t draft_setup_smem_bytes(int d) { return (size_t)d * (4 + kRmax * 4 + kRmax * 2); }

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
  bf16* fcin;            // [R][2d] high parts
  bf16* fcin_lo;         // [R][2d] low parts
  PassRows* rows;        // written
  const PassRows* rows_prev;  // mode 1: rows of the previous recursion (last_row)
  int* status;
};



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

// Greedy acceptance of every slot given the verifier tokens g (in shared or
// global memory) by nthreads cooperating threads; sync() spans exactly them.
// Thread b < B reads its slot's proposals and state before using any of them.
// copy_hidden: also copy the verifier residual rows of each slot into hpend
// (callers that copy them elsewhere pass false).
template <class Sync>
__device__ void accept_rows(const AcceptParams& p, const int* g_all, int tid, int nthreads, Sync sync,
                            bool copy_hidden) {
  __shared__ int s_a[kRmax];
  const int K1 = p.k + 1;
  if (tid < p.B) {
    const int b = tid;
    const int* g = g_all + b * K1;
    int prop[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) prop[j] = j < p.k ? p.proposals[b * p.k + j] : -1;
    SlotState* sp = p.slots + b;
    const SlotState st = *sp;
    int a = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (a == j && j < p.k && prop[j] == g[j]) a = j + 1;
    const int n = st.kv_len;
    for (int i = 0; i <= p.k; ++i) p.committed[b * K1 + i] = i <= a ? g[i] : -1;
    for (int i = 0; i <= a; ++i) p.hist[b * p.hist_ld + n + 1 + i] = g[i];
    p.n_committed[b] = a + 1;
    sp->kv_len = n + a + 1;
    sp->n_generated = st.n_generated + a + 1;
    sp->bonus = g[a];
    sp->steps = st.steps + 1;
    sp->tau_sum = st.tau_sum + a + 1;
    sp->hist[a] = st.hist[a] + 1;
    sp->pending = a + 1;
    sp->pend_pos = n;
    s_a[b] = a;
  }
  if (!copy_hidden) return;
  sync();
  for (int b = 0; b < p.B; ++b)
    for (int idx = tid; idx < (s_a[b] + 1) * p.d; idx += nthreads) {
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



}  // namespace ocrdec
