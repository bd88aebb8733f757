// GEMV epilogue that finishes a pass step in the GEMV's last CTA: greedy
// acceptance after the verifier's LM-head argmax (saves one launch per step).
#pragma once

#include "gemv.cuh"
#include "step_kernels.cuh"

namespace ocrdec {

// LM-head argmax, then - in the last CTA - acceptance, commit and rollback.
struct EpiArgmaxAccept {
  struct Params {
    EpiArgmax::Params am;
    AcceptParams accept;
  };
  __device__ static void apply(const Params& p, const GemvShape& s, const WarpOut& o, const RowSet& rs, int lane) {
    EpiArgmax::apply(p.am, s, o, rs, lane);
  }
  __device__ static void finish(const Params& p, const GemvShape& s, int R, int tid) {
    __shared__ int s_tok[kRmax];
    // every CTA copies its share of the verifier residual rows of all k + 1
    // positions into hpend (the accepted ones are used; the rest is ignored),
    // so the last CTA keeps only the acceptance bookkeeping
    {
      const AcceptParams& a = p.accept;
      const int K1 = a.k + 1, total = a.B * K1 * a.d;
      const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
      for (int idx = (int)blockIdx.x * per + tid; idx < min(total, ((int)blockIdx.x + 1) * per); idx += kConsumers) {
        const int row = idx / a.d, n = idx - row * a.d, b = row / K1, i = row - b * K1;
        a.hpend[((long long)b * (a.max_k + 1) + i) * a.d + n] = a.x[(long long)row * a.d + n];
      }
    }
    if (!EpiArgmax::merge(p.am, s, R, tid, s_tok)) return;
    named_sync(1, kConsumers);
    accept_rows(p.accept, s_tok, tid, kConsumers, ConsumerBarrier{}, false);
  }
};

template <>
__device__ __forceinline__ void epi_init<EpiArgmaxAccept>(int tid) { EpiArgmax::init(tid); }

}  // namespace ocrdec
