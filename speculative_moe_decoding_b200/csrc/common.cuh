// Device helpers shared by the ocrdec kernels (sm_100a).
//
// Bulk (TMA) copies global -> shared with mbarrier completion, bounded waits
// that report a status code instead of hanging, bfloat16 unpacking, and the
// sticky device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ocrdec.h"

namespace ocrdec {

typedef __nv_bfloat16 bf16;

// Upper bound of try_wait rounds before a wait is declared stuck.  Each round
// suspends for up to the hardware's time slice, so this is well above a second.
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr int kRmax = 8;  // rows per pass (pass rows are the 8 MMA columns)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ bool status_bad(const int* status) {
  return status && *(volatile const int*)status != 0;
}

// ---- timeline tracer ---------------------------------------------------------
// The status word heads a small region: status[1] != 0 enables tracing,
// status[2] counts records, and TraceRec entries start 256 bytes in.  Each
// traced CTA appends (start time, duration, kernel tag, SM) when it finishes.
constexpr int kTraceCap = 1 << 19;
struct TraceRec {
  unsigned long long t0;   // the CTA passed its dependency wait
  unsigned int d1, d2, d3; // ns from t0 to the end of phases 1, 2, 3 (3 = CTA end)
  unsigned short tag;
  unsigned short sm;
};

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned int sm_id() {
  unsigned int r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

// Phase marks of one CTA (kept by the thread that records).
struct TraceMarks {
  unsigned long long t0 = 0, t1 = 0, t2 = 0;
};

__device__ __forceinline__ void trace_end(int* status, int tag, const TraceMarks& m) {
  if (!status || !*(volatile int*)(status + 1)) return;
  unsigned int i = atomicAdd(reinterpret_cast<unsigned int*>(status + 2), 1u);
  if (i >= (unsigned)kTraceCap) return;
  TraceRec* r = reinterpret_cast<TraceRec*>(reinterpret_cast<char*>(status) + 256) + i;
  const unsigned long long t3 = gtimer();
  r->t0 = m.t0;
  r->d1 = (unsigned int)((m.t1 ? m.t1 : t3) - m.t0);
  r->d2 = (unsigned int)((m.t2 ? m.t2 : t3) - m.t0);
  r->d3 = (unsigned int)(t3 - m.t0);
  r->tag = (unsigned short)tag;
  r->sm = (unsigned short)sm_id();
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false (and
// records OCRDEC_ETIMEOUT) if it does not complete within kSpinLimit rounds.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  set_status(status, OCRDEC_ETIMEOUT);
  return false;
}

// ---- bulk copy global -> shared (TMA unit, no multicast) ------------------
// L2 policy for data read once per step (weights): their lines are the first
// to be evicted, so the step's reused data - KV caches, activations, kernel
// code - stays in L2 while gigabytes of weights stream past.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---- programmatic dependent launch ----------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- consumer-only named barrier ------------------------------------------
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- bfloat16 ---------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ float bf2f(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ bf16 f2bf(float v) { return __float2bfloat16_rn(v); }
__device__ __forceinline__ float round_bf(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// 16 bytes = 8 bfloat16 -> 8 floats
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf_lo(u.x); f[1] = bf_hi(u.x);
  f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
  f[4] = bf_lo(u.z); f[5] = bf_hi(u.z);
  f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
  uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(b));
  return lo | (hi << 16);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Plain (coherent) 16-byte global load, for data written by earlier kernels of
// the same stream (never stale through the non-coherent path).
__device__ __forceinline__ uint4 ld_v4(const void* p) { return *reinterpret_cast<const uint4*>(p); }

}  // namespace ocrdec
