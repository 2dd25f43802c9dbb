// Small device helpers for the sm_100a engine: inline PTX for mbarriers, bulk
// copies, scoped loads/reductions, packed fp32 FMA, and warp reductions.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace fmoe {

// Device status word (one per GPU that loads the library).  Kernels OR error
// bits into it; fmoe_get_status() reads and clears it.
__device__ unsigned int g_fmoe_status = 0;

enum : unsigned {
  kStatusGridBarrierTimeout = 1u,  // a grid-wide wait ran past its time limit
  kStatusCopyTimeout = 2u,         // a bulk copy did not complete in time
  kStatusCtaWaitTimeout = 4u,      // an intra-CTA hand-off ran past its time limit
  kStatusMmaTimeout = 8u,          // tensor-core work did not complete in time
};

__device__ __forceinline__ void set_status(unsigned bits) { atomicOr(&g_fmoe_status, bits); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)::"memory");
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier (CTA scope) ---------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// Test phase `parity` of `bar`; if it is not complete the thread may sleep in
// hardware for up to ~suspend_ns (it wakes early when the phase completes).
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t suspend_ns = 20000) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}
#ifdef FMOE_TRACE_BUILD
// Trace builds count wait-loop iterations: [0] mbarrier waits, [1] activation
// polls, [2] routing polls.
__device__ unsigned long long g_fmoe_spins[4];
#define FMOE_SPIN(i) atomicAdd(&g_fmoe_spins[i], 1ull)
#else
#define FMOE_SPIN(i) do { } while (0)
#endif

// Wait for phase `parity` of `bar` to complete, for at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    FMOE_SPIN(0);
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// ---- bulk copies (no tensor map; each copy lands in this CTA only) ------------
// Order this thread's earlier generic-proxy shared-memory accesses before
// subsequent async-proxy (bulk copy) writes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Order this thread's earlier generic-proxy accesses of global memory (and
// what it acquired) before its subsequent async-proxy accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// this CTA's shared memory; completion is signalled on `bar` as tx bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch: let the next grid on the stream be
// scheduled (its CTAs start as this grid's CTAs leave), and wait until the
// previous grid on the stream has completed with its writes visible (no-op
// when the launch had no programmatic dependency).
__device__ __forceinline__ void grid_dep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Prefetch `bytes` (multiple of 16, 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- scoped global accesses ---------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
// Two consecutive 64-bit words (16-byte aligned), each read single-copy atomically.
__device__ __forceinline__ void ld_relaxed_gpu_v2u64(const unsigned long long* p, unsigned long long& a,
                                                     unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0,%1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ void st_relaxed_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Read-only input either in shared memory (plain load) or in global memory
// written by an earlier kernel (non-coherent cached load).
template <bool kGlobal, typename T>
__device__ __forceinline__ T ld_in(const T* p) {
  if constexpr (kGlobal) return __ldg(p);
  else return *p;
}

// ---- packed fp32 pairs (sm_100 f32x2) -------------------------------------------
__device__ __forceinline__ uint64_t pk_u32(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float2 unpk_f32(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
// acc.{lo,hi} = a.{lo,hi} * b.{lo,hi} + acc.{lo,hi}, round to nearest, denormals kept.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// ---- reductions -------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Two warp sums at once: returns the sum of `a` over the warp on lanes 0..15
// and the sum of `b` on lanes 16..31 (5 shuffles instead of 10).
__device__ __forceinline__ float warp_sum2_split(float a, float b, int lane) {
  const bool hi = (lane & 16) != 0;
  float keep = hi ? b : a;
  keep += __shfl_xor_sync(0xffffffffu, hi ? a : b, 16);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
  return keep;
}
// Four warp sums at once: lane l returns the sum of y[(l >> 3) & 3] over the
// warp (so lanes 0, 8, 16, 24 hold rows 0..3; 6 shuffles instead of 20).
__device__ __forceinline__ float warp_sum4_split(const float (&y)[4], int lane) {
  const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0;
  float k0 = b4 ? y[2] : y[0], k1 = b4 ? y[3] : y[1];
  k0 += __shfl_xor_sync(0xffffffffu, b4 ? y[0] : y[2], 16);
  k1 += __shfl_xor_sync(0xffffffffu, b4 ? y[1] : y[3], 16);
  float keep = b3 ? k1 : k0;
  keep += __shfl_xor_sync(0xffffffffu, b3 ? k0 : k1, 8);
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) keep += __shfl_xor_sync(0xffffffffu, keep, o);
  return keep;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---- bf16 -------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t f32_to_bf16_rne(float f) {
  const uint32_t u = __float_as_uint(f);
  return (uint32_t)(((uint64_t)u + 0x7FFFull + ((u >> 16) & 1u)) >> 16) & 0xFFFFu;
}

// 2^e as a float for e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

}  // namespace fmoe
