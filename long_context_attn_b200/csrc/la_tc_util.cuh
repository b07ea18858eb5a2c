// Small device helpers shared by the tensor-core kernels: shared/global memory accesses
// with explicit cache behaviour, the fp64 and counter atomics of the cross-head norm
// exchange, bounded mbarrier waits and the SiLU of two packed bf16 values.
#pragma once

#include <stdint.h>

#include "la_common.cuh"
#include "la_sm100.cuh"

namespace la {
namespace tcu {
namespace {   // internal linkage: every kernel file gets its own copy

using namespace sm100;

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Streaming 16-byte store that does not allocate in L1.
__device__ __forceinline__ void st_global_na(void* p, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
// 16-byte load from L2 (never a stale L1 line: the data may have been written by another SM).
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_cg_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ uint4 ld_nc_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// 32-byte accesses (one full sector per thread).
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
__device__ __forceinline__ void st_na_v8(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ double ld_cg_f64(const double* p) {
  double v;
  asm volatile("ld.global.cg.f64 %0, [%1];" : "=d"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_add_f64(double* p, double v) {
  asm volatile("red.relaxed.gpu.global.add.f64 [%0], %1;" ::"l"(p), "d"(v) : "memory");
}
__device__ __forceinline__ void red_add_relaxed_u32(unsigned int* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_release_u32(unsigned int* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// Bounded wait for phase `parity` of an mbarrier (acquire at CTA scope).  Returns false, after
// recording a timeout or because another role already did, when the CTA is aborting.
// The polling loop is out of line so that only the first test is inlined at each site.
// The polling thread suspends in each test (up to 20 us), so that waiting warps leave the
// issue slots to the warps that work.
constexpr uint32_t kSuspendNs = 20000;
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, int* abort_flag, ErrRec* err, uint32_t site,
                                       uint32_t index) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = wait_limit_ns(err);
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
    if (globaltimer_ns() - t0 > lim) {
      report(err, LA_ERR_TIMEOUT, site, index, parity);
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, int* abort_flag, ErrRec* err, uint32_t site,
                                     uint32_t index) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, err, site, index);
}
// The same wait taken by every lane of a warp; the outcome is warp-uniform so that the
// .sync.aligned tcgen05 instructions that follow see a converged warp.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, int* abort_flag, ErrRec* err,
                                          uint32_t site, uint32_t index) {
  const bool ok = wait(bar, parity, abort_flag, err, site, index);
  return __all_sync(0xFFFFFFFFu, ok);
}
// Wait used only to drain work already issued (bounded, never records).
__device__ __noinline__ void drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}
// Bounded poll (one thread) until the counter at c reaches W; false when the CTA is
// aborting or the wait ran out (recorded).
__device__ __noinline__ bool poll_count(unsigned int* c, uint32_t W, int* abort_flag, ErrRec* err, uint32_t index) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = wait_limit_ns(err);
  for (uint32_t ns = 32; ld_acquire_gpu(c) < W; ns = ns < 256 ? 2 * ns : ns) {
    __nanosleep(ns);
    if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
    if (globaltimer_ns() - t0 > lim) {
      report(err, LA_ERR_TIMEOUT, SITE_TC_NORM_WAIT, index, ld_acquire_gpu(c));
      *reinterpret_cast<volatile int*>(abort_flag) = 1;
      return false;
    }
  }
  return true;
}

// SiLU of the two bf16 values packed in x, in packed bf16 arithmetic, from
// sigmoid(x) = (1 + tanh(x/2)) / 2:  h = x/2 (exact), t = tanh(h) (tanh.approx.bf16x2: one
// MUFU op for both halves, t rounded to bf16), SiLU(x) = h + h t (one fused multiply-add,
// rounded once to bf16).  Three instructions per pair: the tensor-core kernels run their
// feature map on warps that share the SM's issue slots with the latency-critical roles.
__device__ __forceinline__ uint32_t silu2_bf16(uint32_t x) {
  uint32_t h, t, r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(h) : "r"(x), "r"(0x3F003F00u));
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(h));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(h), "r"(t), "r"(h));
  return r;
}
__device__ __forceinline__ uint4 silu8(uint4 v) {
  return make_uint4(silu2_bf16(v.x), silu2_bf16(v.y), silu2_bf16(v.z), silu2_bf16(v.w));
}

}  // namespace
}  // namespace tcu
}  // namespace la
