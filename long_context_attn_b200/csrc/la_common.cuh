// Shared device helpers of the Lightning Attention CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/lightning_attn.h"

namespace la {

// ---------------------------------------------------------------------------------------
// Error record: the first 256 bytes of every workspace.  The first failing site wins.
// ---------------------------------------------------------------------------------------
struct ErrRec {
  unsigned int status;   // la_status, 0 = no error
  unsigned int site;     // where (see Site)
  unsigned int index;    // work item / tile / sequence
  unsigned int extra;    // site-specific detail
  unsigned int timeout_ms;   // optional override of the bounded-wait limit (0 = default)
  unsigned int inject;       // host-injected fault for failure tests (0 = none)
  unsigned int pad[58];
};
static_assert(sizeof(ErrRec) == 256, "error record is 256 bytes");

enum Site : unsigned int {
  SITE_NONE = 0,
  SITE_TC_PRODUCER = 1,
  SITE_TC_MMA = 2,
  SITE_TC_TRANSFORM = 3,
  SITE_TC_CONVERT = 4,
  SITE_TC_EPILOGUE = 5,
  SITE_TC_NORM_WAIT = 6,
  SITE_VARLEN_CU = 7,
  SITE_TC_TEARDOWN = 8,
};

enum Inject : unsigned int {
  INJECT_NONE = 0,
  // The CTA of work column 0 never publishes its norm partials: every other CTA's
  // bounded wait on that tile must run out and report LA_ERR_TIMEOUT.
  INJECT_SKIP_PUBLISH = 1,
};

__device__ __forceinline__ void report(ErrRec* rec, unsigned int status, unsigned int site,
                                       unsigned int index, unsigned int extra) {
  if (rec == nullptr) return;
  if (atomicCAS(&rec->status, 0u, status) == 0u) {
    rec->site = site;
    rec->index = index;
    rec->extra = extra;
    __threadfence();
  }
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Default limit of every device-side wait.  A correct run never comes close; the limit
// only turns a logic error into an error status instead of a hung GPU.
constexpr uint64_t kDefaultWaitNs = 4000000000ull;

__device__ __forceinline__ uint64_t wait_limit_ns(const ErrRec* rec) {
  unsigned int ms = rec ? rec->timeout_ms : 0u;
  return ms ? static_cast<uint64_t>(ms) * 1000000ull : kDefaultWaitNs;
}

// ---------------------------------------------------------------------------------------
// Element conversions
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

template <typename T> __device__ __forceinline__ float load_elem(const T* p, int64_t i);
template <> __device__ __forceinline__ float load_elem<float>(const float* p, int64_t i) { return p[i]; }
template <> __device__ __forceinline__ float load_elem<uint16_t>(const uint16_t* p, int64_t i) {
  return bf16_bits_to_f32(p[i]);
}

template <typename T> __device__ __forceinline__ void store_elem(T* p, int64_t i, float v);
template <> __device__ __forceinline__ void store_elem<float>(float* p, int64_t i, float v) { p[i] = v; }
template <> __device__ __forceinline__ void store_elem<uint16_t>(uint16_t* p, int64_t i, float v) {
  p[i] = f32_to_bf16_bits(v);
}

// ---------------------------------------------------------------------------------------
// Feature map and gate.
// "MiniMax-Text-01 405B MoE模型架构与训练策略解析", section 2.1: phi = SiLU, gate = sigmoid.
// ---------------------------------------------------------------------------------------
// Accurate forms (fp32 paths, decode, norm): SiLU(x) = x / (1 + e^-x).
__device__ __forceinline__ float silu_accurate(float x) { return x / (1.0f + expf(-x)); }
__device__ __forceinline__ float sigmoid_accurate(float x) { return 1.0f / (1.0f + expf(-x)); }

// One-MUFU forms for the bf16 tensor-core path, from the identity
// sigmoid(x) = (1 + tanh(x/2)) / 2, so SiLU(x) = h + h * tanh(h) with h = x/2.
// tanh.approx.f32 has a relative error near 2^-11, below the bf16 rounding that follows.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_fast(float x) {
  const float h = 0.5f * x;
  return fmaf(h, tanh_approx(h), h);
}
__device__ __forceinline__ float sigmoid_fast(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

// Largest sum of squares over the head concatenation the norm modes accept (H*D).
constexpr int kMaxNormWidth = 16384;

}  // namespace la
