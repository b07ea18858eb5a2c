// 8-element vectors (16 bytes of bf16, 32 bytes of fp32) for the streaming kernels.
#pragma once

#include "la_common.cuh"

namespace la {

template <typename T> struct Vec8;
// Raw: the vector as loaded (kept in registers until it is needed as floats).
template <> struct Vec8<uint16_t> {
  using Raw = uint4;
  __device__ __forceinline__ static Raw load_raw(const uint16_t* p) { return *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ static void load(const uint16_t* p, float* f) { unpack(load_raw(p), f); }
  __device__ __forceinline__ static void unpack(const Raw& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16_bits_to_f32(static_cast<uint16_t>(w[i] & 0xFFFFu));
      f[2 * i + 1] = bf16_bits_to_f32(static_cast<uint16_t>(w[i] >> 16));
    }
  }
  __device__ __forceinline__ static void store(uint16_t* p, const float* f) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]);
    u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]);
    u.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <> struct Vec8<float> {
  struct Raw {
    float4 a, b;
  };
  __device__ __forceinline__ static Raw load_raw(const float* p) {
    return Raw{*reinterpret_cast<const float4*>(p), *reinterpret_cast<const float4*>(p + 4)};
  }
  __device__ __forceinline__ static void load(const float* p, float* f) { unpack(load_raw(p), f); }
  __device__ __forceinline__ static void unpack(const Raw& r, float* f) {
    f[0] = r.a.x; f[1] = r.a.y; f[2] = r.a.z; f[3] = r.a.w;
    f[4] = r.b.x; f[5] = r.b.y; f[6] = r.b.z; f[7] = r.b.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
};

}  // namespace la
