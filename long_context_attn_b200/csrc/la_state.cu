// Sequence-parallel prefill support: the state entering one rank's chunk of a sequence.
//
// "MiniMax-01系列大模型：超长上下文与多模态能力深度解析与部署指南", section 2.1.3 (LASP+:
// sequence parallelism made for Lightning Attention) splits one long sequence across GPUs.
// The state of "六十四：MiniMax-01" section 3 is a plain sum, S_t = S0 + sum_{i <= t}
// phi(k_i) v_i^T, so the state entering chunk r is S0 plus the sum of the states that the
// chunks before it reach from a zero state.  After every rank has computed its chunk state
// and the states have been gathered, this kernel forms that exclusive prefix, adding in
// rank order so every rank gets the same bits for the same prefix.
#include "la_common.cuh"

namespace la {

__global__ void __launch_bounds__(256) state_prefix_kernel(const float4* __restrict__ gathered, int rank,
                                                           const float4* __restrict__ state0,
                                                           float4* __restrict__ out, int64_t n4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = state0 ? state0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < rank; ++r) {
      const float4 b = gathered[static_cast<int64_t>(r) * n4 + i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    out[i] = a;
  }
}

}  // namespace la

extern "C" la_status lightning_attn_state_prefix(const float* gathered, int world, int rank, const float* state0,
                                                 float* out, int H, int D, la_stream_t stream) {
  if (!gathered || !out || world < 1 || rank < 0 || rank >= world || H < 1 || D < 1) return LA_ERR_INVALID_ARG;
  const int64_t n = static_cast<int64_t>(H) * D * D;
  if (n % 4 != 0) return LA_ERR_INVALID_ARG;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(gathered) || !a16(out) || (state0 && !a16(state0))) return LA_ERR_INVALID_ARG;
  const int64_t n4 = n / 4;
  const int blocks = static_cast<int>(n4 / 256 < 2048 ? (n4 + 255) / 256 : 2048);
  la::state_prefix_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(gathered), rank, reinterpret_cast<const float4*>(state0),
      reinterpret_cast<float4*>(out), n4);
  return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
