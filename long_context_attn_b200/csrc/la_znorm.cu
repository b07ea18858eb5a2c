// Normalised variant of the Lightning Attention forward ("六十四：MiniMax-01", section 3): the
// linear-attention form with its normaliser, which the deployment drops in favour of
// RMSNorm.  Alongside S the recurrence carries z_t = z_{t-1} + phi(k_t) and
//     y_t = phi(q_t)^T S_t / (phi(q_t) . z_t),
// after which the usual output transform (raw, RMSNorm, RMSNorm * sigmoid(g)) applies.
//
// The numerator is the plain raw-mode prefill (the tensor-core or CUDA-core kernel, which
// also carries S).  The denominators need only phi(k) summed over the tokens, so they come
// from a chunked scan here, HBM-streaming and parallel over (sequence, head, chunk):
//   z_chunk_sum_kernel   sum of phi(k) over each chunk of kChunk tokens
//   z_den_kernel         z entering the chunk (z0 + earlier chunks), then token by token
//                        z_t += phi(k_t) and den_t = phi(q_t) . z_t; z_out from the last chunk
//   znorm_transform_kernel  per token: y / den per head, then the output transform, in place
#include "la_common.cuh"

namespace la {
namespace {

constexpr int kChunk = 256;     // tokens per scan chunk
constexpr int kBatch = 16;      // tokens per inner batch of z_den_kernel

template <typename T> __device__ __forceinline__ float ld(const T* p) { return load_elem<T>(p, 0); }

__device__ __forceinline__ float feat(float x, int phi_identity) { return phi_identity ? x : silu_accurate(x); }

// Rows [lo, lo + len) of sequence s; false if they do not lie inside [0, tokens) (a malformed
// cu_seqlens, which the prefill pass reports), in which case the caller touches nothing.
__device__ __forceinline__ bool seq_rows(const int* cu, int T_fixed, int s, int64_t tokens, int64_t& lo,
                                         int64_t& len) {
  if (cu) {
    lo = __ldg(cu + s);
    len = static_cast<int64_t>(__ldg(cu + s + 1)) - lo;
  } else {
    lo = static_cast<int64_t>(s) * T_fixed;
    len = T_fixed;
  }
  return lo >= 0 && len >= 0 && lo + len <= tokens;
}

// grid (max_chunks, H, nseq), D threads: thread d sums phi(k)[., h, d] over the chunk.
template <typename T, int D>
__global__ void __launch_bounds__(D) z_chunk_sum_kernel(const T* __restrict__ k, float* __restrict__ sums,
                                                        const int* cu, int T_fixed, int64_t tokens, int H,
                                                        int max_chunks, int phi_identity) {
  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z, d = threadIdx.x;
  int64_t lo, len;
  if (!seq_rows(cu, T_fixed, s, tokens, lo, len)) return;
  const int64_t t0 = static_cast<int64_t>(c) * kChunk;
  if (t0 >= len) return;
  const int64_t t1 = t0 + kChunk < len ? t0 + kChunk : len;
  float acc = 0.f;
  const int64_t stride = static_cast<int64_t>(H) * D;
  const T* p = k + (lo + t0) * stride + static_cast<int64_t>(h) * D + d;
#pragma unroll 8
  for (int64_t t = t0; t < t1; ++t, p += stride) acc += feat(ld(p), phi_identity);
  sums[((static_cast<int64_t>(s) * H + h) * max_chunks + c) * D + d] = acc;
}

// grid (max_chunks, H, nseq), D threads.  den [tokens, H] fp32; z_out [nseq, H, D] or null.
template <typename T, int D>
__global__ void __launch_bounds__(D) z_den_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                  const float* __restrict__ sums, const float* __restrict__ z_in,
                                                  float* __restrict__ den, float* __restrict__ z_out, const int* cu,
                                                  int T_fixed, int64_t tokens, int H, int max_chunks,
                                                  int phi_identity) {
  constexpr int kWarps = D / 32;
  __shared__ float red[kWarps][kBatch];
  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z, d = threadIdx.x;
  const int lane = d & 31, warp = d >> 5;
  int64_t lo, len;
  if (!seq_rows(cu, T_fixed, s, tokens, lo, len)) return;
  const int64_t nchunks = (len + kChunk - 1) / kChunk;
  const bool last = c == (nchunks > 0 ? nchunks - 1 : 0);
  const int64_t t0 = static_cast<int64_t>(c) * kChunk;
  if (t0 >= len && !last) return;
  const int64_t sh = static_cast<int64_t>(s) * H + h;
  float z = z_in ? z_in[sh * D + d] : 0.f;
  for (int j = 0; j < c; ++j) z += sums[(sh * max_chunks + j) * D + d];
  const int64_t t1 = t0 + kChunk < len ? t0 + kChunk : len;
  const int64_t stride = static_cast<int64_t>(H) * D;
  for (int64_t b0 = t0; b0 < t1; b0 += kBatch) {
    const int n = static_cast<int>(t1 - b0 < kBatch ? t1 - b0 : kBatch);
    float part[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      part[i] = 0.f;
      if (i < n) {
        const int64_t off = (lo + b0 + i) * stride + static_cast<int64_t>(h) * D + d;
        z += feat(ld(k + off), phi_identity);
        part[i] = feat(ld(q + off), phi_identity) * z;
      }
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part[i] += __shfl_xor_sync(0xffffffffu, part[i], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kBatch; ++i) red[warp][i] = part[i];
    }
    __syncthreads();
    if (d < n) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) t += red[w][d];
      den[(lo + b0 + d) * H + h] = t;
    }
    __syncthreads();
  }
  if (last && z_out) z_out[sh * D + d] = z;
}

// One CTA per token: y / den per head, then RAW / RMSNORM / RMSNORM_GATE, in place on io.
template <typename T>
__global__ void __launch_bounds__(256) znorm_transform_kernel(T* io, const float* __restrict__ den,
                                                              const T* __restrict__ g, const float* __restrict__ w,
                                                              int H, int D, int mode, float eps) {
  __shared__ float red[8];
  const int64_t row = blockIdx.x;
  const int HD = H * D;
  T* y = io + row * HD;
  const float* dn = den + row * H;
  if (mode == LA_OUT_RAW) {
    for (int c = threadIdx.x; c < HD; c += blockDim.x) store_elem<T>(y, c, load_elem<T>(y, c) / dn[c / D]);
    return;
  }
  float ss = 0.f;
  for (int c = threadIdx.x; c < HD; c += blockDim.x) {
    const float x = load_elem<T>(y, c) / dn[c / D];
    ss = fmaf(x, x, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) tot += red[i];
  const float r = 1.0f / sqrtf(tot / static_cast<float>(HD) + eps);
  for (int c = threadIdx.x; c < HD; c += blockDim.x) {
    float o = load_elem<T>(y, c) / dn[c / D] * r;
    if (w) o *= __ldg(w + c);
    if (mode == LA_OUT_RMSNORM_GATE) o *= sigmoid_accurate(load_elem<T>(g, row * HD + c));
    store_elem<T>(y, c, o);
  }
}

template <typename T, int D>
cudaError_t launch_scan_t(const void* q, const void* k, const float* z_in, float* sums, float* den, float* z_out,
                          const int* cu, int nseq, int T_fixed, int64_t tokens, int H, int max_chunks,
                          int phi_identity, cudaStream_t stream) {
  const dim3 grid(max_chunks, H, nseq);
  z_chunk_sum_kernel<T, D><<<grid, D, 0, stream>>>(static_cast<const T*>(k), sums, cu, T_fixed, tokens, H,
                                                   max_chunks, phi_identity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  z_den_kernel<T, D><<<grid, D, 0, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k), sums, z_in, den,
                                             z_out, cu, T_fixed, tokens, H, max_chunks, phi_identity);
  return cudaGetLastError();
}

}  // namespace

int znorm_max_chunks(int max_len) { return max_len > 0 ? (max_len + kChunk - 1) / kChunk : 1; }

cudaError_t launch_znorm_scan(const void* q, const void* k, const float* z_in, float* sums, float* den, float* z_out,
                              const int* cu, int nseq, int T_fixed, int max_len, int64_t tokens, int H, int D,
                              la_dtype dt, int phi_identity, cudaStream_t stream) {
  const int mc = znorm_max_chunks(max_len);
  if (dt == LA_BF16)
    return D == 128 ? launch_scan_t<uint16_t, 128>(q, k, z_in, sums, den, z_out, cu, nseq, T_fixed, tokens, H, mc,
                                                   phi_identity, stream)
                    : launch_scan_t<uint16_t, 64>(q, k, z_in, sums, den, z_out, cu, nseq, T_fixed, tokens, H, mc,
                                                  phi_identity, stream);
  return D == 128 ? launch_scan_t<float, 128>(q, k, z_in, sums, den, z_out, cu, nseq, T_fixed, tokens, H, mc,
                                              phi_identity, stream)
                  : launch_scan_t<float, 64>(q, k, z_in, sums, den, z_out, cu, nseq, T_fixed, tokens, H, mc,
                                             phi_identity, stream);
}

cudaError_t launch_znorm_transform(void* io, const float* den, const void* g, const float* w, int64_t tokens, int H,
                                   int D, int mode, float eps, la_dtype dt, cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  if (dt == LA_BF16)
    znorm_transform_kernel<uint16_t><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
        static_cast<uint16_t*>(io), den, static_cast<const uint16_t*>(g), w, H, D, mode, eps);
  else
    znorm_transform_kernel<float><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
        static_cast<float*>(io), den, static_cast<const float*>(g), w, H, D, mode, eps);
  return cudaGetLastError();
}

}  // namespace la
