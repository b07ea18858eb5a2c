// Normalised variant of the Lightning Attention forward ("六十四：MiniMax-01", section 3): the
// linear-attention form with its normaliser, which the deployment drops in favour of
// RMSNorm.  Alongside S the recurrence carries z_t = z_{t-1} + phi(k_t) and
//     y_t = phi(q_t)^T S_t / (phi(q_t) . z_t),
// after which the usual output transform (raw, RMSNorm, RMSNorm * sigmoid(g)) applies.
//
// The numerator is the plain raw-mode prefill (the tensor-core or CUDA-core kernel, which
// also carries S).  The denominators need only phi(k) summed over the tokens, so they come
// from a chunked scan here, HBM-streaming and parallel over (sequence, head, chunk):
//   z_chunk_sum_kernel   sum of phi(k) over each chunk of kChunk tokens (16-byte vectors)
//   z_prefix_kernel      those sums turned into their exclusive prefix over the chunks
//   z_den_kernel         z entering the chunk (z0 + earlier chunks), then token by token
//                        z_t += phi(k_t) and den_t = phi(q_t) . z_t; z_out from the last chunk
//                        (8 dimensions per lane, the dot product reduced across a lane group)
//   znorm_transform_kernel  per token: y / den per head, then the output transform (in place
//                        or into another buffer)
#include "la_common.cuh"
#include "la_vec.cuh"

namespace la {
namespace {

constexpr int kChunk = 256;     // tokens per scan chunk

template <typename T> __device__ __forceinline__ float ld(const T* p) { return load_elem<T>(p, 0); }

// SiLU for the scan, x / (1 + e^-x), from the CUDA fast intrinsics (__expf, __fdividef: a few
// ulp; the exponent is clamped so the divisor stays below 2^126, where __fdividef is exact
// enough).  The scan evaluates phi three times per element of q and k, and the accurate
// form (expf and an IEEE division) made it instruction-bound.
__device__ __forceinline__ float feat(float x, int phi_identity) {
  return phi_identity ? x : __fdividef(x, 1.0f + __expf(fminf(-x, 80.0f)));
}

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

// grid (max_chunks, H, nseq), 256 threads: D/8 threads cover a row with 8-element vectors,
// 256/(D/8) row groups stride through the chunk, and the groups' partial sums of phi(k) are
// added in shared memory (fixed order).
template <typename T, int D>
__global__ void __launch_bounds__(256) z_chunk_sum_kernel(const T* __restrict__ k, float* __restrict__ sums,
                                                          const int* cu, int T_fixed, int64_t tokens, int H,
                                                          int max_chunks, int phi_identity) {
  constexpr int kTpr = D / 8, kGroups = 256 / kTpr;
  __shared__ float part[kGroups][D];
  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int grp = threadIdx.x / kTpr, col = (threadIdx.x % kTpr) * 8;
  int64_t lo, len;
  if (!seq_rows(cu, T_fixed, s, tokens, lo, len)) return;
  const int64_t t0 = static_cast<int64_t>(c) * kChunk;
  if (t0 >= len) return;
  const int64_t t1 = t0 + kChunk < len ? t0 + kChunk : len;
  const int64_t stride = static_cast<int64_t>(H) * D;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int64_t t = t0 + grp; t < t1; t += kGroups) {
    float x[8];
    Vec8<T>::load(k + (lo + t) * stride + static_cast<int64_t>(h) * D + col, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += feat(x[i], phi_identity);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[grp][col + i] = acc[i];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float t = 0.f;
    for (int gI = 0; gI < kGroups; ++gI) t += part[gI][d];
    sums[((static_cast<int64_t>(s) * H + h) * max_chunks + c) * D + d] = t;
  }
}

// grid (H, nseq), D threads: the chunk sums of one (sequence, head) become their exclusive
// prefix, in place (chunk c then holds the sum of phi(k) over the chunks before it).
__global__ void __launch_bounds__(128) z_prefix_kernel(float* __restrict__ sums, const int* cu, int T_fixed,
                                                       int64_t tokens, int H, int D, int max_chunks) {
  const int h = blockIdx.x, s = blockIdx.y;
  int64_t lo, len;
  if (!seq_rows(cu, T_fixed, s, tokens, lo, len)) return;
  const int nch = static_cast<int>((len + kChunk - 1) / kChunk);
  float* p = sums + (static_cast<int64_t>(s) * H + h) * max_chunks * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float run = 0.f;
#pragma unroll 8
    for (int c = 0; c < nch; ++c) {
      const float t = p[static_cast<int64_t>(c) * D + d];
      p[static_cast<int64_t>(c) * D + d] = run;
      run += t;
    }
  }
}

// grid (ceil(max_chunks / kItems), H, nseq), 256 threads.  One item = one (chunk, head) of a
// sequence, served by D/8 lanes of one warp, each owning 8 of the D dimensions of z.  The
// item's lanes add the earlier chunks' sum (the prefix) to z_in, then walk the chunk token by token
// (loads of 4 tokens in flight): z += phi(k_t), den_t = phi(q_t) . z reduced over the lanes.
// den [tokens, H] fp32; z_out [nseq, H, D] from the last chunk (a zero-length sequence has
// one, which copies z_in).  No block-wide barrier: items finish independently.
template <typename T, int D>
__global__ void __launch_bounds__(256, 2) z_den_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                    const float* __restrict__ sums, const float* __restrict__ z_in,
                                                    float* __restrict__ den, float* __restrict__ z_out, const int* cu,
                                                    int T_fixed, int64_t tokens, int H, int max_chunks,
                                                    int phi_identity) {
  constexpr int kTpr = D / 8, kItems = 256 / kTpr, kAhead = 4;
  const int h = blockIdx.y, s = blockIdx.z;
  const int c = blockIdx.x * kItems + threadIdx.x / kTpr;
  const int j = threadIdx.x % kTpr;
  const int lane = threadIdx.x & 31;
  const unsigned gmask = ((kTpr == 32) ? 0xffffffffu : ((1u << kTpr) - 1u)) << (lane & ~(kTpr - 1));
  int64_t lo, len;
  if (c >= max_chunks || !seq_rows(cu, T_fixed, s, tokens, lo, len)) return;
  const int64_t nchunks = (len + kChunk - 1) / kChunk;
  const bool last = c == (nchunks > 0 ? nchunks - 1 : 0);
  const int64_t t0 = static_cast<int64_t>(c) * kChunk;
  if (t0 >= len && !last) return;
  const int64_t sh = static_cast<int64_t>(s) * H + h;
  float z[8];
  if (z_in) {
    Vec8<float>::load(z_in + sh * D + 8 * j, z);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] = 0.f;
  }
  if (c < nchunks) {   // the exclusive prefix of the chunk sums (z_prefix_kernel)
    float a[8];
    Vec8<float>::load(sums + (sh * max_chunks + c) * D + 8 * j, a);
#pragma unroll
    for (int i = 0; i < 8; ++i) z[i] += a[i];
  }
  const int64_t t1 = t0 + kChunk < len ? t0 + kChunk : len;
  const int64_t stride = static_cast<int64_t>(H) * D;
  const int64_t col = static_cast<int64_t>(h) * D + 8 * j;
  for (int64_t b0 = t0; b0 < t1; b0 += kAhead) {
    const int n = static_cast<int>(t1 - b0 < kAhead ? t1 - b0 : kAhead);
    float kr[kAhead][8], qr[kAhead][8];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (u < n) {
        Vec8<T>::load(k + (lo + b0 + u) * stride + col, kr[u]);
        Vec8<T>::load(q + (lo + b0 + u) * stride + col, qr[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (u < n) {
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          z[i] += feat(kr[u][i], phi_identity);
          part = fmaf(feat(qr[u][i], phi_identity), z[i], part);
        }
#pragma unroll
        for (int o = kTpr / 2; o > 0; o >>= 1) part += __shfl_xor_sync(gmask, part, o);
        if (j == 0) den[(lo + b0 + u) * H + h] = part;
      }
    }
  }
  if (last && z_out) Vec8<float>::store(z_out + sh * D + 8 * j, z);
}

// One CTA per token: y / den per head, then RAW / RMSNORM / RMSNORM_GATE, in place on io.
// 8-element vectors; the H reciprocals of the token's denominators sit in shared memory.
// With den null it is the output transform alone (the prefill's norm when too many heads
// for the fused exchange).  sigmoid(g) from the fast intrinsics (a few ulp, exponent
// clamped), as in the scan.
template <typename T, int D>
__global__ void __launch_bounds__(256) znorm_transform_kernel(const T* src, T* dst, const float* __restrict__ den,
                                                              const T* __restrict__ g, const float* __restrict__ w,
                                                              int H, int mode, float eps) {
  constexpr int kV = 8;
  __shared__ float rden[kMaxNormWidth / 64];
  __shared__ float red[8];
  const int64_t row = blockIdx.x;
  const int HD = H * D;
  const T* y = src + row * HD;   // src and dst may be the same buffer (each element is read
  T* yo = dst + row * HD;        // by the thread that writes it, after the row's reduction)
  for (int h = threadIdx.x; h < H; h += blockDim.x) rden[h] = den ? 1.0f / den[row * H + h] : 1.0f;
  __syncthreads();
  float r = 1.0f;
  if (mode != LA_OUT_RAW) {
    float ss = 0.f;
    for (int c = threadIdx.x * kV; c < HD; c += blockDim.x * kV) {
      float x[kV];
      Vec8<T>::load(y + c, x);
      const float s = rden[c / D];
#pragma unroll
      for (int i = 0; i < kV; ++i) ss = fmaf(x[i] * s, x[i] * s, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) tot += red[i];
    r = 1.0f / sqrtf(tot / static_cast<float>(HD) + eps);
  }
  for (int c = threadIdx.x * kV; c < HD; c += blockDim.x * kV) {
    float x[kV], gv[kV];
    Vec8<T>::load(y + c, x);
    if (mode == LA_OUT_RMSNORM_GATE) Vec8<T>::load(g + row * HD + c, gv);
    const float s = rden[c / D] * r;
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      float o = x[i] * s;
      if (mode != LA_OUT_RAW && w) o *= __ldg(w + c + i);
      if (mode == LA_OUT_RMSNORM_GATE) o *= __fdividef(1.0f, 1.0f + __expf(fminf(-gv[i], 80.0f)));
      x[i] = o;
    }
    Vec8<T>::store(yo + c, x);
  }
}

template <typename T, int D>
cudaError_t launch_scan_t(const void* q, const void* k, const float* z_in, float* sums, float* den, float* z_out,
                          const int* cu, int nseq, int T_fixed, int64_t tokens, int H, int max_chunks,
                          int phi_identity, cudaStream_t stream) {
  const dim3 grid(max_chunks, H, nseq);
  z_chunk_sum_kernel<T, D><<<grid, 256, 0, stream>>>(static_cast<const T*>(k), sums, cu, T_fixed, tokens, H,
                                                   max_chunks, phi_identity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  z_prefix_kernel<<<dim3(H, nseq), D, 0, stream>>>(sums, cu, T_fixed, tokens, H, D, max_chunks);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 grid_den((max_chunks + 256 / (D / 8) - 1) / (256 / (D / 8)), H, nseq);
  z_den_kernel<T, D><<<grid_den, 256, 0, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k), sums, z_in, den,
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

cudaError_t launch_output_transform(const void* src, void* dst, const float* den, const void* g, const float* w,
                                    int64_t tokens, int H, int D, int mode, float eps, la_dtype dt,
                                    cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  const unsigned n = static_cast<unsigned>(tokens);
  if (dt == LA_BF16) {
    auto* a = static_cast<const uint16_t*>(src);
    auto* b = static_cast<uint16_t*>(dst);
    auto* gg = static_cast<const uint16_t*>(g);
    if (D == 128) znorm_transform_kernel<uint16_t, 128><<<n, 256, 0, stream>>>(a, b, den, gg, w, H, mode, eps);
    else znorm_transform_kernel<uint16_t, 64><<<n, 256, 0, stream>>>(a, b, den, gg, w, H, mode, eps);
  } else {
    auto* a = static_cast<const float*>(src);
    auto* b = static_cast<float*>(dst);
    auto* gg = static_cast<const float*>(g);
    if (D == 128) znorm_transform_kernel<float, 128><<<n, 256, 0, stream>>>(a, b, den, gg, w, H, mode, eps);
    else znorm_transform_kernel<float, 64><<<n, 256, 0, stream>>>(a, b, den, gg, w, H, mode, eps);
  }
  return cudaGetLastError();
}

cudaError_t launch_znorm_transform(void* io, const float* den, const void* g, const float* w, int64_t tokens, int H,
                                   int D, int mode, float eps, la_dtype dt, cudaStream_t stream) {
  return launch_output_transform(io, io, den, g, w, tokens, H, D, mode, eps, dt, stream);
}

}  // namespace la
