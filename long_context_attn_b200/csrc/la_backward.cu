// Backward pass of the Lightning Attention forward: the element-wise and per-token kernels
// around three causal linear-attention passes (which run on the prefill kernels).
//
// The pages give no gradient formulas ("MiniMax-Text-01 405B MoE模型架构与训练策略解析",
// section 2.1, names the operator used in training); the chain rule through the forward
// of "六十四：MiniMax-01" section 3 (S_t = S0 + sum_{i<=t} phi(k_i) v_i^T, y_t = S_t^T phi(q_t))
// gives, per head, with dy the gradient of the raw output:
//   dphi(q_t) = sum_{i<=t} (dy_t . v_i) phi(k_i) + S0 dy_t
//   dphi(k_i) = sum_{t>=i} (v_i . dy_t) phi(q_t)
//   dv_i      = sum_{t>=i} (phi(k_i) . phi(q_t)) dy_t
//   dS0       = sum_t phi(q_t) dy_t^T
// Each line is a causal linear attention with the identity feature map: the first runs
// forward in time (queries dy, keys v, values phi(k), initial state S0^T); the other two
// run on the time-reversed sequences (queries rho(v), keys rho(dy), values rho(phi(q)); and
// queries rho(phi(k)), keys rho(phi(q)), values rho(dy), whose final state is dS0).  The
// kernels here supply what those passes take and finish what they give:
//   bwd_norm_gate_token_kernel  dy and dg from dout through RMSNorm(y) * w * sigmoid(g)
//   bwd_norm_gate_kernel  the same with the norm weight's gradient (CTAs over blocks of tokens)
//   bwd_prep_kernel       phi(k) and the reversed copies rho(v), rho(dy), rho(phi(q)), rho(phi(k))
//   bwd_post_kernel       dq = dphi(q) * phi'(q); un-reverses dk (times phi'(k)) and dv in place
//   transpose_states      S0^T for the first pass
// When the prefill kernel can walk time backwards itself (the tensor-core path), the
// reversed copies are not needed: bwd_feat_kernel writes phi(q) and phi(k), the last two
// passes run in reverse time (the third taking phi on the raw k and q in the kernel), and
// bwd_scale_kernel multiplies dq and dk by phi'.
// All of them are HBM-streaming kernels: 16-byte vectors, grid-stride loops over rows.
#include "la_common.cuh"
#include "la_vec.cuh"

namespace la {
namespace {

constexpr int kVec = 8;   // elements per vector (16 bytes of bf16)

// sigmoid(x) = 1 / (1 + e^-x) from the CUDA fast intrinsics (__expf, __fdividef: a few ulp;
// the exponent is clamped so the divisor stays below 2^126).  These streaming kernels
// evaluate it once or twice per element; the accurate form (expf and an IEEE division)
// left them instruction-bound below the HBM rate.
__device__ __forceinline__ float sig(float x) { return __fdividef(1.0f, 1.0f + __expf(fminf(-x, 80.0f))); }
__device__ __forceinline__ float feature(float x, int phi_identity) { return phi_identity ? x : x * sig(x); }
// d/dx [x sigmoid(x)] = sigmoid(x) (1 + x (1 - sigmoid(x)))
__device__ __forceinline__ float dfeature(float x, int phi_identity) {
  if (phi_identity) return 1.0f;
  const float s = sig(x);
  return s * (1.0f + x * (1.0f - s));
}

// Row `row` of the packed tokens: first row and one-past-last row of its sequence.
__device__ __forceinline__ void seq_bounds(const int* cu, int nseq, int T_fixed, int64_t row, int64_t& lo,
                                           int64_t& hi) {
  if (!cu) {
    const int64_t s = row / T_fixed;
    lo = s * T_fixed;
    hi = lo + T_fixed;
    return;
  }
  int a = 0, b = nseq;   // largest s with cu[s] <= row; empty sequences are skipped
  while (b - a > 1) {
    const int m = (a + b) >> 1;
    if (__ldg(cu + m) <= row) a = m; else b = m;
  }
  lo = __ldg(cu + a);
  hi = __ldg(cu + a + 1);
}

// dy and dg alone (no dw), one CTA per token: many short CTAs per SM keep more rows in
// flight than the token-blocked kernel below can, whose raw vectors fill the registers
// (measured on the 128K-token, H*D = 8192 backward: 2.7 ms against 3.4 ms).  Same formulas;
// the second loop re-reads the row (from L1/L2).
template <typename T>
__global__ void __launch_bounds__(256) bwd_norm_gate_token_kernel(const T* y, const T* __restrict__ g,
                                                            const T* __restrict__ dout, const float* __restrict__ w,
                                                            T* dy, T* __restrict__ dg, int HD, int gate, float eps) {
  __shared__ float red[2][8];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * HD;
  float ss = 0.f, su = 0.f;
  for (int c = threadIdx.x * kVec; c < HD; c += blockDim.x * kVec) {
    float yv[kVec], dv[kVec], gv[kVec];
    Vec8<T>::load(y + base + c, yv);
    Vec8<T>::load(dout + base + c, dv);
    if (gate) Vec8<T>::load(g + base + c, gv);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const float s = gate ? sig(gv[i]) : 1.0f;
      const float u = dv[i] * (w ? __ldg(w + c + i) : 1.0f) * s;
      ss = fmaf(yv[i], yv[i], ss);
      su = fmaf(u, yv[i], su);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    su += __shfl_xor_sync(0xffffffffu, su, o);
  }
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) { red[0][warp] = ss; red[1][warp] = su; }
  __syncthreads();
  ss = 0.f; su = 0.f;
  for (int i = 0; i < nw; ++i) { ss += red[0][i]; su += red[1][i]; }
  const float r = 1.0f / sqrtf(ss / static_cast<float>(HD) + eps);
  const float coef = r * r * r * su / static_cast<float>(HD);
  for (int c = threadIdx.x * kVec; c < HD; c += blockDim.x * kVec) {
    float yv[kVec], dv[kVec], gv[kVec], o[kVec], og[kVec];
    Vec8<T>::load(y + base + c, yv);
    Vec8<T>::load(dout + base + c, dv);
    if (gate) Vec8<T>::load(g + base + c, gv);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const float s = gate ? sig(gv[i]) : 1.0f;
      const float wc = w ? __ldg(w + c + i) : 1.0f;
      o[i] = r * dv[i] * wc * s - coef * yv[i];
      og[i] = dv[i] * yv[i] * r * wc * s * (1.0f - s);
    }
    Vec8<T>::store(dy + base + c, o);
    if (gate) Vec8<T>::store(dg + base + c, og);
  }
}

// The same for bf16 rows of exactly 2048 VPT elements (H * D = 8192 at 64 heads of 128):
// each thread keeps its VPT vectors of y, dout and g, and the gate's sigmoid, in registers
// between the two sums and the outputs, so every row is read from memory once.
template <int VPT>
__global__ void __launch_bounds__(256) bwd_norm_gate_row_kernel(const uint16_t* y, const uint16_t* __restrict__ g,
                                                          const uint16_t* __restrict__ dout,
                                                          const float* __restrict__ w, uint16_t* dy,
                                                          uint16_t* __restrict__ dg, int gate, float eps) {
  constexpr int HD = 256 * kVec * VPT;
  __shared__ float red[2][8];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * HD;
  uint4 yr[VPT], dr[VPT], gr[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int c = (threadIdx.x + 256 * j) * kVec;
    yr[j] = Vec8<uint16_t>::load_raw(y + base + c);
    dr[j] = Vec8<uint16_t>::load_raw(dout + base + c);
    gr[j] = gate ? Vec8<uint16_t>::load_raw(g + base + c) : make_uint4(0, 0, 0, 0);
  }
  float sg[VPT][kVec];
  float ss = 0.f, su = 0.f;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int c = (threadIdx.x + 256 * j) * kVec;
    float yv[kVec], dv[kVec], gv[kVec];
    Vec8<uint16_t>::unpack(yr[j], yv);
    Vec8<uint16_t>::unpack(dr[j], dv);
    Vec8<uint16_t>::unpack(gr[j], gv);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      sg[j][i] = gate ? sig(gv[i]) : 1.0f;
      const float u = dv[i] * (w ? __ldg(w + c + i) : 1.0f) * sg[j][i];
      ss = fmaf(yv[i], yv[i], ss);
      su = fmaf(u, yv[i], su);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    su += __shfl_xor_sync(0xffffffffu, su, o);
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { red[0][warp] = ss; red[1][warp] = su; }
  __syncthreads();
  ss = 0.f; su = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) { ss += red[0][i]; su += red[1][i]; }
  const float r = 1.0f / sqrtf(ss / static_cast<float>(HD) + eps);
  const float coef = r * r * r * su / static_cast<float>(HD);
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int c = (threadIdx.x + 256 * j) * kVec;
    float yv[kVec], dv[kVec], o[kVec], og[kVec];
    Vec8<uint16_t>::unpack(yr[j], yv);
    Vec8<uint16_t>::unpack(dr[j], dv);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const float s = sg[j][i];
      const float wc = w ? __ldg(w + c + i) : 1.0f;
      o[i] = r * dv[i] * wc * s - coef * yv[i];
      og[i] = dv[i] * yv[i] * r * wc * s * (1.0f - s);
    }
    Vec8<uint16_t>::store(dy + base + c, o);
    if (gate) Vec8<uint16_t>::store(dg + base + c, og);
  }
}

// The norm/gate backward with the norm weight's gradient, in one pass over the tokens.  RAW
// is not launched (dy = dout).  With r = 1/sqrt(mean(y^2) + eps), s = sigmoid(g) (1 without
// the gate) and u = dout * w * s, per token:
//   dy = r u - r^3 y (sum u y) / HD,    dg = dout * y * r * w * s * (1 - s),
// and per column dw_c = sum over tokens of dout_c * y_c * r * s_c.
// CTA b takes the contiguous tokens [b * per, min((b + 1) * per, tokens)); thread j owns the
// columns (j + i * blockDim.x) * 8 .. + 7, i < kV.  Per token each thread loads its vectors of
// y, dout and g once (kept raw in registers), the CTA reduces sum(y^2) and sum(u y), and the
// thread writes dy and dg and adds its dw terms in registers.  Several CTAs per SM keep
// enough loads in flight; the reduction buffer alternates between two halves by token
// parity, so one barrier per token suffices.  With `partial` set, the CTA's dw column sums
// go to partial[b] (summed over b in order by bwd_norm_weight_sum_kernel: deterministic).
// y and dy may be the same buffer (each element is read by the thread that writes it).
template <typename T, int kV>
__global__ void __launch_bounds__(512) bwd_norm_gate_kernel(const T* y, const T* __restrict__ g,
                                                            const T* __restrict__ dout, const float* __restrict__ w,
                                                            T* dy, T* __restrict__ dg, float* __restrict__ partial,
                                                            int64_t tokens, int64_t per, int HD, int gate, float eps) {
  using Raw = typename Vec8<T>::Raw;
  __shared__ float2 red[2][16];
  const int nwarp = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t t1 = t0 + per < tokens ? t0 + per : tokens;
  const float inv_hd = 1.0f / static_cast<float>(HD);
  float acc[kV][kVec];
#pragma unroll
  for (int i = 0; i < kV; ++i)
#pragma unroll
    for (int e = 0; e < kVec; ++e) acc[i][e] = 0.f;
  int par = 0;
  for (int64_t t = t0; t < t1; ++t, par ^= 1) {
    const int64_t base = t * HD;
    Raw ry[kV], rd[kV], rg[kV];
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int c = (threadIdx.x + i * blockDim.x) * kVec;
      if (c < HD) {
        ry[i] = Vec8<T>::load_raw(y + base + c);
        rd[i] = Vec8<T>::load_raw(dout + base + c);
        if (gate) rg[i] = Vec8<T>::load_raw(g + base + c);
      }
    }
    float ss = 0.f, su = 0.f;
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int c = (threadIdx.x + i * blockDim.x) * kVec;
      if (c < HD) {
        float yv[kVec], dv[kVec], gv[kVec];
        Vec8<T>::unpack(ry[i], yv);
        Vec8<T>::unpack(rd[i], dv);
        if (gate) Vec8<T>::unpack(rg[i], gv);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          const float u = dv[e] * (w ? __ldg(w + c + e) : 1.0f) * (gate ? sig(gv[e]) : 1.0f);
          ss = fmaf(yv[e], yv[e], ss);
          su = fmaf(u, yv[e], su);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      su += __shfl_xor_sync(0xffffffffu, su, o);
    }
    if (lane == 0) red[par][warp] = make_float2(ss, su);
    __syncthreads();
    ss = 0.f;
    su = 0.f;
    for (int i = 0; i < nwarp; ++i) {
      const float2 x = red[par][i];
      ss += x.x;
      su += x.y;
    }
    const float r = 1.0f / sqrtf(ss * inv_hd + eps);
    const float coef = r * r * r * su * inv_hd;
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int c = (threadIdx.x + i * blockDim.x) * kVec;
      if (c < HD) {
        float yv[kVec], dv[kVec], gv[kVec], o[kVec], og[kVec];
        Vec8<T>::unpack(ry[i], yv);
        Vec8<T>::unpack(rd[i], dv);
        if (gate) Vec8<T>::unpack(rg[i], gv);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          const float sg = gate ? sig(gv[e]) : 1.0f;
          const float wc = w ? __ldg(w + c + e) : 1.0f;
          const float n = dv[e] * yv[e] * r * sg;   // dout * y * r * s: dw's term
          o[e] = r * dv[e] * wc * sg - coef * yv[e];
          og[e] = n * wc * (1.0f - sg);
          acc[i][e] += n;
        }
        Vec8<T>::store(dy + base + c, o);
        if (gate) Vec8<T>::store(dg + base + c, og);
      }
    }
  }
  if (!partial) return;
  float* out = partial + static_cast<int64_t>(blockIdx.x) * HD;
#pragma unroll
  for (int i = 0; i < kV; ++i) {
    const int c = (threadIdx.x + i * blockDim.x) * kVec;
    if (c < HD) Vec8<float>::store(out + c, acc[i]);
  }
}

// dw[c] = sum of the CTAs' partial sums in CTA order.
__global__ void __launch_bounds__(256) bwd_norm_weight_sum_kernel(const float* __restrict__ partial, int nblocks,
                                                                  int HD, float* __restrict__ dw) {
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < HD; c += gridDim.x * blockDim.x) {
    float a = 0.f;
    for (int b = 0; b < nblocks; ++b) a += partial[static_cast<int64_t>(b) * HD + c];
    dw[c] = a;
  }
}

// Per 8-element vector of row `row`: fk[row] = phi(k); at the mirrored row m of the same
// sequence, rv[m] = v, rdy[m] = dy, rfq[m] = phi(q), rfk[m] = phi(k).
template <typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const T* __restrict__ dy,
                                                       T* __restrict__ fk, T* __restrict__ rv, T* __restrict__ rdy,
                                                       T* __restrict__ rfq, T* __restrict__ rfk, const int* cu,
                                                       int nseq, int T_fixed, int64_t tokens, int HD,
                                                       int phi_identity) {
  const int vpr = HD / kVec;
  const int64_t n = tokens * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / vpr;
    const int c = static_cast<int>(i - row * vpr) * kVec;
    int64_t lo, hi;
    seq_bounds(cu, nseq, T_fixed, row, lo, hi);
    const int64_t m = lo + hi - 1 - row;
    if (row < lo || row >= hi || m < 0 || m >= tokens) continue;   // malformed cu_seqlens (the passes report it)
    const int64_t src = row * HD + c, dst = m * HD + c;
    float a[kVec], b[kVec];
    Vec8<T>::load(q + src, a);
    Vec8<T>::load(k + src, b);
#pragma unroll
    for (int j = 0; j < kVec; ++j) { a[j] = feature(a[j], phi_identity); b[j] = feature(b[j], phi_identity); }
    Vec8<T>::store(fk + src, b);
    Vec8<T>::store(rfk + dst, b);
    Vec8<T>::store(rfq + dst, a);
    Vec8<T>::load(v + src, a);
    Vec8<T>::store(rv + dst, a);
    Vec8<T>::load(dy + src, a);
    Vec8<T>::store(rdy + dst, a);
  }
}

// dq *= phi'(q) in place.  dk and dv hold the reversed-time results: the thread of the
// earlier row of each mirrored pair swaps the pair (dk times phi'(k) at its new row).
template <typename T>
__global__ void __launch_bounds__(256) bwd_post_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       T* __restrict__ dq, T* __restrict__ dk, T* __restrict__ dv,
                                                       const int* cu, int nseq, int T_fixed, int64_t tokens,
                                                       int HD, int phi_identity) {
  const int vpr = HD / kVec;
  const int64_t n = tokens * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / vpr;
    const int c = static_cast<int>(i - row * vpr) * kVec;
    int64_t lo, hi;
    seq_bounds(cu, nseq, T_fixed, row, lo, hi);
    const int64_t m = lo + hi - 1 - row;
    if (row < lo || row >= hi || m < 0 || m >= tokens) continue;   // malformed cu_seqlens (the passes report it)
    const int64_t a0 = row * HD + c, b0 = m * HD + c;
    float x[kVec], d[kVec];
    if (!phi_identity) {
      Vec8<T>::load(q + a0, x);
      Vec8<T>::load(dq + a0, d);
#pragma unroll
      for (int j = 0; j < kVec; ++j) d[j] *= dfeature(x[j], 0);
      Vec8<T>::store(dq + a0, d);
    }
    if (row > m) continue;
    float ka[kVec], kb[kVec], da[kVec], db[kVec];
    Vec8<T>::load(dk + a0, da);
    Vec8<T>::load(dk + b0, db);
    if (!phi_identity) {
      Vec8<T>::load(k + a0, ka);
      Vec8<T>::load(k + b0, kb);
#pragma unroll
      for (int j = 0; j < kVec; ++j) { db[j] *= dfeature(ka[j], 0); da[j] *= dfeature(kb[j], 0); }
    }
    Vec8<T>::store(dk + a0, db);
    if (row != m) Vec8<T>::store(dk + b0, da);
    if (row != m) {
      Vec8<T>::load(dv + a0, da);
      Vec8<T>::load(dv + b0, db);
      Vec8<T>::store(dv + a0, db);
      Vec8<T>::store(dv + b0, da);
    }
  }
}

// Reverse-time composition (the prefill kernel walks time backwards itself): phi(q) and
// phi(k) in place of the reversed copies, 16-byte vectors.
template <typename T>
__global__ void __launch_bounds__(256) bwd_feat_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       T* __restrict__ fq, T* __restrict__ fk, int64_t n8,
                                                       int phi_identity) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float a[kVec];
    Vec8<T>::load(q + i * kVec, a);
#pragma unroll
    for (int j = 0; j < kVec; ++j) a[j] = feature(a[j], phi_identity);
    Vec8<T>::store(fq + i * kVec, a);
    Vec8<T>::load(k + i * kVec, a);
#pragma unroll
    for (int j = 0; j < kVec; ++j) a[j] = feature(a[j], phi_identity);
    Vec8<T>::store(fk + i * kVec, a);
  }
}

// ... and its finish: dq *= phi'(q), dk *= phi'(k), in place (dv needs nothing).
template <typename T>
__global__ void __launch_bounds__(256) bwd_scale_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        T* __restrict__ dq, T* __restrict__ dk, int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float x[kVec], d[kVec];
    Vec8<T>::load(q + i * kVec, x);
    Vec8<T>::load(dq + i * kVec, d);
#pragma unroll
    for (int j = 0; j < kVec; ++j) d[j] *= dfeature(x[j], 0);
    Vec8<T>::store(dq + i * kVec, d);
    Vec8<T>::load(k + i * kVec, x);
    Vec8<T>::load(dk + i * kVec, d);
#pragma unroll
    for (int j = 0; j < kVec; ++j) d[j] *= dfeature(x[j], 0);
    Vec8<T>::store(dk + i * kVec, d);
  }
}

__global__ void __launch_bounds__(256) transpose_states_kernel(const float* __restrict__ in, float* __restrict__ out,
                                                               int64_t nmat, int D) {
  const int64_t n = nmat * D * D;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t mtx = i / (static_cast<int64_t>(D) * D);
    const int r = static_cast<int>((i / D) % D), c = static_cast<int>(i % D);
    out[(mtx * D + c) * D + r] = in[i];
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;   // 8 resident CTAs of 256 threads per SM
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

// The norm/gate kernel's launch shape: kvmax vectors of 8 per thread at most (4 of bf16, 2
// of fp32: the raw vectors stay in registers), threads a multiple of 32 (<= 512), kV = the
// vectors each thread takes; CTAs = the resident CTAs of the whole GPU (at most
// kNormGateMaxBlocks, at most one per token).
constexpr int kNormGateMaxBlocks = 1024;
struct NormGateShape {
  int threads, kv;
};
NormGateShape norm_gate_shape(int HD, int kvmax) {
  const int vecs = HD / kVec;
  int threads = (vecs + kvmax - 1) / kvmax;
  threads = ((threads + 31) / 32) * 32;
  if (threads > 512) threads = 512;
  return {threads, (vecs + threads - 1) / threads};
}

}  // namespace

int64_t norm_weight_partial_floats(int64_t tokens, int HD) {
  const int64_t nb = tokens < kNormGateMaxBlocks ? tokens : kNormGateMaxBlocks;
  return nb * HD;
}

namespace {
template <typename T, int kV>
cudaError_t launch_norm_gate_t(const void* y, const void* g, const void* dout, const float* w, void* dy, void* dg,
                               float* partial, float* dw, int64_t tokens, int threads, int HD, int gate, float eps,
                               cudaStream_t stream) {
  auto kern = bwd_norm_gate_kernel<T, kV>;
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
  if (e != cudaSuccess) return e;
  int64_t nb = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
  if (nb > kNormGateMaxBlocks) nb = kNormGateMaxBlocks;
  if (nb > tokens) nb = tokens;
  const int64_t per = (tokens + nb - 1) / nb;
  nb = (tokens + per - 1) / per;
  kern<<<static_cast<unsigned>(nb), threads, 0, stream>>>(static_cast<const T*>(y), static_cast<const T*>(g),
                                                          static_cast<const T*>(dout), w, static_cast<T*>(dy),
                                                          static_cast<T*>(dg), dw ? partial : nullptr, tokens, per,
                                                          HD, gate, eps);
  if ((e = cudaGetLastError()) != cudaSuccess || !dw) return e;
  bwd_norm_weight_sum_kernel<<<(HD + 255) / 256, 256, 0, stream>>>(partial, static_cast<int>(nb), HD, dw);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_norm_gate_dt(const void* y, const void* g, const void* dout, const float* w, void* dy, void* dg,
                                float* partial, float* dw, int64_t tokens, int HD, int gate, float eps,
                                cudaStream_t stream) {
  const NormGateShape sh = norm_gate_shape(HD, sizeof(T) == 2 ? 4 : 2);
  switch (sh.kv) {
    case 1: return launch_norm_gate_t<T, 1>(y, g, dout, w, dy, dg, partial, dw, tokens, sh.threads, HD, gate, eps, stream);
    case 2: return launch_norm_gate_t<T, 2>(y, g, dout, w, dy, dg, partial, dw, tokens, sh.threads, HD, gate, eps, stream);
    case 3: return launch_norm_gate_t<T, 3>(y, g, dout, w, dy, dg, partial, dw, tokens, sh.threads, HD, gate, eps, stream);
    default: return launch_norm_gate_t<T, 4>(y, g, dout, w, dy, dg, partial, dw, tokens, sh.threads, HD, gate, eps, stream);
  }
}
}  // namespace

cudaError_t launch_bwd_norm_gate(const void* y, const void* g, const void* dout, const float* w, void* dy, void* dg,
                                 float* partial, float* dw, int64_t tokens, int HD, int gate, float eps, la_dtype dt,
                                 cudaStream_t stream) {
  if (tokens == 0) {   // no tokens: the gradient of the norm weight is zero
    if (dw) bwd_norm_weight_sum_kernel<<<(HD + 255) / 256, 256, 0, stream>>>(partial, 0, HD, dw);
    return cudaGetLastError();
  }
  if (!dw) {
    if (dt == LA_BF16 && (HD == 4096 || HD == 8192)) {
      const auto yb = static_cast<const uint16_t*>(y), gb = static_cast<const uint16_t*>(g),
                 db = static_cast<const uint16_t*>(dout);
      auto dyb = static_cast<uint16_t*>(dy), dgb = static_cast<uint16_t*>(dg);
      if (HD == 8192)
        bwd_norm_gate_row_kernel<4><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(yb, gb, db, w, dyb, dgb, gate,
                                                                                        eps);
      else
        bwd_norm_gate_row_kernel<2><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(yb, gb, db, w, dyb, dgb, gate,
                                                                                        eps);
    } else if (dt == LA_BF16)
      bwd_norm_gate_token_kernel<uint16_t><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
          static_cast<const uint16_t*>(y), static_cast<const uint16_t*>(g), static_cast<const uint16_t*>(dout), w,
          static_cast<uint16_t*>(dy), static_cast<uint16_t*>(dg), HD, gate, eps);
    else
      bwd_norm_gate_token_kernel<float><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
          static_cast<const float*>(y), static_cast<const float*>(g), static_cast<const float*>(dout), w,
          static_cast<float*>(dy), static_cast<float*>(dg), HD, gate, eps);
    return cudaGetLastError();
  }
  if (dt == LA_BF16) return launch_norm_gate_dt<uint16_t>(y, g, dout, w, dy, dg, partial, dw, tokens, HD, gate, eps, stream);
  return launch_norm_gate_dt<float>(y, g, dout, w, dy, dg, partial, dw, tokens, HD, gate, eps, stream);
}

cudaError_t launch_bwd_prep(const void* q, const void* k, const void* v, const void* dy, void* fk, void* rv,
                            void* rdy, void* rfq, void* rfk, const int* cu, int nseq, int T_fixed, int64_t tokens,
                            int HD, int phi_identity, la_dtype dt, cudaStream_t stream) {
  const int64_t n = tokens * (HD / kVec);
  if (n == 0) return cudaSuccess;
  if (dt == LA_BF16)
    bwd_prep_kernel<uint16_t><<<grid_for(n), 256, 0, stream>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v),
        static_cast<const uint16_t*>(dy), static_cast<uint16_t*>(fk), static_cast<uint16_t*>(rv),
        static_cast<uint16_t*>(rdy), static_cast<uint16_t*>(rfq), static_cast<uint16_t*>(rfk), cu, nseq, T_fixed,
        tokens, HD, phi_identity);
  else
    bwd_prep_kernel<float><<<grid_for(n), 256, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<const float*>(dy), static_cast<float*>(fk), static_cast<float*>(rv), static_cast<float*>(rdy),
        static_cast<float*>(rfq), static_cast<float*>(rfk), cu, nseq, T_fixed, tokens, HD, phi_identity);
  return cudaGetLastError();
}

cudaError_t launch_bwd_post(const void* q, const void* k, void* dq, void* dk, void* dv, const int* cu, int nseq,
                            int T_fixed, int64_t tokens, int HD, int phi_identity, la_dtype dt, cudaStream_t stream) {
  const int64_t n = tokens * (HD / kVec);
  if (n == 0) return cudaSuccess;
  if (dt == LA_BF16)
    bwd_post_kernel<uint16_t><<<grid_for(n), 256, 0, stream>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<uint16_t*>(dq),
        static_cast<uint16_t*>(dk), static_cast<uint16_t*>(dv), cu, nseq, T_fixed, tokens, HD, phi_identity);
  else
    bwd_post_kernel<float><<<grid_for(n), 256, 0, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<float*>(dq),
        static_cast<float*>(dk), static_cast<float*>(dv), cu, nseq, T_fixed, tokens, HD, phi_identity);
  return cudaGetLastError();
}

cudaError_t launch_bwd_feat(const void* q, const void* k, void* fq, void* fk, int64_t elems, int phi_identity,
                            la_dtype dt, cudaStream_t stream) {
  const int64_t n8 = elems / kVec;
  if (n8 == 0) return cudaSuccess;
  if (dt == LA_BF16)
    bwd_feat_kernel<uint16_t><<<grid_for(n8), 256, 0, stream>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<uint16_t*>(fq),
        static_cast<uint16_t*>(fk), n8, phi_identity);
  else
    bwd_feat_kernel<float><<<grid_for(n8), 256, 0, stream>>>(static_cast<const float*>(q),
                                                             static_cast<const float*>(k), static_cast<float*>(fq),
                                                             static_cast<float*>(fk), n8, phi_identity);
  return cudaGetLastError();
}

cudaError_t launch_bwd_scale(const void* q, const void* k, void* dq, void* dk, int64_t elems, la_dtype dt,
                             cudaStream_t stream) {
  const int64_t n8 = elems / kVec;
  if (n8 == 0) return cudaSuccess;
  if (dt == LA_BF16)
    bwd_scale_kernel<uint16_t><<<grid_for(n8), 256, 0, stream>>>(
        static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<uint16_t*>(dq),
        static_cast<uint16_t*>(dk), n8);
  else
    bwd_scale_kernel<float><<<grid_for(n8), 256, 0, stream>>>(static_cast<const float*>(q),
                                                              static_cast<const float*>(k), static_cast<float*>(dq),
                                                              static_cast<float*>(dk), n8);
  return cudaGetLastError();
}

cudaError_t launch_transpose_states(const float* in, float* out, int64_t nmat, int D, cudaStream_t stream) {
  const int64_t n = nmat * D * D;
  if (n == 0) return cudaSuccess;
  transpose_states_kernel<<<grid_for(n), 256, 0, stream>>>(in, out, nmat, D);
  return cudaGetLastError();
}

}  // namespace la
