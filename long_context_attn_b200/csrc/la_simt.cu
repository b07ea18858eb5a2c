// Block-wise Lightning Attention prefill on CUDA cores (fp32 arithmetic throughout).
//
// This is the path for fp32 inputs (where the 1e-4 relative tolerance rules out a
// one-pass TF32 or bf16 tensor-core product) and for shapes the tensor-core kernel does
// not take.  It computes the block-wise form of the recurrence exactly as the pages
// structure it ("MiniMax-01技术报告解读（二）计算优化", section 3: block size C; the
// intra-block masked product plus the inter-block read of the carried state), with the
// state S of "六十四：MiniMax-01" section 3 held in shared memory in fp32:
//   y_t = sum_{i in block, i <= t} (phi(q_t).phi(k_i)) v_i + phi(q_t)^T S_prev
//   S_prev += sum_{i in block} phi(k_i) v_i^T          (after the whole block)
// One CTA owns one (sequence, head) chain and walks it block by block in 32-row
// sub-tiles.  The RMSNorm * sigmoid(g) output transform ("MiniMax-Text-01 405B MoE模型
// 架构与训练策略解析", section 2.1) runs afterwards in norm_gate_kernel, one CTA per token.
#include "la_common.cuh"

namespace la {

constexpr int kSimtThreads = 256;
constexpr int kSub = 32;  // rows per sub-tile

template <int D>
struct SimtSmem {
  float S[D][D];
  float Q[kSub][D + 1];
  float K[kSub][D + 1];
  float V[kSub][D + 1];
  float P[kSub][kSub + 1];
};

template <typename T, int D>
__device__ __forceinline__ void load_rows(float (*dst)[D + 1], const T* src, int64_t row0, int nrows,
                                          int H, int h, bool feat, bool phi_identity) {
  for (int e = threadIdx.x; e < kSub * D; e += kSimtThreads) {
    const int r = e / D, c = e % D;
    float x = 0.f;
    if (r < nrows) {
      x = load_elem<T>(src, ((row0 + r) * H + h) * static_cast<int64_t>(D) + c);
      if (feat && !phi_identity) x = silu_accurate(x);
    }
    dst[r][c] = x;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
simt_prefill_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    T* __restrict__ out, float* __restrict__ y_ws, const float* state_in,
                    float* state_out, const int* __restrict__ cu, int T_fixed, int H,
                    int C, int phi_identity, int64_t total_rows, ErrRec* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem_raw);
  const int h = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;

  int64_t row0;
  int L;
  if (cu) {
    row0 = cu[s];
    L = cu[s + 1] - cu[s];
    if (L < 0 || row0 < 0 || row0 + L > total_rows) {
      if (tid == 0) report(err, LA_ERR_DEVICE, SITE_VARLEN_CU, s, 0);
      return;
    }
  } else {
    row0 = static_cast<int64_t>(s) * T_fixed;
    L = T_fixed;
  }

  const int64_t st_off = (static_cast<int64_t>(s) * H + h) * D * D;
  for (int e = tid; e < D * D; e += kSimtThreads)
    sm.S[e / D][e % D] = state_in ? state_in[st_off + e] : 0.f;

  // Output ownership: row r = tid / 8, columns c = tid % 8 + 8 m.
  constexpr int kOC = D / 8;
  const int orow = tid / 8, ocol = tid % 8;
  // State-update ownership: column c = tid % D, rows i = tid / D + (256 / D) m.
  constexpr int kRowStep = kSimtThreads / D;
  constexpr int kSR = D / kRowStep;
  const int scol = tid % D, srow = tid / D;
  const int HD = H * D;

  for (int b0 = 0; b0 < L; b0 += C) {
    const int n = min(C, L - b0);
    for (int q0 = 0; q0 < n; q0 += kSub) {
      __syncthreads();
      load_rows<T, D>(sm.Q, q, row0 + b0 + q0, min(kSub, n - q0), H, h, true, phi_identity);
      __syncthreads();
      float acc[kOC];
#pragma unroll
      for (int m = 0; m < kOC; ++m) acc[m] = 0.f;
      // inter: phi(q) S_prev
      for (int i = 0; i < D; ++i) {
        const float a = sm.Q[orow][i];
#pragma unroll
        for (int m = 0; m < kOC; ++m) acc[m] = fmaf(a, sm.S[i][ocol + 8 * m], acc[m]);
      }
      // intra: masked (phi(q) phi(k)^T) v over the key sub-tiles of this block up to q0
      for (int k0 = 0; k0 <= q0; k0 += kSub) {
        __syncthreads();
        load_rows<T, D>(sm.K, k, row0 + b0 + k0, min(kSub, n - k0), H, h, true, phi_identity);
        load_rows<T, D>(sm.V, v, row0 + b0 + k0, min(kSub, n - k0), H, h, false, phi_identity);
        __syncthreads();
        for (int jj = 0; jj < 4; ++jj) {
          const int j = ocol + 8 * jj;
          float p = 0.f;
          for (int i = 0; i < D; ++i) p = fmaf(sm.Q[orow][i], sm.K[j][i], p);
          sm.P[orow][j] = (k0 + j <= q0 + orow) ? p : 0.f;
        }
        __syncthreads();
        for (int j = 0; j < kSub; ++j) {
          const float p = sm.P[orow][j];
#pragma unroll
          for (int m = 0; m < kOC; ++m) acc[m] = fmaf(p, sm.V[j][ocol + 8 * m], acc[m]);
        }
      }
      if (q0 + orow < n) {
        const int64_t row = row0 + b0 + q0 + orow;
#pragma unroll
        for (int m = 0; m < kOC; ++m) {
          const int64_t idx = row * HD + h * D + ocol + 8 * m;
          if (y_ws) y_ws[idx] = acc[m];
          else store_elem<T>(out, idx, acc[m]);
        }
      }
    }
    // carry: S_prev += phi(K_block)^T V_block
    float sacc[kSR];
#pragma unroll
    for (int m = 0; m < kSR; ++m) sacc[m] = 0.f;
    for (int k0 = 0; k0 < n; k0 += kSub) {
      __syncthreads();
      load_rows<T, D>(sm.K, k, row0 + b0 + k0, min(kSub, n - k0), H, h, true, phi_identity);
      load_rows<T, D>(sm.V, v, row0 + b0 + k0, min(kSub, n - k0), H, h, false, phi_identity);
      __syncthreads();
      for (int j = 0; j < kSub; ++j) {
        const float vv = sm.V[j][scol];
#pragma unroll
        for (int m = 0; m < kSR; ++m) sacc[m] = fmaf(sm.K[j][srow + kRowStep * m], vv, sacc[m]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kSR; ++m) sm.S[srow + kRowStep * m][scol] += sacc[m];
  }
  __syncthreads();
  if (state_out)
    for (int e = tid; e < D * D; e += kSimtThreads) state_out[st_off + e] = sm.S[e / D][e % D];
}

// One CTA per token: o = y * rsqrt(mean(y^2) + eps) * w [* sigmoid(g)] over the H*D row.
template <typename T>
__global__ void __launch_bounds__(256)
norm_gate_kernel(const float* __restrict__ y, const T* __restrict__ g, T* __restrict__ out, int HD,
                 int mode, float eps, const float* __restrict__ w) {
  __shared__ float s_part[8];
  const int64_t row = static_cast<int64_t>(blockIdx.x) * HD;
  float ss = 0.f;
  for (int c = threadIdx.x; c < HD; c += 256) {
    const float x = y[row + c];
    ss = fmaf(x, x, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += s_part[i];
  const float r = 1.0f / sqrtf(tot / static_cast<float>(HD) + eps);
  for (int c = threadIdx.x; c < HD; c += 256) {
    float o = y[row + c] * r;
    if (w) o *= w[c];
    if (mode == LA_OUT_RMSNORM_GATE) o *= sigmoid_accurate(load_elem<T>(g, row + c));
    store_elem<T>(out, row + c, o);
  }
}

size_t simt_smem_bytes(int D) { return D == 128 ? sizeof(SimtSmem<128>) : sizeof(SimtSmem<64>); }

template <typename T, int D>
static cudaError_t launch_simt_t(const void* q, const void* k, const void* v, void* out, float* y_ws,
                                 const float* state_in, float* state_out, const int* cu, int nseq, int Tlen,
                                 int H, int C, int phi_identity, int64_t total_rows, ErrRec* err,
                                 cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<D>);
  cudaError_t e = cudaFuncSetAttribute(simt_prefill_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(H, nseq);
  simt_prefill_kernel<T, D><<<grid, kSimtThreads, smem, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(out),
      y_ws, state_in, state_out, cu, Tlen, H, C, phi_identity, total_rows, err);
  return cudaGetLastError();
}

cudaError_t launch_simt_prefill(const void* q, const void* k, const void* v, void* out, float* y_ws,
                                const float* state_in, float* state_out, const int* cu, int nseq, int T,
                                int H, int D, int C, la_dtype dt, int phi_identity, int64_t total_rows,
                                ErrRec* err, cudaStream_t stream) {
  if (dt == LA_BF16) {
    if (D == 128) return launch_simt_t<uint16_t, 128>(q, k, v, out, y_ws, state_in, state_out, cu, nseq, T, H, C, phi_identity, total_rows, err, stream);
    return launch_simt_t<uint16_t, 64>(q, k, v, out, y_ws, state_in, state_out, cu, nseq, T, H, C, phi_identity, total_rows, err, stream);
  }
  if (D == 128) return launch_simt_t<float, 128>(q, k, v, out, y_ws, state_in, state_out, cu, nseq, T, H, C, phi_identity, total_rows, err, stream);
  return launch_simt_t<float, 64>(q, k, v, out, y_ws, state_in, state_out, cu, nseq, T, H, C, phi_identity, total_rows, err, stream);
}

cudaError_t launch_norm_gate(const float* y, const void* g, void* out, int64_t tokens, int HD, int mode,
                             float eps, const float* w, la_dtype dt, cudaStream_t stream) {
  if (tokens <= 0) return cudaSuccess;
  if (dt == LA_BF16)
    norm_gate_kernel<uint16_t><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
        y, static_cast<const uint16_t*>(g), static_cast<uint16_t*>(out), HD, mode, eps, w);
  else
    norm_gate_kernel<float><<<static_cast<unsigned>(tokens), 256, 0, stream>>>(
        y, static_cast<const float*>(g), static_cast<float*>(out), HD, mode, eps, w);
  return cudaGetLastError();
}

}  // namespace la
