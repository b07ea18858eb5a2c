// Single-token decode step of Lightning Attention (sm_100a).
//
// "六十四：MiniMax-01", section 3: a new token only updates the running state and reads
// it -- S <- S + phi(k) v^T, y = phi(q)^T S (update first, so the token sees itself).
// "MiniMax-Text-01 405B MoE模型架构与训练策略解析", section 2.1: o = RMSNorm(y) * sigmoid(g),
// the norm taken over the concatenation of all heads of the sequence.
//
// The step is bound by HBM: per (sequence, head) the D x D fp32 state is read and written
// once (128 KiB at D = 128) against ~1 KiB of token data.  One CTA owns one (b, h) state;
// each warp streams whole 512-byte rows with 128-bit accesses, every thread keeps all
// of its rows in flight at once, and the update and the read happen in the same pass.
// The cross-head norm needs all H heads of a sequence: each CTA publishes its y and its
// sum of squares, and the last CTA of the sequence to arrive (a counter per sequence)
// normalises the whole H*D row.  Nobody waits, so no co-residency is needed, and the
// counter is reset by that last CTA, which leaves the workspace zeroed.
#include "la_common.cuh"

namespace la {

struct DecodeWs {
  int* count;      // [B] arrivals per sequence (zero between calls)
  float* y;        // [B, H, D] raw outputs
  float* part;     // [B, H] per-head sums of squares
  const int* row_index;    // optional [B]: token row of item b in q, k, v, g, out (else b)
  const int* state_index;  // optional [B]: state slot of item b (else b)
  float* z;                // optional [slots, H, D]: normaliser of the normalised variant (in place)
};

template <typename T, int D>
__global__ void __launch_bounds__(256)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const T* __restrict__ g, T* __restrict__ out, float* __restrict__ state, int B,
                   int H, int phi_identity, int mode, float eps, const float* __restrict__ norm_w,
                   DecodeWs ws) {
  constexpr int kThreads = 256;
  constexpr int kVecPerRow = D / 4;                  // float4 per state row
  constexpr int kRowsPerPass = kThreads / kVecPerRow;
  constexpr int kPasses = D / kRowsPerPass;          // rows each thread owns
  static_assert(kThreads % kVecPerRow == 0 && D % kRowsPerPass == 0, "tiling");

  __shared__ float s_fq[D], s_fk[D], s_v[D];
  __shared__ float s_red[kRowsPerPass][D];
  __shared__ float s_ss[kThreads / 32];
  __shared__ int s_last;

  const int bh = blockIdx.x;            // b * H + h
  const int b = bh / H;
  const int h = bh % H;
  const int tid = threadIdx.x;
  // Item b's token row and state slot (a mixed step gathers its one-token sequences).
  const int64_t trow = ws.row_index ? __ldg(ws.row_index + b) : b;
  const int64_t slot = ws.state_index ? __ldg(ws.state_index + b) : b;
  const int64_t tok = (trow * H + h) * D;

  for (int i = tid; i < D; i += kThreads) {
    const float xq = load_elem<T>(q, tok + i), xk = load_elem<T>(k, tok + i);
    s_fq[i] = phi_identity ? xq : silu_accurate(xq);
    s_fk[i] = phi_identity ? xk : silu_accurate(xk);
    s_v[i] = load_elem<T>(v, tok + i);
  }

  // Issue every state load of this thread before the first use.
  const int c4 = tid % kVecPerRow;
  const int r0 = tid / kVecPerRow;
  float4* S = reinterpret_cast<float4*>(state + (slot * H + h) * D * D);
  float4 s[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) s[p] = __ldcs(&S[(r0 + p * kRowsPerPass) * kVecPerRow + c4]);
  __syncthreads();

  const float4 vv = make_float4(s_v[4 * c4], s_v[4 * c4 + 1], s_v[4 * c4 + 2], s_v[4 * c4 + 3]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int row = r0 + p * kRowsPerPass;
    const float a = s_fk[row], c = s_fq[row];
    s[p].x = fmaf(a, vv.x, s[p].x); s[p].y = fmaf(a, vv.y, s[p].y);
    s[p].z = fmaf(a, vv.z, s[p].z); s[p].w = fmaf(a, vv.w, s[p].w);
    acc.x = fmaf(c, s[p].x, acc.x); acc.y = fmaf(c, s[p].y, acc.y);
    acc.z = fmaf(c, s[p].z, acc.z); acc.w = fmaf(c, s[p].w, acc.w);
    __stcs(&S[row * kVecPerRow + c4], s[p]);
  }
  s_red[r0][4 * c4 + 0] = acc.x; s_red[r0][4 * c4 + 1] = acc.y;
  s_red[r0][4 * c4 + 2] = acc.z; s_red[r0][4 * c4 + 3] = acc.w;
  __syncthreads();

  // y[j] = sum over the row groups, in a fixed order.
  float y = 0.f;
  if (tid < D) {
#pragma unroll
    for (int r = 0; r < kRowsPerPass; ++r) y += s_red[r][tid];
  }
  const int HD = H * D;
  if (ws.z) {
    // Normalised variant ("六十四：MiniMax-01", section 3): z <- z + phi(k), y <- y / (phi(q) . z).
    float zp = 0.f;
    if (tid < D) {
      float* zr = ws.z + (slot * H + h) * D;
      const float zn = zr[tid] + s_fk[tid];
      zr[tid] = zn;
      zp = s_fq[tid] * zn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zp += __shfl_xor_sync(0xffffffffu, zp, o);
    if ((tid & 31) == 0) s_ss[tid >> 5] = zp;
    __syncthreads();
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) den += s_ss[w];
    __syncthreads();   // s_ss is reused for the sum of squares below
    y /= den;
  }
  if (mode == LA_OUT_RAW) {
    if (tid < D) store_elem<T>(out, trow * HD + h * D + tid, y);
    return;
  }

  // Publish y and this head's sum of squares (fixed-order reduction).
  float sq = (tid < D) ? y * y : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if ((tid & 31) == 0) s_ss[tid >> 5] = sq;
  if (tid < D) ws.y[static_cast<int64_t>(bh) * D + tid] = y;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) t += s_ss[w];
    ws.part[bh] = t;
    __threadfence();
    const int prev = atomicAdd(&ws.count[b], 1);
    s_last = (prev == H - 1);
  }
  __syncthreads();
  if (!s_last) return;

  // Last arriver of sequence b: normalise the whole H*D row.
  __threadfence();
  if (tid == 0) {
    float t = 0.f;
    for (int h = 0; h < H; ++h) t += __ldcg(&ws.part[b * H + h]);
    s_ss[0] = 1.0f / sqrtf(t / static_cast<float>(HD) + eps);
    ws.count[b] = 0;  // leave the workspace zeroed for the next call
  }
  __syncthreads();
  const float r = s_ss[0];
  const int64_t yrow = static_cast<int64_t>(b) * HD;
  const int64_t row = trow * HD;
  for (int c = tid; c < HD; c += kThreads) {
    float o = __ldcg(&ws.y[yrow + c]) * r;
    if (norm_w) o *= norm_w[c];
    if (mode == LA_OUT_RMSNORM_GATE) o *= sigmoid_accurate(load_elem<T>(g, row + c));
    store_elem<T>(out, row + c, o);
  }
}

size_t decode_workspace_bytes(int B, int H, int D) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  return 256 + up(sizeof(int) * size_t(B)) + up(sizeof(float) * size_t(B) * H * D) +
         up(sizeof(float) * size_t(B) * H);
}

static DecodeWs carve_decode_ws(void* workspace, int B, int H, int D, const int* row_index,
                                const int* state_index, float* z) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  char* p = static_cast<char*>(workspace) + 256;
  DecodeWs ws;
  ws.count = reinterpret_cast<int*>(p);
  p += up(sizeof(int) * size_t(B));
  ws.y = reinterpret_cast<float*>(p);
  p += up(sizeof(float) * size_t(B) * H * D);
  ws.part = reinterpret_cast<float*>(p);
  ws.row_index = row_index;
  ws.state_index = state_index;
  ws.z = z;
  return ws;
}

template <typename T, int D>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, const void* g, void* out,
                                   float* state, int B, int H, int phi_identity, int mode, float eps,
                                   const float* w, void* workspace, const int* row_index,
                                   const int* state_index, float* z, cudaStream_t stream) {
  DecodeWs ws = carve_decode_ws(workspace, B, H, D, row_index, state_index, z);
  decode_step_kernel<T, D><<<B * H, 256, 0, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(g), static_cast<T*>(out), state, B, H, phi_identity, mode, eps, w, ws);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, void* out, float* state,
                          int B, int H, int D, la_dtype dt, int phi_identity, int mode, float eps,
                          const float* w, void* workspace, cudaStream_t stream, const int* row_index,
                          const int* state_index, float* z) {
  if (dt == LA_BF16) {
    if (D == 128)
      return launch_decode_t<uint16_t, 128>(q, k, v, g, out, state, B, H, phi_identity, mode, eps, w, workspace,
                                            row_index, state_index, z, stream);
    return launch_decode_t<uint16_t, 64>(q, k, v, g, out, state, B, H, phi_identity, mode, eps, w, workspace,
                                         row_index, state_index, z, stream);
  }
  if (D == 128)
    return launch_decode_t<float, 128>(q, k, v, g, out, state, B, H, phi_identity, mode, eps, w, workspace,
                                       row_index, state_index, z, stream);
  return launch_decode_t<float, 64>(q, k, v, g, out, state, B, H, phi_identity, mode, eps, w, workspace,
                                    row_index, state_index, z, stream);
}

// Mixed step: the one-token sequences of cu_seqlens (in sequence order) become the items
// of a decode batch: item j gets the token row cu[s] and the state slot state_slot[s] of
// the j-th such sequence.  One CTA; a block-wide prefix count per chunk of 1024 keeps the
// order deterministic.
__global__ void __launch_bounds__(1024) gather_single_token_kernel(const int* __restrict__ cu,
                                                                     const int* __restrict__ state_slot, int n,
                                                                     int* __restrict__ row_index,
                                                                     int* __restrict__ state_index) {
  __shared__ int warp_tot[32];
  __shared__ int base;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) base = 0;
  __syncthreads();
  for (int s0 = 0; s0 < n; s0 += 1024) {
    const int s = s0 + tid;
    const bool one = s < n && (cu[s + 1] - cu[s]) == 1;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, one);
    const int before = __popc(m & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(m);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += warp_tot[w];
    if (one) {
      row_index[off + before] = cu[s];
      state_index[off + before] = state_slot[s];
    }
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < 32; ++w) t += warp_tot[w];
      base += t;
    }
    __syncthreads();
  }
}

cudaError_t launch_gather_single_token(const int* cu, const int* state_slot, int n, int* row_index,
                                       int* state_index, cudaStream_t stream) {
  gather_single_token_kernel<<<1, 1024, 0, stream>>>(cu, state_slot, n, row_index, state_index);
  return cudaGetLastError();
}

}  // namespace la
