// The state a prefill ends with, without its outputs, on the 5th-generation tensor cores.
//
// The state of "六十四：MiniMax-01" section 3 is a plain sum, S_T = S_0 + sum_t phi(k_t) v_t^T,
// so the state a sequence (or a chunk of one) reaches needs only its keys and values.  This
// is the first step of the sequence-parallel prefill ("MiniMax-01系列大模型：超长上下文与多模态
// 能力深度解析与部署指南", section 2.1.3, LASP+): every rank computes its chunk's state before
// the states are exchanged.  A full prefill would also compute the scores, both output
// products and the outputs; here only phi(K)^T V is accumulated, streamed at HBM speed.
//
// Design (B200, sm_100a):
//  * grid (splits, H, sequences): one CTA sums a contiguous run of 128-row tiles of one
//    (sequence, head) into a 128 x 128 fp32 accumulator in TMEM (d_k lanes x d_v columns).
//    The host picks the split count so that one wave of CTAs covers the SMs; the partial
//    sums are added in a fixed order by a second kernel (with S_0), so the result does not
//    depend on timing.
//  * Warp 0 (one lane) streams K (two 64-column boxes) and V (two boxes) of each tile with
//    TMA (128-byte swizzle) into a three-stage ring; warps 4-11 apply SiLU to the K boxes in
//    place (the same packed-bf16 SiLU as the tensor-core prefill, so both give the same
//    state) and zero the rows past the sequence end in K and V; warp 1 (one lane) issues,
//    per tile, 8 k-steps x 2 MMAs  S[:, 0:64] += phi(K)^T V[:, 0:64],  S[:, 64:128] += ...
//    (both operands MN-major, M = d_k = 128, N = 64, K = 16 tokens); warps 0-3 (one per
//    TMEM lane quarter) finally write the partial state.
//  * Every wait is bounded (globaltimer); a wait that runs out records LA_ERR_TIMEOUT, the
//    CTA drains its issued loads and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "la_common.cuh"
#include "la_sm100.cuh"
#include "la_tc_util.cuh"

namespace la {
using namespace sm100;

namespace {

constexpr int kD = 128;
constexpr int kTile = 128;
constexpr int kStages = 3;
constexpr int kThreads = 384;                    // 12 warps
constexpr int kXfWarp0 = 4;
constexpr int kXfThreads = 256;                  // warps 4..11
constexpr uint32_t kBoxBytes = kTile * 64 * 2;   // 128 rows x 64 bf16 columns = 16 KiB
constexpr uint32_t kStageBytes = 4 * kBoxBytes;  // K box 0, K box 1, V box 0, V box 1
constexpr uint32_t OFF_KS = 0;                   // offsets inside a stage
constexpr uint32_t OFF_VS = 2 * kBoxBytes;
constexpr uint32_t OFF_BARS = kStages * kStageBytes;
constexpr uint32_t kTmemCols = 128;

struct Bars {
  uint64_t full[kStages], xf[kStages], empty[kStages], done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kSmemBytes = OFF_BARS + sizeof(Bars) + 1024;   // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

// MN-major operand descriptor template, 128-byte swizzle, 64-element chunks kBoxBytes apart
// along M / N, 8-row groups 1024 bytes apart (start address added per operand).
constexpr uint64_t kDescMN = (static_cast<uint64_t>((kBoxBytes >> 4) & 0x3FFFu) << 16) |
                             (static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
__device__ __forceinline__ uint64_t desc_at(uint64_t tmpl, uint32_t a) { return tmpl + ((a >> 4) & 0x3FFFu); }
constexpr uint32_t kIdesc = make_idesc_bf16(128, 64, 1, 1);

struct StateParams {
  float* partial;          // [splits, nseq, H, D, D] fp32
  const int* cu;           // [nseq + 1] device, or null (fixed length T)
  int nseq, T, H, splits, rows_per_split, phi_identity;
  int64_t tokens;
  ErrRec* err;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Bounded wait; false once the CTA is aborting (this wait ran out, or another role's did).
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, int* abort_flag, ErrRec* err, uint32_t site,
                                       uint32_t index) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = wait_limit_ns(err);
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;   // suspends: no issue slots used
    if ((n & 3u) == 0) {
      if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
      if (globaltimer_ns() - t0 > lim) {
        report(err, LA_ERR_TIMEOUT, site, index, parity);
        *reinterpret_cast<volatile int*>(abort_flag) = 1;
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars& B, ErrRec* err, uint32_t site,
                                         uint32_t index) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, &B.abort_flag, err, site, index);
}
// Wait used only to drain work already issued (bounded, never records).
__device__ __noinline__ void drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const StateParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  Bars& B = *reinterpret_cast<Bars*>(smem + OFF_BARS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;

  // This CTA's rows: [r0, r1) of sequence s, whose first packed row is lo.
  int64_t lo, L;
  if (p.cu) {
    lo = __ldg(p.cu + s);
    L = static_cast<int64_t>(__ldg(p.cu + s + 1)) - lo;
  } else {
    lo = static_cast<int64_t>(s) * p.T;
    L = p.T;
  }
  if (lo < 0 || L < 0 || lo + L > p.tokens) {   // malformed cu_seqlens: no rows, and say so
    if (tid == 0) report(p.err, LA_ERR_DEVICE, SITE_VARLEN_CU, static_cast<unsigned>(s), 0);
    L = 0;
  }
  const int64_t r0 = static_cast<int64_t>(split) * p.rows_per_split;
  const int64_t r1 = min(L, r0 + p.rows_per_split);
  const int n = r1 > r0 ? static_cast<int>((r1 - r0 + kTile - 1) / kTile) : 0;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&B.full[i], 1);
      mbar_init(&B.xf[i], kXfThreads);
      mbar_init(&B.empty[i], 1);
    }
    mbar_init(&B.done, 1);
    B.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<kTmemCols>(&B.tmem_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B.tmem_base;

  if (warp == 0) {
    // TMA producer (one lane): K and V boxes of tile j into stage j % 3.
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t pol = policy_evict_first();
      const int32_t x0 = h * kD;
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !wait_bar(&B.empty[st], ((j / kStages) - 1) & 1, B, p.err, SITE_TC_PRODUCER, j)) break;
        const int32_t row = static_cast<int32_t>(lo + r0 + static_cast<int64_t>(j) * kTile);
        uint8_t* stg = smem + st * kStageBytes;
        mbar_arrive_expect_tx(&B.full[st], kStageBytes);
        tma_load_2d(stg + OFF_KS, &tm_k, x0, row, &B.full[st], pol);
        tma_load_2d(stg + OFF_KS + kBoxBytes, &tm_k, x0 + 64, row, &B.full[st], pol);
        tma_load_2d(stg + OFF_VS, &tm_v, x0, row, &B.full[st], pol);
        tma_load_2d(stg + OFF_VS + kBoxBytes, &tm_v, x0 + 64, row, &B.full[st], pol);
        issued = j + 1;
      }
      // Every issued load lands before this CTA's shared memory can go away.
      for (int j = issued - 1; j >= 0 && j >= issued - kStages; --j) drain(&B.full[j % kStages], (j / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // MMA issuer (one lane).
    if (lane == 0 && n > 0) {
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        if (!wait_bar(&B.xf[st], (j / kStages) & 1, B, p.err, SITE_TC_MMA, j)) break;
        tc_fence_after();
        const uint32_t a = sbase + st * kStageBytes;
        const uint64_t kd = desc_at(kDescMN, a + OFF_KS);
        const uint64_t v0 = desc_at(kDescMN, a + OFF_VS);
        const uint64_t v1 = desc_at(kDescMN, a + OFF_VS + kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem, kd + 128 * kk, v0 + 128 * kk, kIdesc, acc);
          mma_ss(tmem + 64, kd + 128 * kk, v1 + 128 * kk, kIdesc, acc);
        }
        mma_commit(&B.empty[st]);
      }
      mma_commit(&B.done);   // every MMA issued above has completed when this arrives
      drain(&B.done, 0);
    }
    __syncwarp();
  } else if (warp >= kXfWarp0) {
    // SiLU of the K boxes in place; rows past the sequence end zeroed in K and V.
    const int wt = tid - 32 * kXfWarp0;
    constexpr int kChunks = static_cast<int>(kBoxBytes / 16);   // 16-byte chunks per box
    for (int j = 0; j < n; ++j) {
      const int st = j % kStages;
      const bool ok = wait_bar(&B.full[st], (j / kStages) & 1, B, p.err, SITE_TC_TRANSFORM, j);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const int64_t left = r1 - r0 - static_cast<int64_t>(j) * kTile;
      const int vr = left < kTile ? static_cast<int>(left) : kTile;
      const uint32_t a = sbase + st * kStageBytes;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint32_t box = a + OFF_KS + b * kBoxBytes;
        for (int c0 = wt; c0 < kChunks; c0 += 4 * kXfThreads) {
          uint4 x[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) x[u] = lds128(box + 16u * (c0 + u * kXfThreads));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c0 + u * kXfThreads;
            uint4 y = x[u];
            if ((c >> 3) >= vr) {
              y = make_uint4(0, 0, 0, 0);
            } else if (!p.phi_identity) {
              y = tcu::silu8(y);
            }
            sts128(box + 16u * c, y);
          }
        }
      }
      if (vr < kTile) {
        for (int c = wt; c < 2 * kChunks; c += kXfThreads)
          if (((c % kChunks) >> 3) >= vr) sts128(a + OFF_VS + 16u * c, make_uint4(0, 0, 0, 0));
      }
      fence_proxy_async_smem();   // the tensor core reads what these threads wrote
      mbar_arrive(&B.xf[st]);
    }
  }

  // Epilogue: warps 0-3, one per TMEM lane quarter (lane = row of S = d_k index).
  if (warp < 4) {
    const bool have = n > 0 && wait_bar(&B.done, 0, B, p.err, SITE_TC_EPILOGUE, 0);
    const bool go = __all_sync(0xFFFFFFFFu, have && !*reinterpret_cast<volatile int*>(&B.abort_flag));
    const int row = 32 * warp + lane;
    float* dst = p.partial + ((static_cast<int64_t>(split) * p.nseq + s) * p.H + h) * kD * kD +
                 static_cast<int64_t>(row) * kD;
    if (go) tc_fence_after();
#pragma unroll 1
    for (int cg = 0; cg < kD / 32; ++cg) {
      uint32_t r[32];
      if (go) {
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * cg, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(dst + 32 * cg + i) =
            make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                        __uint_as_float(r[i + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<kTmemCols>(tmem);
}

// out = state_in (or zeros) + the split partials, added in split order.  state_in and out
// may be the same buffer (each element is read once by the thread that writes it).
__global__ void __launch_bounds__(256) state_reduce_kernel(const float4* __restrict__ partial, int splits,
                                                           const float4* state_in, float4* out, int64_t n4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = state_in ? state_in[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < splits; ++sp) {
      const float4 b = partial[static_cast<int64_t>(sp) * n4 + i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    out[i] = a;
  }
}

// Chunk boundaries of B sequences of T tokens cut into S chunks of Tc tokens (the last
// chunks of a sequence may be shorter or empty): cu[b * S + c] = b * T + min(c * Tc, T).
__global__ void chunk_cu_kernel(int* cu, int B, int T, int Tc, int S) {
  const int n = B * S;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x) {
    if (i == n) {
      cu[i] = B * T;
    } else {
      const int b = i / S, c = i % S;
      const int64_t off = static_cast<int64_t>(c) * Tc;
      cu[i] = b * T + static_cast<int>(off < T ? off : T);
    }
  }
}

// prefix[b, c] = S0[b] + sum_{c' < c} cs[b, c'] (in chunk order) and out[b] = S0[b] + all of
// them: the initial state of every chunk of a sequence and its final state.  With time
// running backwards the chunks are taken from the last: prefix[b, c] = S0[b] + sum_{c' > c}.
// s0 and out may be the same buffer (a call's state_in and state_out): each element is read
// once, by the thread that later writes it, so neither is declared __restrict__.
__global__ void __launch_bounds__(256) chunk_prefix_kernel(const float4* __restrict__ cs, const float4* s0,
                                                           float4* __restrict__ prefix, float4* out,
                                                           int B, int S, int64_t n4, int reverse) {
  const int64_t total = static_cast<int64_t>(B) * n4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / n4, e = i % n4;
    float4 run = s0 ? s0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < S; ++j) {
      const int c = reverse ? S - 1 - j : j;
      const int64_t at = (b * S + c) * n4 + e;
      prefix[at] = run;
      const float4 x = cs[at];
      run.x += x.x; run.y += x.y; run.z += x.z; run.w += x.w;
    }
    if (out) out[i] = run;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [rows, cols] bf16 row-major, box 64 columns x 128 rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kTile)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

// Splits per (sequence, head): one wave of CTAs over the SMs, whole tiles per split.
int chunk_state_splits(int nseq, int H, int max_len, int num_sms) {
  const int tiles = (max_len + kTile - 1) / kTile;
  const int64_t items = static_cast<int64_t>(nseq) * H;
  int sp = items >= num_sms ? 1 : static_cast<int>(num_sms / items);
  if (sp > tiles) sp = tiles;
  return sp < 1 ? 1 : sp;
}

cudaError_t launch_chunk_state_tc(const void* k, const void* v, const float* state_in, float* state_out,
                                  float* partial, const int* cu, int nseq, int T, int max_len, int64_t tokens, int H,
                                  int phi_identity, int num_sms, ErrRec* err, cudaStream_t stream) {
  const int splits = chunk_state_splits(nseq, H, max_len, num_sms);
  const int tiles = (max_len + kTile - 1) / kTile;
  StateParams p{};
  p.partial = partial;
  p.cu = cu;
  p.nseq = nseq;
  p.T = T;
  p.H = H;
  p.splits = splits;
  p.rows_per_split = ((tiles + splits - 1) / splits) * kTile;
  if (p.rows_per_split == 0) p.rows_per_split = kTile;
  p.phi_identity = phi_identity;
  p.tokens = tokens;
  p.err = err;
  const int64_t cols = static_cast<int64_t>(H) * kD;
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, tokens, cols) || !make_map(&mv, v, tokens, cols)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  chunk_state_tc_kernel<<<dim3(splits, H, nseq), kThreads, kSmemBytes, stream>>>(mk, mv, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t n4 = static_cast<int64_t>(nseq) * H * kD * kD / 4;
  const int blocks = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, static_cast<int64_t>(num_sms) * 8));
  state_reduce_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(partial), splits,
                                                  reinterpret_cast<const float4*>(state_in),
                                                  reinterpret_cast<float4*>(state_out), n4);
  return cudaGetLastError();
}

cudaError_t launch_chunk_cu(int* cu, int B, int T, int Tc, int S, cudaStream_t stream) {
  chunk_cu_kernel<<<(B * S + 256) / 256, 256, 0, stream>>>(cu, B, T, Tc, S);
  return cudaGetLastError();
}

cudaError_t launch_chunk_prefix(const float* cs, const float* s0, float* prefix, float* out, int B, int S, int H,
                                int reverse, int num_sms, cudaStream_t stream) {
  const int64_t n4 = static_cast<int64_t>(H) * kD * kD / 4;
  const int64_t total = static_cast<int64_t>(B) * n4;
  const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(num_sms) * 8));
  chunk_prefix_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(cs),
                                                  reinterpret_cast<const float4*>(s0),
                                                  reinterpret_cast<float4*>(prefix), reinterpret_cast<float4*>(out),
                                                  B, S, n4, reverse);
  return cudaGetLastError();
}

}  // namespace la
