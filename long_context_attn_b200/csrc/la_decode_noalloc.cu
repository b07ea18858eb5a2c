// Decode step for callers that cannot allocate device memory.
//
// lightning_attn_decode_step needs a caller-provided workspace (error record, one counter
// per sequence, the raw per-head outputs and per-head sums of squares).  Some callers
// cannot provide one: their device memory is owned entirely by another allocator (a
// serving engine that reserves nearly all of HBM up front for its cache and state pools,
// so an extra cudaMalloc fails or fragments the pool), or they run a latency-critical
// decode loop in which cudaMalloc, which can synchronise the device, is not allowed.
// lightning_attn_decode_step_noalloc gives them the same computation with its scratch in
// a fixed-size array compiled into this library instead.
//
// Rules of that array:
//  * It is a file-scope __device__ array of LA_DECODE_NOALLOC_SCRATCH_BYTES bytes; every GPU
//    that loads the library holds one copy until the process exits.
//  * Host code must not pass the array's name to a kernel (on the host that name is only a
//    stand-in).  Its device address is taken with cudaGetSymbolAddress, once per device,
//    with that device current, during the first call on that device; that first call should
//    therefore come before any stream capture.
//  * Every call shares the array and it keeps the previous call's contents, so each call
//    clears the per-sequence counters (the only part that must start at zero) with an
//    asynchronous memset on its stream.  Calls that overlap on the GPU (different streams,
//    or different host threads without ordering) race on the array.
//  * Sizes whose scratch would not fit are rejected with LA_ERR_UNSUPPORTED before anything
//    is enqueued.  Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
//  * The address is cached per device index for the life of the process: a device reset
//    (cudaDeviceReset) unmaps the array and makes the cached address stale, so the entry
//    point must not be called again after one.
//  * The error record lives in the array and is not visible to lightning_attn_check; the
//    decode kernel has no bounded waits, so the launch status is the whole error report.
#include <mutex>

#include "la_common.cuh"

namespace la {
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, void* out, float* state,
                          int B, int H, int D, la_dtype dt, int phi_identity, int mode, float eps,
                          const float* w, void* workspace, cudaStream_t stream,
                          const int* row_index = nullptr, const int* state_index = nullptr,
                          float* z = nullptr);
size_t decode_workspace_bytes(int B, int H, int D);
void set_last_path(const char* path);
}  // namespace la

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[LA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
la_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return LA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LA_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" la_status lightning_attn_decode_step_noalloc(const void* q, const void* k, const void* v, const void* g,
                                                        void* out, float* state, int B, int H, int D,
                                                        la_dtype dtype, la_feature_map phi, la_out_mode mode,
                                                        float eps, const float* norm_weight, la_stream_t stream) {
  if ((dtype != LA_F32 && dtype != LA_BF16) || (phi != LA_PHI_SILU && phi != LA_PHI_IDENTITY) ||
      (mode != LA_OUT_RAW && mode != LA_OUT_RMSNORM && mode != LA_OUT_RMSNORM_GATE))
    return LA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || (D != 64 && D != 128)) return LA_ERR_INVALID_ARG;
  if (mode != LA_OUT_RAW && (static_cast<int64_t>(H) * D > la::kMaxNormWidth || !(eps > 0.0f)))
    return LA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !state) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return LA_ERR_INVALID_ARG;
  if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  if (norm_weight && !aligned16(norm_weight)) return LA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H * D > (int64_t{1} << 40) ||
      la::decode_workspace_bytes(B, H, D) > LA_DECODE_NOALLOC_SCRATCH_BYTES)
    return LA_ERR_UNSUPPORTED;  // the fixed scratch is too small for this batch

  void* scratch = nullptr;
  const la_status st = scratch_address(&scratch);
  if (st != LA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Per-sequence counters follow the 256-byte error record and must start at zero.
  if (cudaMemsetAsync(static_cast<char*>(scratch) + 256, 0, sizeof(int) * static_cast<size_t>(B), s) != cudaSuccess)
    return LA_ERR_CUDA;
  const cudaError_t e = la::launch_decode(q, k, v, g, out, state, B, H, D, dtype, phi == LA_PHI_IDENTITY ? 1 : 0,
                                          static_cast<int>(mode), eps, norm_weight, scratch, s);
  if (e != cudaSuccess) return LA_ERR_CUDA;
  la::set_last_path("decode");
  return LA_OK;
}
