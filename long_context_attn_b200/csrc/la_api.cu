// C ABI of the Lightning Attention library: argument validation, kernel selection,
// workspace carving and the device error record.  Every compute step runs in the
// kernels of la_decode.cu, la_simt.cu and la_prefill_pair.cu; there is no CPU path.
#include <algorithm>
#include <cstdint>
#include <cstring>

#include "la_common.cuh"
#include "la_prefill_tc.h"

namespace la {
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, void* out, float* state,
                          int B, int H, int D, la_dtype dt, int phi_identity, int mode, float eps,
                          const float* w, void* workspace, cudaStream_t stream,
                          const int* row_index = nullptr, const int* state_index = nullptr,
                          float* z = nullptr);
size_t decode_workspace_bytes(int B, int H, int D);
cudaError_t launch_gather_single_token(const int* cu, const int* state_slot, int n, int* row_index,
                                       int* state_index, cudaStream_t stream);
cudaError_t launch_simt_prefill(const void* q, const void* k, const void* v, void* out, float* y_ws,
                                const float* state_in, float* state_out, const int* cu, int nseq, int T,
                                int H, int D, int C, la_dtype dt, int phi_identity, int64_t total_rows,
                                ErrRec* err, cudaStream_t stream);
cudaError_t launch_norm_gate(const float* y, const void* g, void* out, int64_t tokens, int HD, int mode,
                             float eps, const float* w, la_dtype dt, cudaStream_t stream);
cudaError_t launch_bwd_norm_gate(const void* y, const void* g, const void* dout, const float* w, void* dy, void* dg,
                                 float* partial, float* dw, int64_t tokens, int HD, int gate, float eps, la_dtype dt,
                                 cudaStream_t stream);
cudaError_t launch_bwd_prep(const void* q, const void* k, const void* v, const void* dy, void* fk, void* rv,
                            void* rdy, void* rfq, void* rfk, const int* cu, int nseq, int T_fixed, int64_t tokens,
                            int HD, int phi_identity, la_dtype dt, cudaStream_t stream);
cudaError_t launch_bwd_post(const void* q, const void* k, void* dq, void* dk, void* dv, const int* cu, int nseq,
                            int T_fixed, int64_t tokens, int HD, int phi_identity, la_dtype dt, cudaStream_t stream);
cudaError_t launch_transpose_states(const float* in, float* out, int64_t nmat, int D, cudaStream_t stream);
cudaError_t launch_bwd_feat(const void* q, const void* k, void* fq, void* fk, int64_t elems, int phi_identity,
                            la_dtype dt, cudaStream_t stream);
int64_t norm_weight_partial_floats(int64_t tokens, int HD);
cudaError_t launch_bwd_scale(const void* q, const void* k, void* dq, void* dk, int64_t elems, la_dtype dt,
                             cudaStream_t stream);
int znorm_max_chunks(int max_len);
int chunk_state_splits(int nseq, int H, int max_len, int num_sms);
cudaError_t launch_chunk_cu(int* cu, int B, int T, int Tc, int S, cudaStream_t stream);
cudaError_t launch_chunk_prefix(const float* cs, const float* s0, float* prefix, float* out, int B, int S, int H,
                                int reverse, int num_sms, cudaStream_t stream);
cudaError_t launch_chunk_state_tc(const void* k, const void* v, const float* state_in, float* state_out,
                                  float* partial, const int* cu, int nseq, int T, int max_len, int64_t tokens, int H,
                                  int phi_identity, int num_sms, ErrRec* err, cudaStream_t stream);
cudaError_t launch_znorm_scan(const void* q, const void* k, const float* z_in, float* sums, float* den, float* z_out,
                              const int* cu, int nseq, int T_fixed, int max_len, int64_t tokens, int H, int D,
                              la_dtype dt, int phi_identity, cudaStream_t stream);
cudaError_t launch_znorm_transform(void* io, const float* den, const void* g, const float* w, int64_t tokens, int H,
                                   int D, int mode, float eps, la_dtype dt, cudaStream_t stream);
cudaError_t launch_output_transform(const void* src, void* dst, const float* den, const void* g, const float* w,
                                    int64_t tokens, int H, int D, int mode, float eps, la_dtype dt,
                                    cudaStream_t stream);
}  // namespace la

namespace {

thread_local const char* g_last_path = "none";

constexpr size_t kErrBytes = sizeof(la::ErrRec);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

bool valid_enums(la_dtype dt, la_feature_map phi, la_out_mode mode) {
  return (dt == LA_F32 || dt == LA_BF16) && (phi == LA_PHI_SILU || phi == LA_PHI_IDENTITY) &&
         (mode == LA_OUT_RAW || mode == LA_OUT_RMSNORM || mode == LA_OUT_RMSNORM_GATE);
}

bool valid_head(int H, int D, la_out_mode mode, float eps) {
  if (H < 1 || (D != 64 && D != 128)) return false;
  if (mode != LA_OUT_RAW && (static_cast<int64_t>(H) * D > la::kMaxNormWidth || !(eps > 0.0f))) return false;
  return true;
}

int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0;
}

// Which prefill kernel a call takes.
// kTc: the tensor-core kernel with the norm fused (all of a tile's heads resident at once);
// kTcSplit: more heads than fit at once in a norm mode -- the tensor-core kernel in raw
// mode, then the norm and gate per token in place; kSimt: the CUDA-core kernel.
enum class Path { kTc, kTcSplit, kSimt };

Path choose_path(la_dtype dt, int H, int D, int C, la_out_mode mode) {
  if (!device_is_sm100()) return Path::kSimt;
  la::TcShape s{H, D, C, dt == LA_BF16, static_cast<int>(mode)};
  if (la::tc_eligible(s, current_sm_count())) return Path::kTc;
  la::TcShape raw{H, D, C, dt == LA_BF16, static_cast<int>(LA_OUT_RAW)};
  if (mode != LA_OUT_RAW && la::tc_eligible(raw, current_sm_count())) return Path::kTcSplit;
  return Path::kSimt;
}

// Long sequences with few heads (tensor-core path, fixed length): each of the B sequences
// is cut into S chunks of Tc tokens (a multiple of the tile) that run as separate
// sequences in parallel CTA-pair groups, each chunk starting from the state the chunks
// before it reach -- after it, when time runs backwards -- (their states from the
// chunk-state kernel, summed in order).
constexpr int kSplitMinChunk = 1024;
struct SplitPlan {
  int S, Tc;
};
// 2G workers per head, each owning whole sequences.  With fewer sequences than workers,
// each sequence is cut into S chunks (whole blocks of C rows) so that every worker has one:
// chunk c starts from S0 plus the states of the chunks before it (after it, when time runs
// backwards) -- the chunk-state kernel, then the ordered prefix -- and the sequence's final
// state comes from its last chunk (backwards: from the prefix).
SplitPlan chunk_plan(int B, int T, int H, int D, int C) {
  SplitPlan sp{1, T};
  if (D != 128 || B < 1 || H < 1 || T < 2 * kSplitMinChunk) return sp;
  const int workers = 2 * std::max(1, la::pair_max_active_clusters() / H);
  if (B >= workers) return sp;
  const int S = std::min((workers + B - 1) / B, T / kSplitMinChunk);
  if (S < 2) return sp;
  const int align = C > 128 ? C : 128;
  sp.Tc = ((T + S - 1) / S + align - 1) / align * align;
  sp.S = (T + sp.Tc - 1) / sp.Tc;
  if (sp.S < 2) return SplitPlan{1, T};
  return sp;
}
// Workspace of a split call after the error record: [tensor-core part for the B * S chunks]
// [chunk cu_seqlens] [chunk states] [chunk initial states] [chunk-state split partials].
struct SplitLayout {
  size_t tc, cu, st, part, total;
};
SplitLayout split_layout(const SplitPlan& sp, int B, int64_t tokens, int H, int D, int C) {
  SplitLayout l{};
  const int n = B * sp.S;
  l.tc = la::tc_workspace_bytes(n, sp.Tc, tokens, H, D, C);
  l.cu = up256(sizeof(int) * static_cast<size_t>(n + 1));
  l.st = up256(sizeof(float) * static_cast<size_t>(n) * H * D * D);
  // Chunk-state partials: the launch covers n chunks, or n - 1 when a single forward-time
  // sequence skips its last chunk, and fewer chunks may take more splits each.
  const int sms = current_sm_count();
  size_t units = static_cast<size_t>(la::chunk_state_splits(n, H, sp.Tc, sms)) * n;
  if (n > 1) units = std::max(units, static_cast<size_t>(la::chunk_state_splits(n - 1, H, sp.Tc, sms)) * (n - 1));
  l.part = up256(sizeof(float) * units * H * D * D);
  l.total = l.tc + l.cu + 2 * l.st + l.part;
  return l;
}

size_t prefill_ws_bytes(Path p, int nseq, int max_len, int64_t tokens, int H, int D, int C, la_out_mode mode) {
  if (p == Path::kTc || p == Path::kTcSplit) {
    // A fixed-length call may split (B = nseq, T = max_len); room for that is reserved here
    // (a packed call never splits and at most over-reserves).
    size_t n = la::tc_workspace_bytes(nseq, max_len, tokens, H, D, C);
    const SplitPlan fp = chunk_plan(nseq, max_len, H, D, C);
    if (fp.S > 1) n = std::max(n, split_layout(fp, nseq, tokens, H, D, C).total);
    return kErrBytes + n;
  }
  size_t y = (mode == LA_OUT_RAW) ? 0 : up256(sizeof(float) * static_cast<size_t>(tokens) * H * D);
  return kErrBytes + y;
}

la_status common_prefill(const void* q, const void* k, const void* v, const void* g, void* out,
                         const float* state_in, float* state_out, const int* cu, int nseq, int T_fixed,
                         int max_len, int64_t tokens, int H, int D, int C, la_dtype dt, la_feature_map phi,
                         la_out_mode mode, float eps, const float* w, void* workspace, size_t ws_bytes,
                         cudaStream_t stream, bool reverse = false) {
  if (!valid_enums(dt, phi, mode) || !valid_head(H, D, mode, eps)) return LA_ERR_INVALID_ARG;
  if (C < 1 || C > 1024 || nseq < 1 || tokens < 0 || max_len < 0) return LA_ERR_INVALID_ARG;
  if (tokens > 0) {
    if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  }
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)) ||
      (w && !aligned16(w)))
    return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;

  const Path path = choose_path(dt, H, D, C, mode);
  if (reverse && (path != Path::kTc || mode != LA_OUT_RAW)) return LA_ERR_UNSUPPORTED;   // internal use only
  if (ws_bytes < prefill_ws_bytes(path, nseq, max_len, tokens, H, D, C, mode)) return LA_ERR_INVALID_ARG;
  la::ErrRec* err = static_cast<la::ErrRec*>(workspace);
  char* ws = static_cast<char*>(workspace) + kErrBytes;
  const int phi_id = (phi == LA_PHI_IDENTITY) ? 1 : 0;
  cudaError_t e = cudaSuccess;
  if (path == Path::kTc || path == Path::kTcSplit) {
    const bool split = path == Path::kTcSplit;
    la::TcArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.out = out;
    a.state_in = state_in; a.state_out = state_out; a.cu = cu;
    a.nseq = nseq; a.T = T_fixed; a.max_len = max_len; a.tokens = tokens;
    a.H = H; a.D = D; a.C = C; a.phi_identity = phi_id;
    a.mode = static_cast<int>(split ? LA_OUT_RAW : mode);
    a.eps = eps; a.w = split ? nullptr : w; a.err = err; a.ws = ws;
    a.reverse = reverse ? 1 : 0;
    const bool fixed = !cu && T_fixed > 0;
    const SplitPlan sp = !fixed ? SplitPlan{1, T_fixed}
                                : chunk_plan(nseq, T_fixed, H, D, C);
    if (sp.S > 1) {
      const SplitLayout sl = split_layout(sp, nseq, tokens, H, D, C);
      char* x = ws + sl.tc;
      int* ccu = reinterpret_cast<int*>(x);
      float* cst = reinterpret_cast<float*>(x + sl.cu);
      float* cin = reinterpret_cast<float*>(x + sl.cu + sl.st);
      float* cpart = reinterpret_cast<float*>(x + sl.cu + 2 * sl.st);
      const int n = nseq * sp.S;
      e = la::launch_chunk_cu(ccu, nseq, T_fixed, sp.Tc, sp.S, stream);
      // One sequence: the state of the chunk that ends the walk (the last, or the first when
      // time runs backwards) is never needed -- the kernel ends that chunk with the sequence's
      // final state -- and the other S - 1 chunks are contiguous, so only they are summed.
      const bool skip_one = nseq == 1;
      const size_t chunk_floats = static_cast<size_t>(H) * D * D;
      if (e == cudaSuccess)
        e = la::launch_chunk_state_tc(k, v, nullptr, (skip_one && reverse) ? cst + chunk_floats : cst, cpart,
                                      (skip_one && reverse) ? ccu + 1 : ccu, skip_one ? n - 1 : n, 0, sp.Tc, tokens,
                                      H, phi_id, current_sm_count(), err, stream);
      if (e == cudaSuccess)   // chunk initial states (and, reverse time with several sequences, their final states)
        e = la::launch_chunk_prefix(cst, state_in, cin, (reverse && !skip_one) ? state_out : nullptr, nseq, sp.S, H,
                                    reverse ? 1 : 0, current_sm_count(), stream);
      a.cu = ccu;
      a.nseq = n;
      a.T = 0;
      a.max_len = sp.Tc;
      a.state_in = cin;
      if (reverse && !skip_one) {
        a.state_out = nullptr;
      } else {
        a.chunk_div = sp.S;   // the kernel writes the sequence's final state from the chunk ending the walk
      }
    }
    if (e == cudaSuccess) e = la::launch_tc_prefill(a, current_sm_count(), stream);
    if (e == cudaSuccess && split)   // the norm (and gate) per token, over the raw output in place
      e = la::launch_znorm_transform(out, nullptr, g, w, tokens, H, D, static_cast<int>(mode), eps, dt, stream);
    g_last_path = sp.S > 1 ? (split ? "tcgen05+norm+chunks" : "tcgen05+chunks") : (split ? "tcgen05+norm" : "tcgen05");
  } else {
    float* y_ws = (mode == LA_OUT_RAW) ? nullptr : reinterpret_cast<float*>(ws);
    e = la::launch_simt_prefill(q, k, v, out, y_ws, state_in, state_out, cu, nseq, T_fixed, H, D, C, dt, phi_id,
                                tokens, err, stream);
    if (e == cudaSuccess && y_ws)
      e = la::launch_norm_gate(y_ws, g, out, tokens, H * D, static_cast<int>(mode), eps, w, dt, stream);
    g_last_path = "simt";
  }
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

// Mixed step workspace: [prefill part (error record + counters + sums)] [decode part]
// [decode item token rows] [decode item state slots].  Sized for N decode items at most.
struct MixedLayout {
  size_t pre, dec, idx, total;
};
MixedLayout mixed_layout(int n, int max_pre, int64_t total, int H, int D, int C, la_out_mode mode) {
  MixedLayout m{};
  m.pre = max_pre > 1 ? prefill_ws_bytes(Path::kTc, n, max_pre, total, H, D, C, mode) : kErrBytes;
  m.dec = la::decode_workspace_bytes(n, H, D);
  m.idx = 2 * up256(sizeof(int) * static_cast<size_t>(n));
  m.total = m.pre + m.dec + m.idx;
  return m;
}

// Backward workspace: [prefill part of the raw-mode passes (error record first)] [token
// buffers] [S0^T] [dS_T^T] [dw block partials].  The token buffers are dy, phi(k), phi(q) when the tensor-core
// kernel walks time backwards itself (rev), else dy, phi(k), rho(v), rho(dy), rho(phi(q)),
// rho(phi(k)) (rho: each sequence reversed).
struct BwdLayout {
  bool rev;
  int nbuf;
  size_t pre, buf, st, part, total;
};
BwdLayout bwd_layout(int nseq, int max_len, int64_t tokens, int H, int D, int C, la_dtype dt) {
  BwdLayout b{};
  const Path raw = choose_path(dt, H, D, C, LA_OUT_RAW);
  b.rev = raw == Path::kTc;
  b.nbuf = b.rev ? 3 : 6;
  b.pre = prefill_ws_bytes(raw, nseq, max_len, tokens, H, D, C, LA_OUT_RAW);
  b.buf = up256(static_cast<size_t>(tokens) * H * D * (dt == LA_BF16 ? 2 : 4));
  b.st = up256(sizeof(float) * static_cast<size_t>(nseq) * H * D * D);
  b.part = up256(sizeof(float) * static_cast<size_t>(la::norm_weight_partial_floats(tokens, H * D)));
  b.total = b.pre + b.nbuf * b.buf + 2 * b.st + b.part;
  return b;
}

// The backward as a sequence of launches on one stream (see la_backward.cu for the
// derivation): [forward recompute of raw y, then dy/dg per token] -> prep -> three
// raw-mode identity-feature passes of the prefill kernel -> post.
la_status common_backward(const void* q, const void* k, const void* v, const void* g, const void* dout,
                          const float* state_in, const float* dstate_out, const void* y_saved, void* dq, void* dk,
                          void* dv, void* dg, float* dstate, float* dnorm_weight,
                          const int* cu, int nseq, int T_fixed, int max_len, int64_t tokens, int H, int D, int C,
                          la_dtype dt, la_feature_map phi, la_out_mode mode, float eps, const float* w,
                          void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!valid_enums(dt, phi, mode) || !valid_head(H, D, mode, eps)) return LA_ERR_INVALID_ARG;
  if (C < 1 || C > 1024 || nseq < 1 || tokens < 0 || max_len < 0) return LA_ERR_INVALID_ARG;
  if (tokens > 0) {
    for (const void* p : {q, k, v, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
      if (!p || !aligned16(p)) return LA_ERR_INVALID_ARG;
    if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g) || !dg || !aligned16(dg))) return LA_ERR_INVALID_ARG;
  }
  if ((state_in && !aligned16(state_in)) || (dstate && !aligned16(dstate)) || (w && !aligned16(w)) ||
      (dstate_out && !aligned16(dstate_out)) || (y_saved && !aligned16(y_saved)) ||
      (dnorm_weight && !aligned16(dnorm_weight)))
    return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(nseq, max_len, tokens, H, D, C, dt);
  if (ws_bytes < L.total) return LA_ERR_INVALID_ARG;

  char* base = static_cast<char*>(workspace);
  void* buf[6] = {};
  for (int i = 0; i < L.nbuf; ++i) buf[i] = base + L.pre + i * L.buf;
  float* s0t = reinterpret_cast<float*>(base + L.pre + L.nbuf * L.buf);
  float* dstt = reinterpret_cast<float*>(base + L.pre + L.nbuf * L.buf + L.st);
  float* wpart = reinterpret_cast<float*>(base + L.pre + L.nbuf * L.buf + 2 * L.st);
  void *dybuf = buf[0], *fk = buf[1], *rv = buf[2], *rdy = buf[3], *rfq = buf[4], *rfk = buf[5];
  void* fq = buf[2];   // the reverse-time composition's third buffer
  const int HD = H * D;
  const int phi_id = (phi == LA_PHI_IDENTITY) ? 1 : 0;
  auto pass = [&](const void* qq, const void* kk, const void* vv, void* out, const float* sin,
                  float* sout, la_feature_map f, bool rev = false) {
    return common_prefill(qq, kk, vv, nullptr, out, sin, sout, cu, nseq, T_fixed, max_len, tokens, H, D, C, dt, f,
                          LA_OUT_RAW, eps, nullptr, workspace, L.pre, stream, rev);
  };
  la_status st;
  const void* dy = dout;
  if (dnorm_weight && mode == LA_OUT_RAW &&   // the raw output has no norm weight
      cudaMemsetAsync(dnorm_weight, 0, sizeof(float) * static_cast<size_t>(HD), stream) != cudaSuccess)
    return LA_ERR_CUDA;
  if (mode != LA_OUT_RAW) {
    // the forward's raw y (saved by the caller, else recomputed from the same initial
    // state), then dy and dg
    const void* yv = y_saved;
    if (!yv) {
      if ((st = pass(q, k, v, dybuf, state_in, nullptr, phi)) != LA_OK) return st;
      yv = dybuf;
    }
    // dy and dg, and the norm weight's gradient when asked for
    if (la::launch_bwd_norm_gate(yv, g, dout, w, dybuf, dg, wpart, dnorm_weight, tokens, HD,
                                 mode == LA_OUT_RMSNORM_GATE ? 1 : 0, eps, dt, stream) != cudaSuccess)
      return LA_ERR_CUDA;
    dy = dybuf;
  }
  const float* s0 = nullptr;
  if (state_in) {
    if (la::launch_transpose_states(state_in, s0t, static_cast<int64_t>(nseq) * H, D, stream) != cudaSuccess)
      return LA_ERR_CUDA;
    s0 = s0t;
  }
  // A gradient reaching the final state starts the reverse sums: dphi(k) gets dS_T v, dv gets
  // dS_T^T phi(k), dS0 includes dS_T.
  const float* dsT_t = nullptr;
  if (dstate_out) {
    if (la::launch_transpose_states(dstate_out, dstt, static_cast<int64_t>(nseq) * H, D, stream) != cudaSuccess)
      return LA_ERR_CUDA;
    dsT_t = dstt;
  }
  if (L.rev) {
    // The tensor-core kernel walks time backwards itself: no reversed copies.
    if (la::launch_bwd_feat(q, k, fq, fk, tokens * HD, phi_id, dt, stream) != cudaSuccess) return LA_ERR_CUDA;
    // dphi(q): queries dy, keys v, values phi(k), initial state S0^T, forward in time
    if ((st = pass(dy, v, fk, dq, s0, nullptr, LA_PHI_IDENTITY)) != LA_OK) return st;
    // dphi(k): queries v, keys dy, values phi(q), initial state dS_T^T, backward in time
    if ((st = pass(v, dy, fq, dk, dsT_t, nullptr, LA_PHI_IDENTITY, true)) != LA_OK) return st;
    // dv: queries phi(k), keys phi(q) (the kernel's feature map on the raw k and q), values
    // dy, initial state dS_T, backward in time; its final state is dS0
    if ((st = pass(k, q, dy, dv, dstate_out, dstate, phi, true)) != LA_OK) return st;
    if (!phi_id && la::launch_bwd_scale(q, k, dq, dk, tokens * HD, dt, stream) != cudaSuccess) return LA_ERR_CUDA;
    return LA_OK;
  }
  if (la::launch_bwd_prep(q, k, v, dy, fk, rv, rdy, rfq, rfk, cu, nseq, T_fixed, tokens, HD, phi_id, dt, stream) !=
      cudaSuccess)
    return LA_ERR_CUDA;
  // dphi(q): queries dy, keys v, values phi(k), initial state S0^T
  if ((st = pass(dy, v, fk, dq, s0, nullptr, LA_PHI_IDENTITY)) != LA_OK) return st;
  // reversed dphi(k): queries rho(v), keys rho(dy), values rho(phi(q)), initial state dS_T^T
  if ((st = pass(rv, rdy, rfq, dk, dsT_t, nullptr, LA_PHI_IDENTITY)) != LA_OK) return st;
  // reversed dv: queries rho(phi(k)), keys rho(phi(q)), values rho(dy), initial state dS_T;
  // its final state is dS0
  if ((st = pass(rfk, rfq, rdy, dv, dstate_out, dstate, LA_PHI_IDENTITY)) != LA_OK) return st;
  if (la::launch_bwd_post(q, k, dq, dk, dv, cu, nseq, T_fixed, tokens, HD, phi_id, dt, stream) != cudaSuccess)
    return LA_ERR_CUDA;
  return LA_OK;
}

// Chunk state: the tensor-core kernel (bf16, D = 128, sm_100a) needs the error record and
// one fp32 partial state per split; elsewhere a raw-mode prefill runs with its outputs
// written to scratch (its prefill part, then the scratch outputs).
bool chunk_state_tc(la_dtype dt, int D) { return dt == LA_BF16 && D == 128 && device_is_sm100(); }
constexpr int kChunkFallbackC = 128;
size_t chunk_state_ws_bytes(int nseq, int max_len, int64_t tokens, int H, int D, la_dtype dt) {
  if (chunk_state_tc(dt, D)) {
    const int sp = la::chunk_state_splits(nseq, H, max_len, current_sm_count());
    return kErrBytes + up256(sizeof(float) * static_cast<size_t>(sp) * nseq * H * D * D);
  }
  const Path path = choose_path(dt, H, D, kChunkFallbackC, LA_OUT_RAW);
  return prefill_ws_bytes(path, nseq, max_len, tokens, H, D, kChunkFallbackC, LA_OUT_RAW) +
         up256(static_cast<size_t>(tokens) * H * D * (dt == LA_BF16 ? 2 : 4));
}

// Normalised-variant workspace: [prefill part of the raw pass (error record first)]
// [phi(k) chunk sums: nseq x H x chunks x D fp32] [denominators: tokens x H fp32].
// Normalised-variant workspace: [raw prefill part] [chunk sums of phi(k)] [denominators]
// [a copy of z_in, used when z_out overlaps it].
struct ZLayout {
  size_t pre, sums, den, zin, total;
};
ZLayout z_layout(int nseq, int max_len, int64_t tokens, int H, int D, int C, la_dtype dt) {
  ZLayout z{};
  z.pre = prefill_ws_bytes(choose_path(dt, H, D, C, LA_OUT_RAW), nseq, max_len, tokens, H, D, C, LA_OUT_RAW);
  z.sums = up256(sizeof(float) * static_cast<size_t>(nseq) * H * la::znorm_max_chunks(max_len) * D);
  z.den = up256(sizeof(float) * static_cast<size_t>(tokens) * H);
  z.zin = up256(sizeof(float) * static_cast<size_t>(nseq) * H * D);
  z.total = z.pre + z.sums + z.den + z.zin;
  return z;
}

// y = phi(q)^T S / (phi(q) . z): the raw prefill gives the numerators (and carries S), the
// scan gives the denominators (and carries z), then y / den and the output transform.
la_status common_prefill_znorm(const void* q, const void* k, const void* v, const void* g, void* out,
                               const float* state_in, const float* z_in, float* state_out, float* z_out,
                               const int* cu, int nseq, int T_fixed, int max_len, int64_t tokens, int H, int D,
                               int C, la_dtype dt, la_feature_map phi, la_out_mode mode, float eps, const float* w,
                               void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!valid_enums(dt, phi, mode) || !valid_head(H, D, mode, eps)) return LA_ERR_INVALID_ARG;
  if (C < 1 || C > 1024 || nseq < 1 || nseq > 65535 || tokens < 0 || max_len < 0) return LA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(H) * D > la::kMaxNormWidth) return LA_ERR_UNSUPPORTED;   // per-token reciprocals
  if (tokens > 0 && mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  if ((z_in && !aligned16(z_in)) || (z_out && !aligned16(z_out))) return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  const ZLayout L = z_layout(nseq, max_len, tokens, H, D, C, dt);
  if (ws_bytes < L.total) return LA_ERR_INVALID_ARG;
  char* base = static_cast<char*>(workspace);
  float* sums = reinterpret_cast<float*>(base + L.pre);
  float* den = reinterpret_cast<float*>(base + L.pre + L.sums);
  la_status st = common_prefill(q, k, v, nullptr, out, state_in, state_out, cu, nseq, T_fixed, max_len, tokens, H,
                                D, C, dt, phi, LA_OUT_RAW, eps, nullptr, workspace, L.pre, stream);
  if (st != LA_OK) return st;
  const int phi_id = (phi == LA_PHI_IDENTITY) ? 1 : 0;
  // z_out may be z_in (in place), but the scan's chunk items of a sequence all read z_in
  // while its last item writes z_out, with no order between them: read a copy then.
  const size_t zbytes = sizeof(float) * static_cast<size_t>(nseq) * H * D;
  const uintptr_t zi = reinterpret_cast<uintptr_t>(z_in), zo = reinterpret_cast<uintptr_t>(z_out);
  if (z_in && z_out && zi < zo + zbytes && zo < zi + zbytes) {
    float* zcopy = reinterpret_cast<float*>(base + L.pre + L.sums + L.den);
    if (cudaMemcpyAsync(zcopy, z_in, zbytes, cudaMemcpyDeviceToDevice, stream) != cudaSuccess) return LA_ERR_CUDA;
    z_in = zcopy;
  }
  if (la::launch_znorm_scan(q, k, z_in, sums, den, z_out, cu, nseq, T_fixed, max_len, tokens, H, D, dt, phi_id,
                            stream) != cudaSuccess)
    return LA_ERR_CUDA;
  if (la::launch_znorm_transform(out, den, g, w, tokens, H, D, static_cast<int>(mode), eps, dt, stream) !=
      cudaSuccess)
    return LA_ERR_CUDA;
  return LA_OK;
}

// The output transform's backward: the norm weight's gradient as per-CTA partial rows.
size_t output_transform_backward_ws_bytes(int64_t tokens, int HD) {
  return std::max<size_t>(256, up256(sizeof(float) * static_cast<size_t>(la::norm_weight_partial_floats(tokens, HD))));
}

}  // namespace

namespace la {
// Lets entry points defined in other files record their path (the workspace-free decode).
void set_last_path(const char* path) { g_last_path = path; }
}  // namespace la

extern "C" {

la_status lightning_attn_prefill(const void* q, const void* k, const void* v, const void* g, void* out,
                                 const float* state_in, float* state_out, int B, int T, int H, int D,
                                 int block_size, la_dtype dtype, la_feature_map phi, la_out_mode mode,
                                 float eps, const float* norm_weight, void* workspace, size_t workspace_bytes,
                                 la_stream_t stream) {
  if (B < 1 || T < 0) return LA_ERR_INVALID_ARG;
  const int64_t tokens = static_cast<int64_t>(B) * T;
  if (tokens > INT32_MAX) return LA_ERR_UNSUPPORTED;
  return common_prefill(q, k, v, g, out, state_in, state_out, nullptr, B, T, T, tokens, H, D, block_size, dtype,
                        phi, mode, eps, norm_weight, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_backward(const void* q, const void* k, const void* v, const void* g, const void* dout,
                                  const float* state_in, const float* dstate_out, const void* y, void* dq, void* dk,
                                  void* dv, void* dg, float* dstate_in, float* dnorm_weight,
                                  int B, int T, int H, int D, int block_size, la_dtype dtype, la_feature_map phi,
                                  la_out_mode mode, float eps, const float* norm_weight, void* workspace,
                                  size_t workspace_bytes, la_stream_t stream) {
  if (B < 1 || T < 0) return LA_ERR_INVALID_ARG;
  const int64_t tokens = static_cast<int64_t>(B) * T;
  if (tokens > INT32_MAX) return LA_ERR_UNSUPPORTED;
  return common_backward(q, k, v, g, dout, state_in, dstate_out, y, dq, dk, dv, dg, dstate_in, dnorm_weight, nullptr,
                         B, T, T, tokens, H, D, block_size, dtype, phi, mode, eps, norm_weight, workspace,
                         workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_backward_varlen(const void* q, const void* k, const void* v, const void* g,
                                         const void* dout, const float* state_in, const float* dstate_out,
                                         const void* y, void* dq, void* dk, void* dv, void* dg, float* dstate_in,
                                         float* dnorm_weight, const int* cu_seqlens, int num_seqs,
                                         int max_seqlen, int total_tokens, int H, int D, int block_size,
                                         la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                         const float* norm_weight, void* workspace, size_t workspace_bytes,
                                         la_stream_t stream) {
  if (num_seqs < 1 || !cu_seqlens || !aligned16(cu_seqlens) || total_tokens < 0 || max_seqlen < 0)
    return LA_ERR_INVALID_ARG;
  return common_backward(q, k, v, g, dout, state_in, dstate_out, y, dq, dk, dv, dg, dstate_in, dnorm_weight,
                         cu_seqlens, num_seqs, 0, max_seqlen, total_tokens, H, D, block_size, dtype, phi, mode, eps,
                         norm_weight, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_output_transform(const void* y, const void* g, void* out, int tokens, int H, int D,
                                          la_dtype dtype, la_out_mode mode, float eps, const float* norm_weight,
                                          la_stream_t stream) {
  if (tokens < 0 || H < 1 || (D != 64 && D != 128) || static_cast<int64_t>(H) * D > la::kMaxNormWidth)
    return LA_ERR_INVALID_ARG;
  if (!valid_enums(dtype, LA_PHI_SILU, mode) || (mode != LA_OUT_RAW && !(eps > 0.0f))) return LA_ERR_INVALID_ARG;
  if (tokens > 0) {
    if (!y || !out || !aligned16(y) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  }
  if (norm_weight && !aligned16(norm_weight)) return LA_ERR_INVALID_ARG;
  const cudaError_t e = la::launch_output_transform(y, out, nullptr, g, norm_weight, tokens, H, D,
                                                    static_cast<int>(mode), eps, dtype,
                                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status lightning_attn_output_transform_backward(const void* y, const void* g, const void* dout, void* dy, void* dg,
                                                   float* dnorm_weight, int tokens, int H, int D, la_dtype dtype,
                                                   la_out_mode mode, float eps, const float* norm_weight,
                                                   void* workspace, size_t workspace_bytes, la_stream_t stream) {
  if (tokens < 0 || H < 1 || (D != 64 && D != 128) || static_cast<int64_t>(H) * D > la::kMaxNormWidth)
    return LA_ERR_INVALID_ARG;
  if (!valid_enums(dtype, LA_PHI_SILU, mode) || (mode != LA_OUT_RAW && !(eps > 0.0f))) return LA_ERR_INVALID_ARG;
  if (tokens > 0) {
    if (!dout || !dy || !aligned16(dout) || !aligned16(dy)) return LA_ERR_INVALID_ARG;
    if (mode != LA_OUT_RAW && (!y || !aligned16(y))) return LA_ERR_INVALID_ARG;
    if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g) || !dg || !aligned16(dg))) return LA_ERR_INVALID_ARG;
    if (dy == dout || (mode == LA_OUT_RMSNORM_GATE && (dy == g || dg == y || dg == dout || dg == dy)))
      return LA_ERR_INVALID_ARG;
  }
  if ((norm_weight && !aligned16(norm_weight)) || (dnorm_weight && !aligned16(dnorm_weight)))
    return LA_ERR_INVALID_ARG;
  const int HD = H * D;
  const bool want_dw = dnorm_weight && mode != LA_OUT_RAW;
  if (want_dw && (!workspace || !aligned256(workspace) ||
                  workspace_bytes < output_transform_backward_ws_bytes(tokens, HD)))
    return LA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (mode == LA_OUT_RAW) {   // dy = dout; the raw output has no norm weight
    const size_t bytes = static_cast<size_t>(tokens) * HD * (dtype == LA_BF16 ? 2 : 4);
    if (bytes && cudaMemcpyAsync(dy, dout, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return LA_ERR_CUDA;
    if (dnorm_weight && cudaMemsetAsync(dnorm_weight, 0, sizeof(float) * HD, st) != cudaSuccess) return LA_ERR_CUDA;
    return LA_OK;
  }
  const cudaError_t e = la::launch_bwd_norm_gate(y, g, dout, norm_weight, dy, dg,
                                                 want_dw ? static_cast<float*>(workspace) : nullptr,
                                                 want_dw ? dnorm_weight : nullptr, tokens, HD,
                                                 mode == LA_OUT_RMSNORM_GATE ? 1 : 0, eps, dtype, st);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status lightning_attn_chunk_state(const void* k, const void* v, const float* state_in, float* state_out, int B,
                                     int T, int H, int D, la_dtype dtype, la_feature_map phi, void* workspace,
                                     size_t workspace_bytes, la_stream_t stream) {
  if (B < 1 || B > 65535 || T < 0 || H < 1 || H > 65535 || (D != 64 && D != 128)) return LA_ERR_INVALID_ARG;
  if ((dtype != LA_F32 && dtype != LA_BF16) || (phi != LA_PHI_SILU && phi != LA_PHI_IDENTITY))
    return LA_ERR_INVALID_ARG;
  const int64_t tokens = static_cast<int64_t>(B) * T;
  if (tokens > INT32_MAX) return LA_ERR_UNSUPPORTED;
  if (!state_out || !aligned16(state_out) || (state_in && !aligned16(state_in))) return LA_ERR_INVALID_ARG;
  if (tokens > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  if (workspace_bytes < chunk_state_ws_bytes(B, T, tokens, H, D, dtype)) return LA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (chunk_state_tc(dtype, D)) {
    la::ErrRec* err = static_cast<la::ErrRec*>(workspace);
    float* partial = reinterpret_cast<float*>(static_cast<char*>(workspace) + kErrBytes);
    const cudaError_t e = la::launch_chunk_state_tc(k, v, state_in, state_out, partial, nullptr, B, T, T, tokens, H,
                                                    phi == LA_PHI_IDENTITY ? 1 : 0, current_sm_count(), err, st);
    g_last_path = "tcgen05-state";
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }
  // Elsewhere: the raw prefill of (k, k, v) from state_in; its outputs go to scratch.
  const Path path = choose_path(dtype, H, D, kChunkFallbackC, LA_OUT_RAW);
  const size_t pre = prefill_ws_bytes(path, B, T, tokens, H, D, kChunkFallbackC, LA_OUT_RAW);
  void* scratch = static_cast<char*>(workspace) + pre;
  return common_prefill(k, k, v, nullptr, scratch, state_in, state_out, nullptr, B, T, T, tokens, H, D,
                        kChunkFallbackC, dtype, phi, LA_OUT_RAW, 1e-6f, nullptr, workspace, pre, st);
}

la_status lightning_attn_prefill_znorm(const void* q, const void* k, const void* v, const void* g, void* out,
                                       const float* state_in, const float* z_in, float* state_out, float* z_out,
                                       int B, int T, int H, int D, int block_size, la_dtype dtype,
                                       la_feature_map phi, la_out_mode mode, float eps, const float* norm_weight,
                                       void* workspace, size_t workspace_bytes, la_stream_t stream) {
  if (B < 1 || T < 0) return LA_ERR_INVALID_ARG;
  const int64_t tokens = static_cast<int64_t>(B) * T;
  if (tokens > INT32_MAX) return LA_ERR_UNSUPPORTED;
  return common_prefill_znorm(q, k, v, g, out, state_in, z_in, state_out, z_out, nullptr, B, T, T, tokens, H, D,
                              block_size, dtype, phi, mode, eps, norm_weight, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_prefill_znorm_varlen(const void* q, const void* k, const void* v, const void* g, void* out,
                                              const float* state_in, const float* z_in, float* state_out,
                                              float* z_out, const int* cu_seqlens, int num_seqs, int max_seqlen,
                                              int total_tokens, int H, int D, int block_size, la_dtype dtype,
                                              la_feature_map phi, la_out_mode mode, float eps,
                                              const float* norm_weight, void* workspace, size_t workspace_bytes,
                                              la_stream_t stream) {
  if (num_seqs < 1 || !cu_seqlens || !aligned16(cu_seqlens) || total_tokens < 0 || max_seqlen < 0)
    return LA_ERR_INVALID_ARG;
  return common_prefill_znorm(q, k, v, g, out, state_in, z_in, state_out, z_out, cu_seqlens, num_seqs, 0,
                              max_seqlen, total_tokens, H, D, block_size, dtype, phi, mode, eps, norm_weight,
                              workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_decode_step_znorm(const void* q, const void* k, const void* v, const void* g, void* out,
                                           float* state, float* z, int B, int H, int D, la_dtype dtype,
                                           la_feature_map phi, la_out_mode mode, float eps, const float* norm_weight,
                                           void* workspace, size_t workspace_bytes, la_stream_t stream) {
  if (!z || !aligned16(z)) return LA_ERR_INVALID_ARG;
  if (!valid_enums(dtype, phi, mode) || !valid_head(H, D, mode, eps) || B < 1) return LA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H > INT32_MAX / 2) return LA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !state) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return LA_ERR_INVALID_ARG;
  if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  if (norm_weight && !aligned16(norm_weight)) return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  if (workspace_bytes < la::decode_workspace_bytes(B, H, D)) return LA_ERR_INVALID_ARG;
  cudaError_t e = la::launch_decode(q, k, v, g, out, state, B, H, D, dtype, phi == LA_PHI_IDENTITY ? 1 : 0,
                                    static_cast<int>(mode), eps, norm_weight, workspace,
                                    reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, z);
  g_last_path = "decode";
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status lightning_attn_prefill_varlen(const void* q, const void* k, const void* v, const void* g, void* out,
                                        const float* state_in, float* state_out, const int* cu_seqlens,
                                        int num_seqs, int max_seqlen, int total_tokens, int H, int D,
                                        int block_size, la_dtype dtype, la_feature_map phi, la_out_mode mode,
                                        float eps, const float* norm_weight, void* workspace,
                                        size_t workspace_bytes, la_stream_t stream) {
  if (num_seqs < 1 || !cu_seqlens || !aligned16(cu_seqlens) || total_tokens < 0 || max_seqlen < 0)
    return LA_ERR_INVALID_ARG;
  return common_prefill(q, k, v, g, out, state_in, state_out, cu_seqlens, num_seqs, 0, max_seqlen, total_tokens,
                        H, D, block_size, dtype, phi, mode, eps, norm_weight, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

la_status lightning_attn_decode_step(const void* q, const void* k, const void* v, const void* g, void* out,
                                     float* state, int B, int H, int D, la_dtype dtype, la_feature_map phi,
                                     la_out_mode mode, float eps, const float* norm_weight, void* workspace,
                                     size_t workspace_bytes, la_stream_t stream) {
  if (!valid_enums(dtype, phi, mode) || !valid_head(H, D, mode, eps) || B < 1) return LA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H > INT32_MAX / 2) return LA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !state) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state))
    return LA_ERR_INVALID_ARG;
  if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  if (norm_weight && !aligned16(norm_weight)) return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  if (workspace_bytes < la::decode_workspace_bytes(B, H, D)) return LA_ERR_INVALID_ARG;
  cudaError_t e = la::launch_decode(q, k, v, g, out, state, B, H, D, dtype, phi == LA_PHI_IDENTITY ? 1 : 0,
                                    static_cast<int>(mode), eps, norm_weight, workspace,
                                    reinterpret_cast<cudaStream_t>(stream));
  g_last_path = "decode";
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status lightning_attn_mixed_step(const void* q, const void* k, const void* v, const void* g, void* out,
                                    const int* cu_seqlens, const int* cu_seqlens_host, float* state_pool,
                                    const int* state_slot, int num_seqs, int H, int D, int block_size,
                                    la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                    const float* norm_weight, void* workspace, size_t workspace_bytes,
                                    la_stream_t prefill_stream, la_stream_t decode_stream) {
  if (!valid_enums(dtype, phi, mode) || !valid_head(H, D, mode, eps)) return LA_ERR_INVALID_ARG;
  if (num_seqs < 1 || !cu_seqlens || !cu_seqlens_host || !state_pool || !state_slot || !aligned16(cu_seqlens) ||
      !aligned16(state_pool))
    return LA_ERR_INVALID_ARG;
  if (block_size < 1 || block_size > 1024) return LA_ERR_INVALID_ARG;
  // The split: one-token sequences decode, longer ones prefill.
  int n_dec = 0, max_pre = 0;
  if (cu_seqlens_host[0] < 0) return LA_ERR_INVALID_ARG;
  for (int s = 0; s < num_seqs; ++s) {
    const int L = cu_seqlens_host[s + 1] - cu_seqlens_host[s];
    if (L < 0) return LA_ERR_INVALID_ARG;
    if (L == 1) ++n_dec;
    if (L > max_pre) max_pre = L;
  }
  const int64_t total = cu_seqlens_host[num_seqs];
  if (total > 0) {
    if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_INVALID_ARG;
    if (mode == LA_OUT_RMSNORM_GATE && (!g || !aligned16(g))) return LA_ERR_INVALID_ARG;
  }
  if (norm_weight && !aligned16(norm_weight)) return LA_ERR_INVALID_ARG;
  if (!workspace || !aligned256(workspace)) return LA_ERR_INVALID_ARG;
  if (choose_path(dtype, H, D, block_size, mode) != Path::kTc) return LA_ERR_UNSUPPORTED;
  const MixedLayout lay = mixed_layout(num_seqs, max_pre, total, H, D, block_size, mode);
  if (workspace_bytes < lay.total) return LA_ERR_INVALID_ARG;

  char* base = static_cast<char*>(workspace);
  la::ErrRec* err = reinterpret_cast<la::ErrRec*>(base);
  const int phi_id = (phi == LA_PHI_IDENTITY) ? 1 : 0;
  cudaStream_t ps = reinterpret_cast<cudaStream_t>(prefill_stream);
  cudaStream_t ds = reinterpret_cast<cudaStream_t>(decode_stream);
  cudaError_t e = cudaSuccess;
  if (max_pre > 1) {
    la::TcArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.out = out;
    a.state_in = state_pool; a.state_out = state_pool; a.cu = cu_seqlens;
    a.nseq = num_seqs; a.T = 0; a.max_len = max_pre; a.tokens = total;
    a.H = H; a.D = D; a.C = block_size; a.phi_identity = phi_id; a.mode = static_cast<int>(mode);
    a.eps = eps; a.w = norm_weight; a.err = err; a.ws = base + kErrBytes;
    a.state_index = state_slot;
    a.skip_single = 1;
    e = la::launch_tc_prefill(a, current_sm_count(), ps);
  }
  if (e == cudaSuccess && n_dec > 0) {
    char* dws = base + lay.pre;
    int* rows = reinterpret_cast<int*>(base + lay.pre + lay.dec);
    int* slots = reinterpret_cast<int*>(base + lay.pre + lay.dec + lay.idx / 2);
    // The decode counters live where the previous step's layout may have left other data.
    e = cudaMemsetAsync(dws, 0, lay.dec, ds);
    if (e == cudaSuccess) e = la::launch_gather_single_token(cu_seqlens, state_slot, num_seqs, rows, slots, ds);
    if (e == cudaSuccess)
      e = la::launch_decode(q, k, v, g, out, state_pool, n_dec, H, D, dtype, phi_id, static_cast<int>(mode), eps,
                            norm_weight, dws, ds, rows, slots);
  }
  g_last_path = "mixed";
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

size_t lightning_attn_workspace_size(la_op op, int B_or_N, int T_or_max, int total_tokens, int H, int D,
                                     int block_size, la_dtype dtype, la_out_mode mode) {
  if (op == LA_OP_OUTPUT_TRANSFORM_BACKWARD) {   // B_or_N = tokens
    if (B_or_N < 0 || H < 1 || (D != 64 && D != 128)) return 0;
    return output_transform_backward_ws_bytes(B_or_N, H * D);
  }
  if (B_or_N < 1 || T_or_max < 0 || H < 1 || (D != 64 && D != 128)) return 0;
  if (op == LA_OP_DECODE) return la::decode_workspace_bytes(B_or_N, H, D);
  if (op == LA_OP_MIXED) {
    if (total_tokens < 0 || block_size < 1 || block_size > 1024) return 0;
    return mixed_layout(B_or_N, T_or_max, total_tokens, H, D, block_size, mode).total;
  }
  if (op == LA_OP_CHUNK_STATE)   // no block size: the state does not depend on it
    return chunk_state_ws_bytes(B_or_N, T_or_max, static_cast<int64_t>(B_or_N) * T_or_max, H, D, dtype);
  if (block_size < 1 || block_size > 1024) return 0;
  const Path path = choose_path(dtype, H, D, block_size, mode);
  if (op == LA_OP_PREFILL)
    return prefill_ws_bytes(path, B_or_N, T_or_max, static_cast<int64_t>(B_or_N) * T_or_max, H, D, block_size,
                            mode);
  if (op == LA_OP_PREFILL_VARLEN) {
    if (total_tokens < 0) return 0;
    return prefill_ws_bytes(path, B_or_N, T_or_max, total_tokens, H, D, block_size, mode);
  }
  if (op == LA_OP_PREFILL_ZNORM)
    return z_layout(B_or_N, T_or_max, static_cast<int64_t>(B_or_N) * T_or_max, H, D, block_size, dtype).total;
  if (op == LA_OP_PREFILL_ZNORM_VARLEN) {
    if (total_tokens < 0) return 0;
    return z_layout(B_or_N, T_or_max, total_tokens, H, D, block_size, dtype).total;
  }
  if (op == LA_OP_BACKWARD)
    return bwd_layout(B_or_N, T_or_max, static_cast<int64_t>(B_or_N) * T_or_max, H, D, block_size, dtype).total;
  if (op == LA_OP_BACKWARD_VARLEN) {
    if (total_tokens < 0) return 0;
    return bwd_layout(B_or_N, T_or_max, total_tokens, H, D, block_size, dtype).total;
  }
  return 0;
}

la_status lightning_attn_check(void* workspace, la_stream_t stream, unsigned int* detail) {
  if (!workspace) return LA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LA_ERR_CUDA;
  unsigned int rec[4] = {0, 0, 0, 0};
  if (cudaMemcpy(rec, workspace, sizeof(rec), cudaMemcpyDeviceToHost) != cudaSuccess) return LA_ERR_CUDA;
  if (detail) std::memcpy(detail, rec, sizeof(rec));
  if (rec[0] == 0) return LA_OK;
  if (cudaMemset(workspace, 0, sizeof(rec)) != cudaSuccess) return LA_ERR_CUDA;
  return static_cast<la_status>(rec[0]);
}

const char* lightning_attn_status_string(la_status s) {
  switch (s) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
    case LA_ERR_CUDA: return "LA_ERR_CUDA";
    case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    case LA_ERR_DEVICE: return "LA_ERR_DEVICE";
  }
  return "LA_ERR_UNKNOWN";
}

const char* lightning_attn_last_path(void) { return g_last_path; }

}  // extern "C"
