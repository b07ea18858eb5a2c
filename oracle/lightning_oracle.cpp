// Lightning Attention forward -- plain fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline / reference arm may load or run this code.  It shares no code,
// header, table or helper with the CUDA library, and it never routes product calls.
//
// Sources (web pages; cited by title and section):
//   [Tut64]  "六十四：MiniMax-01" (LLM tutorial, lesson 64), section 3 "Lightning Attention 的定位":
//            linear attention as a running state, S_t = S_{t-1} + phi(k_t) v_t^T, and the
//            output read from the state, phi(q_t)^T S_t (sum over i <= t: causal, inclusive);
//            in its normalised form also z_t = z_{t-1} + phi(k_t) and the division by
//            phi(q_t)^T z_t.
//   [Arch]   "MiniMax-Text-01 405B MoE模型架构与训练策略解析", section 2.1 "Lightning Attention-2":
//            Q, K, V = SiLU(X);  Y = Q * (K^T * V);  output = RMSNorm(Y) * sigmoid(X).
//   [Ops]    "MiniMax-01技术报告解读（二）计算优化", section 3: lightning_attention_chunk_size 256 and
//            lightning_attention_pad_options [32, 64, 128] (block size and tail padding).
//
// Readings taken where the pages are silent or disagree (each is listed with the design notes):
//   * phi = SiLU on q and k only; v is used raw (the workload statement applies SiLU to Q, K).
//   * No normaliser z and no denominator: [Arch] feeds Y straight into RMSNorm.
//   * No decay factor and no 1/sqrt(d) scaling (neither appears in the linear form).
//   * Causal mask inclusive (i <= t); a decode step updates S first, then reads it.
//   * RMSNorm over the concatenation of all heads of a token (H*D values), eps inside the
//     square root: r = 1/sqrt(mean(y^2) + eps); then multiply by weight w and sigmoid(g).
//
// Every function computes in fp64 from the exact widening of the stored inputs
// (bf16 bits or fp32).  Layouts: q, k, v [tokens, H, D]; g and out [tokens, H*D];
// states [seq, H, D(k), D(v)] row-major.

#include <omp.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

namespace {

enum { DT_F32 = 0, DT_BF16 = 1 };
enum { PHI_SILU = 0, PHI_IDENTITY = 1 };
enum { MODE_RAW = 0, MODE_RMSNORM = 1, MODE_RMSNORM_GATE = 2 };

inline double widen(const void* base, int dtype, int64_t i) {
  if (dtype == DT_BF16) {
    uint32_t u = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[i]) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return static_cast<double>(f);
  }
  return static_cast<double>(static_cast<const float*>(base)[i]);
}

// [Arch] 2.1: SiLU(x) = x * sigmoid(x) = x / (1 + e^-x).
inline double silu(double x) { return x / (1.0 + std::exp(-x)); }
inline double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }
inline double feature(double x, int phi) { return phi == PHI_SILU ? silu(x) : x; }

// Token-by-token recurrence for one head over rows [row0, row0 + n) of the packed
// [tokens, H, D] inputs.  S (D x D, fp64) enters as the state before the first
// token and leaves as the state after the last.  y receives, for each token, the
// D values phi(q_t)^T S_t at y[(t * H + h) * D + j]  ([Tut64] section 3).
void recur_head(const void* q, const void* k, const void* v, int dtype, int64_t row0, int64_t n,
                int H, int D, int h, int phi, double* S, double* y) {
  std::vector<double> fq(D), fk(D), vv(D), acc(D);
  for (int64_t t = 0; t < n; ++t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      fq[i] = feature(widen(q, dtype, base + i), phi);
      fk[i] = feature(widen(k, dtype, base + i), phi);
      vv[i] = widen(v, dtype, base + i);
      acc[i] = 0.0;
    }
    // S_t = S_{t-1} + phi(k_t) v_t^T, then y_t = phi(q_t)^T S_t.
    for (int i = 0; i < D; ++i) {
      double* Si = S + static_cast<int64_t>(i) * D;
      const double a = fk[i], b = fq[i];
      for (int j = 0; j < D; ++j) {
        Si[j] += a * vv[j];
        acc[j] += b * Si[j];
      }
    }
    double* yt = y + (t * H + h) * static_cast<int64_t>(D);
    for (int j = 0; j < D; ++j) yt[j] = acc[j];
  }
}

// Output transform of one token ([Arch] 2.1): concatenate the H heads (index h*D + j),
// then RAW: o = y; RMSNORM: o = y * r * w; RMSNORM_GATE: o = y * r * w * sigmoid(g),
// with r = 1 / sqrt(mean(y^2) + eps) over the H*D values.
void transform_token(const double* y, int HD, int mode, double eps, const float* w,
                     const void* g, int dtype, int64_t grow, double* o) {
  if (mode == MODE_RAW) {
    for (int c = 0; c < HD; ++c) o[c] = y[c];
    return;
  }
  double ss = 0.0;
  for (int c = 0; c < HD; ++c) ss += y[c] * y[c];
  const double r = 1.0 / std::sqrt(ss / HD + eps);
  for (int c = 0; c < HD; ++c) {
    double val = y[c] * r * (w ? static_cast<double>(w[c]) : 1.0);
    if (mode == MODE_RMSNORM_GATE) val *= sigmoid(widen(g, dtype, grow * HD + c));
    o[c] = val;
  }
}

// Comparison accumulator for the streaming check of a candidate output.
struct Cmp {
  double max_ref = 0.0, max_err = 0.0;
  int64_t argmax = -1, nonfinite = 0;
};

inline void cmp_update(Cmp& c, double ref, double cand, int64_t idx) {
  if (!std::isfinite(cand)) { c.nonfinite++; return; }
  c.max_ref = std::max(c.max_ref, std::fabs(ref));
  double e = std::fabs(ref - cand);
  if (e > c.max_err) { c.max_err = e; c.argmax = idx; }
}

// One packed sequence: rows [row0, row0 + L).  The H recurrences run in parallel
// over token chunks; each chunk's outputs are transformed and either stored
// (out != nullptr) or compared against `cand` (a dtype tensor [tokens, H*D]).
void run_sequence(const void* q, const void* k, const void* v, const void* g, int dtype,
                  int64_t row0, int64_t L, int H, int D, int phi, int mode, double eps,
                  const float* w, std::vector<double>& states /* H*D*D, in/out */,
                  double* out, const void* cand, Cmp* cmp) {
  const int HD = H * D;
  const int64_t CH = 256;
  std::vector<double> y(static_cast<size_t>(CH) * HD);
  std::vector<double> o(static_cast<size_t>(CH) * HD);
  for (int64_t c0 = 0; c0 < L; c0 += CH) {
    const int64_t n = std::min(CH, L - c0);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h)
      recur_head(q, k, v, dtype, row0 + c0, n, H, D, h, phi,
                 states.data() + static_cast<size_t>(h) * D * D, y.data());
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
      double* ot = out ? out + (row0 + c0 + t) * HD : o.data() + t * HD;
      transform_token(y.data() + t * HD, HD, mode, eps, w, g, dtype, row0 + c0 + t, ot);
    }
    if (cand) {
      Cmp local;
      for (int64_t t = 0; t < n; ++t) {
        const int64_t grow = row0 + c0 + t;
        const double* ot = out ? out + grow * HD : o.data() + t * HD;
        for (int c = 0; c < HD; ++c)
          cmp_update(local, ot[c], widen(cand, dtype, grow * HD + c), grow * HD + c);
      }
      cmp->max_ref = std::max(cmp->max_ref, local.max_ref);
      cmp->nonfinite += local.nonfinite;
      if (local.max_err > cmp->max_err) { cmp->max_err = local.max_err; cmp->argmax = local.argmax; }
    }
  }
}

void load_states(std::vector<double>& st, const float* state_in, int64_t seq, int H, int D) {
  const int64_t n = static_cast<int64_t>(H) * D * D;
  st.assign(n, 0.0);
  if (state_in)
    for (int64_t i = 0; i < n; ++i) st[i] = static_cast<double>(state_in[seq * n + i]);
}

void finish_states(const std::vector<double>& st, int64_t seq, int H, int D, double* state_out,
                   const float* cand_state, Cmp* scmp) {
  const int64_t n = static_cast<int64_t>(H) * D * D;
  if (state_out)
    for (int64_t i = 0; i < n; ++i) state_out[seq * n + i] = st[i];
  if (cand_state && scmp)
    for (int64_t i = 0; i < n; ++i)
      cmp_update(*scmp, st[i], static_cast<double>(cand_state[seq * n + i]), seq * n + i);
}

void write_stats(double* stats, const Cmp& o, const Cmp& s) {
  if (!stats) return;
  stats[0] = o.max_ref; stats[1] = o.max_err; stats[2] = static_cast<double>(o.argmax);
  stats[3] = static_cast<double>(o.nonfinite);
  stats[4] = s.max_ref; stats[5] = s.max_err; stats[6] = static_cast<double>(s.argmax);
  stats[7] = static_cast<double>(s.nonfinite);
}

// ---------------------------------------------------------------------------------------
// Backward pass.  The pages print no gradient formulas (training used this operator, per
// [Arch] section 2.1); what follows is the chain rule applied to the forward above, step
// by step, in fp64.  For a loss L with dL/do = dO given:
//
//   output transform (per token, c over the H*D concatenation, s_c = sigmoid(g_c) with the
//   gate and 1 without, r = 1/sqrt(mean(y^2) + eps), u_c = dO_c w_c s_c):
//     RAW:            dy = dO
//     RMSNORM(_GATE): dy_c = r u_c - r^3 y_c (sum_c' u_c' y_c') / (H*D)
//     gate:           dg_c = dO_c y_c r w_c s_c (1 - s_c)
//     norm weight:    dw_c = sum over tokens of dO_c y_c r s_c
//   recurrence (per head; S_t = S0 + sum_{i<=t} phi(k_i) v_i^T, y_t = S_t^T phi(q_t)), with
//   dS_T the gradient reaching the final state (zero unless given):
//     dphi(q_t) = S_t dy_t
//     F_t = dS_T + sum_{i>=t} phi(q_i) dy_i^T      (the same sum taken from the end)
//     dphi(k_t) = F_t v_t,   dv_t = F_t^T phi(k_t),   dS0 = F_0
//   feature map: dq = dphi(q) * phi'(q), phi'(x) = sigmoid(x) (1 + x (1 - sigmoid(x))) for
//   SiLU and 1 for the identity; likewise dk.

// d/dx [x * sigmoid(x)] = sigmoid(x) + x * sigmoid(x) * (1 - sigmoid(x)).
inline double dfeature(double x, int phi) {
  if (phi != PHI_SILU) return 1.0;
  const double s = sigmoid(x);
  return s * (1.0 + x * (1.0 - s));
}

// Backward of transform_token for one token: dy (H*D), with the gate dg (H*D), and this
// token's terms of dw (H*D, added into dwt if non-null).
void transform_token_backward(const double* y, const void* dout, const void* g, int dtype, int64_t grow,
                              int HD, int mode, double eps, const float* w, double* dy, double* dg,
                              double* dwt) {
  if (mode == MODE_RAW) {
    for (int c = 0; c < HD; ++c) dy[c] = widen(dout, dtype, grow * HD + c);
    return;
  }
  double ss = 0.0;
  for (int c = 0; c < HD; ++c) ss += y[c] * y[c];
  const double r = 1.0 / std::sqrt(ss / HD + eps);
  double dot = 0.0;
  std::vector<double> u(HD);
  for (int c = 0; c < HD; ++c) {
    const double s = (mode == MODE_RMSNORM_GATE) ? sigmoid(widen(g, dtype, grow * HD + c)) : 1.0;
    const double wc = w ? static_cast<double>(w[c]) : 1.0;
    const double d = widen(dout, dtype, grow * HD + c);
    u[c] = d * wc * s;
    dot += u[c] * y[c];
    if (mode == MODE_RMSNORM_GATE && dg) dg[c] = d * y[c] * r * wc * s * (1.0 - s);
    if (dwt) dwt[c] = d * y[c] * r * s;
  }
  for (int c = 0; c < HD; ++c) dy[c] = r * u[c] - r * r * r * y[c] * dot / HD;
}

// Recurrence backward for one head over rows [row0, row0 + n).  S enters as S0 (D x D) and
// F as dST (D x D, the final state's gradient; null for zero);
// dy is the fp64 [tokens, H, D] gradient of the raw output.  Writes dq, dk, dv at the
// same packed positions and dS0 (D x D).  dy is indexed from the sequence's first row:
// dy[(t * H + h) * D + j].
void recur_head_backward(const void* q, const void* k, const void* v, int dtype, int64_t row0, int64_t n,
                         int H, int D, int h, int phi, const double* S0, const double* dST, const double* dy,
                         double* dq, double* dk, double* dv, double* dS0) {
  std::vector<double> S(S0, S0 + static_cast<size_t>(D) * D);
  std::vector<double> fk(D), vv(D);
  // forward in time: dphi(q_t) = S_t dy_t, S_t including token t
  for (int64_t t = 0; t < n; ++t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      fk[i] = feature(widen(k, dtype, base + i), phi);
      vv[i] = widen(v, dtype, base + i);
    }
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < D; ++j) S[static_cast<size_t>(i) * D + j] += fk[i] * vv[j];
    for (int i = 0; i < D; ++i) {
      double a = 0.0;
      for (int j = 0; j < D; ++j) a += S[static_cast<size_t>(i) * D + j] * dy[(t * H + h) * D + j];
      dq[base + i] = a * dfeature(widen(q, dtype, base + i), phi);
    }
  }
  // backward in time: F_t = dS_T + sum_{i >= t} phi(q_i) dy_i^T
  std::vector<double> F(static_cast<size_t>(D) * D, 0.0), fq(D);
  if (dST)
    for (size_t i = 0; i < F.size(); ++i) F[i] = dST[i];
  for (int64_t t = n - 1; t >= 0; --t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      fq[i] = feature(widen(q, dtype, base + i), phi);
      fk[i] = feature(widen(k, dtype, base + i), phi);
      vv[i] = widen(v, dtype, base + i);
    }
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < D; ++j) F[static_cast<size_t>(i) * D + j] += fq[i] * dy[(t * H + h) * D + j];
    for (int i = 0; i < D; ++i) {
      double b = 0.0;
      for (int j = 0; j < D; ++j) b += F[static_cast<size_t>(i) * D + j] * vv[j];
      dk[base + i] = b * dfeature(widen(k, dtype, base + i), phi);
    }
    for (int j = 0; j < D; ++j) {
      double c = 0.0;
      for (int i = 0; i < D; ++i) c += F[static_cast<size_t>(i) * D + j] * fk[i];
      dv[base + j] = c;
    }
  }
  for (size_t i = 0; i < F.size(); ++i) dS0[i] = F[i];
}

// ---------------------------------------------------------------------------------------
// Normalised variant ([Tut64] section 3, the linear-attention form before the deployment
// drops the denominator): alongside S the recurrence carries z_t = z_{t-1} + phi(k_t), and
//   y_t = phi(q_t)^T S_t / (phi(q_t) . z_t)
// (the denominator is the normaliser that stands in for softmax's row sum).  The output
// transform is then applied to y as in the plain form.  One head over rows [row0, row0+n);
// S (D x D) and z (D) enter as the initial state and leave as the final one.
void recur_head_znorm(const void* q, const void* k, const void* v, int dtype, int64_t row0, int64_t n, int H,
                      int D, int h, int phi, double* S, double* z, double* y, double* dens = nullptr) {
  std::vector<double> fq(D), fk(D), vv(D), acc(D);
  for (int64_t t = 0; t < n; ++t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      fq[i] = feature(widen(q, dtype, base + i), phi);
      fk[i] = feature(widen(k, dtype, base + i), phi);
      vv[i] = widen(v, dtype, base + i);
      acc[i] = 0.0;
    }
    double den = 0.0;
    for (int i = 0; i < D; ++i) {
      double* Si = S + static_cast<int64_t>(i) * D;
      z[i] += fk[i];
      den += fq[i] * z[i];
      for (int j = 0; j < D; ++j) {
        Si[j] += fk[i] * vv[j];
        acc[j] += fq[i] * Si[j];
      }
    }
    double* yt = y + (t * H + h) * static_cast<int64_t>(D);
    for (int j = 0; j < D; ++j) yt[j] = acc[j] / den;
    if (dens) dens[t * H + h] = den;
  }
}

// Backward of the normalised variant's denominator for one head, after the numerator's
// part has gone through recur_head_backward (which assigned dq, dk).  With d_t = phi(q_t) . z_t
// and dd_t the gradient reaching d_t (for y_t = n_t / d_t: dd_t = -(dy_t . y_t) / d_t):
//   dphi(q_t) += dd_t z_t           (z_t including token t)
//   dphi(k_i) += dz_T + sum_{t >= i} dd_t phi(q_t),    dz0 = dz_T + sum_t dd_t phi(q_t)
// through phi' as in the plain backward.  dd is indexed [t * H + h] from the sequence's
// first row; z0 and dzT (nullable) are this head's D-vectors; dz0 receives D values.
void znorm_head_backward_den(const void* q, const void* k, int dtype, int64_t row0, int64_t n, int H, int D, int h,
                             int phi, const double* z0, const double* dzT, const double* dd, double* dq, double* dk,
                             double* dz0) {
  std::vector<double> z(z0, z0 + D);
  for (int64_t t = 0; t < n; ++t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      z[i] += feature(widen(k, dtype, base + i), phi);
      dq[base + i] += dd[t * H + h] * z[i] * dfeature(widen(q, dtype, base + i), phi);
    }
  }
  std::vector<double> acc(D, 0.0);
  if (dzT)
    for (int i = 0; i < D; ++i) acc[i] = dzT[i];
  for (int64_t t = n - 1; t >= 0; --t) {
    const int64_t base = ((row0 + t) * H + h) * static_cast<int64_t>(D);
    for (int i = 0; i < D; ++i) {
      acc[i] += dd[t * H + h] * feature(widen(q, dtype, base + i), phi);
      dk[base + i] += acc[i] * dfeature(widen(k, dtype, base + i), phi);
    }
  }
  for (int i = 0; i < D; ++i) dz0[i] = acc[i];
}

}  // namespace

extern "C" {

// Packed-sequence forward ([Tut64] section 3 recurrence, [Arch] 2.1 output transform).
// cu: N + 1 row offsets into the packed tensors (sequence s = rows cu[s] .. cu[s+1]).
// Each sequence starts from state_in[s] (zeros if state_in is null); its final state
// goes to state_out[s].  If `out` is non-null the fp64 result [tokens, H*D] is stored.
// If `cand_out` / `cand_state` are non-null they are compared instead (streaming: no
// fp64 copy of the output is kept) and stats[0..7] receive
// {max|o_ref|, max|o_ref - o_cand|, argmax, nonfinite, same four for the state}.
int oracle_forward_packed(const void* q, const void* k, const void* v, const void* g, int dtype,
                          const int32_t* cu, int N, int H, int D, const float* state_in, int phi,
                          int mode, double eps, const float* w, double* out, double* state_out,
                          const void* cand_out, const float* cand_state, double* stats) {
  if (N < 0 || H <= 0 || D <= 0) return 1;
  if (mode == MODE_RMSNORM_GATE && !g) return 1;
  Cmp ocmp, scmp;
  std::vector<double> st;
  for (int s = 0; s < N; ++s) {
    const int64_t L = static_cast<int64_t>(cu[s + 1]) - cu[s];
    if (L < 0) return 1;
    load_states(st, state_in, s, H, D);
    run_sequence(q, k, v, g, dtype, cu[s], L, H, D, phi, mode, eps, w, st, out, cand_out, &ocmp);
    finish_states(st, s, H, D, state_out, cand_state, &scmp);
  }
  write_stats(stats, ocmp, scmp);
  return 0;
}

// Fixed-length batch [B, T, H, D]: the packed form with cu[b] = b * T.
int oracle_prefill(const void* q, const void* k, const void* v, const void* g, int dtype, int B,
                   int T, int H, int D, const float* state_in, int phi, int mode, double eps,
                   const float* w, double* out, double* state_out, const void* cand_out,
                   const float* cand_state, double* stats) {
  if (B < 0 || T < 0) return 1;
  std::vector<int32_t> cu(B + 1);
  for (int b = 0; b <= B; ++b) cu[b] = b * T;
  return oracle_forward_packed(q, k, v, g, dtype, cu.data(), B, H, D, state_in, phi, mode, eps, w,
                               out, state_out, cand_out, cand_state, stats);
}

// One decode step for B sequences: q, k, v [B, H, D], g [B, H*D], state [B, H, D, D] fp32.
// [Tut64] section 3: each new token only updates the state, S <- S + phi(k) v^T, and is
// read from it, y = phi(q)^T S; then the [Arch] 2.1 output transform.
int oracle_decode(const void* q, const void* k, const void* v, const void* g, int dtype, int B, int H,
                  int D, const float* state_in, int phi, int mode, double eps, const float* w,
                  double* out, double* state_out, const void* cand_out, const float* cand_state,
                  double* stats) {
  return oracle_prefill(q, k, v, g, dtype, B, 1, H, D, state_in, phi, mode, eps, w, out, state_out,
                        cand_out, cand_state, stats);
}

// Independent restatement R1 ([Tut64] section 3, the sum form before it is folded into
// a state): y_t = sum_{i <= t} (phi(q_t) . phi(k_i)) v_i, i.e. Y = (phi(Q) phi(K)^T (.) M) V
// with M_ti = [i <= t].  O(T^2 D) per head; tiny inputs only.  One sequence [T, H, D];
// y receives the raw (untransformed) [T, H, D] result.
int oracle_quadratic(const void* q, const void* k, const void* v, int dtype, int T, int H, int D,
                     int phi, double* y) {
  if (T < 0 || H <= 0 || D <= 0) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int h = 0; h < H; ++h) {
    std::vector<double> fq(static_cast<size_t>(T) * D), fk(static_cast<size_t>(T) * D),
        vv(static_cast<size_t>(T) * D);
    for (int t = 0; t < T; ++t)
      for (int i = 0; i < D; ++i) {
        const int64_t idx = (static_cast<int64_t>(t) * H + h) * D + i;
        fq[static_cast<size_t>(t) * D + i] = feature(widen(q, dtype, idx), phi);
        fk[static_cast<size_t>(t) * D + i] = feature(widen(k, dtype, idx), phi);
        vv[static_cast<size_t>(t) * D + i] = widen(v, dtype, idx);
      }
    for (int t = 0; t < T; ++t) {
      double* yt = y + (static_cast<int64_t>(t) * H + h) * D;
      for (int j = 0; j < D; ++j) yt[j] = 0.0;
      for (int i = 0; i <= t; ++i) {
        double p = 0.0;
        for (int c = 0; c < D; ++c) p += fq[static_cast<size_t>(t) * D + c] * fk[static_cast<size_t>(i) * D + c];
        for (int j = 0; j < D; ++j) yt[j] += p * vv[static_cast<size_t>(i) * D + j];
      }
    }
  }
  return 0;
}

// Independent restatement R2: the block-wise form with block size C (any C >= 1).
// For each block of C tokens (the last one may be shorter):
//   intra:  y_t = sum_{i in block, i <= t} (phi(q_t) . phi(k_i)) v_i
//   inter:  y_t += phi(q_t)^T S_prev            (S_prev = state before the block)
//   carry:  S_prev += sum_{i in block} phi(k_i) v_i^T
// [Ops] section 3 fixes the block size the deployment uses (256).  One sequence
// [T, H, D] starting from s0 [H, D, D] (zeros if null); y receives the raw result and
// state_out [H, D, D] the final state.
int oracle_chunked(const void* q, const void* k, const void* v, int dtype, int T, int H, int D, int C,
                   int phi, const double* s0, double* y, double* state_out) {
  if (T < 0 || H <= 0 || D <= 0 || C < 1) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int h = 0; h < H; ++h) {
    std::vector<double> S(static_cast<size_t>(D) * D, 0.0);
    if (s0)
      for (int i = 0; i < D * D; ++i) S[i] = s0[static_cast<size_t>(h) * D * D + i];
    std::vector<double> fq(static_cast<size_t>(C) * D), fk(static_cast<size_t>(C) * D),
        vv(static_cast<size_t>(C) * D);
    for (int b0 = 0; b0 < T; b0 += C) {
      const int n = std::min(C, T - b0);
      for (int t = 0; t < n; ++t)
        for (int i = 0; i < D; ++i) {
          const int64_t idx = (static_cast<int64_t>(b0 + t) * H + h) * D + i;
          fq[static_cast<size_t>(t) * D + i] = feature(widen(q, dtype, idx), phi);
          fk[static_cast<size_t>(t) * D + i] = feature(widen(k, dtype, idx), phi);
          vv[static_cast<size_t>(t) * D + i] = widen(v, dtype, idx);
        }
      for (int t = 0; t < n; ++t) {
        double* yt = y + (static_cast<int64_t>(b0 + t) * H + h) * D;
        for (int j = 0; j < D; ++j) {
          double inter = 0.0;
          for (int i = 0; i < D; ++i) inter += fq[static_cast<size_t>(t) * D + i] * S[static_cast<size_t>(i) * D + j];
          yt[j] = inter;
        }
        for (int i = 0; i <= t; ++i) {
          double p = 0.0;
          for (int c = 0; c < D; ++c) p += fq[static_cast<size_t>(t) * D + c] * fk[static_cast<size_t>(i) * D + c];
          for (int j = 0; j < D; ++j) yt[j] += p * vv[static_cast<size_t>(i) * D + j];
        }
      }
      for (int t = 0; t < n; ++t)
        for (int i = 0; i < D; ++i) {
          const double a = fk[static_cast<size_t>(t) * D + i];
          for (int j = 0; j < D; ++j) S[static_cast<size_t>(i) * D + j] += a * vv[static_cast<size_t>(t) * D + j];
        }
    }
    if (state_out)
      for (int i = 0; i < D * D; ++i) state_out[static_cast<size_t>(h) * D * D + i] = S[i];
  }
  return 0;
}

// The output transform alone ([Arch] 2.1), for tests of the norm and gate on given y.
int oracle_transform(const double* y, int64_t tokens, int H, int D, int mode, double eps,
                     const float* w, const void* g, int dtype, double* out) {
  const int HD = H * D;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < tokens; ++t) transform_token(y + t * HD, HD, mode, eps, w, g, dtype, t, out + t * HD);
  return 0;
}

// The output transform's backward alone ([Arch] 2.1, by the chain rule), for tests of a
// backward whose first step it is: per token, dy (fp64 [tokens, H*D]) from the raw output y
// (fp64 [tokens, H*D]) and dout (dtype), dg in gate mode, and dw [H*D] summed over the tokens
// in token order (zero in raw mode).  dg and dw may be null.
int oracle_transform_backward(const double* y, const void* dout, const void* g, int dtype, int64_t tokens, int H,
                              int D, int mode, double eps, const float* w, double* dy, double* dg, double* dw) {
  if (tokens < 0 || H <= 0 || D <= 0 || !dout || !dy) return 1;
  if (mode != MODE_RAW && !y) return 1;
  if (mode == MODE_RMSNORM_GATE && !g) return 1;
  const int HD = H * D;
  const bool want_dw = dw && mode != MODE_RAW;
  std::vector<double> dwt(want_dw ? static_cast<size_t>(tokens) * HD : 0);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < tokens; ++t)
    transform_token_backward(mode == MODE_RAW ? nullptr : y + t * HD, dout, g, dtype, t, HD, mode, eps, w,
                             dy + t * HD, (mode == MODE_RMSNORM_GATE && dg) ? dg + t * HD : nullptr,
                             want_dw ? dwt.data() + t * HD : nullptr);
  if (dw) {
    for (int c = 0; c < HD; ++c) dw[c] = 0.0;
    if (want_dw)
      for (int64_t t = 0; t < tokens; ++t)
        for (int c = 0; c < HD; ++c) dw[c] += dwt[static_cast<size_t>(t) * HD + c];
  }
  return 0;
}

// Backward of oracle_forward_packed for the loss whose output gradient is dout [tokens, H*D]
// (same dtype as q) and whose final-state gradient is dstate_out [N, H, D, D] fp32 (null for
// zero).  Recomputes the raw forward y, applies the transform backward per token, then the
// recurrence backward per head.  Outputs fp64: dq, dk, dv [tokens, H, D], dg [tokens, H*D]
// (gate mode; may be null otherwise), dstate [N, H, D, D] (the gradient of each sequence's
// initial state; may be null), dw [H*D] (the norm weight's gradient, zero in raw mode; may
// be null).
int oracle_backward_packed(const void* q, const void* k, const void* v, const void* g, const void* dout,
                           int dtype, const int32_t* cu, int N, int H, int D, const float* state_in,
                           const float* dstate_out, int phi, int mode, double eps, const float* w, double* dq,
                           double* dk, double* dv, double* dg, double* dstate, double* dw) {
  if (N < 0 || H <= 0 || D <= 0 || !dout || !dq || !dk || !dv) return 1;
  if (mode == MODE_RMSNORM_GATE && (!g || !dg)) return 1;
  const int HD = H * D;
  if (dw)
    for (int c = 0; c < HD; ++c) dw[c] = 0.0;
  const int64_t nst = static_cast<int64_t>(H) * D * D;
  for (int s = 0; s < N; ++s) {
    const int64_t row0 = cu[s], L = static_cast<int64_t>(cu[s + 1]) - cu[s];
    if (L < 0) return 1;
    std::vector<double> S0(nst, 0.0);
    if (state_in)
      for (int64_t i = 0; i < nst; ++i) S0[i] = static_cast<double>(state_in[s * nst + i]);
    // raw forward y, from S0
    std::vector<double> st(S0), y(static_cast<size_t>(L) * HD), dy(static_cast<size_t>(L) * HD);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h)
      recur_head(q, k, v, dtype, row0, L, H, D, h, phi, st.data() + static_cast<size_t>(h) * D * D, y.data());
    // transform backward per token (dy indexed from the sequence's first row); each token's
    // dw terms kept apart and added afterwards in token order
    const bool want_dw = dw && mode != MODE_RAW;
    std::vector<double> dwt(want_dw ? static_cast<size_t>(L) * HD : 0);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < L; ++t)
      transform_token_backward(y.data() + t * HD, dout, g, dtype, row0 + t, HD, mode, eps, w,
                               dy.data() + t * HD, dg ? dg + (row0 + t) * HD : nullptr,
                               want_dw ? dwt.data() + t * HD : nullptr);
    if (want_dw)
      for (int64_t t = 0; t < L; ++t)
        for (int c = 0; c < HD; ++c) dw[c] += dwt[static_cast<size_t>(t) * HD + c];
    std::vector<double> dS0(nst), dST;
    if (dstate_out) {
      dST.resize(nst);
      for (int64_t i = 0; i < nst; ++i) dST[i] = static_cast<double>(dstate_out[s * nst + i]);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h)
      recur_head_backward(q, k, v, dtype, row0, L, H, D, h, phi, S0.data() + static_cast<size_t>(h) * D * D,
                          dstate_out ? dST.data() + static_cast<size_t>(h) * D * D : nullptr, dy.data(), dq, dk,
                          dv, dS0.data() + static_cast<size_t>(h) * D * D);
    if (dstate)
      for (int64_t i = 0; i < nst; ++i) dstate[s * nst + i] = dS0[i];
  }
  return 0;
}

// Packed-sequence forward of the normalised variant.  As oracle_forward_packed, plus the
// normaliser state: z_in [N, H, D] (zeros if null) and z_out [N, H, D] (may be null).
// out receives the transformed fp64 result [tokens, H*D].
int oracle_forward_znorm_packed(const void* q, const void* k, const void* v, const void* g, int dtype,
                                const int32_t* cu, int N, int H, int D, const float* state_in, const float* z_in,
                                int phi, int mode, double eps, const float* w, double* out, double* state_out,
                                double* z_out) {
  if (N < 0 || H <= 0 || D <= 0 || !out) return 1;
  if (mode == MODE_RMSNORM_GATE && !g) return 1;
  const int HD = H * D;
  const int64_t nst = static_cast<int64_t>(H) * D * D, nz = static_cast<int64_t>(H) * D;
  for (int s = 0; s < N; ++s) {
    const int64_t row0 = cu[s], L = static_cast<int64_t>(cu[s + 1]) - cu[s];
    if (L < 0) return 1;
    std::vector<double> S(nst, 0.0), z(nz, 0.0), y(static_cast<size_t>(L) * HD);
    if (state_in)
      for (int64_t i = 0; i < nst; ++i) S[i] = static_cast<double>(state_in[s * nst + i]);
    if (z_in)
      for (int64_t i = 0; i < nz; ++i) z[i] = static_cast<double>(z_in[s * nz + i]);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h)
      recur_head_znorm(q, k, v, dtype, row0, L, H, D, h, phi, S.data() + static_cast<size_t>(h) * D * D,
                       z.data() + static_cast<size_t>(h) * D, y.data());
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < L; ++t)
      transform_token(y.data() + t * HD, HD, mode, eps, w, g, dtype, row0 + t, out + (row0 + t) * HD);
    if (state_out)
      for (int64_t i = 0; i < nst; ++i) state_out[s * nst + i] = S[i];
    if (z_out)
      for (int64_t i = 0; i < nz; ++i) z_out[s * nz + i] = z[i];
  }
  return 0;
}

// Backward of oracle_forward_znorm_packed for the loss with output gradient dout [tokens, H*D]
// (dtype of q) and final-state gradients dstate_out [N, H, D, D], dz_out [N, H, D] (fp32, null
// for zero).  Recomputes the forward (y and each token's denominators), applies the transform
// backward per token, splits each head's raw-output gradient into the numerator's
// dn_t = dy_t / d_t and the denominator's dd_t = -(dy_t . y_t) / d_t, runs the plain recurrence
// backward on dn and adds the denominator's terms.  Outputs fp64: dq, dk, dv [tokens, H, D],
// dg [tokens, H*D] (gate mode), dstate [N, H, D, D], dz [N, H, D], dw [H*D] (may be null
// but dq, dk, dv).
int oracle_backward_znorm_packed(const void* q, const void* k, const void* v, const void* g, const void* dout,
                                 int dtype, const int32_t* cu, int N, int H, int D, const float* state_in,
                                 const float* z_in, const float* dstate_out, const float* dz_out, int phi, int mode,
                                 double eps, const float* w, double* dq, double* dk, double* dv, double* dg,
                                 double* dstate, double* dz, double* dw) {
  if (N < 0 || H <= 0 || D <= 0 || !dout || !dq || !dk || !dv) return 1;
  if (mode == MODE_RMSNORM_GATE && (!g || !dg)) return 1;
  const int HD = H * D;
  if (dw)
    for (int c = 0; c < HD; ++c) dw[c] = 0.0;
  const int64_t nst = static_cast<int64_t>(H) * D * D, nz = static_cast<int64_t>(H) * D;
  for (int s = 0; s < N; ++s) {
    const int64_t row0 = cu[s], L = static_cast<int64_t>(cu[s + 1]) - cu[s];
    if (L < 0) return 1;
    std::vector<double> S0(nst, 0.0), z0(nz, 0.0), dST, dzT;
    if (state_in)
      for (int64_t i = 0; i < nst; ++i) S0[i] = static_cast<double>(state_in[s * nst + i]);
    if (z_in)
      for (int64_t i = 0; i < nz; ++i) z0[i] = static_cast<double>(z_in[s * nz + i]);
    if (dstate_out) {
      dST.resize(nst);
      for (int64_t i = 0; i < nst; ++i) dST[i] = static_cast<double>(dstate_out[s * nst + i]);
    }
    if (dz_out) {
      dzT.resize(nz);
      for (int64_t i = 0; i < nz; ++i) dzT[i] = static_cast<double>(dz_out[s * nz + i]);
    }
    // forward recompute: y and the denominators
    std::vector<double> S(S0), z(z0), y(static_cast<size_t>(L) * HD), den(static_cast<size_t>(L) * H);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h)
      recur_head_znorm(q, k, v, dtype, row0, L, H, D, h, phi, S.data() + static_cast<size_t>(h) * D * D,
                       z.data() + static_cast<size_t>(h) * D, y.data(), den.data());
    // transform backward per token (dw terms kept per token, added in token order)
    const bool want_dw = dw && mode != MODE_RAW;
    std::vector<double> dy(static_cast<size_t>(L) * HD), dwt(want_dw ? static_cast<size_t>(L) * HD : 0);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < L; ++t)
      transform_token_backward(y.data() + t * HD, dout, g, dtype, row0 + t, HD, mode, eps, w, dy.data() + t * HD,
                               dg ? dg + (row0 + t) * HD : nullptr, want_dw ? dwt.data() + t * HD : nullptr);
    if (want_dw)
      for (int64_t t = 0; t < L; ++t)
        for (int c = 0; c < HD; ++c) dw[c] += dwt[static_cast<size_t>(t) * HD + c];
    // numerator and denominator parts of each head's raw-output gradient
    std::vector<double> dn(static_cast<size_t>(L) * HD), dd(static_cast<size_t>(L) * H);
    for (int64_t t = 0; t < L; ++t)
      for (int h = 0; h < H; ++h) {
        const double d = den[t * H + h];
        double dot = 0.0;
        for (int j = 0; j < D; ++j) {
          const int64_t at = (t * H + h) * static_cast<int64_t>(D) + j;
          dot += dy[at] * y[at];
          dn[at] = dy[at] / d;
        }
        dd[t * H + h] = -dot / d;
      }
    std::vector<double> dS0(nst), dz0(nz);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
      recur_head_backward(q, k, v, dtype, row0, L, H, D, h, phi, S0.data() + static_cast<size_t>(h) * D * D,
                          dstate_out ? dST.data() + static_cast<size_t>(h) * D * D : nullptr, dn.data(), dq, dk, dv,
                          dS0.data() + static_cast<size_t>(h) * D * D);
      znorm_head_backward_den(q, k, dtype, row0, L, H, D, h, phi, z0.data() + static_cast<size_t>(h) * D,
                              dz_out ? dzT.data() + static_cast<size_t>(h) * D : nullptr, dd.data(), dq, dk,
                              dz0.data() + static_cast<size_t>(h) * D);
    }
    if (dstate)
      for (int64_t i = 0; i < nst; ++i) dstate[s * nst + i] = dS0[i];
    if (dz)
      for (int64_t i = 0; i < nz; ++i) dz[s * nz + i] = dz0[i];
  }
  return 0;
}

// Number of OpenMP threads the oracle's parallel loops use (reported with CPU timings).
int oracle_num_threads() { return omp_get_max_threads(); }

}  // extern "C"
