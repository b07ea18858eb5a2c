// Host-side dispatch of the tensor-core prefill: eligibility, workspace size and launch.
// The kernel itself (both directions of time, every output mode) is in la_prefill_pair.cu.
#include <algorithm>

#include "la_common.cuh"
#include "la_prefill_tc.h"

namespace la {
namespace {
constexpr int kD = 128;
}  // namespace

int max_active_clusters() { return pair_max_active_clusters(); }

bool tc_eligible(const TcShape& s, int num_sms) {
  (void)num_sms;
  if (!s.bf16 || s.D != kD || (s.C != 128 && s.C != 256) || s.H < 1) return false;
  // The cross-head norm exchange needs every head's CTA pair resident at once.
  if (s.mode != LA_OUT_RAW && s.H > max_active_clusters()) return false;
  return true;
}

size_t tc_workspace_bytes(int nseq, int max_len, int64_t tokens, int H, int D, int C) {
  (void)D;
  (void)C;
  return pair_workspace_bytes(nseq, max_len, tokens, H);
}

cudaError_t launch_tc_prefill(const TcArgs& a, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  return launch_pair_prefill(a, stream);
}

}  // namespace la
