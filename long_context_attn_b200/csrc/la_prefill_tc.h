// Host interface of the tcgen05 (5th-generation tensor core) prefill kernel.
#pragma once

#include <cstddef>
#include <cstdint>

#include "la_common.cuh"

namespace la {

struct TcShape {
  int H, D, C;
  bool bf16;
  int mode;
};

struct TcArgs {
  const void *q, *k, *v, *g;
  void* out;
  const float* state_in;
  float* state_out;
  const int* cu;       // device cu_seqlens (varlen) or nullptr (fixed length T)
  int nseq, T, max_len;
  int64_t tokens;
  int H, D, C, phi_identity, mode;
  int reverse;         // nonzero: time runs backwards (raw mode only)
  float eps;
  const float* w;
  ErrRec* err;
  char* ws;            // workspace after the error record
  const int* state_index;  // optional [nseq] device: state slot of each sequence (else s)
  int skip_single;         // nonzero: sequences of exactly one token are left alone entirely
  int chunk_div;           // > 1: sequence s is chunk s % chunk_div of sequence s / chunk_div;
                           // only the chunk that ends the walk (the last one, or the first when
                           // time runs backwards) writes state_out (at s / chunk_div)
};

// True when the tensor-core kernel handles this shape on a GPU with `num_sms` SMs.
bool tc_eligible(const TcShape& s, int num_sms);
// Workspace bytes after the 256-byte error record.
size_t tc_workspace_bytes(int nseq, int max_len, int64_t tokens, int H, int D, int C);
cudaError_t launch_tc_prefill(const TcArgs& a, int num_sms, cudaStream_t stream);
// CTA pairs (heads x groups) that fit on the current device at once.
int max_active_clusters();

// The kernel (la_prefill_pair.cu): each CTA of a head's pair is a worker that owns whole
// sequences (or chunks of one) with the state in its TMEM; time runs either way.
cudaError_t launch_pair_prefill(const TcArgs& a, cudaStream_t stream);
size_t pair_workspace_bytes(int nseq, int max_len, int64_t tokens, int H);
int pair_max_active_clusters();
// Sequence groups of the pair kernel for a call (2 workers per head and group).
int pair_groups(int nseq, int H);

}  // namespace la
