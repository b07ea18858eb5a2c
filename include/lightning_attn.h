/*
 * lightning_attn.h -- C ABI of the Lightning Attention forward on B200 (sm_100a).
 *
 * What the library computes (sources are web pages, cited by title and section):
 *
 *   "六十四：MiniMax-01" (LLM tutorial, lesson 64), section 3 "Lightning Attention 的定位":
 *     linear attention keeps a running state per head,
 *         S_t = S_{t-1} + phi(k_t) v_t^T,        y_t = phi(q_t)^T S_t,
 *     (the sum runs over i <= t: causal, diagonal included), and a decode step only
 *     updates the state and reads it.
 *   "MiniMax-Text-01 405B MoE模型架构与训练策略解析", section 2.1 "Lightning Attention-2":
 *     phi = SiLU, Y = Q (K^T V), output = RMSNorm(Y) * sigmoid(gate).
 *   "MiniMax-01技术报告解读（二）计算优化", section 3: the block (chunk) size is 256 and the
 *     tail block is padded to one of 32 / 64 / 128 rows; section 6: prefill and decode run
 *     as separate paths on separate CUDA streams.
 *
 * Readings where the pages are silent: phi is applied to q and k only (v raw); there is
 * no normaliser denominator, no decay and no 1/sqrt(d) scale; the RMSNorm runs over the
 * concatenation of the H heads of a token (H*D values) with eps inside the square root,
 *     o = y * rsqrt(mean(y^2) + eps) * w * sigmoid(g).
 * The block size changes rounding and work, not the exact result.
 *
 * Tensor layouts (all row-major, contiguous, device memory unless stated):
 *   q, k, v   [B, T, H, D] (prefill), [total_tokens, H, D] (varlen), [B, H, D] (decode)
 *   g, out    [B, T, H*D],            [total_tokens, H*D],             [B, H*D]
 *   states    fp32 [B or N, H, D, D]: state[s][h][i][j] multiplies phi(q)[i] to give y[j]
 * q, k, v, g and out share one element type (la_dtype); states are always fp32.
 * All device pointers must be 16-byte aligned.
 *
 * Calls are asynchronous on `stream`.  Arguments are validated on the host before any
 * launch; a rejected call launches nothing and returns its status.  Failures detected
 * on the device (a bounded wait that ran out, decreasing cu_seqlens) are recorded in
 * the workspace and reported by lightning_attn_check().  Ownership: the caller owns
 * every buffer, including the workspace; the library allocates nothing and keeps no
 * per-call state, so calls on different streams with different workspaces are
 * independent.  Calls that share a workspace must be ordered on one stream.
 */
#ifndef LIGHTNING_ATTN_H_
#define LIGHTNING_ATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (the same type as cudaStream_t / CUstream). NULL = legacy stream. */
typedef struct CUstream_st* la_stream_t;

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1,  /* a pointer, size, alignment or enum value is invalid          */
  LA_ERR_UNSUPPORTED = 2,  /* valid, but no kernel of the library handles the combination */
  LA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a kernel launch failed         */
  LA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (reported by _check)      */
  LA_ERR_DEVICE = 5        /* a device-side argument check failed (reported by _check)     */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/* RAW: out = y.  RMSNORM: out = y * r * w.  RMSNORM_GATE: out = y * r * w * sigmoid(g). */
typedef enum { LA_OUT_RAW = 0, LA_OUT_RMSNORM = 1, LA_OUT_RMSNORM_GATE = 2 } la_out_mode;

/* SILU: phi(x) = x * sigmoid(x) on q and k.  IDENTITY: phi(x) = x (exact-integer tests). */
typedef enum { LA_PHI_SILU = 0, LA_PHI_IDENTITY = 1 } la_feature_map;

typedef enum {
  LA_OP_PREFILL = 0,
  LA_OP_PREFILL_VARLEN = 1,
  LA_OP_DECODE = 2,
  LA_OP_MIXED = 3,
  LA_OP_BACKWARD = 4,
  LA_OP_BACKWARD_VARLEN = 5,
  LA_OP_PREFILL_ZNORM = 6,
  LA_OP_PREFILL_ZNORM_VARLEN = 7,
  LA_OP_CHUNK_STATE = 8,
  LA_OP_OUTPUT_TRANSFORM_BACKWARD = 9
} la_op;

/*
 * Causal block-wise prefill of B sequences of T tokens each.
 * Source: "六十四：MiniMax-01" section 3 (recurrence), "MiniMax-Text-01 405B MoE模型架构与训练
 * 策略解析" section 2.1 (SiLU, RMSNorm * sigmoid gate), "MiniMax-01技术报告解读（二）计算优化"
 * section 3 (block size 256, tail pads 32/64/128).
 *
 *   q, k, v      [B, T, H, D], dtype; read only.
 *   g            [B, T, H*D], dtype; required iff mode == LA_OUT_RMSNORM_GATE, else ignored.
 *   out          [B, T, H*D], dtype; written.  May not alias any input.
 *   state_in     fp32 [B, H, D, D] initial state per sequence, or NULL for zeros.
 *   state_out    fp32 [B, H, D, D] final state, or NULL.  May equal state_in (in place).
 *   B, T         B >= 1, T >= 0 (T == 0: no output; state_out = state_in or zeros).
 *   H, D         H >= 1; D in {64, 128}.  The RMSNorm modes need H*D <= 16384.
 *   block_size   the block (chunk) size C, 1..1024.  bf16 with D = 128 and C in {128, 256} runs
 *                on the tcgen05 tensor-core kernel; every other valid combination runs on the
 *                CUDA-core kernel (fp32 arithmetic).  lightning_attn_last_path() names the one used.
 *                On the tensor-core kernel each CTA of a head's pair is a worker that owns
 *                whole sequences (with few heads, several groups of pairs share them); when a
 *                call has fewer sequences than workers per head, a sequence of T >= 2048 is
 *                cut into chunks that run in parallel from the states of the chunks before
 *                them ("tcgen05+chunks": at 64 heads, two chunks); in a norm mode with more
 *                heads than CTA pairs fit at once, the norm runs as a second per-token pass
 *                ("tcgen05+norm").  The result is the same up to rounding.
 *   eps          RMSNorm epsilon (> 0 for the norm modes).
 *   norm_weight  fp32 [H*D] RMSNorm weight, or NULL for ones.
 *   workspace    device scratch of >= lightning_attn_workspace_size(LA_OP_PREFILL, ...)
 *                bytes, 256-byte aligned.  Its first 256 bytes hold the error record
 *                (words 0-3: status, site, index, detail -- read and cleared by
 *                lightning_attn_check; word 4: bounded-wait limit in ms, 0 = default 4 s;
 *                word 5: fault-injection selector for failure tests, 0 = none).  The call
 *                clears the rest of the workspace itself.
 * Returns LA_OK after enqueueing, or an error status with nothing enqueued.
 */
LA_API la_status lightning_attn_prefill(const void* q, const void* k, const void* v, const void* g, void* out,
                                 const float* state_in, float* state_out, int B, int T, int H, int D,
                                 int block_size, la_dtype dtype, la_feature_map phi, la_out_mode mode,
                                 float eps, const float* norm_weight, void* workspace,
                                 size_t workspace_bytes, la_stream_t stream);

/*
 * Prefill of N variable-length sequences packed along the token axis.
 * Source: as lightning_attn_prefill; packing with cu_seqlens follows the varlen
 * treatment of "MiniMax-01系列大模型：超长上下文与多模态能力深度解析与部署指南" section 2.1.3.
 *
 *   q, k, v      [total_tokens, H, D]; g, out [total_tokens, H*D].
 *   cu_seqlens   DEVICE int32 [N + 1], cu_seqlens[0] == 0, non-decreasing,
 *                cu_seqlens[N] == total_tokens.  Sequence s is rows cu[s] .. cu[s+1]-1.
 *                Violations found on the device are reported by lightning_attn_check.
 *   state_in / state_out  fp32 [N, H, D, D] or NULL.  Each sequence starts from its own
 *                state (zeros if NULL) -- states never flow between sequences.
 *   max_seqlen   an upper bound on every sequence length (sizes the workspace).
 *   Tail blocks are padded to the smallest of 32 / 64 / 128 that fits.
 * Other arguments as lightning_attn_prefill.
 */
LA_API la_status lightning_attn_prefill_varlen(const void* q, const void* k, const void* v, const void* g,
                                        void* out, const float* state_in, float* state_out,
                                        const int* cu_seqlens, int num_seqs, int max_seqlen,
                                        int total_tokens, int H, int D, int block_size,
                                        la_dtype dtype, la_feature_map phi, la_out_mode mode,
                                        float eps, const float* norm_weight, void* workspace,
                                        size_t workspace_bytes, la_stream_t stream);

/*
 * One decode step for B sequences, one new token each.
 * Source: "六十四：MiniMax-01" section 3 (each new token only updates the state and is
 * read from it: S <- S + phi(k) v^T, y = phi(q)^T S -- update first, then read), and
 * "MiniMax-Text-01 405B MoE模型架构与训练策略解析" section 2.1 (output transform).
 *
 *   q, k, v      [B, H, D]; g, out [B, H*D].
 *   state        fp32 [B, H, D, D], updated IN PLACE.
 *   workspace    >= lightning_attn_workspace_size(LA_OP_DECODE, ...) bytes, 256-byte aligned,
 *                zero-filled before its first use; every completed call leaves it zeroed.
 * Other arguments as lightning_attn_prefill.
 */
LA_API la_status lightning_attn_decode_step(const void* q, const void* k, const void* v, const void* g,
                                     void* out, float* state, int B, int H, int D, la_dtype dtype,
                                     la_feature_map phi, la_out_mode mode, float eps,
                                     const float* norm_weight, void* workspace, size_t workspace_bytes,
                                     la_stream_t stream);

/* Size of the scratch array compiled into the library for
 * lightning_attn_decode_step_noalloc: 8.25 MiB + 256 bytes, which holds the decode scratch
 * of every batch with B*H*D <= 2^21 (e.g. 256 sequences x 64 heads x 128, or 32768
 * sequences x 1 head x 64): 256 + 4B + 4*B*H*D + 4*B*H bytes, each part rounded up to 256. */
#define LA_DECODE_NOALLOC_SCRATCH_BYTES 8651008u

/*
 * Decode step that allocates nothing and takes no workspace (the pages have no
 * counterpart: this entry point exists for callers of this library that cannot allocate).
 * It is for callers whose device memory is owned entirely by another allocator (e.g. a
 * serving engine that reserves nearly all of HBM for its cache and state pools, where an
 * extra cudaMalloc fails or fragments the pool) and for latency-critical decode loops in
 * which cudaMalloc, which can synchronise the device, is not allowed.
 *
 * Same computation, arguments and results as lightning_attn_decode_step, without
 * `workspace` / `workspace_bytes`.  Its scratch is a fixed array of
 * LA_DECODE_NOALLOC_SCRATCH_BYTES bytes inside the library (one copy per GPU that loads the
 * library, held until the process exits):
 *   - The first call on each device looks up the array's device address (with that device
 *     current); make that first call before any stream capture.
 *   - Every call shares the array: each call clears the per-sequence counters on its stream,
 *     and calls that overlap on the GPU (other streams, unordered host threads) race.
 *   - Batches whose scratch would exceed the array (decode_workspace bytes > the size above)
 *     return LA_ERR_UNSUPPORTED with nothing enqueued.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - The error record sits in the library's array, where lightning_attn_check cannot
 *     reach it: device-side errors of this call are not reported to the caller (the decode
 *     kernel has no bounded waits, so the only such errors would be the CUDA launch errors
 *     that the return status already carries).
 *   - The array's address is kept per device for the life of the process; after a
 *     cudaDeviceReset (or any other teardown of the device's primary context) this entry
 *     point must not be called again in that process.
 *   - q, k, v, g, out, state and norm_weight must live on the current device.
 * On success lightning_attn_last_path() returns "decode".
 */
LA_API la_status lightning_attn_decode_step_noalloc(const void* q, const void* k, const void* v, const void* g,
                                                    void* out, float* state, int B, int H, int D, la_dtype dtype,
                                                    la_feature_map phi, la_out_mode mode, float eps,
                                                    const float* norm_weight, la_stream_t stream);

/*
 * Mixed serving step over N sequences packed back to back: "MiniMax-01技术报告解读（二）
 * 计算优化", sections 3 and 6 (chunked prefill; prefill and decode on separate streams).
 * A sequence with exactly one new token is decoded (lightning_attn_decode_step: S is
 * updated, then read); a sequence with more new tokens is prefilled as a continuation
 * (lightning_attn_prefill_varlen with S0 = its current state, which is then replaced by
 * the state after its last token).  Results are those of the two calls.
 *   q, k, v          packed [total, H, D] device; g, out packed [total, H*D] (g when gated)
 *   cu_seqlens       [N+1] int32 device: token offsets of the sequences (non-decreasing)
 *   cu_seqlens_host  [N+1] int32 host: the same values (they decide the split and sizes)
 *   state_pool       fp32 device [P, H, D, D]: the caller's state pool, updated in place
 *   state_slot       [N] int32 device: pool slot of each sequence; slots must be distinct
 *   prefill_stream   runs the prefill kernel; decode_stream runs the decode kernels (the
 *                    two may be the same stream).  Nothing is ordered between them: the
 *                    caller synchronises both before reading the results or reusing
 *                    `workspace`.
 *   workspace        >= lightning_attn_workspace_size(LA_OP_MIXED, N, max_prefill_len,
 *                    total, ...) bytes, 256-byte aligned; the error record is shared by
 *                    both streams (read it with lightning_attn_check after syncing both).
 * Only the tensor-core configuration (bf16, D = 128, block 128 or 256, and for the norm
 * modes all heads' CTA pairs resident at once) is supported, else LA_ERR_UNSUPPORTED with
 * nothing enqueued; sequences of length 0 are allowed and left alone.  Invalid arguments
 * (including host cu_seqlens that decrease) return LA_ERR_INVALID_ARG and enqueue nothing.
 */
LA_API la_status lightning_attn_mixed_step(const void* q, const void* k, const void* v, const void* g, void* out,
                                           const int* cu_seqlens, const int* cu_seqlens_host, float* state_pool,
                                           const int* state_slot, int num_seqs, int H, int D, int block_size,
                                           la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                           const float* norm_weight, void* workspace, size_t workspace_bytes,
                                           la_stream_t prefill_stream, la_stream_t decode_stream);

/*
 * Sequence-parallel prefill ("MiniMax-01系列大模型：超长上下文与多模态能力深度解析与部署指南",
 * section 2.1.3, LASP+): one sequence is split into contiguous chunks, one per rank.  The
 * state is a plain sum, so the state entering chunk `rank` is state0 plus the sum of the
 * states the earlier chunks reach from a zero state.  Given those chunk states gathered in
 * rank order, this writes the prefix for `rank` (adding in rank order: deterministic).
 *   gathered  fp32 device [world, H, D, D] (chunk states, rank order)
 *   state0    fp32 device [H, D, D] or NULL (zero): the state before the whole sequence
 *   out       fp32 device [H, D, D] (may not alias `gathered`)
 * The host side of a sequence-parallel prefill is long_context_attn_b200.sequence_parallel:
 * a raw-mode prefill of the chunk from a zero state, an all-gather of the chunk states,
 * this prefix, then the chunk's prefill from the prefix.
 */
LA_API la_status lightning_attn_state_prefix(const float* gathered, int world, int rank, const float* state0,
                                             float* out, int H, int D, la_stream_t stream);

/*
 * Normalised variant of lightning_attn_prefill ("六十四：MiniMax-01" section 3, the linear-
 * attention form with its normaliser): besides S each sequence carries z, the running sum
 * of phi(k), and the raw output is divided by phi(q) . z before the output transform:
 *   S_t = S_{t-1} + phi(k_t) v_t^T,  z_t = z_{t-1} + phi(k_t),
 *   y_t = phi(q_t)^T S_t / (phi(q_t) . z_t),  out = transform(y) as lightning_attn_prefill.
 * The denominator is not guarded: with phi = SiLU (which takes negative values) it can be
 * zero or negative, and the result then is whatever the division gives.
 *   z_in    fp32 [B, H, D] initial normaliser per sequence, or NULL (zeros).
 *   z_out   fp32 [B, H, D] final normaliser, or NULL.  May equal z_in.
 *   workspace  >= lightning_attn_workspace_size(LA_OP_PREFILL_ZNORM, B, T, 0, ...) bytes.
 * Needs H*D <= 16384 in every output mode (LA_ERR_UNSUPPORTED otherwise).  Other arguments
 * (state_in / state_out: the same S) as lightning_attn_prefill.
 */
LA_API la_status lightning_attn_prefill_znorm(const void* q, const void* k, const void* v, const void* g, void* out,
                                              const float* state_in, const float* z_in, float* state_out,
                                              float* z_out, int B, int T, int H, int D, int block_size,
                                              la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                              const float* norm_weight, void* workspace, size_t workspace_bytes,
                                              la_stream_t stream);

/*
 * The normalised variant over N packed sequences (cu_seqlens as lightning_attn_prefill_varlen;
 * z_in / z_out fp32 [N, H, D] or NULL).  Workspace: LA_OP_PREFILL_ZNORM_VARLEN.
 */
LA_API la_status lightning_attn_prefill_znorm_varlen(const void* q, const void* k, const void* v, const void* g,
                                                     void* out, const float* state_in, const float* z_in,
                                                     float* state_out, float* z_out, const int* cu_seqlens,
                                                     int num_seqs, int max_seqlen, int total_tokens, int H, int D,
                                                     int block_size, la_dtype dtype, la_feature_map phi,
                                                     la_out_mode mode, float eps, const float* norm_weight,
                                                     void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * One decode step of the normalised variant: as lightning_attn_decode_step, and z (fp32
 * [B, H, D], required, updated in place) becomes z + phi(k); the raw output is divided by
 * phi(q) . z before the output transform.  Workspace: LA_OP_DECODE.
 */
LA_API la_status lightning_attn_decode_step_znorm(const void* q, const void* k, const void* v, const void* g,
                                                  void* out, float* state, float* z, int B, int H, int D,
                                                  la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                                  const float* norm_weight, void* workspace, size_t workspace_bytes,
                                                  la_stream_t stream);

/*
 * Backward pass of lightning_attn_prefill: the gradients of a loss with respect to q, k, v,
 * the gate and the initial state, given the gradient `dout` of its output and (optionally)
 * the gradient `dstate_out` reaching its final state (a later chunk that continued from it).  The pages give
 * no gradient formulas ("MiniMax-Text-01 405B MoE模型架构与训练策略解析" section 2.1 names the
 * operator as trained); they follow from the forward of "六十四：MiniMax-01" section 3 by the
 * chain rule.  Per head, with dy the gradient of the raw output y (dy = dout in RAW mode;
 * through RMSNorm * w * sigmoid(g) otherwise, recomputing y from q, k, v, state_in):
 *   dphi(q_t) = sum_{i<=t} (dy_t . v_i) phi(k_i) + S0 dy_t
 *   dphi(k_i) = sum_{t>=i} (v_i . dy_t) phi(q_t)
 *   dv_i      = sum_{t>=i} (phi(k_i) . phi(q_t)) dy_t,      dS0 = sum_t phi(q_t) dy_t^T
 * plus, with dS_T = dstate_out:  dphi(k_i) += dS_T v_i,  dv_i += dS_T^T phi(k_i),  dS0 += dS_T
 * and dq = dphi(q) * phi'(q), dk = dphi(k) * phi'(k).  The three sums run as causal
 * linear-attention passes of the prefill kernels (the last two on time-reversed copies).
 *
 *   q, k, v       [B, T, H, D] dtype, the forward's inputs; dout [B, T, H*D] dtype.
 *   g             [B, T, H*D] dtype, required iff mode == LA_OUT_RMSNORM_GATE.
 *   state_in      fp32 [B, H, D, D] the forward's initial states, or NULL (zeros).
 *   dstate_out    fp32 [B, H, D, D] gradient of the final states, or NULL (zeros).
 *   y             [B, T, H*D] dtype: the forward's raw output (its y before the norm, as
 *                 lightning_attn_prefill in LA_OUT_RAW mode gives it), or NULL.  In the norm
 *                 modes the backward needs y; given, it is used, else it is recomputed (one
 *                 more pass of the prefill kernel).  Ignored in LA_OUT_RAW mode.
 *   dq, dk, dv    [B, T, H, D] dtype, written (none may alias an input or each other).
 *   dg            [B, T, H*D] dtype, written iff mode == LA_OUT_RMSNORM_GATE (else ignored).
 *   dstate_in     fp32 [B, H, D, D] gradient of the initial states, or NULL.
 *   dnorm_weight  fp32 [H*D], written with the norm weight's gradient summed over all tokens
 *                 (dw = sum_t dout_t * y_t * r_t [* sigmoid(g_t)], deterministic order), or
 *                 NULL; zeros in LA_OUT_RAW mode.
 *   norm_weight   as the forward.
 *   workspace     >= lightning_attn_workspace_size(LA_OP_BACKWARD, B, T, 0, H, D, block_size,
 *                 dtype, mode) bytes, 256-byte aligned; the error record as for the prefill.
 * Other arguments as lightning_attn_prefill (block_size selects the passes' kernel the same
 * way).  Returns LA_OK after enqueueing, or an error status with nothing enqueued.
 */
LA_API la_status lightning_attn_backward(const void* q, const void* k, const void* v, const void* g,
                                         const void* dout, const float* state_in, const float* dstate_out,
                                         const void* y, void* dq, void* dk, void* dv, void* dg, float* dstate_in,
                                         float* dnorm_weight, int B, int T, int H, int D, int block_size,
                                         la_dtype dtype, la_feature_map phi, la_out_mode mode, float eps,
                                         const float* norm_weight, void* workspace, size_t workspace_bytes,
                                         la_stream_t stream);

/*
 * Backward of lightning_attn_prefill_varlen: as lightning_attn_backward over N packed
 * sequences (q, k, v, dq, dk, dv [total, H, D]; g, dout, dg [total, H*D]; cu_seqlens DEVICE
 * int32 [N + 1] as for the forward; state_in, dstate_out, dstate_in [N, H, D, D] or NULL; y
 * [total, H*D] or NULL; dnorm_weight [H*D] or NULL).  Time is reversed within each sequence.  Workspace: LA_OP_BACKWARD_VARLEN with N, max_seqlen,
 * total_tokens.
 */
LA_API la_status lightning_attn_backward_varlen(const void* q, const void* k, const void* v, const void* g,
                                                const void* dout, const float* state_in, const float* dstate_out,
                                                const void* y, void* dq, void* dk, void* dv, void* dg,
                                                float* dstate_in, float* dnorm_weight, const int* cu_seqlens,
                                                int num_seqs, int max_seqlen, int total_tokens, int H, int D,
                                                int block_size, la_dtype dtype, la_feature_map phi,
                                                la_out_mode mode, float eps, const float* norm_weight,
                                                void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * The output transform alone ("MiniMax-Text-01 405B MoE模型架构与训练策略解析" section 2.1), per
 * token over the H*D concatenation:  RAW: out = y;  RMSNORM: out = y * r * w;
 * RMSNORM_GATE: out = y * r * w * sigmoid(g), with r = 1 / sqrt(mean(y^2) + eps).
 * With lightning_attn_prefill in LA_OUT_RAW mode it gives the normalised output while
 * keeping y (for lightning_attn_backward's `y`).
 *   y, out      [tokens, H*D] dtype, device; out may equal y (in place).
 *   g           [tokens, H*D] dtype, required iff mode == LA_OUT_RMSNORM_GATE.
 *   H*D <= 16384; norm_weight fp32 [H*D] or NULL (ones).
 */
LA_API la_status lightning_attn_output_transform(const void* y, const void* g, void* out, int tokens, int H, int D,
                                                 la_dtype dtype, la_out_mode mode, float eps,
                                                 const float* norm_weight, la_stream_t stream);

/*
 * Backward of lightning_attn_output_transform: given the gradient dout of its output, the
 * gradient dy of the raw output y, the gate's gradient dg and the norm weight's gradient
 * (the chain rule through the transform of "MiniMax-Text-01 405B MoE模型架构与训练策略解析"
 * section 2.1, as inside lightning_attn_backward).  Per token, with r = 1/sqrt(mean(y^2) +
 * eps), s = sigmoid(g) (1 without the gate) and u = dout * w * s:
 *   dy = r u - r^3 y (sum over the row of u y) / (H*D),   dg = dout * y * r * w * s * (1 - s),
 *   dnorm_weight = sum over tokens of dout * y * r * s.
 * RAW: dy = dout (copied), dnorm_weight zeros.  It is the first step of a backward whose
 * linear-attention part runs elsewhere (lightning_attn_backward in LA_OUT_RAW mode given dy,
 * e.g. each rank of a sequence-parallel backward).
 *   y, g, dout    [tokens, H*D] dtype, device (y ignored in RAW; g iff RMSNORM_GATE).
 *   dy            [tokens, H*D] dtype, written; may equal y, not dout or g.
 *   dg            [tokens, H*D] dtype, written iff RMSNORM_GATE; distinct from the others.
 *   dnorm_weight  fp32 [H*D] or NULL; summed in a fixed order (deterministic).
 *   workspace     needed iff dnorm_weight is given in a norm mode: >= lightning_attn_workspace_size(
 *                 LA_OP_OUTPUT_TRANSFORM_BACKWARD, tokens, 0, 0, H, D, 0, dtype, mode) bytes,
 *                 256-byte aligned.
 * H*D <= 16384.  Returns LA_OK after enqueueing, or an error status with nothing enqueued.
 */
LA_API la_status lightning_attn_output_transform_backward(const void* y, const void* g, const void* dout, void* dy,
                                                          void* dg, float* dnorm_weight, int tokens, int H, int D,
                                                          la_dtype dtype, la_out_mode mode, float eps,
                                                          const float* norm_weight, void* workspace,
                                                          size_t workspace_bytes, la_stream_t stream);

/*
 * The state lightning_attn_prefill would end with, without computing its outputs:
 *   state_out[b] = state_in[b] + sum_t phi(k_t) v_t^T      ("六十四：MiniMax-01" section 3:
 * the state is a plain sum over the sequence).  Step 1 of the sequence-parallel prefill
 * ("MiniMax-01系列大模型：超长上下文与多模态能力深度解析与部署指南" section 2.1.3, LASP+): each
 * rank's chunk state before the exchange.  Reads only k and v.
 *   k, v        [B, T, H, D] dtype, device.
 *   state_in    fp32 [B, H, D, D] or NULL (zeros).  state_out fp32 [B, H, D, D]; may equal
 *               state_in.
 *   workspace   >= lightning_attn_workspace_size(LA_OP_CHUNK_STATE, B, T, 0, H, D, 0, dtype, 0)
 *               bytes, 256-byte aligned; error record as for the prefill.
 * bf16 with D = 128 on sm_100a runs a tensor-core kernel (phi(K)^T V accumulated in TMEM,
 * split over the tokens, the splits added in a fixed order); elsewhere a raw-mode prefill
 * runs with its outputs written to the workspace.  The result equals the prefill's final
 * state up to rounding order.
 */
LA_API la_status lightning_attn_chunk_state(const void* k, const void* v, const float* state_in, float* state_out,
                                            int B, int T, int H, int D, la_dtype dtype, la_feature_map phi,
                                            void* workspace, size_t workspace_bytes, la_stream_t stream);

/*
 * Workspace bytes needed by one call (0 on invalid arguments).
 *   op == LA_OP_PREFILL:         B_or_N = B, T_or_max = T, total_tokens ignored.
 *   op == LA_OP_PREFILL_VARLEN:  B_or_N = N, T_or_max = max_seqlen, total_tokens.
 *   op == LA_OP_DECODE:          B_or_N = B, the rest ignored except H, D, dtype, mode.
 *   op == LA_OP_MIXED:           B_or_N = N, T_or_max = longest sequence with more than
 *                                one token (0 if none), total_tokens = all packed tokens.
 *   op == LA_OP_BACKWARD:        as LA_OP_PREFILL.
 *   op == LA_OP_BACKWARD_VARLEN: as LA_OP_PREFILL_VARLEN.
 *   op == LA_OP_PREFILL_ZNORM:   as LA_OP_PREFILL.
 *   op == LA_OP_PREFILL_ZNORM_VARLEN: as LA_OP_PREFILL_VARLEN.
 *   op == LA_OP_CHUNK_STATE:     B_or_N = B, T_or_max = T (block_size and mode ignored).
 *   op == LA_OP_OUTPUT_TRANSFORM_BACKWARD: B_or_N = tokens (>= 0), H, D; the rest ignored.
 * The size depends on the kernel the call will select (which depends on the device), so
 * query it with the target device current.
 */
LA_API size_t lightning_attn_workspace_size(la_op op, int B_or_N, int T_or_max, int total_tokens, int H, int D,
                                     int block_size, la_dtype dtype, la_out_mode mode);

/*
 * Synchronises `stream`, then reads and clears the error record in `workspace`.
 * Returns LA_OK, LA_ERR_TIMEOUT, LA_ERR_DEVICE, or LA_ERR_CUDA (stream error).
 * `detail` (may be NULL) receives 4 words: {status, site, index, extra}.
 */
LA_API la_status lightning_attn_check(void* workspace, la_stream_t stream, unsigned int* detail);

/* Static, human-readable name of a status. */
LA_API const char* lightning_attn_status_string(la_status s);

/* Name of the kernel path the last successful call on this thread selected (diagnostic):
 * "tcgen05", "tcgen05+chunks", "tcgen05+norm", "tcgen05+norm+chunks", "simt", "decode",
 * "mixed", "tcgen05-state". */
LA_API const char* lightning_attn_last_path(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_ATTN_H_ */
