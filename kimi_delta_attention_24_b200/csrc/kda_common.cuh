// Shared host/device definitions of the KDA forward library (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

constexpr int kHeadDim = 128;        // K = V = 128, the only supported head size
constexpr float kL2Eps = 1e-6f;      // inside the square root of the q/k L2 norm

// Device status word (first 4 bytes of the workspace), sticky until read by the host.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadSeqlens = 2u;  // cu_seqlens not ordered as 0 = cu[0] <= ... <= cu[N] = T
constexpr uint32_t kStatusBadIndex = 4u;    // a decode state index at or past the pool's slot count

// Input-transform flags (public values in kda.h).
constexpr uint32_t kFlagGatePrecomputed = KDA_FLAG_GATE_PRECOMPUTED;  // g holds fp32 log alpha
constexpr uint32_t kFlagNoQkL2Norm = KDA_FLAG_NO_QK_L2NORM;           // q, k used as given
constexpr uint32_t kFlagBetaPrecomputed = KDA_FLAG_BETA_PRECOMPUTED;  // beta holds fp32 beta
constexpr uint32_t kFlagMask = kFlagGatePrecomputed | kFlagNoQkL2Norm | kFlagBetaPrecomputed;
constexpr size_t kWorkspaceHeader = 256;  // status word + padding; the rest is per-unit tables

// Arguments of one forward call, after host-side validation.
struct FwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* g;
  const __nv_bfloat16* beta;
  __nv_bfloat16* out;
  const float* A_log;
  const float* dt_bias;
  const float* initial_state;  // may be null
  float* final_state;          // may be null
  const int32_t* cu_seqlens;   // null: batch mode
  int64_t seqlen;              // batch mode: tokens per sequence
  int32_t num_heads;
  int32_t num_seqs;
  float scale;
  float lower_bound;
  int32_t state_transposed;
  uint32_t* status;            // workspace status word, may be null (recurrent path)
  uint32_t flags = 0;          // kFlag* input transforms switched off (split path only)
};

// Token range [bos, eos) of sequence n, clamped to the call's T tokens so that a malformed
// cu_seqlens (which the host cannot read without a sync) never sends a kernel outside the token
// tensors; the kernels report it through kStatusBadSeqlens.
__device__ __forceinline__ void seq_range(const FwdParams& p, int n, int64_t& bos, int64_t& eos) {
  if (p.cu_seqlens) {
    const int64_t b = p.cu_seqlens[n], e = p.cu_seqlens[n + 1];
    bos = b < 0 ? 0 : (b > p.seqlen ? p.seqlen : b);
    eos = e < bos ? bos : (e > p.seqlen ? p.seqlen : e);
  } else {
    bos = (int64_t)n * p.seqlen;
    eos = bos + p.seqlen;
  }
}

// Whether sequence n's entries of cu_seqlens are in order: cu[n] <= cu[n + 1], cu[0] = 0 and
// cu[N] = T.  Together over all n they say that the documents tile the T tokens.
__device__ __forceinline__ bool seq_entries_ok(const FwdParams& p, int n) {
  if (!p.cu_seqlens) return true;
  const int64_t b = p.cu_seqlens[n], e = p.cu_seqlens[n + 1];
  return b <= e && (n > 0 || b == 0) && (n + 1 < p.num_seqs || e == p.seqlen);
}

// Whether every entry of cu_seqlens is in order, computed by the whole CTA (every thread must call
// it, with the same answer for all).  Kernels that own one (sequence, head) unit per CTA use it to
// apply the empty-document rule: when the offsets do not tile the T tokens in order, every document
// is treated as empty (no token read, no output row written, final state = initial state).
__device__ __forceinline__ bool cta_seqlens_ok(const FwdParams& p) {
  bool bad = false;
  if (p.cu_seqlens)
    for (int n = threadIdx.x; n < p.num_seqs; n += blockDim.x) bad |= !seq_entries_ok(p, n);
  return __syncthreads_or(bad) == 0;
}

// Launchers (defined in the kernel translation units).  Return the launch's cudaError_t.
cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream);
// The fused single-kernel chunked path (one CTA per (sequence, head); needs only the status word).
cudaError_t launch_chunked(const FwdParams& p, cudaStream_t stream);
// The split chunked path: chunk table, chunk-parallel intra-chunk kernel, recurrence kernel.
// ckpt (optional): also store the state at the start of every 64-token chunk (S^T, fp32) there.
cudaError_t launch_split(const FwdParams& p, void* workspace, cudaStream_t stream, float* ckpt = nullptr);
size_t checkpoint_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);
size_t split_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);
int split_launch_count(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);
// The segment map (M, B) of every unit: the split path with the recurrence in map mode.
cudaError_t launch_segment_map(const FwdParams& p, void* workspace, float* map_M, float* map_B,
                               cudaStream_t stream);
// S_out = M S_in + B for `units` (sequence, head) units (S_in null: zero).
cudaError_t launch_state_affine(const float* M, const float* B, const float* S_in, float* S_out, int64_t units,
                                int32_t transposed, cudaStream_t stream);
// Zero padding of head sizes below 128 (kda_pad.cu): rows of w elements of esz bytes to / from
// 128-wide rows, and [R][C] states to / from 128 x 128 ones.
cudaError_t launch_pad_rows(const void* src, void* dst, int64_t rows, int w, int esz, cudaStream_t stream);
// (rows are copied only if `nonzero` is null or *nonzero != 0)
cudaError_t launch_unpad_rows(const void* src, void* dst, int64_t rows, int w, int esz, cudaStream_t stream,
                              const int32_t* nonzero = nullptr);
cudaError_t launch_pad_state(const float* src, float* dst, int64_t units, int R, int C, cudaStream_t stream);
cudaError_t launch_unpad_state(const float* src, float* dst, int64_t units, int R, int C, cudaStream_t stream);
// The backward pass (kda_bwd): workspace bytes, and the launch (zeroes dA_log / ddt_bias first).
size_t bwd_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);
cudaError_t launch_bwd(const FwdParams& f, const __nv_bfloat16* d_out, const float* d_final, __nv_bfloat16* dq,
                       __nv_bfloat16* dk, __nv_bfloat16* dv, __nv_bfloat16* dg, __nv_bfloat16* dbeta, float* dA_log,
                       float* ddt_bias, float* d_initial, const float* checkpoints, void* workspace,
                       cudaStream_t stream);
// The batched recurrent decode step (kda_decode).
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                          void* out, const float* A_log, const float* dt_bias, float lower_bound,
                          const float* state_in, float* state_out, const int32_t* state_indices, int32_t batch,
                          int32_t seqlen, int32_t num_heads, int64_t num_slots, int32_t state_transposed,
                          uint32_t flags, uint32_t* status, cudaStream_t stream);
// One CTA whose bounded wait on a never-completed phase runs out after limit_ns (self-test).
cudaError_t launch_wait_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);

// Validates the arguments of a forward call, rejects more than max_units (sequence, head) units with
// KDA_ERR_WORKSPACE_TOO_SMALL, and only then clears the device status word `status` and launches
// the fused chunked path with it (used by kda_fwd_static_workspace).  A rejected call enqueues
// nothing.
kda_status_t fwd_fused(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                       void* out, const float* A_log, const float* dt_bias, float lower_bound,
                       const float* initial_state, float* final_state, const int32_t* cu_seqlens, int32_t batch,
                       int64_t seqlen, int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs,
                       int32_t state_transposed, uint32_t* status, int64_t max_units, cudaStream_t stream);

}  // namespace kda
