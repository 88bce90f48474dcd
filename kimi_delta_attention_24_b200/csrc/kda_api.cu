// C ABI of the KDA forward library: argument validation, workspace layout and launches.
// The declarations and the contract live in include/kda.h.
#include <math.h>

#include "kda_common.cuh"

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Shape {
  int64_t total_tokens;
  int32_t num_seqs;
};

// Validates everything the host can check without touching device memory.
kda_status_t validate(const void* q, const void* k, const void* v, const void* g, const void* beta,
                      const void* out, const float* A_log, const float* dt_bias, float lower_bound,
                      const float* initial_state, const float* final_state,
                      const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                      int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs,
                      int32_t state_transposed, float scale, Shape* shape, uint32_t flags = 0,
                      bool need_out = true) {
  if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) return KDA_ERR_UNSUPPORTED;
  if (!(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_UNSUPPORTED;
  if ((flags & ~kda::kFlagMask) != 0) return KDA_ERR_INVALID_ARGUMENT;
  const bool gate_in_kernel = !(flags & kda::kFlagGatePrecomputed);
  if (!q || !k || !v || !g || !beta || (need_out && !out)) return KDA_ERR_INVALID_ARGUMENT;
  if (gate_in_kernel && (!A_log || !dt_bias)) return KDA_ERR_INVALID_ARGUMENT;
  if (batch < 0 || seqlen < 0 || num_heads <= 0 || num_seqs < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (state_transposed != 0 && state_transposed != 1) return KDA_ERR_INVALID_ARGUMENT;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARGUMENT;
  const void* vec[] = {q, k, v, g, out};
  for (const void* p : vec)
    if (!aligned(p, 16)) return KDA_ERR_INVALID_ARGUMENT;
  if (!aligned(beta, (flags & kda::kFlagBetaPrecomputed) ? 4 : 2)) return KDA_ERR_INVALID_ARGUMENT;
  if (gate_in_kernel && (!aligned(A_log, 4) || !aligned(dt_bias, 16))) return KDA_ERR_INVALID_ARGUMENT;
  if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
    return KDA_ERR_INVALID_ARGUMENT;
  if (cu_seqlens) {
    if (!aligned(cu_seqlens, 4) || batch != 1) return KDA_ERR_INVALID_ARGUMENT;
    if (seqlen > INT32_MAX) return KDA_ERR_INVALID_ARGUMENT;  // cu_seqlens is int32
    shape->num_seqs = num_seqs;
  } else {
    if (num_seqs != 0 && num_seqs != batch) return KDA_ERR_INVALID_ARGUMENT;
    shape->num_seqs = batch;
  }
  shape->total_tokens = (int64_t)batch * seqlen;
  if (shape->total_tokens > INT32_MAX) return KDA_ERR_INVALID_ARGUMENT;  // token coordinates are int32
  if ((int64_t)shape->num_seqs * num_heads > INT32_MAX) return KDA_ERR_INVALID_ARGUMENT;
  return KDA_OK;
}

kda::FwdParams make_params(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, float scale, void* out, const float* A_log,
                           const float* dt_bias, float lower_bound, const float* initial_state,
                           float* final_state, const int32_t* cu_seqlens, int64_t seqlen,
                           int32_t num_heads, int32_t num_seqs, int32_t state_transposed,
                           uint32_t* status) {
  kda::FwdParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = static_cast<const __nv_bfloat16*>(g);
  p.beta = static_cast<const __nv_bfloat16*>(beta);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.initial_state = initial_state;
  p.final_state = final_state;
  p.cu_seqlens = cu_seqlens;
  p.seqlen = seqlen;
  p.num_heads = num_heads;
  p.num_seqs = num_seqs;
  p.scale = scale;
  p.lower_bound = lower_bound;
  p.state_transposed = state_transposed;
  p.status = status;
  return p;
}

}  // namespace

kda_status_t kda::fwd_fused(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            float scale, void* out, const float* A_log, const float* dt_bias, float lower_bound,
                            const float* initial_state, float* final_state, const int32_t* cu_seqlens,
                            int32_t batch, int64_t seqlen, int32_t num_heads, int32_t head_dim_k,
                            int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed, uint32_t* status,
                            int64_t max_units, cudaStream_t stream) {
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, out, A_log, dt_bias, lower_bound, initial_state,
                             final_state, cu_seqlens, batch, seqlen, num_heads, head_dim_k,
                             head_dim_v, num_seqs, state_transposed, scale, &shape);
  if (st != KDA_OK) return st;
  const int64_t units = (int64_t)shape.num_seqs * num_heads;
  if (units > max_units) return KDA_ERR_WORKSPACE_TOO_SMALL;
  if (!status) return KDA_ERR_INVALID_ARGUMENT;
  if (units == 0) return KDA_OK;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
                                 initial_state, final_state, cu_seqlens, seqlen, num_heads,
                                 shape.num_seqs, state_transposed, status);
  // stream-ordered: a time-out recorded by an earlier call does not leak into this one
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), stream) != cudaSuccess) return KDA_ERR_CUDA;
  return kda::launch_chunked(p, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" {

int kda_is_supported(int head_dim, int dtype_is_bf16, float lower_bound) {
  return head_dim == kda::kHeadDim && dtype_is_bf16 != 0 && lower_bound >= -5.0f &&
         lower_bound <= 0.0f;
}

size_t kda_workspace_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::split_workspace_bytes(total_tokens, num_heads, num_seqs);
}

int kda_fwd_launch_count(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::split_launch_count(total_tokens, num_heads, num_seqs);
}

kda_status_t kda_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        float scale, void* out, void* workspace, size_t workspace_bytes,
                        const float* A_log, const float* dt_bias, float lower_bound,
                        const float* initial_state, float* final_state, const int32_t* cu_seqlens,
                        int32_t batch, int64_t seqlen, int32_t num_heads, int32_t head_dim_k,
                        int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed, uint32_t flags,
                        kda_stream_t stream) {
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, out, A_log, dt_bias, lower_bound, initial_state,
                             final_state, cu_seqlens, batch, seqlen, num_heads, head_dim_k,
                             head_dim_v, num_seqs, state_transposed, scale, &shape, flags);
  if (st != KDA_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_workspace_size(shape.total_tokens, num_heads, shape.num_seqs))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
                                 initial_state, final_state, cu_seqlens, seqlen, num_heads,
                                 shape.num_seqs, state_transposed, static_cast<uint32_t*>(workspace));
  p.flags = flags;
  if ((int64_t)shape.num_seqs * num_heads == 0) return KDA_OK;
  return kda::launch_split(p, workspace, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? KDA_OK
                                                                                                 : KDA_ERR_CUDA;
}

kda_status_t kda_segment_map(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             void* workspace, size_t workspace_bytes, const float* A_log,
                             const float* dt_bias, float lower_bound, float* map_M, float* map_B,
                             const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                             int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs, uint32_t flags,
                             kda_stream_t stream) {
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, nullptr, A_log, dt_bias, lower_bound, nullptr, nullptr,
                             cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v, num_seqs, 0, 1.0f,
                             &shape, flags, /*need_out=*/false);
  if (st != KDA_OK) return st;
  if (!map_M || !map_B || !aligned(map_M, 16) || !aligned(map_B, 16)) return KDA_ERR_INVALID_ARGUMENT;
  if (!workspace || !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_workspace_size(shape.total_tokens, num_heads, shape.num_seqs))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, 1.0f, nullptr, A_log, dt_bias, lower_bound, nullptr, nullptr,
                                 cu_seqlens, seqlen, num_heads, shape.num_seqs, 0,
                                 static_cast<uint32_t*>(workspace));
  p.flags = flags;
  if ((int64_t)shape.num_seqs * num_heads == 0) return KDA_OK;
  return kda::launch_segment_map(p, workspace, map_M, map_B, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status_t kda_state_affine(const float* map_M, const float* map_B, const float* state_in, float* state_out,
                              int64_t units, int32_t head_dim, int32_t state_transposed, kda_stream_t stream) {
  if (head_dim != kda::kHeadDim) return KDA_ERR_UNSUPPORTED;
  if (units < 0 || units > INT32_MAX || (state_transposed != 0 && state_transposed != 1))
    return KDA_ERR_INVALID_ARGUMENT;
  if (!map_B || !state_out || (state_in && !map_M)) return KDA_ERR_INVALID_ARGUMENT;
  if (!aligned(map_B, 16) || !aligned(state_out, 16) || (map_M && !aligned(map_M, 16)) ||
      (state_in && !aligned(state_in, 16)))
    return KDA_ERR_INVALID_ARGUMENT;
  return kda::launch_state_affine(map_M, map_B, state_in, state_out, units, state_transposed,
                                  reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status_t kda_fwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                     float scale, void* out, void* workspace, size_t workspace_bytes,
                     const float* A_log, const float* dt_bias, float lower_bound,
                     const float* initial_state, float* final_state, const int32_t* cu_seqlens,
                     int32_t batch, int64_t seqlen, int32_t num_heads, int32_t head_dim_k,
                     int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed,
                     kda_stream_t stream) {
  return kda_fwd_ex(q, k, v, g, beta, scale, out, workspace, workspace_bytes, A_log, dt_bias, lower_bound,
                    initial_state, final_state, cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v,
                    num_seqs, state_transposed, 0u, stream);
}

kda_status_t kda_fwd_recurrent(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, float scale, void* out, void* workspace,
                               size_t workspace_bytes, const float* A_log, const float* dt_bias,
                               float lower_bound, const float* initial_state, float* final_state,
                               const int32_t* cu_seqlens, int32_t batch, int64_t seqlen,
                               int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v,
                               int32_t num_seqs, int32_t state_transposed, kda_stream_t stream) {
  (void)workspace_bytes;
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, out, A_log, dt_bias, lower_bound, initial_state,
                             final_state, cu_seqlens, batch, seqlen, num_heads, head_dim_k,
                             head_dim_v, num_seqs, state_transposed, scale, &shape);
  if (st != KDA_OK) return st;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
                                 initial_state, final_state, cu_seqlens, seqlen, num_heads,
                                 shape.num_seqs, state_transposed, static_cast<uint32_t*>(workspace));
  if ((int64_t)shape.num_seqs * num_heads == 0) return KDA_OK;
  return kda::launch_recurrent(p, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status_t kda_decode(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        float scale, void* out, const float* A_log, const float* dt_bias,
                        float lower_bound, const float* state_in, float* state_out,
                        const int32_t* state_indices, int32_t batch, int32_t seqlen,
                        int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, int64_t num_slots,
                        int32_t state_transposed, uint32_t flags, void* workspace,
                        kda_stream_t stream) {
  if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) return KDA_ERR_UNSUPPORTED;
  if ((flags & ~kda::kFlagMask) != 0) return KDA_ERR_INVALID_ARGUMENT;
  const bool gate_in_kernel = !(flags & kda::kFlagGatePrecomputed);
  if (gate_in_kernel && !(lower_bound >= -5.0f && lower_bound <= 0.0f)) return KDA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !g || !beta || !out) return KDA_ERR_INVALID_ARGUMENT;
  if (gate_in_kernel && (!A_log || !dt_bias)) return KDA_ERR_INVALID_ARGUMENT;
  if (batch < 0 || seqlen < 0 || num_heads <= 0 || num_slots < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (state_transposed != 0 && state_transposed != 1) return KDA_ERR_INVALID_ARGUMENT;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARGUMENT;
  const void* vec[] = {q, k, v, g, out};
  for (const void* p : vec)
    if (!aligned(p, 16)) return KDA_ERR_INVALID_ARGUMENT;
  if (!aligned(beta, (flags & kda::kFlagBetaPrecomputed) ? 4 : 2)) return KDA_ERR_INVALID_ARGUMENT;
  if (gate_in_kernel && (!aligned(A_log, 4) || !aligned(dt_bias, 16))) return KDA_ERR_INVALID_ARGUMENT;
  if ((state_in && !aligned(state_in, 16)) || (state_out && !aligned(state_out, 16)))
    return KDA_ERR_INVALID_ARGUMENT;
  if (state_indices && !aligned(state_indices, 4)) return KDA_ERR_INVALID_ARGUMENT;
  if (!state_indices && (state_in || state_out) && num_slots < batch) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace && !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if ((int64_t)batch * seqlen > INT32_MAX || (int64_t)batch * num_heads > INT32_MAX)
    return KDA_ERR_INVALID_ARGUMENT;
  return kda::launch_decode(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound, state_in, state_out,
                            state_indices, batch, seqlen, num_heads, num_slots, state_transposed, flags,
                            static_cast<uint32_t*>(workspace), reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

size_t kda_bwd_workspace_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::bwd_workspace_bytes(total_tokens, num_heads, num_seqs);
}

kda_status_t kda_bwd(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                     const float* A_log, const float* dt_bias, float lower_bound, const float* initial_state,
                     const void* d_out, const float* d_final, void* dq, void* dk, void* dv, void* dg, void* dbeta,
                     float* dA_log, float* ddt_bias, float* d_initial, void* workspace, size_t workspace_bytes,
                     const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                     int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs, kda_stream_t stream) {
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, d_out, A_log, dt_bias, lower_bound, initial_state, d_final,
                             cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v, num_seqs, 0, scale,
                             &shape);
  if (st != KDA_OK) return st;
  if (!dq || !dk || !dv || !dg || !dbeta || !dA_log || !ddt_bias) return KDA_ERR_INVALID_ARGUMENT;
  const void* vec[] = {dq, dk, dv, dg, ddt_bias};
  for (const void* p : vec)
    if (!aligned(p, 16)) return KDA_ERR_INVALID_ARGUMENT;
  if (!aligned(dbeta, 2) || !aligned(dA_log, 4) || (d_initial && !aligned(d_initial, 16)))
    return KDA_ERR_INVALID_ARGUMENT;
  if (!workspace || !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_bwd_workspace_size(shape.total_tokens, num_heads, shape.num_seqs))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, nullptr, A_log, dt_bias, lower_bound, initial_state,
                                 nullptr, cu_seqlens, seqlen, num_heads, shape.num_seqs, 0, nullptr);
  return kda::launch_bwd(p, static_cast<const __nv_bfloat16*>(d_out), d_final, static_cast<__nv_bfloat16*>(dq),
                         static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv),
                         static_cast<__nv_bfloat16*>(dg), static_cast<__nv_bfloat16*>(dbeta), dA_log, ddt_bias,
                         d_initial, workspace, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status_t kda_read_device_status(void* workspace, kda_stream_t stream) {
  if (!workspace) return KDA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
  }
  if (word & kda::kStatusTimeout) return KDA_ERR_DEVICE_TIMEOUT;
  return (word & (kda::kStatusBadSeqlens | kda::kStatusBadIndex)) ? KDA_ERR_INVALID_ARGUMENT : KDA_OK;
}

kda_status_t kda_selftest_wait_timeout(void* workspace, uint32_t limit_us, kda_stream_t stream) {
  if (!workspace || !aligned(workspace, 256) || limit_us == 0 || limit_us > 1000000u)
    return KDA_ERR_INVALID_ARGUMENT;
  return kda::launch_wait_timeout(static_cast<uint32_t*>(workspace), (uint64_t)limit_us * 1000u,
                                  reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

const char* kda_status_string(kda_status_t status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARGUMENT: return "KDA_ERR_INVALID_ARGUMENT";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_WORKSPACE_TOO_SMALL: return "KDA_ERR_WORKSPACE_TOO_SMALL";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
  }
  return "KDA_ERR_UNKNOWN";
}

}  // extern "C"
