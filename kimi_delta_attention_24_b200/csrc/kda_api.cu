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

// Head sizes kda_fwd_ex runs by zero padding to 128: multiples of 8 (16-byte bf16 rows) up to 128.
bool padded_head_dim_ok(int32_t d) { return d >= 8 && d <= kda::kHeadDim && d % 8 == 0; }

// Bytes after the split path's workspace that zero padding needs: 128-wide q, k, v, out (bf16), g
// (fp32, the wider of its two types), dt_bias, and the initial and final states.
size_t pad_bytes(int64_t tokens, int32_t H, int32_t N, int32_t K, int32_t V) {
  if (K == kda::kHeadDim && V == kda::kHeadDim) return 0;
  const size_t rows = (size_t)(tokens > 0 ? tokens : 0) * (size_t)(H > 0 ? H : 0);
  const size_t row_bf16 = kda::kHeadDim * 2, row_f32 = kda::kHeadDim * 4;
  const size_t units = (size_t)(N > 0 ? N : 0) * (size_t)(H > 0 ? H : 0);
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  return 4 * up(rows * row_bf16) + up(rows * row_f32) + up((size_t)(H > 0 ? H : 0) * row_f32) +
         2 * up(units * kda::kHeadDim * row_f32);
}

// Validates everything the host can check without touching device memory.
kda_status_t validate(const void* q, const void* k, const void* v, const void* g, const void* beta,
                      const void* out, const float* A_log, const float* dt_bias, float lower_bound,
                      const float* initial_state, const float* final_state,
                      const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                      int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs,
                      int32_t state_transposed, float scale, Shape* shape, uint32_t flags = 0,
                      bool need_out = true, bool any_head_dim = false) {
  if (any_head_dim) {
    if (!padded_head_dim_ok(head_dim_k) || !padded_head_dim_ok(head_dim_v)) return KDA_ERR_UNSUPPORTED;
  } else if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) {
    return KDA_ERR_UNSUPPORTED;
  }
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
  return head_dim == kda::kHeadDim && dtype_is_bf16 != 0 && lower_bound >= -5.0f && lower_bound <= 0.0f;
}

size_t kda_workspace_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::split_workspace_bytes(total_tokens, num_heads, num_seqs);
}

int kda_fwd_launch_count(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::split_launch_count(total_tokens, num_heads, num_seqs);
}

size_t kda_workspace_size_ex(int64_t total_tokens, int32_t num_heads, int32_t num_seqs, int32_t head_dim_k,
                             int32_t head_dim_v) {
  const size_t split = kda::split_workspace_bytes(total_tokens, num_heads, num_seqs);
  if (head_dim_k == kda::kHeadDim && head_dim_v == kda::kHeadDim) return split;
  return (split + 255) / 256 * 256 + pad_bytes(total_tokens, num_heads, num_seqs, head_dim_k, head_dim_v);
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
                             head_dim_v, num_seqs, state_transposed, scale, &shape, flags, true, true);
  if (st != KDA_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_workspace_size_ex(shape.total_tokens, num_heads, shape.num_seqs, head_dim_k,
                                              head_dim_v))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
                                 initial_state, final_state, cu_seqlens, seqlen, num_heads,
                                 shape.num_seqs, state_transposed, static_cast<uint32_t*>(workspace));
  p.flags = flags;
  const int64_t units = (int64_t)shape.num_seqs * num_heads;
  if (units == 0) return KDA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int K = head_dim_k, V = head_dim_v;
  if (K == kda::kHeadDim && V == kda::kHeadDim)
    return kda::launch_split(p, workspace, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;

  // head sizes below 128: zero-pad into the workspace, run the 128-wide path, copy the results out
  const int64_t rows = shape.total_tokens * num_heads;
  const size_t row_bf16 = kda::kHeadDim * 2, row_f32 = kda::kHeadDim * 4;
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  uint8_t* cur = static_cast<uint8_t*>(workspace) +
                 up(kda::split_workspace_bytes(shape.total_tokens, num_heads, shape.num_seqs));
  auto take = [&](size_t bytes) {
    uint8_t* r = cur;
    cur += up(bytes);
    return r;
  };
  void* q2 = take(rows * row_bf16);
  void* k2 = take(rows * row_bf16);
  void* v2 = take(rows * row_bf16);
  void* o2 = take(rows * row_bf16);
  void* g2 = take(rows * row_f32);
  float* dt2 = reinterpret_cast<float*>(take((size_t)num_heads * row_f32));
  float* s02 = reinterpret_cast<float*>(take((size_t)units * kda::kHeadDim * row_f32));
  float* sf2 = reinterpret_cast<float*>(take((size_t)units * kda::kHeadDim * row_f32));
  const bool gate_pre = (flags & kda::kFlagGatePrecomputed) != 0;
  const int R = state_transposed ? V : K, C = state_transposed ? K : V;
  bool ok = kda::launch_pad_rows(q, q2, rows, K, 2, s) == cudaSuccess &&
            kda::launch_pad_rows(k, k2, rows, K, 2, s) == cudaSuccess &&
            kda::launch_pad_rows(v, v2, rows, V, 2, s) == cudaSuccess &&
            kda::launch_pad_rows(g, g2, rows, K, gate_pre ? 4 : 2, s) == cudaSuccess;
  if (ok && !gate_pre) ok = kda::launch_pad_rows(dt_bias, dt2, num_heads, K, 4, s) == cudaSuccess;
  if (ok && initial_state) ok = kda::launch_pad_state(initial_state, s02, units, R, C, s) == cudaSuccess;
  if (!ok) return KDA_ERR_CUDA;
  p.q = static_cast<const __nv_bfloat16*>(q2);
  p.k = static_cast<const __nv_bfloat16*>(k2);
  p.v = static_cast<const __nv_bfloat16*>(v2);
  p.g = static_cast<const __nv_bfloat16*>(g2);
  p.out = static_cast<__nv_bfloat16*>(o2);
  p.dt_bias = gate_pre ? nullptr : dt2;
  p.initial_state = initial_state ? s02 : nullptr;
  p.final_state = final_state ? sf2 : nullptr;
  if (kda::launch_split(p, workspace, s) != cudaSuccess) return KDA_ERR_CUDA;
  // the documents cover every token when cu_seqlens is in order, so every padded output row was
  // written; when it is not, the chunk table is all zero and `out` must stay untouched: the copy
  // reads the chunk table's total first and skips
  const int32_t* chunk_total = reinterpret_cast<const int32_t*>(static_cast<uint8_t*>(workspace) +
                                                                kda::kWorkspaceHeader) + shape.num_seqs;
  if (kda::launch_unpad_rows(o2, out, rows, V, 2, s, chunk_total) != cudaSuccess) return KDA_ERR_CUDA;
  if (final_state && kda::launch_unpad_state(sf2, final_state, units, R, C, s) != cudaSuccess) return KDA_ERR_CUDA;
  return KDA_OK;
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
  if (head_dim_k != kda::kHeadDim || head_dim_v != kda::kHeadDim) return KDA_ERR_UNSUPPORTED;
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
  if (batch < 0 || seqlen < 0 || num_heads <= 0 || num_slots < 0) return KDA_ERR_INVALID_ARGUMENT;
  // with no token nothing of the token tensors is read: they may be null (empty tensors)
  if (seqlen > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_INVALID_ARGUMENT;
  if (seqlen > 0 && gate_in_kernel && (!A_log || !dt_bias)) return KDA_ERR_INVALID_ARGUMENT;
  if (state_transposed != 0 && state_transposed != 1) return KDA_ERR_INVALID_ARGUMENT;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARGUMENT;
  const void* vec[] = {q, k, v, g, out};
  for (const void* p : vec)
    if (!aligned(p, 16)) return KDA_ERR_INVALID_ARGUMENT;
  if (!aligned(beta, (flags & kda::kFlagBetaPrecomputed) ? 4 : 2)) return KDA_ERR_INVALID_ARGUMENT;
  if (gate_in_kernel && seqlen > 0 && (!aligned(A_log, 4) || !aligned(dt_bias, 16))) return KDA_ERR_INVALID_ARGUMENT;
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

size_t kda_checkpoint_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return kda::checkpoint_bytes(total_tokens, num_heads, num_seqs);
}

kda_status_t kda_fwd_checkpointed(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                  float scale, void* out, void* workspace, size_t workspace_bytes,
                                  const float* A_log, const float* dt_bias, float lower_bound,
                                  const float* initial_state, float* final_state, float* checkpoints,
                                  size_t checkpoint_bytes, const int32_t* cu_seqlens, int32_t batch, int64_t seqlen,
                                  int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs,
                                  kda_stream_t stream) {
  Shape shape;
  kda_status_t st = validate(q, k, v, g, beta, out, A_log, dt_bias, lower_bound, initial_state, final_state,
                             cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v, num_seqs, 0, scale,
                             &shape);
  if (st != KDA_OK) return st;
  if (!workspace || !aligned(workspace, 256) || !checkpoints || !aligned(checkpoints, 16))
    return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_workspace_size(shape.total_tokens, num_heads, shape.num_seqs) ||
      checkpoint_bytes < kda_checkpoint_size(shape.total_tokens, num_heads, shape.num_seqs))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound,
                                 initial_state, final_state, cu_seqlens, seqlen, num_heads,
                                 shape.num_seqs, 0, static_cast<uint32_t*>(workspace));
  if ((int64_t)shape.num_seqs * num_heads == 0) return KDA_OK;
  return kda::launch_split(p, workspace, reinterpret_cast<cudaStream_t>(stream), checkpoints) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

kda_status_t kda_bwd(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                     const float* A_log, const float* dt_bias, float lower_bound, const float* initial_state,
                     const void* d_out, const float* d_final, const float* checkpoints, void* dq, void* dk,
                     void* dv, void* dg, void* dbeta,
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
  if (!aligned(dbeta, 2) || !aligned(dA_log, 4) || (d_initial && !aligned(d_initial, 16)) ||
      (checkpoints && !aligned(checkpoints, 16)))
    return KDA_ERR_INVALID_ARGUMENT;
  if (!workspace || !aligned(workspace, 256)) return KDA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < kda_bwd_workspace_size(shape.total_tokens, num_heads, shape.num_seqs))
    return KDA_ERR_WORKSPACE_TOO_SMALL;
  kda::FwdParams p = make_params(q, k, v, g, beta, scale, nullptr, A_log, dt_bias, lower_bound, initial_state,
                                 nullptr, cu_seqlens, seqlen, num_heads, shape.num_seqs, 0, nullptr);
  return kda::launch_bwd(p, static_cast<const __nv_bfloat16*>(d_out), d_final, static_cast<__nv_bfloat16*>(dq),
                         static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv),
                         static_cast<__nv_bfloat16*>(dg), static_cast<__nv_bfloat16*>(dbeta), dA_log, ddt_bias,
                         d_initial, checkpoints, workspace, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
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
