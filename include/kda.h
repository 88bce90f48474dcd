/*
 * kda.h — C ABI of the B200 (sm_100a) Kimi Delta Attention forward library (libkda_b200.so).
 *
 * The operation.  Kimi Delta Attention is a gated delta rule with a per-channel decay:
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = scale * S_t^T q_t
 * with, applied inside the kernels (the flags use_qk_l2norm_in_kernel, use_beta_sigmoid_in_kernel,
 * use_gate_in_kernel and safe_gate of fla's chunk_kda, all on):
 *     q <- q / sqrt(|q|^2 + 1e-6),  k likewise,  beta <- sigmoid(beta),
 *     log alpha_c = lower_bound * sigmoid(exp(A_log[h]) * (g_c + dt_bias[h, c])).
 * The argument order of kda_fwd follows FlashKDA's `fwd` (q, k, v, g, beta, scale, out, workspace,
 * A_log, dt_bias, lower_bound, initial_state, final_state, cu_seqlens) as printed in the vLLM PR
 * #54859 report ("[Kimi-K3] Bump FlashKDA to fix unstable inverse", section 关键源码片段); the
 * workspace query follows `get_workspace_size(T, H, N)` on the same page; the support predicate
 * follows `is_flashkda_supported(128, torch.bfloat16, lower_bound)` there.  Shapes and the
 * batch-mode call (cu_seqlens = None) follow "What CUDA Version Is Required to Use FlashKDA?",
 * section Usage Examples.  This C ABI adds explicit sizes and a stream.
 *
 * Layouts (all contiguous, row-major, device memory; q, k, v, g, out, dt_bias and the states
 * 16-byte aligned, beta 2-byte, A_log and cu_seqlens 4-byte; batch * seqlen < 2^31 tokens):
 *   q, k, g   bf16  [batch, seqlen, H, K]      (packed varlen: batch = 1, seqlen = total tokens)
 *   v, out    bf16  [batch, seqlen, H, V]
 *   beta      bf16  [batch, seqlen, H]          raw, before the sigmoid
 *   A_log     fp32  [H];    dt_bias fp32 [H, K]
 *   initial_state / final_state  fp32 [N, H, K, V] holding S[k][v]   (state_transposed = 0)
 *                                fp32 [N, H, V, K] holding S^T        (state_transposed = 1)
 *   cu_seqlens int32 [N + 1]: cu[0] = 0, non-decreasing, cu[N] = seqlen (batch must be 1)
 * K = V = 128 is the supported head size; lower_bound must lie in [-5, 0].
 *
 * Ownership.  The caller owns every buffer.  The library allocates no device memory, keeps no
 * per-call state, never synchronises the stream and never copies device data to the host
 * (except kda_read_device_status, which exists to do exactly that).  Outputs are written in
 * place on `stream`.  initial_state may alias final_state: each unit reads its state before
 * writing it.  Rows of `out` outside [0, cu[N]) are not touched.
 *
 * Errors.  Argument problems are found on the host before anything is launched and nothing is
 * written.  A launch failure returns KDA_ERR_CUDA.  The chunked kernel bounds every wait it
 * performs; if a bound is exceeded it records KDA_ERR_DEVICE_TIMEOUT in the workspace status
 * word and the affected work is skipped — read it with kda_read_device_status.  The contents of
 * cu_seqlens live on the device, so they are checked there: unless 0 = cu[0] <= cu[1] <= ... <=
 * cu[N] = seqlen, the kernels record KDA_ERR_INVALID_ARGUMENT in the status word, never read or
 * write outside the T tokens, and treat every document as empty (out is not written,
 * final_state receives initial_state).
 */
#ifndef KDA_B200_H_
#define KDA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad shape, misaligned pointer, bad flag */
  KDA_ERR_UNSUPPORTED = 2,        /* head dim != 128 or lower_bound outside [-5, 0] */
  KDA_ERR_WORKSPACE_TOO_SMALL = 3,
  KDA_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
  KDA_ERR_DEVICE_TIMEOUT = 5      /* a bounded device-side wait ran out (see kda_read_device_status) */
} kda_status_t;

/* Input-transform flags (fla chunk_kda's use_gate_in_kernel, use_qk_l2norm_in_kernel and
 * use_beta_sigmoid_in_kernel, as listed in "What CUDA Version Is Required to Use FlashKDA?",
 * Usage Examples; 0 means all three transforms run in the kernel, as in kda_fwd).
 *   KDA_FLAG_GATE_PRECOMPUTED  g holds fp32 log alpha [tokens, H, K] (natural log, <= 0): the safe
 *                              gate is not applied and A_log / dt_bias are not read (may be NULL).
 *                              kda_fwd_ex clamps it to [lower_bound, 0] (the safe-gate range);
 *                              kda_decode uses it as given.
 *   KDA_FLAG_NO_QK_L2NORM      q and k are used as given (no L2 normalisation).
 *   KDA_FLAG_BETA_PRECOMPUTED  beta holds fp32 beta [tokens, H] (no sigmoid). */
enum {
  KDA_FLAG_GATE_PRECOMPUTED = 1,
  KDA_FLAG_NO_QK_L2NORM = 2,
  KDA_FLAG_BETA_PRECOMPUTED = 4
};

/* 1 when (head_dim, dtype, lower_bound) is a configuration this library runs: head_dim = 128,
 * bf16 inputs (dtype_is_bf16 != 0) and -5 <= lower_bound <= 0; otherwise 0.  Mirrors
 * is_flashkda_supported(128, torch.bfloat16, lower_bound). */
int kda_is_supported(int head_dim, int dtype_is_bf16, float lower_bound);

/* Bytes of device workspace kda_fwd needs for (total tokens T, heads H, sequences N), as
 * get_workspace_size(T, H, N): a 256-byte header (the sticky device status word and two item
 * counters), the chunk table, 82,944 bytes of intermediates per (chunk, head) for at most
 * (T + 63 N) / 64 chunks, and one 64 KB fp32 state per head for the sequence that is cut between
 * two stages (4.08 GB at T = 32768, H = 96, N = 1).  Depends only on its arguments.  Only the
 * header needs initialisation by the caller: zero it once before first use. */
size_t kda_workspace_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);

/* Number of kernel launches one kda_fwd call with these sizes enqueues on the current device:
 * 3 (chunk table, intra-chunk kernel, recurrence kernel), 5 when the call runs in two stages
 * (N * H below the device's SM count: the chunk range is cut in two and the second intra-chunk
 * launch overlaps the first recurrence), 2 when there are no chunks, 0 when N * H = 0.
 * -1 if the device cannot be queried. */
int kda_fwd_launch_count(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);

/* The chunked forward pass (the product path): chunk table, then the chunk-parallel intra-chunk
 * kernel and the per-(sequence, head) recurrence kernel over one or two ranges of chunks, all on
 * `stream` (launches after the first intra-chunk one are programmatic dependents of the launch
 * before them: they may start while it drains and wait in-kernel for what they read).
 *   scale          multiplies the output (o = scale * S^T qhat); it never enters the state.
 *   workspace      device buffer of at least kda_workspace_size(batch*seqlen, H, N) bytes, its
 *                  first 256 bytes zeroed once by the caller before its first use; calls that
 *                  share a workspace must be ordered (the same stream, or events).
 *   initial_state  NULL means a zero state.   final_state  NULL means it is not written.
 *   cu_seqlens     NULL selects batch mode: N = batch sequences of length seqlen each.
 *   num_seqs       N; with cu_seqlens it must be the number of documents, without it batch
 *                  (0 is accepted and means batch).
 *   state_transposed  0: state is S[k][v];  1: state is stored transposed (S^T, [V][K]).
 * Returns KDA_OK once the work is enqueued on `stream`. */
kda_status_t kda_fwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                     float scale, void* out, void* workspace, size_t workspace_bytes,
                     const float* A_log, const float* dt_bias, float lower_bound,
                     const float* initial_state, float* final_state, const int32_t* cu_seqlens,
                     int32_t batch, int64_t seqlen, int32_t num_heads, int32_t head_dim_k,
                     int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed,
                     kda_stream_t stream);

/* Bytes of workspace kda_fwd_ex needs for head sizes (K, V): kda_workspace_size(T, H, N) when
 * K = V = 128; for smaller head sizes also 128-wide copies of q, k, v, g, out, dt_bias and the
 * states, into which the inputs are zero-padded. */
size_t kda_workspace_size_ex(int64_t total_tokens, int32_t num_heads, int32_t num_seqs, int32_t head_dim_k,
                             int32_t head_dim_v);

/* kda_fwd with the input transforms selectable (fla chunk_kda's use_gate_in_kernel,
 * use_qk_l2norm_in_kernel and use_beta_sigmoid_in_kernel; "What CUDA Version Is Required to Use
 * FlashKDA?", Usage Examples): `flags` is a combination of the KDA_FLAG_* values, 0 giving
 * kda_fwd.  With KDA_FLAG_GATE_PRECOMPUTED, g is fp32 log alpha [batch, seqlen, H, K] (16-byte
 * aligned), A_log and dt_bias may be NULL, and each log alpha is clamped to [lower_bound, 0] (the
 * range whose per-16-token exponent span the chunked kernels keep inside float range); with
 * KDA_FLAG_BETA_PRECOMPUTED beta is fp32 [batch, seqlen, H] (4-byte aligned).
 * Head sizes: besides K = V = 128, any K and V that are multiples of 8 up to 128 (fla's chunk_kda
 * takes any head size).  Those run the same kernels on zero-padded 128-wide copies made in the
 * workspace (size from kda_workspace_size_ex), which is exact: padded key channels are zero in q
 * and k, padded value channels zero in v, so they add nothing and their state entries stay zero;
 * layouts are the same with K and V in place of 128.  Same errors as kda_fwd otherwise. */
kda_status_t kda_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        float scale, void* out, void* workspace, size_t workspace_bytes,
                        const float* A_log, const float* dt_bias, float lower_bound,
                        const float* initial_state, float* final_state, const int32_t* cu_seqlens,
                        int32_t batch, int64_t seqlen, int32_t num_heads, int32_t head_dim_k,
                        int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed, uint32_t flags,
                        kda_stream_t stream);

/* The segment map of every (sequence, head) unit, for sequence-parallel prefill (KCP, the KDA
 * context parallelism of torchtitan PR #4374): the forward pass is affine in the state a segment
 * starts from, S_out = M S_in + B, with M (K x K) the product of the segment's per-token
 * transitions (I - beta khat khat^T) Diag(alpha) and B (K x V) the state reached from zero.  Same
 * inputs, workspace and flags as kda_fwd_ex (no scale, output or states); writes
 *   map_M  fp32 [N, H, K, K]   (M[k][k'], row-major; 16-byte aligned)
 *   map_B  fp32 [N, H, K, V]   (B[k][v])
 * Runs the chunk table and the intra-chunk kernel once, then one recurrence launch of 2 N H CTAs
 * (B from v and a zero state; M from v = 0 and the identity state).  An empty sequence gets
 * M = I, B = 0.  Errors as kda_fwd. */
kda_status_t kda_segment_map(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             void* workspace, size_t workspace_bytes, const float* A_log,
                             const float* dt_bias, float lower_bound, float* map_M, float* map_B,
                             const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                             int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs, uint32_t flags,
                             kda_stream_t stream);

/* state_out = map_M state_in + map_B for `units` (sequence, head) units of 128 x 128 fp32: the
 * fold of one segment map over a state (KCP's scan step).  map_M and map_B as kda_segment_map
 * writes them; state_in / state_out in the layout `state_transposed` selects (S[k][v], or S^T);
 * state_in NULL means a zero state (then map_M may be NULL too); state_out may alias state_in.
 * One CTA per unit, fp32 on CUDA cores.  KDA_ERR_UNSUPPORTED for head_dim != 128,
 * KDA_ERR_INVALID_ARGUMENT for null or misaligned (16-byte) pointers or a bad flag. */
kda_status_t kda_state_affine(const float* map_M, const float* map_B, const float* state_in, float* state_out,
                              int64_t units, int32_t head_dim, int32_t state_transposed, kda_stream_t stream);

/* The same operation evaluated token by token on CUDA cores (one thread per state column):
 * no chunking, no tensor cores.  Same arguments, layouts and errors as kda_fwd (the workspace
 * may be NULL with workspace_bytes = 0).  It is the GPU restatement of the recurrence and the
 * basis of single-token decoding; it is much slower than kda_fwd on long prefills. */
kda_status_t kda_fwd_recurrent(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, float scale, void* out, void* workspace,
                               size_t workspace_bytes, const float* A_log, const float* dt_bias,
                               float lower_bound, const float* initial_state, float* final_state,
                               const int32_t* cu_seqlens, int32_t batch, int64_t seqlen,
                               int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v,
                               int32_t num_seqs, int32_t state_transposed, kda_stream_t stream);

/* kda_fwd for callers that cannot allocate device memory (for example runtimes that plan every
 * device buffer ahead of time and forbid libraries from calling cudaMalloc, or code that must not
 * trigger cudaMalloc's device-wide synchronisation).  The pages have no counterpart to this entry
 * point.  Same arguments as kda_fwd, minus the workspace: its scratch is a 256-byte device array
 * that lives in the library (held by every GPU that loads it until the process exits), and it
 * allocates nothing.  That array holds no per-chunk intermediates, so it runs the fused
 * single-kernel path (one CTA per (sequence, head), every intermediate on chip): results agree
 * with kda_fwd's to rounding, and it is slower on long prefills.
 *   - At most 4096 (sequence, head) units per call, a fixed limit of this entry point; more
 *     returns KDA_ERR_WORKSPACE_TOO_SMALL.  Arguments are validated first (the same checks and
 *     codes as kda_fwd), and a rejected call enqueues nothing.
 *   - The first call on a device looks up the array's address on that device; make it before any
 *     stream capture.
 *   - All calls share the array: calls that overlap on the GPU race on it.
 *   - Each accepted call clears the array's status word, which is not reported: device time-outs
 *     and out-of-order cu_seqlens go unreported here.  Out-of-order offsets still get kda_fwd's
 *     empty-document rule (out not written, final_state = initial_state). */
kda_status_t kda_fwd_static_workspace(const void* q, const void* k, const void* v, const void* g,
                                      const void* beta, float scale, void* out, const float* A_log,
                                      const float* dt_bias, float lower_bound,
                                      const float* initial_state, float* final_state,
                                      const int32_t* cu_seqlens, int32_t batch, int64_t seqlen,
                                      int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v,
                                      int32_t num_seqs, int32_t state_transposed,
                                      kda_stream_t stream);

/* One recurrent step of a batch of requests, each advancing its own state in a state pool by
 * `seqlen` tokens (1 for plain decoding, a few for speculative tokens): the decode path that
 * serves Kimi-K3 beside the chunked prefill (vLLM PR #54859 report, sections 风险与影响 and
 * 关联脉络).  For each (request b, head h) and each of its tokens in order:
 *     S <- Diag(alpha) S;  delta = beta (v - S^T khat);  S <- S + khat delta^T;  o = scale S^T qhat
 * with the same in-kernel transforms as kda_fwd unless `flags` switches them off (see the
 * KDA_FLAG_* values).  Runs on CUDA cores, one CTA per (request, head), state in registers; bound
 * by the state's HBM traffic (64 KB read + 64 KB written per unit).
 *   q, k, v, out   bf16 [batch, seqlen, H, 128];  g bf16 [batch, seqlen, H, 128] (fp32 with
 *                  KDA_FLAG_GATE_PRECOMPUTED);  beta bf16 [batch, seqlen, H] (fp32 with
 *                  KDA_FLAG_BETA_PRECOMPUTED);  A_log fp32 [H], dt_bias fp32 [H, 128].
 *   state_in / state_out  fp32 pools [num_slots, H, 128, 128] (S[k][v], or S^T with
 *                  state_transposed = 1).  state_in NULL means zero states; state_out NULL means
 *                  no write; they may be the same pool (in-place update).  With seqlen = 0 the
 *                  requests' states are copied from state_in to state_out unchanged (the token
 *                  tensors, A_log and dt_bias are then not read and may be NULL).
 *   state_indices  int32 [batch]: the pool slot of each request; NULL means slot b for request b.
 *                  A negative index skips the request (nothing read or written: padding).  The
 *                  non-negative indices of one call must be distinct.  An index >= num_slots
 *                  also skips the request and records KDA_ERR_INVALID_ARGUMENT in the workspace
 *                  status word when a workspace is given.
 *   workspace      optional (NULL allowed): a device buffer of at least 256 bytes, 256-byte
 *                  aligned, whose first 4 bytes are the sticky status word read by
 *                  kda_read_device_status.
 * Errors as kda_fwd (lower_bound is checked only when the gate is computed in the kernel).
 * Pointers to q, k, v, g, out and the pools are 16-byte aligned, beta 2-byte (4 if fp32). */
kda_status_t kda_decode(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        float scale, void* out, const float* A_log, const float* dt_bias,
                        float lower_bound, const float* state_in, float* state_out,
                        const int32_t* state_indices, int32_t batch, int32_t seqlen,
                        int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, int64_t num_slots,
                        int32_t state_transposed, uint32_t flags, void* workspace,
                        kda_stream_t stream);

/* Bytes of the checkpoints kda_fwd_checkpointed writes for (T, H, N): one fp32 128 x 128 state per
 * (64-token chunk, head) for at most T / 64 + N + 1 chunk slots (3.2 GB at T = 32768, H = 96). */
size_t kda_checkpoint_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);

/* kda_fwd (K = V = 128, the in-kernel transforms on) that also stores, for the backward pass, the
 * state at the start of every 64-token chunk of every (sequence, head): fp32 S^T [v][k], 64 KB per
 * (chunk, head), slot floor(bos_n / 64) + n + c for chunk c of sequence n (bos_n its first token).
 * checkpoints: device, 16-byte aligned, at least kda_checkpoint_size bytes.  Otherwise as kda_fwd. */
kda_status_t kda_fwd_checkpointed(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                  float scale, void* out, void* workspace, size_t workspace_bytes,
                                  const float* A_log, const float* dt_bias, float lower_bound,
                                  const float* initial_state, float* final_state, float* checkpoints,
                                  size_t checkpoint_bytes, const int32_t* cu_seqlens, int32_t batch, int64_t seqlen,
                                  int32_t num_heads, int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs,
                                  kda_stream_t stream);

/* Bytes of device workspace kda_bwd needs for (total tokens T, heads H, sequences N): the forward's
 * workspace and the checkpoints and output it writes (used when the call is given no checkpoints),
 * per (64-token chunk, head) the chunk's factors for the reverse state walk and the gradient kernel
 * (336.5 KB) and dDelta (32 KB), one 128 x 128 state gradient per chunk slot and head, per-token
 * partials (3 x 128 + 1 fp32 per token and head), and a scratch of 369 KB per CTA of the
 * chunk-parallel kernels (at most 296).  Depends
 * only on its arguments; its first 256 bytes hold the status word read by kda_read_device_status. */
size_t kda_bwd_workspace_size(int64_t total_tokens, int32_t num_heads, int32_t num_seqs);

/* The backward pass: gradients of sum(d_out * out) + sum(d_final * final_state) with respect to
 * every input of kda_fwd (torchtitan trains Kimi-K3 through chunk_kda, and its varlen test checks
 * the gradient as well as the forward: torchtitan PR #4374, Results).  Same inputs, layouts and
 * errors as kda_fwd (state_transposed = 0: states and their gradients are [N, H, K, V]), plus
 *   d_out        bf16 [batch, seqlen, H, V]   the output's gradient
 *   d_final      fp32 [N, H, K, V] or NULL (zero)   the final state's gradient
 *   checkpoints  what kda_fwd_checkpointed stored for the same inputs, or NULL: then the backward
 *                first runs the forward itself to make them (in the workspace)
 * and writes
 *   dq, dk, dg   bf16 [batch, seqlen, H, K];  dv bf16 [batch, seqlen, H, V];  dbeta bf16
 *                [batch, seqlen, H] (w.r.t. the raw beta, before the sigmoid; dg w.r.t. the raw gate)
 *   dA_log fp32 [H], ddt_bias fp32 [H, K]  (overwritten: zeroed, then summed over all tokens)
 *   d_initial    fp32 [N, H, K, V] or NULL (not written)
 * In the chunked form, fp32 throughout (products on the tensor cores with tf32 operands split into
 * high and low parts, fp32-level): (without checkpoints) the checkpointing forward; then per
 * 64-token chunk, in parallel, the chunk's factors (gate, norms, decay-weighted Gram products,
 * (I + A)^{-1}); per (sequence, head), from the last chunk to the first, the gradient of the state at
 * every chunk boundary; per chunk, in parallel, the gradients of the chunk's inputs; and a last
 * kernel for the derivatives of the in-kernel transforms.  Gradient pointers are 16-byte aligned
 * (dbeta 2, dA_log 4).  With out-of-order cu_seqlens every document is treated as empty: the token
 * gradients are not written, d_initial = d_final, and the workspace status word records it. */
kda_status_t kda_bwd(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                     const float* A_log, const float* dt_bias, float lower_bound, const float* initial_state,
                     const void* d_out, const float* d_final, const float* checkpoints, void* dq, void* dk,
                     void* dv, void* dg, void* dbeta,
                     float* dA_log, float* ddt_bias, float* d_initial, void* workspace, size_t workspace_bytes,
                     const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
                     int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs, kda_stream_t stream);

/* Synchronises `stream`, reads the workspace's sticky status word, clears it, and returns
 * KDA_OK or the recorded device error: KDA_ERR_DEVICE_TIMEOUT (a bounded wait ran out; reported
 * first when both are recorded) or KDA_ERR_INVALID_ARGUMENT (cu_seqlens out of order, or a decode
 * state index past the pool).
 * KDA_ERR_CUDA if the copy fails. */
kda_status_t kda_read_device_status(void* workspace, kda_stream_t stream);

/* Self-test of the device time-out path.  Enqueues one CTA that waits, with the forward kernels'
 * bounded wait, on a barrier phase that nothing completes; after limit_us microseconds
 * (1 .. 1,000,000) the wait gives up and records KDA_ERR_DEVICE_TIMEOUT in the workspace status
 * word, which kda_read_device_status then returns.  Nothing faults or hangs and the stream stays
 * usable.  KDA_ERR_INVALID_ARGUMENT for a null or misaligned workspace or a limit out of range. */
kda_status_t kda_selftest_wait_timeout(void* workspace, uint32_t limit_us, kda_stream_t stream);

/* A static, human-readable name for a status code. */
const char* kda_status_string(kda_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H_ */
