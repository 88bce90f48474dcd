// kda_fwd_static_workspace: the chunked forward pass for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to allocate device memory while they run this operator: inference
// runtimes that plan every device buffer ahead of time and forbid libraries from calling
// cudaMalloc, or code that must not pay cudaMalloc's implicit device-wide synchronisation.  They
// still own their inputs and outputs, but have nowhere to put kda_fwd's workspace.  This entry
// point uses a workspace that lives in the library itself: a file-scope device array, allocated
// once when the library's device code is loaded on a GPU and held by that GPU until the process
// exits.  That array cannot hold the per-chunk intermediates of kda_fwd's split path (about 81 KB
// per chunk and head), so this entry point runs the fused single-kernel chunked path, which keeps
// every intermediate on chip and needs only the status word; its results agree with kda_fwd's to
// rounding.
//
// Limits and behaviour:
//   - The array holds the workspace of at most kStaticMaxUnits (sequence, head) units; larger
//     problems are rejected with KDA_ERR_WORKSPACE_TOO_SMALL before anything is launched.
//   - The array's device address is looked up once per device, on the first call made with that
//     device current (cudaGetSymbolAddress).  Make that first call before any stream capture.
//   - Every call shares the one array.  Calls whose kernels overlap on the GPU race on it; issue
//     them on one stream, or otherwise order them.
//   - Each call clears the array's status word first (stream-ordered), so a device-side time-out
//     recorded by an earlier call does not leak into the next; the status itself is not reported
//     to the caller by this entry point.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating library routine.
#include <mutex>

#include "kda_common.cuh"

namespace {

constexpr int32_t kStaticMaxUnits = 4096;
constexpr size_t kStaticWorkspaceBytes = kda::kWorkspaceHeader + (size_t)kStaticMaxUnits * sizeof(int32_t);

static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
void* g_static_workspace_ptr[kMaxDevices] = {};
std::mutex g_static_workspace_mutex;

// Device address of g_static_workspace on the current device (looked up once per device).
kda_status_t static_workspace_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_workspace_mutex);
  if (!g_static_workspace_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess || !ptr) return KDA_ERR_CUDA;
    g_static_workspace_ptr[dev] = ptr;
  }
  *out = g_static_workspace_ptr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_fwd_static_workspace(
    const void* q, const void* k, const void* v, const void* g, const void* beta, float scale, void* out,
    const float* A_log, const float* dt_bias, float lower_bound, const float* initial_state,
    float* final_state, const int32_t* cu_seqlens, int32_t batch, int64_t seqlen, int32_t num_heads,
    int32_t head_dim_k, int32_t head_dim_v, int32_t num_seqs, int32_t state_transposed,
    kda_stream_t stream) {
  const int64_t seqs = cu_seqlens ? (int64_t)num_seqs : (int64_t)batch;
  if (seqs < 0 || num_heads < 0) return KDA_ERR_INVALID_ARGUMENT;
  if (seqs * (int64_t)num_heads > kStaticMaxUnits) return KDA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  kda_status_t st = static_workspace_address(&ws);
  if (st != KDA_OK) return st;
  if (cudaMemsetAsync(ws, 0, kda::kWorkspaceHeader, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KDA_ERR_CUDA;
  return kda::fwd_fused(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound, initial_state, final_state,
                        cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v, num_seqs, state_transposed,
                        static_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}
