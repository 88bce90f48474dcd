// kda_fwd_static_workspace: the chunked forward pass for callers that cannot allocate device
// memory.
//
// Some callers are not allowed to allocate device memory while they run this operator: inference
// runtimes that plan every device buffer ahead of time and forbid libraries from calling
// cudaMalloc, or code that must not pay cudaMalloc's implicit device-wide synchronisation.  They
// still own their inputs and outputs, but have nowhere to put kda_fwd's workspace.  This entry
// point uses scratch that lives in the library itself: a file-scope device array, allocated once
// when the library's device code is loaded on a GPU and held by that GPU until the process exits.
// That array cannot hold the per-chunk intermediates of kda_fwd's split path (about 81 KB per
// chunk and head), so this entry point runs the fused single-kernel chunked path, which keeps
// every intermediate on chip; its only scratch is the device status word (the first 4 bytes of
// the array; the rest of its 256 bytes pads it to the status-header size the kernels expect).
//
// Limits and behaviour:
//   - At most kStaticMaxUnits (sequence, head) units per call, a fixed limit of this entry point:
//     every CTA of the fused kernel scans all N + 1 offsets of cu_seqlens to apply the
//     empty-document rule, so the limit also bounds that scan.  Larger problems are rejected with
//     KDA_ERR_WORKSPACE_TOO_SMALL after the arguments have been validated and before anything is
//     enqueued.
//   - The array's device address is looked up once per device, on the first call made with that
//     device current (cudaGetSymbolAddress).  Make that first call before any stream capture.
//   - Every call shares the one array.  Calls whose kernels overlap on the GPU race on it; issue
//     them on one stream, or otherwise order them.
//   - Each call clears the status word (stream-ordered) after validation, so a device-side time-out
//     or malformed-offsets flag recorded by an earlier call does not leak into the next; the status
//     itself is not reported to the caller by this entry point.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating library routine.
#include <mutex>

#include "kda_common.cuh"

namespace {

constexpr int32_t kStaticMaxUnits = 4096;
constexpr size_t kStaticWorkspaceBytes = kda::kWorkspaceHeader;

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
  void* ws = nullptr;
  kda_status_t st = static_workspace_address(&ws);  // host-side lookup; writes no device memory
  if (st != KDA_OK) return st;
  return kda::fwd_fused(q, k, v, g, beta, scale, out, A_log, dt_bias, lower_bound, initial_state, final_state,
                        cu_seqlens, batch, seqlen, num_heads, head_dim_k, head_dim_v, num_seqs, state_transposed,
                        static_cast<uint32_t*>(ws), kStaticMaxUnits, reinterpret_cast<cudaStream_t>(stream));
}
