// Device and host helpers shared by the chunked KDA kernels (fused and split paths).
#pragma once

#include <cuda.h>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {

constexpr int kChunk = 64;                          // chunk length C
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // bound of every device-side wait
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
}
// x as a bf16 pair hi = bf16(x), lo = bf16(x - hi), two values at a time.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
__device__ __forceinline__ float fast_sigmoid(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ uint2 ldg_u2(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const uint2*>(p));
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// First row of the Gram right operand R_I inside its tile: 0, 16, 48, 96 (R_I has 16 (I+1) rows).
__host__ __device__ constexpr uint32_t row_off(int I) { return 8u * I * (I + 1); }

// Bounded wait on a phase.  Returns false on time-out (after raising *abort and the status word)
// or once *abort is up.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             uint32_t* status, uint64_t limit_ns = kWaitLimitNs) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    // sleeps until the phase completes (or 20 us pass), so a waiting thread takes no issue slots
    if (sm100::mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if ((n & 7) == 0) {
      if (*abort) return false;
      if (sm100::globaltimer_ns() - t0 > limit_ns) {
        *abort = 1;
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Bounded wait that polls without suspending (lowest wake-up latency, for the few threads on a
// critical path).  Same contract as bounded_wait.
__device__ __forceinline__ bool bounded_spin(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             uint32_t* status) {
  if (sm100::mbar_test(bar, parity)) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (sm100::mbar_test(bar, parity)) return true;
    if ((n & 255) == 0) {
      if (*abort) return false;
      if (sm100::globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// [tokens, H, 128] bf16 viewed as 3-D (channel, head, token); box 64 channels x 1 head x 64 tokens,
// 128-byte swizzle, zero fill past the last token.
inline bool make_token_map(CUtensorMap* map, const void* base, int64_t tokens, int H) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)(tokens > 0 ? tokens : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kChunk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [tokens, H, 128] fp32 viewed as 3-D (channel, head, token); box 64 channels x 1 head x 64 tokens,
// no swizzle (used only to pull tiles into L2 ahead of plain loads).
inline bool make_token_map_f32(CUtensorMap* map, const void* base, int64_t tokens, int H) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)(tokens > 0 ? tokens : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 4, (cuuint64_t)H * kHeadDim * 4};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kChunk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Number of SMs of the current device (looked up once per device); 0 on error.
inline int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = v;
  }
  return cache[dev];
}

// Sets the dynamic shared-memory limit of `kernel` once per device.
template <typename Kernel>
inline cudaError_t set_smem_once(Kernel kernel, uint32_t bytes, bool (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace kda
