// Head sizes below 128 for the chunked path, by zero padding to 128.
//
// fla's chunk_kda takes any head size (the usage example of "What CUDA Version Is Required to Use
// FlashKDA?" uses K = V = 128); the chunked kernels here are built for 128.  Padding is exact:
//   - key channels k >= K: q, k are 0 there, so the L2 norms, every Gram product, every update
//     k delta^T and every output S^T q are unchanged; those state rows start at 0 and only decay;
//   - value channels v >= V: v is 0 there, so those state columns and output columns stay 0.
// These kernels copy the inputs into 128-wide rows in the workspace (zero tail), and copy the
// 128-wide output and final state back out.  Rows are 16-byte aligned in both layouts (K and V
// are multiples of 8), and every thread moves 16 bytes.
#include "kda_common.cuh"

namespace kda {
namespace {

// dst[row][0 .. 128 * esz) <- src[row][0 .. w * esz), zero tail; esz 2 (bf16) or 4 (fp32).
__global__ void pad_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t rows, int w,
                                int esz) {
  const int chunks_out = kHeadDim * esz / 16, chunks_in = w * esz / 16;
  const int64_t total = rows * chunks_out;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / chunks_out;
    const int c = (int)(i - r * chunks_out);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c < chunks_in) v = *reinterpret_cast<const uint4*>(src + (size_t)r * chunks_in * 16 + (size_t)c * 16);
    *reinterpret_cast<uint4*>(dst + (size_t)r * chunks_out * 16 + (size_t)c * 16) = v;
  }
}

// dst[row][0 .. w * esz) <- src[row][0 .. w * esz) of 128-wide rows; nothing if *nonzero == 0.
__global__ void unpad_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t rows, int w,
                                  int esz, const int32_t* nonzero) {
  if (nonzero && *nonzero == 0) return;
  const int chunks_src = kHeadDim * esz / 16, chunks = w * esz / 16;
  const int64_t total = rows * chunks;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / chunks;
    const int c = (int)(i - r * chunks);
    *reinterpret_cast<uint4*>(dst + (size_t)r * chunks * 16 + (size_t)c * 16) =
        *reinterpret_cast<const uint4*>(src + (size_t)r * chunks_src * 16 + (size_t)c * 16);
  }
}

// A state [R][C] (R x C fp32, R = K, C = V; or R = V, C = K transposed) to / from the 128 x 128 one,
// per (sequence, head): 128 rows of 128, zero outside [R][C].
__global__ void pad_state_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t units, int R, int C) {
  const int64_t total = units * kHeadDim * (kHeadDim / 4);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i / (kHeadDim * kHeadDim / 4);
    const int rem = (int)(i - u * (kHeadDim * kHeadDim / 4));
    const int r = rem / (kHeadDim / 4), c4 = rem % (kHeadDim / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < R && 4 * c4 < C) v = *reinterpret_cast<const float4*>(src + ((size_t)u * R + r) * C + 4 * c4);
    *reinterpret_cast<float4*>(dst + ((size_t)u * kHeadDim + r) * kHeadDim + 4 * c4) = v;
  }
}

__global__ void unpad_state_kernel(const float* __restrict__ src, float* __restrict__ dst, int64_t units, int R,
                                   int C) {
  const int64_t total = units * R * (C / 4);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i / ((int64_t)R * (C / 4));
    const int rem = (int)(i - u * ((int64_t)R * (C / 4)));
    const int r = rem / (C / 4), c4 = rem % (C / 4);
    *reinterpret_cast<float4*>(dst + ((size_t)u * R + r) * C + 4 * c4) =
        *reinterpret_cast<const float4*>(src + ((size_t)u * kHeadDim + r) * kHeadDim + 4 * c4);
  }
}

unsigned grid_for(int64_t work) {
  const int64_t blocks = (work + 255) / 256;
  return (unsigned)(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_pad_rows(const void* src, void* dst, int64_t rows, int w, int esz, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  pad_rows_kernel<<<grid_for(rows * kHeadDim * esz / 16), 256, 0, stream>>>(
      static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), rows, w, esz);
  return cudaGetLastError();
}

cudaError_t launch_unpad_rows(const void* src, void* dst, int64_t rows, int w, int esz, cudaStream_t stream,
                              const int32_t* nonzero) {
  if (rows == 0) return cudaSuccess;
  unpad_rows_kernel<<<grid_for(rows * w * esz / 16), 256, 0, stream>>>(
      static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), rows, w, esz, nonzero);
  return cudaGetLastError();
}

cudaError_t launch_pad_state(const float* src, float* dst, int64_t units, int R, int C, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  pad_state_kernel<<<grid_for(units * kHeadDim * kHeadDim / 4), 256, 0, stream>>>(src, dst, units, R, C);
  return cudaGetLastError();
}

cudaError_t launch_unpad_state(const float* src, float* dst, int64_t units, int R, int C, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  unpad_state_kernel<<<grid_for(units * R * C / 4), 256, 0, stream>>>(src, dst, units, R, C);
  return cudaGetLastError();
}

}  // namespace kda
