// Sequence-parallel prefill (KCP, "KDA Context Parallelism": torchtitan PR #4374, the KCP remark):
// the device-side pieces.
//
// The forward pass is affine in the state a segment starts from: running a segment of tokens from
// S_in gives S_out = M S_in + B, with M (K x K) the product of the segment's per-token transitions
// (I - beta k k^T) Diag(alpha) and B (K x V) the state the segment reaches from zero.  So a sequence
// cut into R segments, one per rank, needs one exchange: every rank computes its segment's (M, B)
// (kda_segment_map, in kda_split.cu's map mode), the ranks all-gather the maps, and rank r folds the
// maps of segments 0 .. r-1 over the sequence's initial state to get the state its segment starts
// from (kda_state_affine, here), then runs the ordinary forward pass on its segment.
//
// kda_state_affine computes S_out = M S_in + B for every (sequence, head) unit: one CTA per unit,
// a 128 x 128 x 128 fp32 product tiled through shared memory (16-deep k tiles, an 8 x 8 block of
// outputs per thread).  It is a few GFLOP per fold at most, far below any other cost of the
// prefill, so it stays in fp32 on CUDA cores.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kAffThreads = 256;
constexpr int kAffK = 16;

// M [u][i][k], B [u][i][j], S [u][k][j] (or S^T [u][j][k] when transposed); S_in may be null
// (zero state: S_out = B) and may equal S_out.
__global__ void __launch_bounds__(kAffThreads) affine_kernel(const float* __restrict__ M, const float* __restrict__ B,
                                                             const float* S_in, float* S_out, int transposed) {
  constexpr int D = kHeadDim;
  __shared__ __align__(16) float sM[kAffK][D + 4];  // sM[kk][i] = M[i][k0 + kk] (padded rows)
  __shared__ __align__(16) float sS[kAffK][D];  // sS[kk][j] = S[k0 + kk][j]
  const size_t uoff = (size_t)blockIdx.x * D * D;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;  // output rows 8 ty .. + 7, columns 8 tx .. + 7
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

  if (S_in) {
    const float* Mu = M + uoff;
    const float* Su = S_in + uoff;
    for (int k0 = 0; k0 < D; k0 += kAffK) {
      // 2048 elements of each tile, 8 per thread
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int idx = tid + kAffThreads * e;  // 0 .. 2047
        {
          const int i = idx >> 4, kk = idx & 15;  // M row i, column k0 + kk
          sM[kk][i] = Mu[(size_t)i * D + k0 + kk];
        }
        if (transposed) {
          const int j = idx >> 4, kk = idx & 15;  // S^T row j, column k0 + kk
          sS[kk][j] = Su[(size_t)j * D + k0 + kk];
        } else {
          const int kk = idx >> 7, j = idx & 127;
          sS[kk][j] = Su[(size_t)(k0 + kk) * D + j];
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kAffK; ++kk) {
        const float4 m0 = *reinterpret_cast<const float4*>(&sM[kk][8 * ty]);
        const float4 m1 = *reinterpret_cast<const float4*>(&sM[kk][8 * ty + 4]);
        const float4 s0 = *reinterpret_cast<const float4*>(&sS[kk][8 * tx]);
        const float4 s1 = *reinterpret_cast<const float4*>(&sS[kk][8 * tx + 4]);
        const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(mv[a], sv[b], acc[a][b]);
      }
      __syncthreads();
    }
  }
  // every read of S_in is done (the last tile sits in shared memory): S_out may alias it
  const float* Bu = B + uoff;
  float* Ou = S_out + uoff;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = 8 * ty + a;
    const float4 b0 = *reinterpret_cast<const float4*>(Bu + (size_t)i * D + 8 * tx);
    const float4 b1 = *reinterpret_cast<const float4*>(Bu + (size_t)i * D + 8 * tx + 4);
    acc[a][0] += b0.x; acc[a][1] += b0.y; acc[a][2] += b0.z; acc[a][3] += b0.w;
    acc[a][4] += b1.x; acc[a][5] += b1.y; acc[a][6] += b1.z; acc[a][7] += b1.w;
  }
  if (!transposed) {
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      float* o = Ou + (size_t)(8 * ty + a) * D + 8 * tx;
      reinterpret_cast<float4*>(o)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      reinterpret_cast<float4*>(o)[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    }
  } else {
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      float* o = Ou + (size_t)(8 * tx + b) * D + 8 * ty;
      reinterpret_cast<float4*>(o)[0] = make_float4(acc[0][b], acc[1][b], acc[2][b], acc[3][b]);
      reinterpret_cast<float4*>(o)[1] = make_float4(acc[4][b], acc[5][b], acc[6][b], acc[7][b]);
    }
  }
}

}  // namespace

cudaError_t launch_state_affine(const float* M, const float* B, const float* S_in, float* S_out, int64_t units,
                                int32_t transposed, cudaStream_t stream) {
  if (units == 0) return cudaSuccess;
  affine_kernel<<<(unsigned)units, kAffThreads, 0, stream>>>(M, B, S_in, S_out, transposed);
  return cudaGetLastError();
}

}  // namespace kda
