// Token-serial KDA forward on CUDA cores.
//
// The recurrence of Kimi Delta Attention (the operator FlashKDA `fwd` and fla `chunk_kda`
// compute; shapes per "What CUDA Version Is Required to Use FlashKDA?", Usage Examples):
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t
// evaluated one token at a time.  The columns of S evolve independently (the update acts on the
// K side only), so a CTA owns one (sequence, head) unit and a slice of kVSlice state columns,
// one column per thread, kept in 128 fp32 registers.  Inputs are staged in shared memory a tile
// of kTile tokens at a time; the L2 norms, the sigmoid of beta and the safe gate are computed
// for the whole tile first (one warp per token row, four channels per lane), then each thread
// walks the tile's tokens over its column.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kTile = 16;
constexpr int kVSlice = 64;

__device__ __forceinline__ float sigmoidf_acc(float x) { return 1.0f / (1.0f + expf(-x)); }

__global__ void __launch_bounds__(kVSlice) recurrent_kernel(FwdParams p) {
  constexpr int K = kHeadDim, V = kHeadDim;
  __shared__ __align__(16) float s_q[kTile][K];
  __shared__ __align__(16) float s_k[kTile][K];
  __shared__ __align__(16) float s_a[kTile][K];
  __shared__ __align__(16) float s_v[kTile][kVSlice];
  __shared__ float s_b[kTile];

  const int H = p.num_heads;
  const int unit = blockIdx.x;
  const int n = unit / H, h = unit % H;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kVSlice / 32;
  const int col = blockIdx.y * kVSlice + tid;

  int64_t bos, eos;
  seq_range(p, n, bos, eos);
  if (tid == 0 && h == 0 && blockIdx.y == 0 && p.status && !seq_entries_ok(p, n))
    atomicOr(p.status, kStatusBadSeqlens);
  // offsets out of order: every document is empty, as in the chunked paths
  if (!cta_seqlens_ok(p)) eos = bos;

  const size_t state_off = ((size_t)n * H + h) * (size_t)K * V;
  float S[K];
#pragma unroll
  for (int c = 0; c < K; ++c) {
    float s = 0.f;
    if (p.initial_state) {
      s = p.state_transposed ? p.initial_state[state_off + (size_t)col * K + c]
                             : p.initial_state[state_off + (size_t)c * V + col];
    }
    S[c] = s;
  }

  const float gate_a = expf(p.A_log[h]);
  const float* dtb = p.dt_bias + (size_t)h * K;
  float4 dt4 = reinterpret_cast<const float4*>(dtb)[lane];

  for (int64_t t0 = bos; t0 < eos; t0 += kTile) {
    const int nt = (int)((eos - t0) < (int64_t)kTile ? (eos - t0) : (int64_t)kTile);
    __syncthreads();
    // Phase A: transform the tile (one warp per token row, 4 channels per lane).
    for (int i = warp; i < nt; i += kWarps) {
      const size_t row = (size_t)(t0 + i) * H + h;
      const uint2 qr = reinterpret_cast<const uint2*>(p.q + row * K)[lane];
      const uint2 kr = reinterpret_cast<const uint2*>(p.k + row * K)[lane];
      const uint2 gr = reinterpret_cast<const uint2*>(p.g + row * K)[lane];
      float qf[4], kf[4], gf[4];
      {
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qr);
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gr);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float2 a = __bfloat1622float2(q2[j]);
          float2 b = __bfloat1622float2(k2[j]);
          float2 c = __bfloat1622float2(g2[j]);
          qf[2 * j] = a.x; qf[2 * j + 1] = a.y;
          kf[2 * j] = b.x; kf[2 * j + 1] = b.y;
          gf[2 * j] = c.x; gf[2 * j + 1] = c.y;
        }
      }
      float sq = 0.f, sk = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sq = fmaf(qf[j], qf[j], sq);
        sk = fmaf(kf[j], kf[j], sk);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
      }
      const float iq = 1.0f / sqrtf(sq + kL2Eps);
      const float ik = 1.0f / sqrtf(sk + kL2Eps);
      const float dts[4] = {dt4.x, dt4.y, dt4.z, dt4.w};
      float4 qo, ko, ao;
      float* qop = &qo.x;
      float* kop = &ko.x;
      float* aop = &ao.x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qop[j] = qf[j] * iq;
        kop[j] = kf[j] * ik;
        aop[j] = expf(p.lower_bound * sigmoidf_acc(gate_a * (gf[j] + dts[j])));
      }
      reinterpret_cast<float4*>(s_q[i])[lane] = qo;
      reinterpret_cast<float4*>(s_k[i])[lane] = ko;
      reinterpret_cast<float4*>(s_a[i])[lane] = ao;
      if (lane == 0) s_b[i] = sigmoidf_acc(__bfloat162float(p.beta[row]));
    }
    for (int i = 0; i < nt; ++i) {
      const size_t row = (size_t)(t0 + i) * H + h;
      s_v[i][tid] = __bfloat162float(p.v[row * V + col]);
    }
    __syncthreads();
    // Phase B: the recurrence over the tile's tokens, one state column per thread.
    for (int i = 0; i < nt; ++i) {
      float pred = 0.f;
#pragma unroll
      for (int c = 0; c < K; c += 4) {
        const float4 a = *reinterpret_cast<const float4*>(&s_a[i][c]);
        const float4 kk = *reinterpret_cast<const float4*>(&s_k[i][c]);
        S[c] *= a.x; S[c + 1] *= a.y; S[c + 2] *= a.z; S[c + 3] *= a.w;
        pred = fmaf(S[c], kk.x, pred);
        pred = fmaf(S[c + 1], kk.y, pred);
        pred = fmaf(S[c + 2], kk.z, pred);
        pred = fmaf(S[c + 3], kk.w, pred);
      }
      const float d = s_b[i] * (s_v[i][tid] - pred);
      float o = 0.f;
#pragma unroll
      for (int c = 0; c < K; c += 4) {
        const float4 kk = *reinterpret_cast<const float4*>(&s_k[i][c]);
        const float4 qq = *reinterpret_cast<const float4*>(&s_q[i][c]);
        S[c] = fmaf(kk.x, d, S[c]);
        S[c + 1] = fmaf(kk.y, d, S[c + 1]);
        S[c + 2] = fmaf(kk.z, d, S[c + 2]);
        S[c + 3] = fmaf(kk.w, d, S[c + 3]);
        o = fmaf(S[c], qq.x, o);
        o = fmaf(S[c + 1], qq.y, o);
        o = fmaf(S[c + 2], qq.z, o);
        o = fmaf(S[c + 3], qq.w, o);
      }
      const size_t row = (size_t)(t0 + i) * H + h;
      p.out[row * V + col] = __float2bfloat16_rn(p.scale * o);
    }
  }

  if (p.final_state) {
#pragma unroll
    for (int c = 0; c < K; ++c) {
      if (p.state_transposed) p.final_state[state_off + (size_t)col * K + c] = S[c];
      else p.final_state[state_off + (size_t)c * V + col] = S[c];
    }
  }
}

}  // namespace

cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream) {
  const int64_t units = (int64_t)p.num_seqs * p.num_heads;
  if (units == 0) return cudaSuccess;
  dim3 grid((unsigned)units, kHeadDim / kVSlice);
  recurrent_kernel<<<grid, kVSlice, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
