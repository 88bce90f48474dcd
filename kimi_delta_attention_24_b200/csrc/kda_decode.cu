// Batched recurrent KDA step for decoding: a few tokens per request, each request's state read
// from and written back to a state pool.
//
// Serving keeps one recurrent state per request in a pool and advances it by one token (or a few,
// e.g. speculative tokens) per step; the vLLM PR #54859 report names this decode path beside the
// chunked prefill (summary section).  Per (request, head) unit the step is
//     for each of the request's T tokens:  S <- Diag(alpha) S,  delta = beta (v - S^T khat),
//                                          S <- S + khat delta^T,  o = scale S^T qhat
// with the in-kernel transforms of the forward pass (L2 norms of q and k, sigmoid of beta, the
// safe gate), each of which a flag can switch off for inputs the caller has already transformed.
//
// The step reads and writes the 64 KB fp32 state once per unit and does ~4 K2 flops per token on
// it, so it is bound by HBM bandwidth: one CTA of 256 threads per unit holds the whole 128 x 128
// state in registers (a 16 x 4 block per thread, loaded with coalesced 16-byte accesses: a warp
// reads one 512-byte state row per instruction), streams it in and out once, and does every
// reduction on chip (shared memory across warps for the untransposed layout, warp shuffles for
// the transposed one).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerWarp = 16;  // 8 warps x 16 state rows

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const void* g;               // bf16 raw gate, or fp32 log alpha (kFlagGatePrecomputed)
  const void* beta;            // bf16 raw beta, or fp32 beta (kFlagBetaPrecomputed)
  __nv_bfloat16* out;
  const float* A_log;
  const float* dt_bias;
  const float* state_in;       // pool [num_slots, H, 128, 128]; null: zero state
  float* state_out;            // pool [num_slots, H, 128, 128]; may alias state_in
  const int32_t* indices;      // [batch] pool slot per request (negative: skip); null: slot = request
  int64_t num_slots;
  int32_t batch, seqlen, num_heads;
  float scale, lower_bound;
  uint32_t flags;
  uint32_t* status;            // may be null
};

__device__ __forceinline__ float sigmoid_acc(float x) { return 1.0f / (1.0f + expf(-x)); }

// Transform one token of one unit into shared memory: qhat, khat, alpha (fp32 [128] each), v, beta.
// Warps 0..3 take q, k, g, v (a lane takes 4 channels); the norms are warp reductions.
__device__ __forceinline__ void load_token(const DecodeParams& p, size_t row, int h, float* s_q, float* s_k,
                                           float* s_a, float* s_v, float* s_b) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int D = kHeadDim;
  if (warp == 0 || warp == 1) {
    const __nv_bfloat16* src = (warp == 0 ? p.q : p.k) + row * D;
    const uint2 u = *reinterpret_cast<const uint2*>(src + 4 * lane);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    float x[4] = {a.x, a.y, b.x, b.y};
    float inv = 1.0f;
    if (!(p.flags & kFlagNoQkL2Norm)) {
      float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      inv = 1.0f / sqrtf(ss + kL2Eps);
    }
    float* dst = warp == 0 ? s_q : s_k;
    reinterpret_cast<float4*>(dst)[lane] = make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
  } else if (warp == 2) {
    float la[4];
    if (p.flags & kFlagGatePrecomputed) {
      const float4 t = reinterpret_cast<const float4*>(static_cast<const float*>(p.g) + row * D)[lane];
      la[0] = t.x; la[1] = t.y; la[2] = t.z; la[3] = t.w;
    } else {
      const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.g) + row * D + 4 * lane);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      const float gv[4] = {a.x, a.y, b.x, b.y};
      const float ga = expf(p.A_log[h]);
      const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
      const float dts[4] = {dt.x, dt.y, dt.z, dt.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) la[j] = p.lower_bound * sigmoid_acc(ga * (gv[j] + dts[j]));
    }
    reinterpret_cast<float4*>(s_a)[lane] = make_float4(expf(la[0]), expf(la[1]), expf(la[2]), expf(la[3]));
  } else if (warp == 3) {
    const uint2 u = *reinterpret_cast<const uint2*>(p.v + row * D + 4 * lane);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    reinterpret_cast<float4*>(s_v)[lane] = make_float4(a.x, a.y, b.x, b.y);
  } else if (warp == 4 && lane == 0) {
    *s_b = (p.flags & kFlagBetaPrecomputed) ? static_cast<const float*>(p.beta)[row]
                                            : sigmoid_acc(__bfloat162float(static_cast<const __nv_bfloat16*>(p.beta)[row]));
  }
}

// Sum over the 32 lanes of 16 values at once: after the exchange, lanes 2 i and 2 i + 1 hold the
// total of value i.
__device__ __forceinline__ float transpose_reduce16(const float (&x)[16], int lane) {
  float w8[8], w4[4], w2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) w8[j] = (b4 ? x[j + 8] : x[j]) + __shfl_xor_sync(0xffffffffu, b4 ? x[j] : x[j + 8], 16);
#pragma unroll
  for (int j = 0; j < 4; ++j) w4[j] = (b3 ? w8[j + 4] : w8[j]) + __shfl_xor_sync(0xffffffffu, b3 ? w8[j] : w8[j + 4], 8);
#pragma unroll
  for (int j = 0; j < 2; ++j) w2[j] = (b2 ? w4[j + 2] : w4[j]) + __shfl_xor_sync(0xffffffffu, b2 ? w4[j] : w4[j + 2], 4);
  float w1 = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? w2[0] : w2[1], 2);
  return w1 + __shfl_xor_sync(0xffffffffu, w1, 1);
}

// One CTA per (request, head) unit.  Thread (warp w, lane l) holds state rows 16 w .. 16 w + 15,
// columns 4 l .. 4 l + 3 of the stored matrix: S[k][v] (kTransposed = false: rows are k) or
// S^T[v][k] (kTransposed = true: rows are v).
template <bool kTransposed>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(DecodeParams p) {
  constexpr int D = kHeadDim;
  __shared__ __align__(16) float s_q[D], s_k[D], s_a[D], s_v[D];
  __shared__ __align__(16) float s_red[2][8][D];  // per-warp partial sums (untransposed layout)
  __shared__ float s_b;

  const int H = p.num_heads;
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t slot = p.indices ? (int64_t)p.indices[b] : (int64_t)b;
  if (slot < 0) return;  // a padding request: nothing read or written
  if (slot >= p.num_slots) {
    if (tid == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
    return;
  }
  const size_t soff = ((size_t)slot * H + h) * (size_t)D * D;
  const int r0 = kRowsPerWarp * warp, c0 = 4 * lane;

  float S[kRowsPerWarp][4];
  if (p.state_in) {
    const float4* src = reinterpret_cast<const float4*>(p.state_in + soff + (size_t)r0 * D + c0);
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const float4 t = __ldcs(src + i * (D / 4));
      S[i][0] = t.x; S[i][1] = t.y; S[i][2] = t.z; S[i][3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) S[i][0] = S[i][1] = S[i][2] = S[i][3] = 0.f;
  }

  for (int t = 0; t < p.seqlen; ++t) {
    const size_t row = ((size_t)b * p.seqlen + t) * H + h;
    __syncthreads();  // the previous token's shared inputs and partial sums have been read
    load_token(p, row, h, s_q, s_k, s_a, s_v, &s_b);
    __syncthreads();
    const float beta = s_b;
    if (!kTransposed) {
      // rows are k: decay, then the prediction S^T khat summed over this thread's rows and the warps
      float pr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        const float a = s_a[r0 + i], kk = s_k[r0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[i][j] *= a;
          pr[j] = fmaf(S[i][j], kk, pr[j]);
        }
      }
      reinterpret_cast<float4*>(s_red[0][warp])[lane] = make_float4(pr[0], pr[1], pr[2], pr[3]);
      __syncthreads();
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float4 t4 = reinterpret_cast<const float4*>(s_red[0][w])[lane];
        d[0] += t4.x; d[1] += t4.y; d[2] += t4.z; d[3] += t4.w;
      }
      const float4 vv = reinterpret_cast<const float4*>(s_v)[lane];
      d[0] = beta * (vv.x - d[0]);
      d[1] = beta * (vv.y - d[1]);
      d[2] = beta * (vv.z - d[2]);
      d[3] = beta * (vv.w - d[3]);
      float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        const float kk = s_k[r0 + i], qq = s_q[r0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[i][j] = fmaf(kk, d[j], S[i][j]);
          o[j] = fmaf(S[i][j], qq, o[j]);
        }
      }
      reinterpret_cast<float4*>(s_red[1][warp])[lane] = make_float4(o[0], o[1], o[2], o[3]);
      __syncthreads();
      if (warp == 0) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const float4 t4 = reinterpret_cast<const float4*>(s_red[1][w])[lane];
          acc[0] += t4.x; acc[1] += t4.y; acc[2] += t4.z; acc[3] += t4.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(p.scale * acc[0], p.scale * acc[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(p.scale * acc[2], p.scale * acc[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&lo);
        u.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(p.out + row * D + c0) = u;
      }
    } else {
      // rows are v, columns k: the sums over k run across the lanes of a warp
      const float4 a4 = reinterpret_cast<const float4*>(s_a)[lane];
      const float4 k4 = reinterpret_cast<const float4*>(s_k)[lane];
      const float4 q4 = reinterpret_cast<const float4*>(s_q)[lane];
      const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      float pr[kRowsPerWarp];
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[i][j] *= av[j];
          acc = fmaf(S[i][j], kv[j], acc);
        }
        pr[i] = acc;
      }
      const float pred = transpose_reduce16(pr, lane);           // row r0 + lane / 2
      const float dl = beta * (s_v[r0 + (lane >> 1)] - pred);
      float o[kRowsPerWarp];
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        const float di = __shfl_sync(0xffffffffu, dl, 2 * i);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[i][j] = fmaf(kv[j], di, S[i][j]);
          acc = fmaf(S[i][j], qv[j], acc);
        }
        o[i] = acc;
      }
      const float ov = transpose_reduce16(o, lane);
      if ((lane & 1) == 0) p.out[row * D + r0 + (lane >> 1)] = __float2bfloat16_rn(p.scale * ov);
    }
  }

  if (p.state_out) {
    float4* dst = reinterpret_cast<float4*>(p.state_out + soff + (size_t)r0 * D + c0);
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) __stcs(dst + i * (D / 4), make_float4(S[i][0], S[i][1], S[i][2], S[i][3]));
  }
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                          void* out, const float* A_log, const float* dt_bias, float lower_bound,
                          const float* state_in, float* state_out, const int32_t* state_indices, int32_t batch,
                          int32_t seqlen, int32_t num_heads, int64_t num_slots, int32_t state_transposed,
                          uint32_t flags, uint32_t* status, cudaStream_t stream) {
  const int64_t units = (int64_t)batch * num_heads;
  if (units == 0) return cudaSuccess;  // (seqlen 0 still runs: state_out receives state_in)
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = g;
  p.beta = beta;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.state_in = state_in;
  p.state_out = state_out;
  p.indices = state_indices;
  p.num_slots = num_slots;
  p.batch = batch;
  p.seqlen = seqlen;
  p.num_heads = num_heads;
  p.scale = scale;
  p.lower_bound = lower_bound;
  p.flags = flags;
  p.status = status;
  if (state_transposed) decode_kernel<true><<<(unsigned)units, kDecThreads, 0, stream>>>(p);
  else decode_kernel<false><<<(unsigned)units, kDecThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
