// Backward pass of the KDA forward (gradients of every input), token by token on CUDA cores.
//
// torchtitan trains Kimi-K3 through chunk_kda, and its varlen test checks the gradient as well
// as the forward (torchtitan PR #4374, Results: test_varlen_matches_independent_documents).  For
// one token, with Stil = Diag(alpha) S_{t-1}, p = Stil^T khat, delta = beta (v - p),
// S_t = Stil + khat delta^T and o_t = scale S_t^T qhat, the reverse-mode step given dS (the
// gradient w.r.t. S_t) and do_t is
//   dS += scale qhat do^T;  dqhat = scale S_t do;  dkhat = dS delta + Stil dp;  ddelta = dS^T khat;
//   dbeta = ddelta . (v - p);  dv = beta ddelta;  dp = -beta ddelta;  dStil = dS + khat dp^T;
//   dalpha_c = sum_j dStil[c][j] S_{t-1}[c][j];  dS_{t-1} = Diag(alpha) dStil,
// followed by the derivatives of the in-kernel transforms (L2 norms, sigmoid of beta, safe gate).
//
// One CTA per (sequence, head) unit (persistent over units), 256 threads, the 128 x 128 state and
// its gradient held in registers (a 16 x 4 block of each per thread, the layout of the decode
// kernel).  The CTA first runs the forward over its sequence, storing the state at the start of
// every 64-token chunk in the workspace; then, chunk by chunk from the last, it reruns the chunk's
// forward from its checkpoint, storing the state before every token in a per-CTA scratch, and walks
// the chunk's tokens backwards.  Sums over the state's rows run through shared memory across the
// warps, sums over its columns through warp shuffles.  dA_log and dt_bias gradients are summed per
// CTA and added to the outputs (zeroed first) with one atomic per value.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdChunk = 64;
constexpr int kRows = 16;  // state rows per thread: warp w holds rows 16 w .. 16 w + 15
constexpr size_t kStateElems = (size_t)kHeadDim * kHeadDim;

struct BwdParams {
  FwdParams f;
  const __nv_bfloat16* d_out;   // [tokens, H, V]
  const float* d_final;         // [N, H, K, V] or null
  __nv_bfloat16* dq;            // [tokens, H, K]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;            // [tokens, H, V]
  __nv_bfloat16* dg;            // [tokens, H, K]
  __nv_bfloat16* dbeta;         // [tokens, H]
  float* dA_log;                // [H], zeroed before the launch
  float* ddt_bias;              // [H, K], zeroed before the launch
  float* d_initial;             // [N, H, K, V] or null
  float* ckpt;                  // (T / 64 + N + 1) x H states: chunk-start checkpoints
  float* scratch;               // gridDim.x x 64 states: the states before each token of a chunk
};

struct TokenIn {
  float q[kHeadDim], k[kHeadDim], a[kHeadDim], x[kHeadDim], sg[kHeadDim], v[kHeadDim], d[kHeadDim];
  float nq, nk, b;
};

__device__ __forceinline__ float sigmoid_acc(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st_bf16x4(__nv_bfloat16* p, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

// The transformed inputs of one token into shared memory (warps 0..5; a lane takes 4 channels).
// `full`: also q, d_out and the gate's intermediates (the backward step); otherwise only what the
// forward step reads (khat, alpha, beta, v).
__device__ __forceinline__ void load_token(const BwdParams& P, size_t row, int h, float ea, TokenIn& s, bool full) {
  const FwdParams& p = P.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int D = kHeadDim;
  if (warp == 0 || warp == 1) {
    if (warp == 0 && !full) return;
    const float4 x4 = ld_bf16x4((warp == 0 ? p.q : p.k) + row * D + 4 * lane);
    float ss = x4.x * x4.x + x4.y * x4.y + x4.z * x4.z + x4.w * x4.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float n = sqrtf(ss + kL2Eps);
    float* dst = warp == 0 ? s.q : s.k;
    reinterpret_cast<float4*>(dst)[lane] = make_float4(x4.x / n, x4.y / n, x4.z / n, x4.w / n);
    if (lane == 0) (warp == 0 ? s.nq : s.nk) = n;
  } else if (warp == 2) {
    const float4 g4 = ld_bf16x4(p.g + row * D + 4 * lane);
    const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
    const float gv[4] = {g4.x, g4.y, g4.z, g4.w}, dts[4] = {dt.x, dt.y, dt.z, dt.w};
    float xs[4], sgs[4], as[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xs[j] = ea * (gv[j] + dts[j]);
      sgs[j] = sigmoid_acc(xs[j]);
      as[j] = expf(p.lower_bound * sgs[j]);
    }
    reinterpret_cast<float4*>(s.a)[lane] = make_float4(as[0], as[1], as[2], as[3]);
    if (full) {
      reinterpret_cast<float4*>(s.x)[lane] = make_float4(xs[0], xs[1], xs[2], xs[3]);
      reinterpret_cast<float4*>(s.sg)[lane] = make_float4(sgs[0], sgs[1], sgs[2], sgs[3]);
    }
  } else if (warp == 3) {
    reinterpret_cast<float4*>(s.v)[lane] = ld_bf16x4(p.v + row * D + 4 * lane);
  } else if (warp == 4) {
    if (full) reinterpret_cast<float4*>(s.d)[lane] = ld_bf16x4(P.d_out + row * D + 4 * lane);
  } else if (warp == 5 && lane == 0) {
    s.b = sigmoid_acc(__bfloat162float(p.beta[row]));
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

// Sum over the 8 warps of each thread's 4 column partials: red[w][4 lane + j].
__device__ __forceinline__ float4 cross_warp_sum(float (*red)[kHeadDim], const float (&x)[4], int warp, int lane) {
  reinterpret_cast<float4*>(red[warp])[lane] = make_float4(x[0], x[1], x[2], x[3]);
  __syncthreads();
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const float4 t = reinterpret_cast<const float4*>(red[w])[lane];
    s.x += t.x; s.y += t.y; s.z += t.z; s.w += t.w;
  }
  return s;
}

__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(BwdParams P) {
  constexpr int D = kHeadDim;
  __shared__ __align__(16) TokenIn s;
  __shared__ __align__(16) float red[2][8][D];
  __shared__ __align__(16) float rows[3][D];  // dqhat, dkhat, dalpha of the token, per state row
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = kRows * warp, c0 = 4 * lane;
  const int64_t units = (int64_t)p.num_seqs * H;
  float* const scr = P.scratch + (size_t)blockIdx.x * kBwdChunk * kStateElems;
  const bool seqlens_ok = cta_seqlens_ok(p);

  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int n = (int)(u / H), h = (int)(u % H);
    int64_t bos, eos;
    seq_range(p, n, bos, eos);
    if (!seqlens_ok) eos = bos;
    const int64_t L = eos - bos;
    const int nch = (int)((L + kBwdChunk - 1) / kBwdChunk);
    const size_t soff = ((size_t)n * H + h) * kStateElems;
    const int64_t ck0 = bos / kBwdChunk + n;  // this sequence's first checkpoint slot
    const float ea = expf(p.A_log[h]);
    auto ck_ptr = [&](int c) { return P.ckpt + ((size_t)(ck0 + c) * H + h) * kStateElems; };

    float S[kRows][4];
    if (p.initial_state) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(p.initial_state + soff + (size_t)(r0 + i) * D + c0);
        S[i][0] = t.x; S[i][1] = t.y; S[i][2] = t.z; S[i][3] = t.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < kRows; ++i) S[i][0] = S[i][1] = S[i][2] = S[i][3] = 0.f;
    }
    auto store_state = [&](float* dst) {
#pragma unroll
      for (int i = 0; i < kRows; ++i)
        *reinterpret_cast<float4*>(dst + (size_t)(r0 + i) * D + c0) = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
    };
    auto load_state = [&](const float* src) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(src + (size_t)(r0 + i) * D + c0);
        S[i][0] = t.x; S[i][1] = t.y; S[i][2] = t.z; S[i][3] = t.w;
      }
    };
    // one forward token on the registers' state (inputs in shared memory)
    auto forward_token = [&]() {
      float pr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float a = s.a[r0 + i], kk = s.k[r0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[i][j] *= a;
          pr[j] = fmaf(S[i][j], kk, pr[j]);
        }
      }
      const float4 pp = cross_warp_sum(red[0], pr, warp, lane);
      const float4 vv = reinterpret_cast<const float4*>(s.v)[lane];
      const float d[4] = {s.b * (vv.x - pp.x), s.b * (vv.y - pp.y), s.b * (vv.z - pp.z), s.b * (vv.w - pp.w)};
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float kk = s.k[r0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) S[i][j] = fmaf(kk, d[j], S[i][j]);
      }
    };

    // ---------------------------------------------------------------- forward with checkpoints
    for (int c = 0; c < nch; ++c) {
      store_state(ck_ptr(c));
      const int64_t t_end = min(bos + (int64_t)(c + 1) * kBwdChunk, eos);
      for (int64_t t = bos + (int64_t)c * kBwdChunk; t < t_end; ++t) {
        __syncthreads();
        load_token(P, (size_t)t * H + h, h, ea, s, false);
        __syncthreads();
        forward_token();
      }
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
    float dS[kRows][4];
    if (P.d_final) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(P.d_final + soff + (size_t)(r0 + i) * D + c0);
        dS[i][0] = t.x; dS[i][1] = t.y; dS[i][2] = t.z; dS[i][3] = t.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < kRows; ++i) dS[i][0] = dS[i][1] = dS[i][2] = dS[i][3] = 0.f;
    }
    float ddt[4] = {0.f, 0.f, 0.f, 0.f}, dA = 0.f;  // warp 2's gate-parameter sums (channels 4 lane ..)

    for (int c = nch - 1; c >= 0; --c) {
      const int64_t t_begin = bos + (int64_t)c * kBwdChunk;
      const int len = (int)min((int64_t)kBwdChunk, eos - t_begin);
      // rerun the chunk's forward from its checkpoint, keeping the state before each token
      load_state(ck_ptr(c));
      for (int i = 0; i < len; ++i) {
        store_state(scr + (size_t)i * kStateElems);
        __syncthreads();
        load_token(P, (size_t)(t_begin + i) * H + h, h, ea, s, false);
        __syncthreads();
        forward_token();
      }
      // the chunk's tokens backwards
      for (int i = len - 1; i >= 0; --i) {
        const size_t row = (size_t)(t_begin + i) * H + h;
        __syncthreads();
        load_token(P, row, h, ea, s, true);
        load_state(scr + (size_t)i * kStateElems);  // S_{t-1}: written by this thread above
        __syncthreads();
        const float b = s.b, scale = p.scale;
        // p = Stil^T khat
        float pr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) {
          const float a = s.a[r0 + ii], kk = s.k[r0 + ii];
#pragma unroll
          for (int j = 0; j < 4; ++j) pr[j] = fmaf(a * S[ii][j], kk, pr[j]);
        }
        const float4 pp = cross_warp_sum(red[0], pr, warp, lane);
        const float4 vv = reinterpret_cast<const float4*>(s.v)[lane];
        const float4 do4 = reinterpret_cast<const float4*>(s.d)[lane];
        const float pj[4] = {pp.x, pp.y, pp.z, pp.w}, vj[4] = {vv.x, vv.y, vv.z, vv.w};
        const float doj[4] = {do4.x, do4.y, do4.z, do4.w};
        float dl[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) dl[j] = b * (vj[j] - pj[j]);
        // dS += scale qhat do^T; dqhat rows = scale S_t do; ddelta = dS^T khat
        float rq[kRows], pd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) {
          const float a = s.a[r0 + ii], kk = s.k[r0 + ii], qq = s.q[r0 + ii];
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float st = fmaf(kk, dl[j], a * S[ii][j]);  // S_t
            acc = fmaf(st, doj[j], acc);
            dS[ii][j] = fmaf(scale * qq, doj[j], dS[ii][j]);
            pd[j] = fmaf(dS[ii][j], kk, pd[j]);
          }
          rq[ii] = scale * acc;
        }
        const float4 dd = cross_warp_sum(red[1], pd, warp, lane);
        const float ddl[4] = {dd.x, dd.y, dd.z, dd.w};
        float dp[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) dp[j] = -b * ddl[j];
        if (warp == 0) {
          // dv, and dbeta through the sigmoid
          st_bf16x4(P.dv + row * D + c0, b * ddl[0], b * ddl[1], b * ddl[2], b * ddl[3]);
          float db = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) db = fmaf(ddl[j], vj[j] - pj[j], db);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
          if (lane == 0) P.dbeta[row] = __float2bfloat16_rn(db * b * (1.f - b));
        }
        // dkhat = dS delta + Stil dp;  dStil = dS + khat dp^T;  dalpha;  dS <- Diag(alpha) dStil
        float rk[kRows], ra[kRows];
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) {
          const float a = s.a[r0 + ii], kk = s.k[r0 + ii];
          float ak = 0.f, aa = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float st = a * S[ii][j];
            ak = fmaf(dS[ii][j], dl[j], ak);
            ak = fmaf(st, dp[j], ak);
            const float dst = fmaf(kk, dp[j], dS[ii][j]);
            aa = fmaf(dst, S[ii][j], aa);
            dS[ii][j] = a * dst;
          }
          rk[ii] = ak;
          ra[ii] = aa;
        }
        const float tq = transpose_reduce16(rq, lane);
        const float tk = transpose_reduce16(rk, lane);
        const float ta = transpose_reduce16(ra, lane);
        if ((lane & 1) == 0) {
          rows[0][r0 + (lane >> 1)] = tq;
          rows[1][r0 + (lane >> 1)] = tk;
          rows[2][r0 + (lane >> 1)] = ta;
        }
        __syncthreads();
        // back through the transforms: warp 0 q, warp 1 k, warp 2 the gate
        if (warp == 0 || warp == 1) {
          const float* xh = warp == 0 ? s.q : s.k;
          const float4 x4 = reinterpret_cast<const float4*>(xh)[lane];
          const float4 g4 = reinterpret_cast<const float4*>(rows[warp])[lane];
          float dot = x4.x * g4.x + x4.y * g4.y + x4.z * g4.z + x4.w * g4.w;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          const float inv = 1.f / (warp == 0 ? s.nq : s.nk);
          st_bf16x4((warp == 0 ? P.dq : P.dk) + row * D + c0, (g4.x - x4.x * dot) * inv, (g4.y - x4.y * dot) * inv,
                    (g4.z - x4.z * dot) * inv, (g4.w - x4.w * dot) * inv);
        } else if (warp == 2) {
          const float4 da4 = reinterpret_cast<const float4*>(rows[2])[lane];
          const float4 a4 = reinterpret_cast<const float4*>(s.a)[lane];
          const float4 x4 = reinterpret_cast<const float4*>(s.x)[lane];
          const float4 s4 = reinterpret_cast<const float4*>(s.sg)[lane];
          const float dal[4] = {da4.x, da4.y, da4.z, da4.w}, al[4] = {a4.x, a4.y, a4.z, a4.w};
          const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
          float dg[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float dx = dal[j] * al[j] * p.lower_bound * sv[j] * (1.f - sv[j]);
            dg[j] = dx * ea;
            ddt[j] += dg[j];
            dA = fmaf(dx, xv[j], dA);
          }
          st_bf16x4(P.dg + row * D + c0, dg[0], dg[1], dg[2], dg[3]);
        }
      }
    }
    if (P.d_initial) {
#pragma unroll
      for (int i = 0; i < kRows; ++i)
        *reinterpret_cast<float4*>(P.d_initial + soff + (size_t)(r0 + i) * D + c0) =
            make_float4(dS[i][0], dS[i][1], dS[i][2], dS[i][3]);
    }
    if (warp == 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) atomicAdd(P.ddt_bias + (size_t)h * D + c0 + j, ddt[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dA += __shfl_xor_sync(0xffffffffu, dA, o);
      if (lane == 0) atomicAdd(P.dA_log + h, dA);
    }
  }
}

}  // namespace

// At most this many persistent CTAs (one per SM; more SMs than this are left to other work), so the
// workspace size depends only on the problem's sizes.
constexpr int64_t kBwdMaxCtas = 256;

size_t bwd_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t t = total_tokens > 0 ? total_tokens : 0, n = num_seqs > 0 ? num_seqs : 0;
  const int64_t hh = num_heads > 0 ? num_heads : 0;
  const int64_t slots = t / kBwdChunk + n + 1;
  const int64_t units = n * hh;
  const int64_t ctas = units < kBwdMaxCtas ? units : kBwdMaxCtas;
  return ((size_t)slots * hh + (size_t)ctas * kBwdChunk) * kStateElems * sizeof(float);
}

cudaError_t launch_bwd(const FwdParams& f, const __nv_bfloat16* d_out, const float* d_final, __nv_bfloat16* dq,
                       __nv_bfloat16* dk, __nv_bfloat16* dv, __nv_bfloat16* dg, __nv_bfloat16* dbeta, float* dA_log,
                       float* ddt_bias, float* d_initial, void* workspace, cudaStream_t stream) {
  const int64_t units = (int64_t)f.num_seqs * f.num_heads;
  int dev = 0, sms = 0;
  cudaError_t qe = cudaGetDevice(&dev);
  if (qe == cudaSuccess) qe = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (qe != cudaSuccess) return qe;
  cudaError_t e = cudaMemsetAsync(dA_log, 0, sizeof(float) * f.num_heads, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ddt_bias, 0, sizeof(float) * f.num_heads * kHeadDim, stream);
  if (e != cudaSuccess || units == 0) return e;
  const int64_t tokens = f.cu_seqlens ? f.seqlen : f.seqlen * f.num_seqs;
  const int64_t slots = tokens / kBwdChunk + f.num_seqs + 1;
  BwdParams P;
  P.f = f;
  P.d_out = d_out;
  P.d_final = d_final;
  P.dq = dq;
  P.dk = dk;
  P.dv = dv;
  P.dg = dg;
  P.dbeta = dbeta;
  P.dA_log = dA_log;
  P.ddt_bias = ddt_bias;
  P.d_initial = d_initial;
  P.ckpt = static_cast<float*>(workspace);
  P.scratch = P.ckpt + (size_t)slots * f.num_heads * kStateElems;
  int64_t grid = units < sms ? units : sms;
  if (grid > kBwdMaxCtas) grid = kBwdMaxCtas;
  bwd_kernel<<<(unsigned)grid, kBwdThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace kda
