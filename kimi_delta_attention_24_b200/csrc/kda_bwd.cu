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
// The columns of the state evolve independently, so one (sequence, head) unit is split over four
// CTAs of 32 state columns each (persistent over (unit, slice) pairs, two CTAs per SM, 256
// threads).  Inside a CTA, warp w owns 4 columns over all 128 rows and lane l rows 4 l .. 4 l + 3,
// so each thread holds a 4 x 4 block of the state and of its gradient, and the sums over rows that
// the token chain needs (the prediction S^T khat and the delta gradient dS^T khat) are warp
// shuffles: a warp runs the token recurrence on its columns without waiting for the others.  A CTA
// first runs the forward over its sequence, storing its slice at the start of every 32-token chunk
// in the workspace; then, chunk by chunk from the last, it reruns the chunk's forward from its
// checkpoint, storing the slice before every token in a per-CTA scratch, and walks the chunk's tokens
// backwards.  Each chunk's inputs are transformed once (norms, gate, sigmoid) into shared memory,
// and the next token's scratch state is fetched during the current one.  What sums over columns
// (dqhat, dkhat, dalpha per channel, dbeta) is added over the CTA's warps through shared memory (one
// barrier per token) and written per slice; a second kernel adds the slices, applies the derivatives
// of the L2 norms, the gate and the sigmoid, and adds the dA_log / dt_bias sums with one atomic per
// value per CTA (the outputs are zeroed first).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdChunk = 64;  // tokens per checkpoint: the forward's chunk, whose start states it can store
constexpr int kStage = 32;     // tokens whose transformed inputs are staged in shared memory at once
constexpr int kSlice = 32;  // state columns per CTA (4 per warp)
constexpr int kSlices = kHeadDim / kSlice;
constexpr size_t kStateElems = (size_t)kHeadDim * kHeadDim;
constexpr size_t kSliceElems = (size_t)kHeadDim * kSlice;

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
  const float* ckpt_in;         // the forward's checkpoints, or null (then computed into ckpt)
  float* ckpt;                  // (T / 64 + N + 1) x H states: chunk-start checkpoints, S^T[v][k]
  float* scratch;               // gridDim.x x 64 slices: the states before each token of a chunk
  float* part;                  // per slice: dqhat, dkhat, dalpha [tokens, H, K]; then dbeta [slice][tokens, H]
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

// Sum over the 32 lanes of a warp, every lane getting the totals.
__device__ __forceinline__ void warp_allsum4(float (&x)[4]) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int j = 0; j < 4; ++j) x[j] += __shfl_xor_sync(0xffffffffu, x[j], o);
}
__device__ __forceinline__ float warp_allsum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Up to kStage tokens' transformed inputs, staged in shared memory (each warp transforms every eighth
// token) and read by all warps: khat, qhat and alpha per channel, v and d_out on the slice's columns,
// beta.
struct ChunkIn {
  float k[kStage][kHeadDim];
  float q[kStage][kHeadDim];
  float a[kStage][kHeadDim];
  float v[kStage][kSlice];
  float d[kStage][kSlice];
  float b[kStage];
};

__device__ __forceinline__ void stage_chunk(const BwdParams& P, ChunkIn& s, int64_t t_begin, int len, int h,
                                            int scol0, float ea, float4 dt, bool full) {
  const FwdParams& p = P.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.num_heads;
  constexpr int D = kHeadDim;
  const float dts[4] = {dt.x, dt.y, dt.z, dt.w};
  for (int i = warp; i < len; i += kBwdThreads / 32) {
    const size_t row = (size_t)(t_begin + i) * H + h;
    const float4 k4 = ld_bf16x4(p.k + row * D + 4 * lane);
    const float4 g4 = ld_bf16x4(p.g + row * D + 4 * lane);
    const float kv[4] = {k4.x, k4.y, k4.z, k4.w}, gv[4] = {g4.x, g4.y, g4.z, g4.w};
    const float nk = sqrtf(warp_allsum(kv[0] * kv[0] + kv[1] * kv[1] + kv[2] * kv[2] + kv[3] * kv[3]) + kL2Eps);
    float av[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) av[j] = expf(p.lower_bound * sigmoid_acc(ea * (gv[j] + dts[j])));
    reinterpret_cast<float4*>(s.k[i])[lane] = make_float4(kv[0] / nk, kv[1] / nk, kv[2] / nk, kv[3] / nk);
    reinterpret_cast<float4*>(s.a[i])[lane] = make_float4(av[0], av[1], av[2], av[3]);
    if (lane < kSlice / 4) reinterpret_cast<float4*>(s.v[i])[lane] = ld_bf16x4(p.v + row * D + scol0 + 4 * lane);
    if (lane == 0) s.b[i] = sigmoid_acc(__bfloat162float(p.beta[row]));
    if (full) {
      const float4 q4 = ld_bf16x4(p.q + row * D + 4 * lane);
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      const float nq = sqrtf(warp_allsum(qv[0] * qv[0] + qv[1] * qv[1] + qv[2] * qv[2] + qv[3] * qv[3]) + kL2Eps);
      reinterpret_cast<float4*>(s.q[i])[lane] = make_float4(qv[0] / nq, qv[1] / nq, qv[2] / nq, qv[3] / nq);
      if (lane < kSlice / 4) reinterpret_cast<float4*>(s.d[i])[lane] = ld_bf16x4(P.d_out + row * D + scol0 + 4 * lane);
    }
  }
}

// One CTA per (unit, slice of 32 state columns); warp w owns columns 4 w .. 4 w + 3 of the slice over
// all 128 rows, lane l rows 4 l .. 4 l + 3 (a 4 x 4 block of the state and of its gradient per
// thread).  The columns of the state evolve independently, so every warp runs the token recurrence
// on its own columns: the sums over rows (the prediction and the delta gradient) are warp shuffles,
// and the token chain needs no barrier of the CTA.  Each chunk's inputs are transformed once into
// shared memory.  What sums over columns (dqhat, dkhat, dalpha per row, dbeta) is summed over the
// CTA's warps through shared memory (one barrier per token) and written per slice for
// bwd_finish_kernel.  Checkpoints and the per-token scratch are stored per thread (16 contiguous
// floats), since every thread reads back only what it wrote.
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_kernel(BwdParams P) {
  constexpr int D = kHeadDim;
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  ChunkIn& s = *reinterpret_cast<ChunkIn*>(bwd_smem);
  float (*part)[8][3][D] = reinterpret_cast<float (*)[8][3][D]>(bwd_smem + sizeof(ChunkIn));  // [buffer][warp]
  float (*part_beta)[8] = reinterpret_cast<float (*)[8]>(bwd_smem + sizeof(ChunkIn) + 2 * 8 * 3 * D * sizeof(float));
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t units = (int64_t)p.num_seqs * H;
  const int64_t work = units * kSlices;
  float* const scr = P.scratch + (size_t)blockIdx.x * kBwdChunk * kSliceElems;
  const bool seqlens_ok = cta_seqlens_ok(p);
  const int64_t rows_total = (p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs) * H;

  for (int64_t wi = blockIdx.x; wi < work; wi += gridDim.x) {
    const int64_t u = wi / kSlices;
    const int sl = (int)(wi - u * kSlices);
    const int n = (int)(u / H), h = (int)(u % H);
    const int scol0 = sl * kSlice;         // the slice's first state column
    const int col0 = scol0 + 4 * warp;     // this warp's first state column (v)
    int64_t bos, eos;
    seq_range(p, n, bos, eos);
    if (!seqlens_ok) eos = bos;
    const int64_t L = eos - bos;
    const int nch = (int)((L + kBwdChunk - 1) / kBwdChunk);
    const size_t soff = ((size_t)n * H + h) * kStateElems;
    const int64_t ck0 = bos / kBwdChunk + n;  // this sequence's first checkpoint slot
    const float ea = expf(p.A_log[h]);
    const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
    float S[4][4];  // S[4 lane + i][col0 + j]
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p.initial_state) t = *reinterpret_cast<const float4*>(p.initial_state + soff + (size_t)(4 * lane + i) * D + col0);
      S[i][0] = t.x; S[i][1] = t.y; S[i][2] = t.z; S[i][3] = t.w;
    }
    // checkpoint of chunk c: the whole state, transposed (S^T[v][k]), as the forward stores it
    const float* ck_base = P.ckpt_in ? P.ckpt_in : P.ckpt;
    auto ck_ptr = [&](int c) { return ck_base + ((size_t)(ck0 + c) * H + h) * kStateElems; };
    auto load_ckpt = [&](const float* base) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 t = *reinterpret_cast<const float4*>(base + (size_t)(col0 + j) * D + 4 * lane);
        S[0][j] = t.x; S[1][j] = t.y; S[2][j] = t.z; S[3][j] = t.w;
      }
    };
    auto store_ckpt = [&](float* base) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<float4*>(base + (size_t)(col0 + j) * D + 4 * lane) = make_float4(S[0][j], S[1][j], S[2][j], S[3][j]);
    };
    float* const part_q = P.part + (size_t)sl * 3 * rows_total * D;
    float* const part_b = P.part + (size_t)kSlices * 3 * rows_total * D + (size_t)sl * rows_total;

    auto store_state = [&](float* base) {
      float4* dst = reinterpret_cast<float4*>(base + (size_t)tid * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
    };
    auto load_state = [&](const float* base) {
      const float4* src = reinterpret_cast<const float4*>(base + (size_t)tid * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = src[i];
        S[i][0] = t.x; S[i][1] = t.y; S[i][2] = t.z; S[i][3] = t.w;
      }
    };
    // the chunk's token i, this thread's rows and the warp's columns
    auto row4 = [&](const float (*m)[D], int i) {
      const float4 t = reinterpret_cast<const float4*>(m[i])[lane];
      return t;
    };
    auto forward_token = [&](int i) {
      const float4 a4 = row4(s.a, i), k4 = row4(s.k, i);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
      const float4 v4 = reinterpret_cast<const float4*>(s.v[i])[warp];
      const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
      const float b = s.b[i];
      float pr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[r][j] *= av[r];
          pr[j] = fmaf(S[r][j], kv[r], pr[j]);
        }
      warp_allsum4(pr);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float d = b * (vv[j] - pr[j]);
#pragma unroll
        for (int r = 0; r < 4; ++r) S[r][j] = fmaf(kv[r], d, S[r][j]);
      }
    };

    // ---------------------------------------------------------------- forward with checkpoints
    // (only without the forward's checkpoints; each CTA writes its own 32 columns of them)
    if (!P.ckpt_in) {
      for (int c = 0; c < nch; ++c) {
        const int64_t t_begin = bos + (int64_t)c * kBwdChunk;
        const int len = (int)min((int64_t)kBwdChunk, eos - t_begin);
        store_ckpt(P.ckpt + ((size_t)(ck0 + c) * H + h) * kStateElems);
        for (int h0 = 0; h0 < len; h0 += kStage) {
          const int hl = min(kStage, len - h0);
          __syncthreads();  // the previously staged inputs are read
          stage_chunk(P, s, t_begin + h0, hl, h, scol0, ea, dt, false);
          __syncthreads();
          for (int i = 0; i < hl; ++i) forward_token(i);
        }
      }
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
    float dS[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
      if (P.d_final) t = *reinterpret_cast<const float4*>(P.d_final + soff + (size_t)(4 * lane + i) * D + col0);
      dS[i][0] = t.x; dS[i][1] = t.y; dS[i][2] = t.z; dS[i][3] = t.w;
    }
    int buf = 0;
    // one backward token: chunk token i (staged at si); S holds its S_{t-1}
    auto backward_token = [&](int64_t t_begin, int i, int si) {
        const size_t row = (size_t)(t_begin + i) * H + h;
        const float4 a4 = row4(s.a, si), k4 = row4(s.k, si), q4 = row4(s.q, si);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
        const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
        const float4 v4 = reinterpret_cast<const float4*>(s.v[si])[warp];
        const float4 d4 = reinterpret_cast<const float4*>(s.d[si])[warp];
        const float vv[4] = {v4.x, v4.y, v4.z, v4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
        const float b = s.b[si], scale = p.scale;
        // p = Stil^T khat (columns), delta
        float pj[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int j = 0; j < 4; ++j) pj[j] = fmaf(av[r] * S[r][j], kv[r], pj[j]);
        warp_allsum4(pj);
        float dl[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) dl[j] = b * (vv[j] - pj[j]);
        // dS += scale qhat do^T;  dqhat rows = scale S_t do;  ddelta = dS^T khat
        float rq[4], dd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc = fmaf(fmaf(kv[r], dl[j], av[r] * S[r][j]), dv[j], acc);
            dS[r][j] = fmaf(scale * qv[r], dv[j], dS[r][j]);
            dd[j] = fmaf(dS[r][j], kv[r], dd[j]);
          }
          rq[r] = scale * acc;
        }
        warp_allsum4(dd);
        float dp[4], db = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dp[j] = -b * dd[j];
          db = fmaf(dd[j], vv[j] - pj[j], db);
        }
        if (lane == 0) st_bf16x4(P.dv + row * D + col0, b * dd[0], b * dd[1], b * dd[2], b * dd[3]);
        // dkhat = dS delta + Stil dp;  dStil = dS + khat dp^T;  dalpha;  dS <- Diag(alpha) dStil
        float rk[4], ra[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float ak = 0.f, aa = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ak = fmaf(dS[r][j], dl[j], ak);
            ak = fmaf(av[r] * S[r][j], dp[j], ak);
            const float dst = fmaf(kv[r], dp[j], dS[r][j]);
            aa = fmaf(dst, S[r][j], aa);
            dS[r][j] = av[r] * dst;
          }
          rk[r] = ak;
          ra[r] = aa;
        }
        if (i > 0) load_state(scr + (size_t)(i - 1) * kSliceElems);  // the next token's S_{t-1}
        // the warps' row partials through shared memory, summed over the slice's 32 columns
        reinterpret_cast<float4*>(part[buf][warp][0])[lane] = make_float4(rq[0], rq[1], rq[2], rq[3]);
        reinterpret_cast<float4*>(part[buf][warp][1])[lane] = make_float4(rk[0], rk[1], rk[2], rk[3]);
        reinterpret_cast<float4*>(part[buf][warp][2])[lane] = make_float4(ra[0], ra[1], ra[2], ra[3]);
        if (lane == 0) part_beta[buf][warp] = db;
        __syncthreads();
        // 384 row sums: thread t sums entries t and t + 256 (of 3 x 128)
        for (int e = tid; e < 3 * D; e += kBwdThreads) {
          const int which = e / D, r = e % D;
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) acc += part[buf][w][which][r];
          part_q[(size_t)which * rows_total * D + row * D + r] = acc;
        }
        if (tid == 0) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) acc += part_beta[buf][w];
          part_b[row] = acc;
        }
        buf ^= 1;  // the next token writes the other buffer; this one is read until the next barrier
    };
    for (int c = nch - 1; c >= 0; --c) {
      const int64_t t_begin = bos + (int64_t)c * kBwdChunk;
      const int len = (int)min((int64_t)kBwdChunk, eos - t_begin);
      const int len0 = min(kStage, len);  // tokens of the first staged half
      // rerun the chunk's forward from its checkpoint, keeping the state before each token; the
      // second half is staged with what the backward needs and walked backwards right away
      load_ckpt(ck_ptr(c));
      __syncthreads();  // the previously staged inputs and partials are read
      stage_chunk(P, s, t_begin, len0, h, scol0, ea, dt, false);
      __syncthreads();
      for (int i = 0; i < len0; ++i) {
        store_state(scr + (size_t)i * kSliceElems);
        forward_token(i);
      }
      if (len > kStage) {
        __syncthreads();
        stage_chunk(P, s, t_begin + kStage, len - kStage, h, scol0, ea, dt, true);
        __syncthreads();
        for (int i = kStage; i < len; ++i) {
          store_state(scr + (size_t)i * kSliceElems);
          forward_token(i - kStage);
        }
        load_state(scr + (size_t)(len - 1) * kSliceElems);
        for (int i = len - 1; i >= kStage; --i) backward_token(t_begin, i, i - kStage);
      } else {
        load_state(scr + (size_t)(len - 1) * kSliceElems);
      }
      // the first half backwards (S holds the state before its last token)
      __syncthreads();
      stage_chunk(P, s, t_begin, len0, h, scol0, ea, dt, true);
      __syncthreads();
      for (int i = len0 - 1; i >= 0; --i) backward_token(t_begin, i, i);
    }
    if (P.d_initial) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<float4*>(P.d_initial + soff + (size_t)(4 * lane + i) * D + col0) =
            make_float4(dS[i][0], dS[i][1], dS[i][2], dS[i][3]);
    }
    __syncthreads();  // shared partials of this item are read before the next item writes them
  }
}

// Per (token, head) row: the slices' partial sums, then the derivatives of the transforms
// (dq and dk through the L2 norms, dg through the gate, dbeta through the sigmoid).  A CTA takes one
// head and a run of tokens (one warp per token at a time, a lane per 4 channels) and adds its sums
// of the gate-parameter gradients with one atomic per value.
__global__ void __launch_bounds__(256) bwd_finish_kernel(BwdParams P, int64_t tokens, int tokens_per_cta) {
  constexpr int D = kHeadDim;
  __shared__ __align__(16) float s_dt[8][D];
  __shared__ float s_dA[8];
  const FwdParams& p = P.f;
  if (!cta_seqlens_ok(p)) return;  // out-of-order offsets: no document ran, nothing to finish
  const int H = p.num_heads;
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows_total = tokens * H;
  const float ea = expf(p.A_log[h]);
  const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
  const float dts[4] = {dt.x, dt.y, dt.z, dt.w};
  float ddt[4] = {0.f, 0.f, 0.f, 0.f}, dA = 0.f;
  const int64_t t_begin = (int64_t)blockIdx.x * tokens_per_cta;
  const int64_t t_end = min(t_begin + tokens_per_cta, tokens);
  for (int64_t t = t_begin + warp; t < t_end; t += 8) {
    const size_t row = (size_t)t * H + h;
    float gq[4] = {0.f, 0.f, 0.f, 0.f}, gk[4] = {0.f, 0.f, 0.f, 0.f}, ga[4] = {0.f, 0.f, 0.f, 0.f}, gb = 0.f;
#pragma unroll
    for (int sl = 0; sl < kSlices; ++sl) {
      const float* base = P.part + (size_t)sl * 3 * rows_total * D + row * D + 4 * lane;
      const float4 a = *reinterpret_cast<const float4*>(base);
      const float4 b = *reinterpret_cast<const float4*>(base + (size_t)rows_total * D);
      const float4 c = *reinterpret_cast<const float4*>(base + 2 * (size_t)rows_total * D);
      gq[0] += a.x; gq[1] += a.y; gq[2] += a.z; gq[3] += a.w;
      gk[0] += b.x; gk[1] += b.y; gk[2] += b.z; gk[3] += b.w;
      ga[0] += c.x; ga[1] += c.y; ga[2] += c.z; ga[3] += c.w;
      gb += P.part[(size_t)kSlices * 3 * rows_total * D + (size_t)sl * rows_total + row];
    }
    // dq, dk: (dxhat - xhat (xhat . dxhat)) / n
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const float4 x4 = ld_bf16x4((which == 0 ? p.q : p.k) + row * D + 4 * lane);
      const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
      float ss = xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float nrm = sqrtf(ss + kL2Eps);
      const float* gx = which == 0 ? gq : gk;
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) dot += (xv[j] / nrm) * gx[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      float r[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) r[j] = (gx[j] - (xv[j] / nrm) * dot) / nrm;
      st_bf16x4((which == 0 ? P.dq : P.dk) + row * D + 4 * lane, r[0], r[1], r[2], r[3]);
    }
    // dg through the gate; the sums for dt_bias and A_log
    {
      const float4 g4 = ld_bf16x4(p.g + row * D + 4 * lane);
      const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
      float dg[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float x = ea * (gv[j] + dts[j]);
        const float sg = sigmoid_acc(x);
        const float al = expf(p.lower_bound * sg);
        const float dx = ga[j] * al * p.lower_bound * sg * (1.f - sg);
        dg[j] = dx * ea;
        ddt[j] += dg[j];
        dA = fmaf(dx, x, dA);
      }
      st_bf16x4(P.dg + row * D + 4 * lane, dg[0], dg[1], dg[2], dg[3]);
    }
    if (lane == 0) {
      const float b = sigmoid_acc(__bfloat162float(p.beta[row]));
      P.dbeta[row] = __float2bfloat16_rn(gb * b * (1.f - b));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dA += __shfl_xor_sync(0xffffffffu, dA, o);
  reinterpret_cast<float4*>(s_dt[warp])[lane] = make_float4(ddt[0], ddt[1], ddt[2], ddt[3]);
  if (lane == 0) s_dA[warp] = dA;
  __syncthreads();
  if (warp == 0) {
    float t[4] = {0.f, 0.f, 0.f, 0.f}, a = 0.f;
    for (int w = 0; w < 8; ++w) {
      const float4 x = reinterpret_cast<const float4*>(s_dt[w])[lane];
      t[0] += x.x; t[1] += x.y; t[2] += x.z; t[3] += x.w;
      a += s_dA[w];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) atomicAdd(P.ddt_bias + (size_t)h * D + 4 * lane + j, t[j]);
    if (lane == 0) atomicAdd(P.dA_log + h, a);
  }
}

}  // namespace

// At most this many persistent CTAs of the slice kernel (two per SM), so that the workspace size
// depends only on the problem's sizes.
constexpr int64_t kBwdMaxCtas = 512;
constexpr int kFinishTokens = 64;  // tokens per CTA of the finishing kernel

size_t bwd_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t t = total_tokens > 0 ? total_tokens : 0, n = num_seqs > 0 ? num_seqs : 0;
  const int64_t hh = num_heads > 0 ? num_heads : 0;
  const int64_t slots = t / kBwdChunk + n + 1;
  const int64_t work = n * hh * kSlices;
  const int64_t ctas = work < kBwdMaxCtas ? work : kBwdMaxCtas;
  const size_t ckpt = (size_t)slots * hh * kStateElems;
  const size_t scratch = (size_t)ctas * kBwdChunk * kSliceElems;
  const size_t part = (size_t)kSlices * (3 * (size_t)t * hh * kHeadDim + (size_t)t * hh);
  return (ckpt + scratch + part) * sizeof(float);
}

cudaError_t launch_bwd(const FwdParams& f, const __nv_bfloat16* d_out, const float* d_final, __nv_bfloat16* dq,
                       __nv_bfloat16* dk, __nv_bfloat16* dv, __nv_bfloat16* dg, __nv_bfloat16* dbeta, float* dA_log,
                       float* ddt_bias, float* d_initial, const float* checkpoints, void* workspace,
                       cudaStream_t stream) {
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
  const int64_t work = units * kSlices;
  int64_t grid = work < 2 * (int64_t)sms ? work : 2 * (int64_t)sms;
  if (grid > kBwdMaxCtas) grid = kBwdMaxCtas;
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
  P.ckpt_in = checkpoints;
  P.ckpt = static_cast<float*>(workspace);
  P.scratch = P.ckpt + (size_t)slots * f.num_heads * kStateElems;
  const int64_t work_cap = work < kBwdMaxCtas ? work : kBwdMaxCtas;
  P.part = P.scratch + (size_t)work_cap * kBwdChunk * kSliceElems;
  const size_t smem = sizeof(ChunkIn) + (2 * 8 * 3 * kHeadDim + 2 * 8) * sizeof(float);
  static bool attr_done[64] = {};
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if ((e = cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    attr_done[dev] = true;
  }
  bwd_kernel<<<(unsigned)grid, kBwdThreads, smem, stream>>>(P);
  if ((e = cudaGetLastError()) != cudaSuccess || tokens == 0) return e;
  const dim3 fgrid((unsigned)((tokens + kFinishTokens - 1) / kFinishTokens), (unsigned)f.num_heads);
  bwd_finish_kernel<<<fgrid, 256, 0, stream>>>(P, tokens, kFinishTokens);
  return cudaGetLastError();
}

}  // namespace kda
