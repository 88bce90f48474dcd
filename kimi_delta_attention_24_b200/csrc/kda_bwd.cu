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
// CTAs of 32 state columns each (persistent over (unit, slice) pairs, two CTAs per SM), 256 threads,
// the slice of the state and of its gradient in registers (16 rows x 1 column per thread).  A CTA
// first runs the forward over its sequence, storing the slice at the start of every 64-token chunk in
// the workspace; then, chunk by chunk from the last, it reruns the chunk's forward from its
// checkpoint, storing the slice before every token in a per-CTA scratch, and walks the chunk's tokens
// backwards.  Sums over the state's rows run through shared memory across the warps, sums over its
// columns through warp shuffles; what sums over all columns (dqhat, dkhat, dalpha per channel and
// dbeta) is written per slice, and a second kernel adds the slices, applies the derivatives of the
// L2 norms, the gate and the sigmoid, and adds the dA_log / dt_bias sums with one atomic per value
// per CTA (the outputs are zeroed first).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdChunk = 64;
constexpr int kRows = 16;  // state rows per thread: warp w holds rows 16 w .. 16 w + 15
constexpr int kSlice = 32;  // state columns per CTA (one per lane)
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
  float* ckpt;                  // (T / 64 + N + 1) x H states: chunk-start checkpoints (by slice)
  float* scratch;               // gridDim.x x 64 slices: the states before each token of a chunk
  float* part;                  // per slice: dqhat, dkhat, dalpha [tokens, H, K]; then dbeta [slice][tokens, H]
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

// One token's raw inputs, split over the CTA: warps 0..4 read 4 channels per lane of q, k, g, v and
// d_out (warp 0 and 4 only for the backward step), lane 0 of warp 5 reads beta.  Fetched one token
// ahead into registers, so that the global loads of token t + 1 overlap the work on token t.
struct RawTok {
  uint2 u;
  float b;
};

__device__ __forceinline__ RawTok fetch_token(const BwdParams& P, size_t row, bool full) {
  const FwdParams& p = P.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int D = kHeadDim;
  RawTok r;
  r.u = make_uint2(0, 0);
  r.b = 0.f;
  const __nv_bfloat16* src = nullptr;
  if (warp == 0 && full) src = p.q;
  else if (warp == 1) src = p.k;
  else if (warp == 2) src = p.g;
  else if (warp == 3) src = p.v;
  else if (warp == 4 && full) src = P.d_out;
  if (src) r.u = *reinterpret_cast<const uint2*>(src + row * D + 4 * lane);
  if (warp == 5 && lane == 0) r.b = __bfloat162float(p.beta[row]);
  return r;
}

__device__ __forceinline__ float4 bf16x4_of(uint2 u) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// The transformed inputs of one token into shared memory, from the fetched raw values.  `full`:
// also qhat, d_out and the gate's intermediates (the backward step); otherwise only what the forward
// step reads (khat, alpha, beta, v).  dt: this lane's 4 channels of dt_bias[h].
__device__ __forceinline__ void stage_token(const BwdParams& P, const RawTok& r, float ea, float4 dt, TokenIn& s,
                                            bool full) {
  const FwdParams& p = P.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 || warp == 1) {
    if (warp == 0 && !full) return;
    const float4 x4 = bf16x4_of(r.u);
    float ss = x4.x * x4.x + x4.y * x4.y + x4.z * x4.z + x4.w * x4.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float n = sqrtf(ss + kL2Eps);
    float* dst = warp == 0 ? s.q : s.k;
    reinterpret_cast<float4*>(dst)[lane] = make_float4(x4.x / n, x4.y / n, x4.z / n, x4.w / n);
    if (lane == 0) (warp == 0 ? s.nq : s.nk) = n;
  } else if (warp == 2) {
    const float4 g4 = bf16x4_of(r.u);
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
    reinterpret_cast<float4*>(s.v)[lane] = bf16x4_of(r.u);
  } else if (warp == 4) {
    if (full) reinterpret_cast<float4*>(s.d)[lane] = bf16x4_of(r.u);
  } else if (warp == 5 && lane == 0) {
    s.b = sigmoid_acc(r.b);
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

// One CTA per (unit, column slice): the state's 128 rows and the slice's kSlice columns (a 16 x 1
// block per thread: warp w holds rows 16 w .. + 15, lane l column l of the slice).  The columns of
// the state evolve independently, so each slice runs the whole token recurrence on its own; what
// sums over columns (dqhat, dkhat, dalpha per row, dbeta) is written per slice and summed by
// bwd_finish_kernel, which also applies the derivatives of the in-kernel transforms.
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_kernel(BwdParams P) {
  constexpr int D = kHeadDim;
  __shared__ __align__(16) TokenIn s;
  __shared__ __align__(16) float red[2][8][kSlice];
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = kRows * warp;
  const int64_t units = (int64_t)p.num_seqs * H;
  const int64_t work = units * kSlices;
  float* const scr = P.scratch + (size_t)blockIdx.x * kBwdChunk * kSliceElems;
  const bool seqlens_ok = cta_seqlens_ok(p);
  const int64_t rows_total = (p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs) * H;

  for (int64_t wi = blockIdx.x; wi < work; wi += gridDim.x) {
    const int64_t u = wi / kSlices;
    const int sl = (int)(wi - u * kSlices);
    const int n = (int)(u / H), h = (int)(u % H);
    const int col = sl * kSlice + lane;  // this thread's state column (v)
    int64_t bos, eos;
    seq_range(p, n, bos, eos);
    if (!seqlens_ok) eos = bos;
    const int64_t L = eos - bos;
    const int nch = (int)((L + kBwdChunk - 1) / kBwdChunk);
    const size_t soff = ((size_t)n * H + h) * kStateElems;
    const int64_t ck0 = bos / kBwdChunk + n;  // this sequence's first checkpoint slot
    const float ea = expf(p.A_log[h]);
    const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
    auto tok_row = [&](int64_t t) { return (size_t)t * H + h; };
    // checkpoint c of this slice: [128 rows][kSlice]
    auto ck_ptr = [&](int c) { return P.ckpt + (((size_t)(ck0 + c) * H + h) * kSlices + sl) * kSliceElems; };
    float* const part_q = P.part + (size_t)sl * 3 * rows_total * D;  // per slice: dqhat, dkhat, dalpha rows
    float* const part_k = part_q + (size_t)rows_total * D;
    float* const part_a = part_k + (size_t)rows_total * D;
    float* const part_b = P.part + (size_t)kSlices * 3 * rows_total * D + (size_t)sl * rows_total;

    float S[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) S[i] = p.initial_state ? p.initial_state[soff + (size_t)(r0 + i) * D + col] : 0.f;
    auto store_state = [&](float* dst) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) dst[(r0 + i) * kSlice + lane] = S[i];
    };
    auto load_state = [&](const float* src) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) S[i] = src[(r0 + i) * kSlice + lane];
    };
    // the sum over the 8 warps of one value per thread (its column): red[w][lane]
    auto col_sum = [&](float (*rd)[kSlice], float x) {
      rd[warp][lane] = x;
      __syncthreads();
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) t += rd[w][lane];
      return t;
    };
    auto forward_token = [&]() {
      float pr = 0.f;
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        S[i] *= s.a[r0 + i];
        pr = fmaf(S[i], s.k[r0 + i], pr);
      }
      const float d = s.b * (s.v[col] - col_sum(red[0], pr));
#pragma unroll
      for (int i = 0; i < kRows; ++i) S[i] = fmaf(s.k[r0 + i], d, S[i]);
    };

    // ---------------------------------------------------------------- forward with checkpoints
    RawTok rt = fetch_token(P, tok_row(bos), false);  // (L = 0: never staged)
    for (int c = 0; c < nch; ++c) {
      store_state(ck_ptr(c));
      const int64_t t_end = min(bos + (int64_t)(c + 1) * kBwdChunk, eos);
      for (int64_t t = bos + (int64_t)c * kBwdChunk; t < t_end; ++t) {
        __syncthreads();
        stage_token(P, rt, ea, dt, s, false);
        if (t + 1 < eos) rt = fetch_token(P, tok_row(t + 1), false);
        __syncthreads();
        forward_token();
      }
    }

    // ---------------------------------------------------------------- backward, chunk by chunk
    float dS[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) dS[i] = P.d_final ? P.d_final[soff + (size_t)(r0 + i) * D + col] : 0.f;

    for (int c = nch - 1; c >= 0; --c) {
      const int64_t t_begin = bos + (int64_t)c * kBwdChunk;
      const int len = (int)min((int64_t)kBwdChunk, eos - t_begin);
      // rerun the chunk's forward from its checkpoint, keeping the state before each token
      load_state(ck_ptr(c));
      RawTok rf = fetch_token(P, tok_row(t_begin), false);
      for (int i = 0; i < len; ++i) {
        store_state(scr + (size_t)i * kSliceElems);
        __syncthreads();
        stage_token(P, rf, ea, dt, s, false);
        if (i + 1 < len) rf = fetch_token(P, tok_row(t_begin + i + 1), false);
        __syncthreads();
        forward_token();
      }
      // the chunk's tokens backwards; S holds S_{t-1} of the token at hand, loaded from the scratch
      // (written by this thread above) during the token after it
      RawTok rb = fetch_token(P, tok_row(t_begin + len - 1), true);
      load_state(scr + (size_t)(len - 1) * kSliceElems);
      for (int i = len - 1; i >= 0; --i) {
        const size_t row = tok_row(t_begin + i);
        __syncthreads();
        stage_token(P, rb, ea, dt, s, true);
        if (i > 0) rb = fetch_token(P, tok_row(t_begin + i - 1), true);
        __syncthreads();
        const float b = s.b, scale = p.scale;
        float pr = 0.f;
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) pr = fmaf(s.a[r0 + ii] * S[ii], s.k[r0 + ii], pr);
        const float pj = col_sum(red[0], pr);
        const float vj = s.v[col], doj = s.d[col];
        const float dl = b * (vj - pj);
        // dS += scale qhat do^T;  dqhat rows (this slice) = scale S_t do;  ddelta = dS^T khat
        float rq[kRows], pd = 0.f;
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) {
          const float kk = s.k[r0 + ii];
          rq[ii] = scale * fmaf(kk, dl, s.a[r0 + ii] * S[ii]) * doj;
          dS[ii] = fmaf(scale * s.q[r0 + ii], doj, dS[ii]);
          pd = fmaf(dS[ii], kk, pd);
        }
        const float tq = transpose_reduce16(rq, lane);
        const float ddl = col_sum(red[1], pd);
        const float dp = -b * ddl;
        if (warp == 0) {
          P.dv[row * D + col] = __float2bfloat16_rn(b * ddl);
          float db = ddl * (vj - pj);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
          if (lane == 0) part_b[row] = db;
        }
        // dkhat = dS delta + Stil dp;  dStil = dS + khat dp^T;  dalpha;  dS <- Diag(alpha) dStil
        float rk[kRows];
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) rk[ii] = fmaf(dS[ii], dl, s.a[r0 + ii] * S[ii] * dp);
        const float tk = transpose_reduce16(rk, lane);
        float ra[kRows];
#pragma unroll
        for (int ii = 0; ii < kRows; ++ii) {
          const float dst = fmaf(s.k[r0 + ii], dp, dS[ii]);
          ra[ii] = dst * S[ii];
          dS[ii] = s.a[r0 + ii] * dst;
        }
        if (i > 0) load_state(scr + (size_t)(i - 1) * kSliceElems);  // the next token's S_{t-1}
        const float ta = transpose_reduce16(ra, lane);
        if ((lane & 1) == 0) {
          const size_t o = row * D + r0 + (lane >> 1);
          part_q[o] = tq;
          part_k[o] = tk;
          part_a[o] = ta;
        }
      }
    }
    if (P.d_initial) {
#pragma unroll
      for (int i = 0; i < kRows; ++i) P.d_initial[soff + (size_t)(r0 + i) * D + col] = dS[i];
    }
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
  P.ckpt = static_cast<float*>(workspace);
  P.scratch = P.ckpt + (size_t)slots * f.num_heads * kStateElems;
  const int64_t work_cap = work < kBwdMaxCtas ? work : kBwdMaxCtas;
  P.part = P.scratch + (size_t)work_cap * kBwdChunk * kSliceElems;
  bwd_kernel<<<(unsigned)grid, kBwdThreads, 0, stream>>>(P);
  if ((e = cudaGetLastError()) != cudaSuccess || tokens == 0) return e;
  const dim3 fgrid((unsigned)((tokens + kFinishTokens - 1) / kFinishTokens), (unsigned)f.num_heads);
  bwd_finish_kernel<<<fgrid, 256, 0, stream>>>(P, tokens, kFinishTokens);
  return cudaGetLastError();
}

}  // namespace kda
