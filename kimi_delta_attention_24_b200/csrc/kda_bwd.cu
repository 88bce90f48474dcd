// Backward pass of the KDA forward (gradients of every input), in the chunked form.
//
// torchtitan trains Kimi-K3 through chunk_kda, and its varlen test checks the gradient as well
// as the forward (torchtitan PR #4374, Results: test_varlen_matches_independent_documents).  The
// forward of one 64-token chunk (rows r, state S at the chunk start; Gamma the in-chunk cumulative
// log-decay, gamma its last row, khat / qhat the normalised keys / queries) is
//   Kg = khat e^Gamma,  Qt = scale qhat e^Gamma,  Kt = khat e^{gamma - Gamma},
//   M_rs = sum_c khat_rc khat_sc e^{Gamma_rc - Gamma_sc},  A = strict_tril(diag(beta) M),
//   P = scale tril(qhat-khat gated the same way),  T = (I + A)^{-1},  T_b = T diag(beta),
//   W = T_b Kg,  U = T_b V,  Delta = U - W S,  O = Qt S + P Delta,  S' = Diag(e^gamma) S + Kt^T Delta.
// Reverse mode, given dO and dS' (the gradient of the chunk's end state):
//   dDelta = P^T dO + Kt dS',   dS = Diag(e^gamma) dS' + (Qt - P W)^T dO - W^T Kt dS'   (to the chunk before),
//   dKt = Delta dS'^T,  dQt = dO S^T + dP Kn,  dP = tril(dO Delta^T),  dW = -dDelta S^T,
//   dT_b = dDelta V^T + dW Kg^T,  dV = T_b^T dDelta,  dKg = T_b^T dW,  dA = strict_tril(-T^T dT T^T)
//   with dT = dT_b diag(beta),  dM = diag(beta) dA,  dbeta = colsum(dT_b o T) + rowsum(dA o M),
// and the decay-weighted products that carry dM and dP back to khat and qhat never form e^{-Gamma}
// alone: X1_r = sum_{s<r} dM_rs khat_s e^{Gamma_r - Gamma_s} and its transposed and P counterparts
// are evaluated per 16-row sub-block against the decays at a sub-block boundary, so that every
// factor lies in [e^{-80}, e^{80}] (|log alpha| <= 5).  Then
//   dkhat = X1 + X2 + X4 + e^Gamma dKg + e^{gamma - Gamma} dKt,   dqhat = scale (X3 + e^Gamma dO S^T),
//   dGamma = khat (X1 + e^Gamma dKg - X2 - X4 - e^{gamma - Gamma} dKt) + qhat dqhat,
//   dlog alpha_r = sum_{r' >= r} dGamma_r' + dgamma,  dgamma = e^gamma rowsum(S o dS') + sum_r khat e^{gamma-Gamma} dKt,
// followed by the derivatives of the in-kernel transforms (L2 norms, sigmoid of beta, safe gate).
//
// Launches: the checkpointing forward when no chunk-start states are given (the split path, which
// stores S at every chunk start); bwd_prep_kernel (chunk-parallel: forms a chunk's factors and stores
// W, Kt, P^T dO, (Qt - P W)^T dO, e^gamma, M, T, T_b, khat, qhat, Gamma and Kg); bwd_state_kernel
// (one CTA per (sequence, head), chunks last to first: dDelta and the state gradient at every chunk
// boundary); bwd_grad_kernel (chunk-parallel: reads the chunk's factors from the prep output and
// forms the gradients above); bwd_finish_kernel (the transforms, and dA_log / dt_bias summed with
// one atomic per value per CTA).  The chunk-parallel kernels are persistent; each CTA keeps one
// chunk's intermediates in its own global scratch (mostly held by L2).  The products run on the
// tensor cores (mma.sync tf32 with hi/lo operands: fp32-level accuracy), the element-wise work in
// fp32 on CUDA cores.
#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

constexpr int kBwdThreads = 256;
constexpr int C = 64;
constexpr int D = kHeadDim;
constexpr int kF = C * D;          // one 64 x 128 fp32 matrix
constexpr int kQ = C * C;          // one 64 x 64 fp32 matrix
constexpr size_t kStateElems = (size_t)D * D;

// per-chunk outputs of bwd_prep_kernel, for bwd_state_kernel (floats)
constexpr int PR_W = 0;            // W [64][128]
constexpr int PR_KT = kF;          // Kt [64][128]
constexpr int PR_PDO = 2 * kF;     // P^T dO [64][128]
constexpr int PR_Y = 3 * kF;       // (Qt - P W)^T dO [128][128]
constexpr int PR_EG = 3 * kF + D * D;  // e^gamma [128]
constexpr int PR_M = PR_EG + D;        // M [64][64] (strict lower) and T = (I + A)^{-1} [64][64], for the gradient kernel
constexpr int PR_T = PR_M + kQ;
constexpr int PR_TB = PR_T + kQ;       // T_b = T diag(beta) [64][64]
constexpr int PR_KH = PR_TB + kQ;      // khat, qhat, Gamma, Kg [64][128] each: the chunk's element-wise factors
constexpr int PR_QH = PR_KH + kF, PR_G = PR_QH + kF, PR_KG = PR_G + kF;
constexpr int kPrepFloats = PR_KG + kF;

// per-CTA scratch (floats).  The chunk's element-wise factors (khat, qhat, Gamma, Kg) live in the
// prep kernel's output, which both chunk kernels read.  Each kernel reuses buffers once they are dead,
// so that the scratch of all its CTAs (at most 370 KB each) mostly stays in L2.  The prep kernel: the
// Gram product's operands and output in V .. DKG (V is not needed there), Qt - P W in V after them.
// The gradient kernel: dv's temporary and the gated products' partial sums in D (Delta), their
// depth-16 right operands in DW, the 128 x 128 temporary in dO and V, the product T^T dA in DTB.
constexpr int SC_L = 0;  // the gradient kernel: the transposed gated products' output
constexpr int SC_DO = kF, SC_V = 2 * kF, SC_W = 3 * kF, SC_D = 4 * kF, SC_DKT = 5 * kF, SC_DQS = 6 * kF;
constexpr int SC_DW = 7 * kF, SC_DKG = 8 * kF;
constexpr int SC_GL = SC_V, SC_GR = SC_D, SC_GO = SC_DQS + kF / 2;  // prep: 128 x 128, 160 x 128, 128 x 160
constexpr int SC_X = SC_V;                                          // prep: Qt - P W
constexpr int SC_P = 9 * kF, SC_TB = SC_P + kQ;  // prep: M, T and T_b go straight to its output
constexpr int SC_DA = SC_TB + kQ, SC_DP = SC_DA + kQ;  // dA (then dM) and dP adjacent: [dM; dP] is 128 x 64
constexpr int SC_DTB = SC_DP + kQ;
constexpr int SC_BETA = SC_DTB + kQ, SC_EG = SC_BETA + C, SC_DGAM = SC_EG + D, SC_DB = SC_DGAM + D;
static_assert(SC_GO + 160 * D <= SC_P, "the Gram product's output ends before P");
static_assert(SC_DO + kF == SC_V, "dO and V adjacent: the gradient kernel's 128 x 128 temporary");
constexpr int kScratchFloats = SC_DB + C + 64;

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
  const float* ckpt;            // chunk-start states, S^T [v][k], slot bos / 64 + n + j for chunk j of sequence n
  const int32_t* chunk_off;     // [N + 1] first global chunk of each sequence
  float* prep;                  // kPrepFloats per (global chunk, head)
  float* dsp;                   // per slot and head: dS' [k][v], the gradient of chunk j's end state (slot of chunk j)
  float* dd;                    // kF per (global chunk, head): dDelta
  float* part;                  // dqhat, dkhat, dlog alpha [tokens, H, K] each; then dbeta [tokens, H]
  float* scratch;               // kScratchFloats per CTA of the chunk-parallel kernels
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

// ------------------------------------------------------------------------- the GEMM routine (fp32 operands)
// An operand: element (i, j) is p[i * ld + j], or p[j * ld + i] when t (transposed).  With p2, the
// depth index k >= k2 reads the second operand p2 at depth k - k2 (two products summed in one).
struct Mat {
  const float* p;
  int ld;
  bool t;
  const float* p2;
  int k2;
};
__device__ __forceinline__ Mat mat(const float* p, int ld, bool t = false) { return Mat{p, ld, t, nullptr, 1 << 30}; }
__device__ __forceinline__ Mat mat2(const float* p, const float* p2, int k2, int ld, bool t) {
  return Mat{p, ld, t, p2, k2};
}

constexpr int GB_K = 32;  // depth of one staged slice
// A slice keeps its operand's memory orientation in shared memory, rows padded so that the
// tensor-core fragment reads (lane (g, t) reads row or column g, depth t) fall in 32 distinct banks:
// along-i slices as [k][i] with 8 floats of padding (bank 8 t + g), along-k slices as [i][k] with 4
// (bank 4 g + t).  Two stages, so that the next slice's copies overlap the current slice's products.
constexpr int LD_K = GB_K + 4;  // [i][k] rows
constexpr int stage_floats(int w) { return w * LD_K > GB_K * (w + 8) ? w * LD_K : GB_K * (w + 8); }
constexpr int kStageA = stage_floats(64);
// NB: the widest B tile (column block) the kernel's products use, 128 or 160
template <int NB>
struct GemmSmemT {
  float a[2][kStageA];
  float b[2][stage_floats(NB)];
};
using GemmSmem = GemmSmemT<128>;

__device__ __forceinline__ void cp_async16(float* dst, const float* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Copies the GB_K x W slice (depth k0.., rows i0..) of an operand into shared memory, zero outside
// rows x depth: element (i, k) is p[k * ld + i] (along i: to s[k][i], row length W + 8) or p[i * ld +
// k] (kmaj: to s[i][k], row length LD_K).
// The threads that run a product together: the whole CTA of 256 threads, or one half of a CTA of 512
// with its own named barrier.
struct AllThreads {
  __device__ static int tid() { return threadIdx.x; }
  __device__ static void sync() { __syncthreads(); }
};
template <int kBar>
struct HalfCta {
  __device__ static int tid() { return threadIdx.x & (kBwdThreads - 1); }
  __device__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(kBar), "n"(kBwdThreads) : "memory"); }
};

template <int W, class Grp = AllThreads>
__device__ __forceinline__ void slice_copy(float* s, const Mat& m, bool kmaj, int i0, int k0, int rows, int depth) {
  const int ld = m.ld;
  constexpr int kVec = GB_K * W / 4;
  const int tid = Grp::tid();
#pragma unroll
  for (int e = 0; e < (kVec + kBwdThreads - 1) / kBwdThreads; ++e) {
    const int idx = tid + e * kBwdThreads;
    if (kVec % kBwdThreads != 0 && idx >= kVec) break;
    if (!kmaj) {
      const int i4 = idx % (W / 4), k = idx / (W / 4), kk = k0 + k;
      const bool ok = kk < depth && i0 + 4 * i4 < rows;
      const float* src = kk < m.k2 ? m.p + (size_t)kk * ld : m.p2 + (size_t)(kk - m.k2) * ld;
      cp_async16(s + k * (W + 8) + 4 * i4, ok ? src + i0 + 4 * i4 : m.p, ok);
    } else {
      const int k4 = idx % (GB_K / 4), i = idx / (GB_K / 4), kk = k0 + 4 * k4;
      const bool ok = i0 + i < rows && kk < depth;
      const float* src = kk < m.k2 ? m.p + kk : m.p2 + (kk - m.k2);
      cp_async16(s + i * LD_K + 4 * k4, ok ? src + (size_t)(i0 + i) * ld : m.p, ok);
    }
  }
}

// The output of a product: load(i, j) reads what the result (i, j .. j + 1) combines with, store(i, j,
// v, l) writes it from the product's value v and that l.  With kLoadsFirst a thread issues all of its
// tile's loads before its stores (more registers; for outputs that combine with other buffers).  The
// default: C[i][j] = alpha v (+ C[i][j] when acc); mask 1 keeps j < i, mask 2 keeps j <= i (the rest
// is written as 0).
struct EpiStore {
  static constexpr bool kLoadsFirst = false;
  float* C;
  int ldc;
  float alpha;
  bool acc;
  int mask;
  __device__ __forceinline__ float2 load(int i, int j) const {
    return acc ? *reinterpret_cast<const float2*>(C + (size_t)i * ldc + j) : make_float2(0.f, 0.f);
  }
  __device__ __forceinline__ void store(int i, int j, float2 v, float2 l) const {
    float2 o = make_float2(fmaf(alpha, v.x, l.x), fmaf(alpha, v.y, l.y));
    if (mask) {
      const int lim = mask == 1 ? i : i + 1;  // keep j < lim
      if (j + 0 >= lim) o.x = 0.f;
      if (j + 1 >= lim) o.y = 0.f;
    }
    *reinterpret_cast<float2*>(C + (size_t)i * ldc + j) = o;
  }
};

// sum_k A(i, k) B(k, j), i < M, j < N, to the output epi.  Output tiles of (16 RM) x NW on the tensor cores:
// mma.sync m16n8k8 with tf32 operands, each operand split into a high and a low tf32 part and the
// three products hi hi, hi lo, lo hi accumulated in fp32 (about 2^-20 relative: fp32-level).  With
// RM = 4 warp (wm, wn) holds rows 32 wm .. + 31 and columns NW / 4 wn .. + NW / 4 - 1 (2 x NW / 32
// fragments), with RM = 1 (NW = 128) warp w columns 16 w .. + 15 (1 x 2).  M, N multiples of 4, K of
// 8; operands 16-byte aligned with ld a multiple of 4.  X marks operands whose values are tf32
// numbers already (bit 1: A, bit 2: B; bf16 inputs), whose low parts are zero: their products with
// the other operand's high part are skipped.  All threads of the CTA call it; it ends with a barrier.
template <int RM, int NW, int NB, class Epi, int X = 0, class Grp = AllThreads>
__device__ void gemm_t(Mat A, Mat B, int M, int N, int K, GemmSmemT<NB>& sm, const Epi& epi) {
  static_assert(NW <= NB && (RM == 4 || NW == 128), "tile width");
  constexpr int BM = 16 * RM;
  constexpr int MT = RM == 4 ? 2 : 1, NT = RM == 4 ? NW / 32 : 2;  // fragments per warp
  const int tid = Grp::tid(), warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int wm = RM == 4 ? (warp & 1) : 0, wn = RM == 4 ? (warp >> 1) : warp;
  const int row0 = RM == 4 ? 32 * wm : 0, col0 = RM == 4 ? (NW / 4) * wn : 16 * wn;
  const bool a_kmaj = !A.t, b_kmaj = B.t;  // A(i, k) runs along k unless transposed; B(k, j) along j unless transposed
  const int nsl = (K + GB_K - 1) / GB_K;
  // element (row, depth) of a stage's A slice and (column, depth) of its B slice
  auto a_at = [&](const float* sa, int r, int k) { return a_kmaj ? sa[r * LD_K + k] : sa[k * (BM + 8) + r]; };
  auto b_at = [&](const float* sb, int n, int k) { return b_kmaj ? sb[n * LD_K + k] : sb[k * (NW + 8) + n]; };
  for (int i0 = 0; i0 < M; i0 += BM) {
    for (int j0 = 0; j0 < N; j0 += NW) {
      float c[MT][NT][4];
#pragma unroll
      for (int a = 0; a < MT; ++a)
#pragma unroll
        for (int b = 0; b < NT; ++b)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[a][b][e] = 0.f;
      slice_copy<BM, Grp>(sm.a[0], A, a_kmaj, i0, 0, M, K);
      slice_copy<NW, Grp>(sm.b[0], B, b_kmaj, j0, 0, N, K);
      cp_async_commit();
      for (int ks = 0; ks < nsl; ++ks) {
        if (ks + 1 < nsl) {
          slice_copy<BM, Grp>(sm.a[(ks + 1) & 1], A, a_kmaj, i0, (ks + 1) * GB_K, M, K);
          slice_copy<NW, Grp>(sm.b[(ks + 1) & 1], B, b_kmaj, j0, (ks + 1) * GB_K, N, K);
          cp_async_commit();
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        Grp::sync();
        const float* sa = sm.a[ks & 1];
        const float* sb = sm.b[ks & 1];
        const int kn = K - ks * GB_K < GB_K ? K - ks * GB_K : GB_K;
        for (int kk = 0; kk < kn; kk += 8) {
          uint32_t ah[MT][4], al[MT][4];
#pragma unroll
          for (int a = 0; a < MT; ++a) {
            const int r = row0 + 16 * a + g;
            sm100::tf32_split(a_at(sa, r, kk + t), ah[a][0], al[a][0]);
            sm100::tf32_split(a_at(sa, r + 8, kk + t), ah[a][1], al[a][1]);
            sm100::tf32_split(a_at(sa, r, kk + t + 4), ah[a][2], al[a][2]);
            sm100::tf32_split(a_at(sa, r + 8, kk + t + 4), ah[a][3], al[a][3]);
          }
#pragma unroll
          for (int b = 0; b < NT; ++b) {
            const int n = col0 + 8 * b + g;
            uint32_t bh0, bl0, bh1, bl1;
            sm100::tf32_split(b_at(sb, n, kk + t), bh0, bl0);
            sm100::tf32_split(b_at(sb, n, kk + t + 4), bh1, bl1);
#pragma unroll
            for (int a = 0; a < MT; ++a) {
              if constexpr (!(X & 2)) sm100::mma_tf32(c[a][b], ah[a], bl0, bl1);
              if constexpr (!(X & 1)) sm100::mma_tf32(c[a][b], al[a], bh0, bh1);
              sm100::mma_tf32(c[a][b], ah[a], bh0, bh1);
            }
          }
        }
        Grp::sync();  // the stage is refilled two slices on
      }
      if constexpr (Epi::kLoadsFirst) {
        float2 l[MT][2][NT];
#pragma unroll
        for (int a = 0; a < MT; ++a)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int b = 0; b < NT; ++b) {
              const int i = i0 + row0 + 16 * a + g + 8 * hr, j = j0 + col0 + 8 * b + 2 * t;
              if (i < M && j < N) l[a][hr][b] = epi.load(i, j);
            }
#pragma unroll
        for (int a = 0; a < MT; ++a)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int b = 0; b < NT; ++b) {
              const int i = i0 + row0 + 16 * a + g + 8 * hr, j = j0 + col0 + 8 * b + 2 * t;
              if (i < M && j < N) epi.store(i, j, make_float2(c[a][b][2 * hr], c[a][b][2 * hr + 1]), l[a][hr][b]);
            }
      } else {
#pragma unroll
        for (int a = 0; a < MT; ++a)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int b = 0; b < NT; ++b) {
              const int i = i0 + row0 + 16 * a + g + 8 * hr, j = j0 + col0 + 8 * b + 2 * t;
              if (i < M && j < N) epi.store(i, j, make_float2(c[a][b][2 * hr], c[a][b][2 * hr + 1]), epi.load(i, j));
            }
      }
    }
  }
  Grp::sync();
}

template <int X = 0, int NB, class Epi>
__device__ __forceinline__ void gemm_e(Mat A, Mat B, int M, int N, int K, GemmSmemT<NB>& sm, const Epi& epi) {
  if (M <= 16) gemm_t<1, 128, NB, Epi, X>(A, B, M, N, K, sm, epi);
  else gemm_t<4, 128, NB, Epi, X>(A, B, M, N, K, sm, epi);
}
template <int X = 0, int NB>
__device__ __forceinline__ void gemm(float* Cp, int ldc, Mat A, Mat B, int M, int N, int K, float alpha, bool acc,
                                     int mask, GemmSmemT<NB>& sm) {
  gemm_e<X>(A, B, M, N, K, sm, EpiStore{Cp, ldc, alpha, acc, mask});
}

// ------------------------------------------------------------------------- element-wise passes
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float4 add4(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 sub4(float4 a, float4 b) { return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 scl4(float4 a, float f) { return make_float4(a.x * f, a.y * f, a.z * f, a.w * f); }
// the decays: exp of a difference of log-decays (exp(-inf) = 0)
__device__ __forceinline__ float dexp(float x) { return __expf(x); }
__device__ __forceinline__ float4 dexp4(float4 x) { return make_float4(dexp(x.x), dexp(x.y), dexp(x.z), dexp(x.w)); }
struct F4x2 {
  float4 a, b;
};
struct F4x4 {
  float4 a, b, c, d;
};

// An element-wise pass over n4 float4 positions, kBatch per thread at a time: each thread evaluates
// f at a batch of its positions (loads and arithmetic) before it stores any of their results with
// st.  The buffers share one allocation, so the compiler would not move a load above an earlier
// store by itself, and every position would cost a round trip to L2.
template <int kBatch, typename F, typename S>
__device__ __forceinline__ void ew(int n4, F f, S st) {
  using V = decltype(f(0));
  for (int base = threadIdx.x; base < n4; base += kBatch * kBwdThreads) {
    V v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = base + b * kBwdThreads;
      if (i < n4) v[b] = f(i);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int i = base + b * kBwdThreads;
      if (i < n4) st(i, v[b]);
    }
  }
}
constexpr int kF4 = kF / 4, kQ4 = kQ / 4;  // float4s in a 64 x 128 / 64 x 64 matrix
// batch sizes for results of 1, 2 and 4 float4s: small, since larger batches spill registers in the
// chunk kernels (128 registers a thread at two CTAs per SM), which costs more than their latency hiding
constexpr int kB1 = 2, kB2 = 1, kB4 = 1;

// ------------------------------------------------------------------------- per-chunk recomputation
struct Chunk {
  int n, h, len;
  int64_t t0, gc, slot;
};

__device__ __forceinline__ int seq_of_chunk(const int32_t* co, int nseq, int64_t gc) {
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)co[mid] <= gc) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ Chunk locate(const BwdParams& P, int64_t item) {
  const int H = P.f.num_heads;
  Chunk c;
  c.gc = item / H;
  c.h = (int)(item - c.gc * H);
  c.n = seq_of_chunk(P.chunk_off, P.f.num_seqs, c.gc);
  int64_t bos, eos;
  seq_range(P.f, c.n, bos, eos);
  const int64_t j = c.gc - P.chunk_off[c.n];
  c.t0 = bos + j * C;
  c.len = (int)(eos - c.t0 < C ? eos - c.t0 : C);
  c.slot = bos / C + c.n + j;
  return c;
}

// Where a chunk's element-wise factors live (the prep kernel's output).
struct Fac {
  float* kh;
  float* qh;
  float* G;
  float* kg;
};
__device__ __forceinline__ Fac fac_of(float* pr) { return Fac{pr + PR_KH, pr + PR_QH, pr + PR_G, pr + PR_KG}; }

// The factors of a chunk that do not involve the state (the prep kernel): khat, qhat, Gamma and Kg
// to F; beta, e^gamma and dO (fp32, rows past the chunk's end zero) into the CTA's scratch s; the
// Gram blocks and (I + A)^{-1}: P (lower, with scale) and T_b into s, M (strict lower),
// T = (I + A)^{-1} and T_b to Mout, Tout and TBout (the prep kernel's output, which the gradient
// kernel reads).  sT, sA: the solve's two 64 x 65 shared-memory tiles.
template <int NB>
__device__ void chunk_factors(const BwdParams& P, const Chunk& ch, float* s, const Fac& F, GemmSmemT<NB>& gsm,
                              float* sT /* shared 64 x 65 */, float* sA /* shared 64 x 65 */, float* Mout = nullptr,
                              float* Tout = nullptr, float* TBout = nullptr) {
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = ch.h, len = ch.len;
  const float ea = expf(p.A_log[h]);
  const float4 dt = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
  const float dts[4] = {dt.x, dt.y, dt.z, dt.w};
  // prologue: warp per row, lane per 4 channels; each warp loads two rows before it stores any
  for (int r0 = warp; r0 < C; r0 += 2 * (kBwdThreads / 32)) {
    float4 k4[2], q4[2], g4[2], o4[2];
    float br[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + u * (kBwdThreads / 32);
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      k4[u] = q4[u] = g4[u] = o4[u] = z;
      br[u] = 0.f;
      if (r < len) {
        const size_t row = (size_t)(ch.t0 + r) * H + h;
        k4[u] = ld_bf16x4(p.k + row * D + 4 * lane);
        q4[u] = ld_bf16x4(p.q + row * D + 4 * lane);
        g4[u] = ld_bf16x4(p.g + row * D + 4 * lane);
        o4[u] = ld_bf16x4(P.d_out + row * D + 4 * lane);
        br[u] = __bfloat162float(p.beta[row]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + u * (kBwdThreads / 32);
      float sk = k4[u].x * k4[u].x + k4[u].y * k4[u].y + k4[u].z * k4[u].z + k4[u].w * k4[u].w;
      float sq = q4[u].x * q4[u].x + q4[u].y * q4[u].y + q4[u].z * q4[u].z + q4[u].w * q4[u].w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float ik = 1.0f / sqrtf(sk + kL2Eps), iq = 1.0f / sqrtf(sq + kL2Eps);
      const float gv[4] = {g4[u].x, g4[u].y, g4[u].z, g4[u].w};
      float la[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        la[j] = r < len ? p.lower_bound * __fdividef(1.f, 1.f + __expf(-ea * (gv[j] + dts[j]))) : 0.f;
      st4(F.kh + r * D + 4 * lane, scl4(k4[u], ik));
      st4(F.qh + r * D + 4 * lane, scl4(q4[u], iq));
      st4(F.G + r * D + 4 * lane, make_float4(la[0], la[1], la[2], la[3]));
      st4(s + SC_DO + r * D + 4 * lane, o4[u]);
      if (lane == 0) s[SC_BETA + r] = r < len ? sigmoid_acc(br[u]) : 0.f;
    }
  }
  __syncthreads();
  // Gamma: running sum down the rows, one thread per channel (16 rows read at a time)
  if (tid < D) {
    float acc = 0.f;
    for (int r0 = 0; r0 < C; r0 += 16) {
      float col[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) col[r] = F.G[(r0 + r) * D + tid];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        acc += col[r];
        F.G[(r0 + r) * D + tid] = acc;
      }
    }
    s[SC_EG + tid] = dexp(acc);
  }
  __syncthreads();
  ew<kB1>(kF4, [&](int i) { return mul4(ld4(F.kh + 4 * i), dexp4(ld4(F.G + 4 * i))); },
            [&](int i, float4 v) { st4(F.kg + 4 * i, v); });
  // M and P: row r of block I = r / 16 takes khat_r e^{Gamma_r - rho_I} (qhat_r for P) against the
  // rows s < 16 (I + 1) of R_I = khat_s e^{rho_I - Gamma_s}, rho_I = Gamma at the end of block I - 1
  // (0 for I = 0).  One product [LK; LQ] (128 x 128) R_all^T, R_all the four R_I stacked (160 rows,
  // R_I from row 8 I (I + 1)), of which each row keeps its own block's segment.
  {
    float* GL = s + SC_GL;  // [LK; LQ]: 128 x 128
    float* GR = s + SC_GR;  // R_all: 160 x 128
    float* GO = s + SC_GO;  // [LK; LQ] R_all^T: 128 x 160
    ew<kB1>(2 * kF4,
            [&](int i) {
              const int e = (4 * i) & (kF - 1), r = e >> 7, c = e & (D - 1), I = r >> 4;
              const float4 r4 = I == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(F.G + (16 * I - 1) * D + c);
              const float4 x = ld4((4 * i < kF ? F.kh : F.qh) + e);
              return mul4(x, dexp4(sub4(ld4(F.G + e), r4)));
            },
            [&](int i, float4 v) { st4(GL + 4 * i, v); });
    ew<kB1>(160 * D / 4,
            [&](int i) {
              const int q = (4 * i) >> 7, c = (4 * i) & (D - 1);
              const int I = q < 16 ? 0 : (q < 48 ? 1 : (q < 96 ? 2 : 3)), srow = q - 8 * I * (I + 1);
              const float4 r4 = I == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(F.G + (16 * I - 1) * D + c);
              return mul4(ld4(F.kh + srow * D + c), dexp4(sub4(r4, ld4(F.G + srow * D + c))));
            },
            [&](int i, float4 v) { st4(GR + 4 * i, v); });
    __syncthreads();
    if constexpr (NB >= 160) gemm_t<4, 160, NB>(mat(GL, D), mat(GR, D, true), 2 * C, 160, D, gsm, EpiStore{GO, 160, 1.f, false, 0});
    else gemm(GO, 160, mat(GL, D), mat(GR, D, true), 2 * C, 160, D, 1.f, false, 0, gsm);
  }
  // M strictly lower, P (times scale) lower with its diagonal, each row from its block's segment
  ew<kB2>(kQ4,
          [&](int i) {
            const int r = (4 * i) >> 6, c = (4 * i) & (C - 1), I = r >> 4;
            float4 m = make_float4(0.f, 0.f, 0.f, 0.f), q = m;
            if (c < 16 * (I + 1)) {
              const float* go = s + SC_GO + r * 160 + 8 * I * (I + 1) + c;
              m = ld4(go);
              q = scl4(ld4(go + 64 * 160), p.scale);
            }
            if (c + 0 >= r) m.x = 0.f;
            if (c + 1 >= r) m.y = 0.f;
            if (c + 2 >= r) m.z = 0.f;
            if (c + 3 >= r) m.w = 0.f;
            if (c + 0 > r) q.x = 0.f;
            if (c + 1 > r) q.y = 0.f;
            if (c + 2 > r) q.z = 0.f;
            if (c + 3 > r) q.w = 0.f;
            return F4x2{m, q};
          },
          [&](int i, F4x2 v) {
            st4(Mout + 4 * i, v.a);
            st4(s + SC_P + 4 * i, v.b);
            const int r = (4 * i) >> 6, c = (4 * i) & (C - 1);
            const float b = s[SC_BETA + r];
            sA[r * 65 + c] = b * v.a.x;
            sA[r * 65 + c + 1] = b * v.a.y;
            sA[r * 65 + c + 2] = b * v.a.z;
            sA[r * 65 + c + 3] = b * v.a.w;
            sT[r * 65 + c] = 0.f;
            sT[r * 65 + c + 1] = 0.f;
            sT[r * 65 + c + 2] = 0.f;
            sT[r * 65 + c + 3] = 0.f;
          });
  __syncthreads();
  // T = (I + A)^{-1}, A = diag(beta) M, in shared memory (leading dimension 65): diagonal 16 x 16
  // blocks by substitution, then the blocks below them by distance, T_IJ = -T_II sum_K A_IK T_KJ
  if (tid < 64) {
    const int I = tid >> 4, j = tid & 15;
    float x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = (m == j) ? 1.f : 0.f;
#pragma unroll
    for (int m = 0; m < 15; ++m) {
      const float xm = x[m];
#pragma unroll
      for (int i = m + 1; i < 16; ++i) x[i] = fmaf(-sA[(16 * I + i) * 65 + 16 * I + m], xm, x[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sT[(16 * I + i) * 65 + 16 * I + j] = x[i];
  }
  __syncthreads();
  for (int dd = 1; dd < 4; ++dd) {
    // Y_IJ = sum_{K=J}^{I-1} A_IK T_KJ for the 4 - dd blocks at this distance, parked in the (zero)
    // blocks above the diagonal (row block J, column block I), which the result never reads
    const int nb = 4 - dd;
    for (int e = tid; e < nb * 256; e += kBwdThreads) {
      const int J = e >> 8, I = J + dd, r = (e >> 4) & 15, c = e & 15;
      float y = 0.f;
      for (int k = 16 * J; k < 16 * I; ++k) y = fmaf(sA[(16 * I + r) * 65 + k], sT[k * 65 + 16 * J + c], y);
      sT[(16 * J + r) * 65 + 16 * I + c] = y;
    }
    __syncthreads();
    for (int e = tid; e < nb * 256; e += kBwdThreads) {
      const int J = e >> 8, I = J + dd, r = (e >> 4) & 15, c = e & 15;
      float t = 0.f;
      for (int k = 0; k <= r; ++k) t = fmaf(sT[(16 * I + r) * 65 + 16 * I + k], sT[(16 * J + k) * 65 + 16 * I + c], t);
      sT[(16 * I + r) * 65 + 16 * J + c] = -t;
    }
    __syncthreads();
    for (int e = tid; e < nb * 256; e += kBwdThreads) {
      const int J = e >> 8, I = J + dd, r = (e >> 4) & 15, c = e & 15;
      sT[(16 * J + r) * 65 + 16 * I + c] = 0.f;
    }
    __syncthreads();
  }
  ew<kB2>(kQ4,
            [&](int i) {
              const int r = (4 * i) >> 6, c = (4 * i) & (C - 1);
              const float4 t = make_float4(sT[r * 65 + c], sT[r * 65 + c + 1], sT[r * 65 + c + 2], sT[r * 65 + c + 3]);
              return F4x2{t, mul4(t, ld4(s + SC_BETA + c))};
            },
            [&](int i, F4x2 v) {
              st4(Tout + 4 * i, v.a);
              st4(s + SC_TB + 4 * i, v.b);
              st4(TBout + 4 * i, v.b);
            });
  __syncthreads();
}

// The gradient kernel's part of a chunk's prologue: V and dO (fp32, rows past the chunk's end zero)
// and beta into the CTA's scratch; the other element-wise factors come from the prep kernel's output.
__device__ void load_v_do_beta(const BwdParams& P, const Chunk& ch, float* s) {
  const FwdParams& p = P.f;
  const int H = p.num_heads, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r0 = warp; r0 < C; r0 += 2 * (kBwdThreads / 32)) {
    float4 v4[2], o4[2];
    float br[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + u * (kBwdThreads / 32);
      v4[u] = o4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      br[u] = 0.f;
      if (r < ch.len) {
        const size_t row = (size_t)(ch.t0 + r) * H + ch.h;
        v4[u] = ld_bf16x4(p.v + row * D + 4 * lane);
        o4[u] = ld_bf16x4(P.d_out + row * D + 4 * lane);
        br[u] = __bfloat162float(p.beta[row]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + u * (kBwdThreads / 32);
      st4(s + SC_V + r * D + 4 * lane, v4[u]);
      st4(s + SC_DO + r * D + 4 * lane, o4[u]);
      if (lane == 0) s[SC_BETA + r] = r < ch.len ? sigmoid_acc(br[u]) : 0.f;
    }
  }
  __syncthreads();
}

// The decay-weighted products of dM and dP (lower triangular, stored adjacent as XX = [dM; dP],
// 128 x 64) with khat, for rows r:  X1[r] = sum_{s<=r} dM[r][s] khat_s e^{Gamma_r - Gamma_s} and
// X3[r] = sum_{s<=r} dP[r][s] khat_s e^{Gamma_r - Gamma_s}, per block J of s against rho_J = Gamma at
// the end of block J: XX[., J cols] (khat_J e^{rho_J - Gamma}) times e^{Gamma_r - rho_J} (the rows
// above block J add zeros).  X3 is added to out2; X1 is added to dkh and khat X1 to dG, row block J
// as soon as block J of s (the last to reach it) is done, the later rows' partial sums kept in acc.
// T: a 128 x 128 temporary.
__device__ void gated_lower2(const Fac& F, float* dkh, float* dG, float* acc, float* out2, const float* XX, float* T,
                             float* R, GemmSmem& gsm) {
  for (int J = 0; J < 4; ++J) {
    const int r0 = 16 * J;
    const float* rho = F.G + (16 * J + 15) * D;
    ew<kB1>(16 * D / 4,
            [&](int i) {
              const int c = (4 * i) & (D - 1), e = r0 * D + 4 * i;
              return mul4(ld4(F.kh + e), dexp4(sub4(ld4(rho + c), ld4(F.G + e))));
            },
            [&](int i, float4 v) { st4(R + 4 * i, v); });
    __syncthreads();
    gemm(T, D, mat(XX + r0, C), mat(R, D), 2 * C, D, 16, 1.f, false, 0, gsm);
    ew<kB4>((C - r0) * D / 4,
            [&](int i) {
              const int c = (4 * i) & (D - 1), e = r0 * D + 4 * i;
              const float4 f = dexp4(sub4(ld4(F.G + e), ld4(rho + c)));
              float4 v1 = mul4(ld4(T + e), f);
              if (J > 0) v1 = add4(v1, ld4(acc + e));
              const float4 v3 = add4(mul4(ld4(T + C * D + e), f), ld4(out2 + e));
              if (i < 16 * D / 4)  // row block J: X1 complete
                return F4x4{add4(ld4(dkh + e), v1), add4(ld4(dG + e), mul4(ld4(F.kh + e), v1)), v3, {}};
              return F4x4{v1, {}, v3, {}};
            },
            [&](int i, F4x4 v) {
              const int e = r0 * D + 4 * i;
              if (i < 16 * D / 4) {
                st4(dkh + e, v.a);
                st4(dG + e, v.b);
              } else {
                st4(acc + e, v.a);
              }
              st4(out2 + e, v.c);
            });
    __syncthreads();
  }
}

// The transposed decay-weighted products, for rows s:  X[s] = sum_{r>=s} (dM[r][s] khat_r + scale
// dP[r][s] qhat_r) e^{Gamma_r - Gamma_s}, per block K of r against rho_K = Gamma at the end of block
// K - 1 (0 for K = 0): the rows s < 16 (K + 1) of dM[K rows, .]^T (khat_K e^{Gamma - rho_K}) +
// dP[K rows, .]^T (scale qhat_K e^{Gamma - rho_K}), times e^{rho_K - Gamma_s}.  X is added to dkh and
// -khat X to dG, row block K as soon as block K of r (the last to reach it) is done, the earlier
// rows' partial sums kept in acc.
__device__ void gated_upper2(const Fac& F, float* dkh, float* dG, float* acc, const float* dM, const float* dP,
                             float scale, float* R, float* L, GemmSmem& gsm) {
  for (int K = 3; K >= 0; --K) {
    const int r0 = 16 * K, ns = 16 * (K + 1);
    const float* rho = F.G + (16 * K - 1) * D;
    ew<kB2>(16 * D / 4,
            [&](int i) {
              const int c = (4 * i) & (D - 1), e = r0 * D + 4 * i;
              const float4 r4 = K == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(rho + c);
              const float4 f = dexp4(sub4(ld4(F.G + e), r4));
              return F4x2{mul4(ld4(F.kh + e), f), scl4(mul4(ld4(F.qh + e), f), scale)};
            },
            [&](int i, F4x2 v) {
              st4(R + 4 * i, v.a);
              st4(R + 16 * D + 4 * i, v.b);
            });
    __syncthreads();
    // [dM[K rows, .]^T | dP[K rows, .]^T] [R_k; R_q]: one product of depth 32
    gemm(L, D, mat2(dM + r0 * C, dP + r0 * C, 16, C, true), mat(R, D), ns, D, 32, 1.f, false, 0, gsm);
    ew<kB2>(ns * D / 4,
            [&](int i) {
              const int c = (4 * i) & (D - 1), e = 4 * i;
              const float4 r4 = K == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : ld4(rho + c);
              float4 v = mul4(ld4(L + 4 * i), dexp4(sub4(r4, ld4(F.G + e))));
              if (K < 3) v = add4(v, ld4(acc + e));
              if (i >= r0 * D / 4)  // row block K: X complete
                return F4x2{add4(ld4(dkh + e), v), sub4(ld4(dG + e), mul4(ld4(F.kh + e), v))};
              return F4x2{v, {}};
            },
            [&](int i, F4x2 v) {
              const int e = 4 * i;
              if (i >= r0 * D / 4) {
                st4(dkh + e, v.a);
                st4(dG + e, v.b);
              } else {
                st4(acc + e, v.a);
              }
            });
    __syncthreads();
  }
}

// ------------------------------------------------------------------------- kernels
__global__ void bwd_chunk_table_kernel(BwdParams P, int32_t* chunk_off) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const FwdParams& p = P.f;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    chunk_off[0] = 0;
  }
  bool bad = false;
  for (int n = tid; n < p.num_seqs; n += 1024) bad |= !seq_entries_ok(p, n);
  if (__syncthreads_or(bad)) {
    for (int n = tid; n <= p.num_seqs; n += 1024) chunk_off[n] = 0;
    if (tid == 0 && p.status) atomicOr(p.status, kStatusBadSeqlens);
    return;
  }
  for (int base = 0; base < p.num_seqs; base += 1024) {
    const int n = base + tid;
    int32_t cnt = 0;
    if (n < p.num_seqs) {
      int64_t bos, eos;
      seq_range(p, n, bos, eos);
      cnt = (int32_t)((eos - bos + C - 1) / C);
    }
    int32_t x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int32_t w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int32_t incl = carry + x + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (n < p.num_seqs) chunk_off[n + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
}

// the prep kernel: the solve's two 64 x 65 tiles live in the staging buffer, which no product uses
// between the Gram product and the W product
using GemmSmemPrep = GemmSmemT<160>;
constexpr size_t kChunkSmem = sizeof(GemmSmemPrep);
static_assert(2 * 64 * 65 * sizeof(float) <= sizeof(GemmSmemPrep), "solve tiles");
constexpr size_t kGradSmem = sizeof(GemmSmem) + 4 * D * sizeof(float);        // + the dgamma partials

// Per chunk: W, Kt, P^T dO, (Qt - P W)^T dO and e^gamma for the state-gradient walk.
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_prep_kernel(BwdParams P, int64_t items) {
  extern __shared__ float4 smem4[];
  GemmSmemPrep& gsm = *reinterpret_cast<GemmSmemPrep*>(smem4);
  float* sT = reinterpret_cast<float*>(smem4);  // the solve's tiles (see kChunkSmem)
  float* sA = sT + 64 * 65;
  float* s = P.scratch + (size_t)blockIdx.x * kScratchFloats;
  const int tid = threadIdx.x;
  const float scale = P.f.scale;
  const int64_t n_items = min(items, (int64_t)P.chunk_off[P.f.num_seqs] * P.f.num_heads);
  for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x) {
    const Chunk ch = locate(P, it);
    float* pr = P.prep + (size_t)it * kPrepFloats;
    const Fac F = fac_of(pr);  // khat, qhat, Gamma and Kg straight to the output (the gradient kernel reads them)
    chunk_factors(P, ch, s, F, gsm, sT, sA, pr + PR_M, pr + PR_T, pr + PR_TB);
    // W = T_b Kg (to the output); Kt = khat e^{gamma - Gamma}; X = Qt - P W
    gemm(pr + PR_W, D, mat(s + SC_TB, C), mat(F.kg, D), C, D, C, 1.f, false, 0, gsm);
    const float* gam = F.G + (C - 1) * D;
    ew<kB2>(kF4,
              [&](int i) {
                const int c = (4 * i) & (D - 1);
                const float4 G = ld4(F.G + 4 * i);
                return F4x2{mul4(ld4(F.kh + 4 * i), dexp4(sub4(ld4(gam + c), G))),
                            scl4(mul4(ld4(F.qh + 4 * i), dexp4(G)), scale)};
              },
              [&](int i, F4x2 v) {
                st4(pr + PR_KT + 4 * i, v.a);
                st4(s + SC_X + 4 * i, v.b);
              });
    if (tid < D) pr[PR_EG + tid] = s[SC_EG + tid];
    __syncthreads();
    gemm(s + SC_X, D, mat(s + SC_P, C), mat(pr + PR_W, D), C, D, C, -1.f, true, 0, gsm);
    gemm<2>(pr + PR_Y, D, mat(s + SC_X, D, true), mat(s + SC_DO, D), D, D, C, 1.f, false, 0, gsm);  // dO: bf16 values
    gemm<2>(pr + PR_PDO, D, mat(s + SC_P, C, true), mat(s + SC_DO, D), C, D, C, 1.f, false, 0, gsm);
  }
}

// The state walk's outputs: E = Kt dS' (to e) and dDelta = P^T dO + E (to dd); the next dS' =
// Diag(e^gamma) dS' + (Qt - P W)^T dO - W^T E.
struct EpiE {
  static constexpr bool kLoadsFirst = true;
  float* e;
  float* dd;
  const float* pdo;
  __device__ __forceinline__ float2 load(int i, int j) const {
    return *reinterpret_cast<const float2*>(pdo + (size_t)i * D + j);
  }
  __device__ __forceinline__ void store(int i, int j, float2 v, float2 l) const {
    *reinterpret_cast<float2*>(e + (size_t)i * D + j) = v;
    *reinterpret_cast<float2*>(dd + (size_t)i * D + j) = make_float2(v.x + l.x, v.y + l.y);
  }
};
struct EpiS {
  static constexpr bool kLoadsFirst = true;
  float* out;
  const float* dsp;
  const float* y;
  const float* eg;
  __device__ __forceinline__ float2 load(int i, int j) const {
    const float2 a = *reinterpret_cast<const float2*>(dsp + (size_t)i * D + j);
    const float2 b = *reinterpret_cast<const float2*>(y + (size_t)i * D + j);
    const float e = eg[i];
    return make_float2(fmaf(e, a.x, b.x), fmaf(e, a.y, b.y));
  }
  __device__ __forceinline__ void store(int i, int j, float2 v, float2 l) const {
    *reinterpret_cast<float2*>(out + (size_t)i * D + j) = make_float2(l.x - v.x, l.y - v.y);
  }
};

// One CTA per (sequence, head): from the last chunk to the first, with dS' the gradient of the
// chunk's end state (d_final, or 0, for the last chunk):
//   E = Kt dS',  dDelta = P^T dO + E,  dS = Diag(e^gamma) dS' + (Qt - P W)^T dO - W^T E.
// dS' of chunk j is kept in the chunk's slot (the input of bwd_grad_kernel); the dS of chunk 0 is
// the initial state's gradient.
// 512 threads: two groups of 8 warps, each with its own staging buffer, run the two halves of each
// product at once (E by column halves, the next dS' by row halves).
__global__ void __launch_bounds__(2 * kBwdThreads, 1) bwd_state_kernel(BwdParams P) {
  extern __shared__ float4 smem4[];
  GemmSmem* gsm = reinterpret_cast<GemmSmem*>(smem4);  // [2]
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int n = blockIdx.x / H, h = blockIdx.x - n * H;
  const int tid = threadIdx.x;
  int64_t bos, eos;
  seq_range(p, n, bos, eos);
  const int64_t c0 = P.chunk_off[n], nch = P.chunk_off[n + 1] - c0;
  const int64_t slot0 = bos / C + n;
  float* e_buf = P.scratch + (size_t)blockIdx.x * kF;  // E
  const float* dfin = P.d_final ? P.d_final + ((size_t)n * H + h) * kStateElems : nullptr;
  float* d_init = P.d_initial ? P.d_initial + ((size_t)n * H + h) * kStateElems : nullptr;
  constexpr int kS4 = (int)kStateElems / 4;
  auto copy_final = [&](float* dst) {
    ew<kB1>(kS4, [&](int i) { return dfin ? ld4(dfin + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f); },
              [&](int i, float4 v) { st4(dst + 4 * i, v); });
  };
  if (nch == 0) {
    if (d_init && tid < kBwdThreads) copy_final(d_init);
    return;
  }
  if (tid < kBwdThreads) copy_final(P.dsp + ((size_t)(slot0 + nch - 1) * H + h) * kStateElems);
  __syncthreads();
  const bool hi = tid >= kBwdThreads;  // the second group
  for (int64_t j = nch - 1; j >= 0; --j) {
    const int64_t it = (c0 + j) * H + h;
    const float* pr = P.prep + (size_t)it * kPrepFloats;
    if (j > 0) {
      // the previous chunk's factors into L2 while this one runs
      const char* nx = reinterpret_cast<const char*>(P.prep + (size_t)(it - H) * kPrepFloats);
      for (int l = tid; l < (int)(PR_M * sizeof(float) / 128); l += 2 * kBwdThreads)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(nx + (size_t)l * 128));
    }
    const float* dsp = P.dsp + ((size_t)(slot0 + j) * H + h) * kStateElems;
    float* nxt = j > 0 ? P.dsp + ((size_t)(slot0 + j - 1) * H + h) * kStateElems : d_init;
    float* dd = P.dd + (size_t)it * kF;
    // E = Kt dS' and dDelta, columns 64 g .. + 63 by group g
    if (!hi)
      gemm_t<4, 64, 128, EpiE, 0, HalfCta<1>>(mat(pr + PR_KT, D), mat(dsp, D), C, 64, D, gsm[0],
                                             EpiE{e_buf, dd, pr + PR_PDO});
    else
      gemm_t<4, 64, 128, EpiE, 0, HalfCta<2>>(mat(pr + PR_KT, D), mat(dsp + 64, D), C, 64, D, gsm[1],
                                             EpiE{e_buf + 64, dd + 64, pr + PR_PDO + 64});
    __syncthreads();
    // the next dS', rows 64 g .. + 63 by group g
    if (nxt) {
      if (!hi)
        gemm_t<4, 128, 128, EpiS, 0, HalfCta<1>>(mat(pr + PR_W, D, true), mat(e_buf, D), C, D, C, gsm[0],
                                                EpiS{nxt, dsp, pr + PR_Y, pr + PR_EG});
      else
        gemm_t<4, 128, 128, EpiS, 0, HalfCta<2>>(mat(pr + PR_W + 64, D, true), mat(e_buf, D), C, D, C, gsm[1],
                                                EpiS{nxt + 64 * D, dsp + 64 * D, pr + PR_Y + 64 * D, pr + PR_EG + 64});
    }
    __syncthreads();
  }
}

// dT_b's second product, which also writes dT = dT_b diag(beta) (to da)
struct EpiDtb {
  static constexpr bool kLoadsFirst = false;
  float* dtb;
  float* da;
  const float* beta;
  __device__ __forceinline__ float2 load(int i, int j) const {
    return *reinterpret_cast<const float2*>(dtb + (size_t)i * C + j);
  }
  __device__ __forceinline__ void store(int i, int j, float2 v, float2 l) const {
    const float2 o = make_float2(v.x + l.x, v.y + l.y);
    *reinterpret_cast<float2*>(dtb + (size_t)i * C + j) = o;
    *reinterpret_cast<float2*>(da + (size_t)i * C + j) = make_float2(o.x * beta[j], o.y * beta[j + 1]);
  }
};
// dv = T_b^T dDelta, rows of the chunk, as bf16 to the output
struct EpiDv {
  static constexpr bool kLoadsFirst = false;
  __nv_bfloat16* dv;  // the chunk's first row of this head
  int64_t row_stride;
  int len;
  __device__ __forceinline__ float2 load(int, int) const { return make_float2(0.f, 0.f); }
  __device__ __forceinline__ void store(int i, int j, float2 v, float2) const {
    if (i < len) *reinterpret_cast<__nv_bfloat162*>(dv + i * row_stride + j) = __floats2bfloat162_rn(v.x, v.y);
  }
};

// Per chunk: the gradients of khat, qhat, log alpha and beta (to the partial buffers) and dv.
__global__ void __launch_bounds__(kBwdThreads, 2) bwd_grad_kernel(BwdParams P, int64_t items) {
  extern __shared__ float4 smem4[];
  GemmSmem& gsm = *reinterpret_cast<GemmSmem*>(smem4);
  float* part = reinterpret_cast<float*>(smem4) + sizeof(GemmSmem) / 4;  // 4 x 128 floats
  float* s = P.scratch + (size_t)blockIdx.x * kScratchFloats;
  const FwdParams& p = P.f;
  const int H = p.num_heads;
  const int tid = threadIdx.x;
  const float scale = p.scale;
  const int64_t rows_total = (p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs) * H;
  const int64_t n_items = min(items, (int64_t)P.chunk_off[p.num_seqs] * H);
  for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x) {
    const Chunk ch = locate(P, it);
    // M, T = (I + A)^{-1}, T_b = T diag(beta), khat, qhat, Gamma and Kg as the prep kernel stored them
    float* pr = P.prep + (size_t)it * kPrepFloats;
    const Fac F = fac_of(pr);
    load_v_do_beta(P, ch, s);
    const float* Mp = pr + PR_M;
    const float* Tp = pr + PR_T;
    const float* TBp = pr + PR_TB;
    const float* S = P.ckpt + ((size_t)ch.slot * H + ch.h) * kStateElems;   // S^T [v][k]: S(k, v) = S[v * 128 + k]
    const float* dSp = P.dsp + ((size_t)ch.slot * H + ch.h) * kStateElems;  // [k][v]
    const float* dD = P.dd + (size_t)it * kF;
    // Delta = T_b V - W S (W = T_b Kg as the prep kernel stored it)
    gemm<2>(s + SC_D, D, mat(TBp, C), mat(s + SC_V, D), C, D, C, 1.f, false, 0, gsm);  // V: bf16 values
    gemm(s + SC_D, D, mat(pr + PR_W, D), mat(S, D, true), C, D, D, -1.f, true, 0, gsm);
    // dKt = Delta dS'^T;  dQs = dO S^T;  dW = -dDelta S^T;  dP = tril(dO Delta^T)
    gemm(s + SC_DKT, D, mat(s + SC_D, D), mat(dSp, D, true), C, D, D, 1.f, false, 0, gsm);
    gemm<1>(s + SC_DQS, D, mat(s + SC_DO, D), mat(S, D), C, D, D, 1.f, false, 0, gsm);  // dO: bf16 values
    gemm(s + SC_DW, D, mat(dD, D), mat(S, D), C, D, D, -1.f, false, 0, gsm);
    gemm<1>(s + SC_DP, C, mat(s + SC_DO, D), mat(s + SC_D, D, true), C, C, D, 1.f, false, 2, gsm);
    // dgamma from the state: e^gamma_k sum_v S(k, v) dS'(k, v): thread k and half h of the v range
    // (reads of S coalesced over k, each thread's row of dS' read in order, 4 values a load)
    {
      const int k = tid & (D - 1), h = tid >> 7;
      float acc = 0.f;
#pragma unroll 4
      for (int v = 64 * h; v < 64 * h + 64; v += 4) {
        const float4 d = ld4(dSp + (size_t)k * D + v);
        acc = fmaf(S[(size_t)v * D + k], d.x, acc);
        acc = fmaf(S[(size_t)(v + 1) * D + k], d.y, acc);
        acc = fmaf(S[(size_t)(v + 2) * D + k], d.z, acc);
        acc = fmaf(S[(size_t)(v + 3) * D + k], d.w, acc);
      }
      if (h == 1) s[SC_DGAM + k] = acc;
      __syncthreads();
      if (h == 0) s[SC_DGAM + k] = pr[PR_EG + k] * (acc + s[SC_DGAM + k]);
    }
    // dT_b = dDelta V^T + dW Kg^T;  dv = T_b^T dDelta;  dKg = T_b^T dW
    gemm<2>(s + SC_DTB, C, mat(dD, D), mat(s + SC_V, D, true), C, C, D, 1.f, false, 0, gsm);
    // with dT = dT_b diag(beta) (to DA)
    gemm_e(mat(s + SC_DW, D), mat(F.kg, D, true), C, C, D, gsm, EpiDtb{s + SC_DTB, s + SC_DA, s + SC_BETA});
    gemm_e(mat(TBp, C, true), mat(dD, D), C, D, C, gsm,
           EpiDv{P.dv + ((size_t)ch.t0 * H + ch.h) * D, (int64_t)H * D, ch.len});
    gemm(s + SC_DKG, D, mat(TBp, C, true), mat(s + SC_DW, D), C, D, C, 1.f, false, 0, gsm);
    // dbeta (columns) = colsum(dT_b o T); dA = strict_tril(-T^T dT T^T)
    {
      // thread (column c, quarter q of the rows), the quarters added by shuffles
      const int c = tid >> 2, q = tid & 3;
      float acc = 0.f;
#pragma unroll
      for (int r = 16 * q; r < 16 * q + 16; ++r) acc = fmaf(s[SC_DTB + r * C + c], Tp[r * C + c], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (q == 0) s[SC_DB + c] = acc;
    }
    __syncthreads();
    // T^T dT into DTB (dead)
    gemm(s + SC_DTB, C, mat(Tp, C, true), mat(s + SC_DA, C), C, C, C, 1.f, false, 0, gsm);
    gemm(s + SC_DA, C, mat(s + SC_DTB, C), mat(Tp, C, true), C, C, C, -1.f, false, 1, gsm);
    // dbeta (rows) += rowsum(dA o M); dM = diag(beta) dA (in place)
    {
      // thread (row r, quarter q of the columns)
      const int r = tid >> 2, q = tid & 3;
      float acc = 0.f;
#pragma unroll
      for (int c = 16 * q; c < 16 * q + 16; ++c) acc = fmaf(s[SC_DA + r * C + c], Mp[r * C + c], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (q == 0) s[SC_DB + r] += acc;
    }
    __syncthreads();
    ew<kB1>(kQ4, [&](int i) { return scl4(ld4(s + SC_DA + 4 * i), s[SC_BETA + ((4 * i) >> 6)]); },
              [&](int i, float4 v) { st4(s + SC_DA + 4 * i, v); });
    // the decay-weighted products: X1 = gated(dM, khat) and X3 = gated(dP, khat) (rows r), X2 = the
    // transposed one of dM with khat and X4 = scale x that of dP with qhat (rows s)
    float* dkh = s + SC_DKG;  // becomes dkhat: e^Gamma dKg first
    float* dqh = s + SC_DQS;  // becomes dqhat / scale: e^Gamma dO S^T first
    float* dG = s + SC_W;     // dGamma
    const float* gam = F.G + (C - 1) * D;
    ew<kB4>(kF4,
              [&](int i) {
                const int c = (4 * i) & (D - 1);
                const float4 G = ld4(F.G + 4 * i), eG = dexp4(G);
                const float4 a = mul4(ld4(dkh + 4 * i), eG);                                   // e^Gamma dKg
                const float4 b = mul4(ld4(s + SC_DKT + 4 * i), dexp4(sub4(ld4(gam + c), G)));  // e^{gamma-Gamma} dKt
                return F4x4{add4(a, b), mul4(ld4(F.kh + 4 * i), sub4(a, b)), b, mul4(ld4(dqh + 4 * i), eG)};
              },
              [&](int i, F4x4 v) {
                st4(dkh + 4 * i, v.a);
                st4(dG + 4 * i, v.b);
                st4(s + SC_DKT + 4 * i, v.c);
                st4(dqh + 4 * i, v.d);
              });
    __syncthreads();
    // X1 (into dkhat and dGamma) and X3 (added to dqhat / scale) in one pass; V and dO are dead: their
    // 2 x 64 x 128 floats hold the 128 x 128 temporary.  Delta and dW are dead as well.
    gated_lower2(F, dkh, dG, s + SC_D, dqh, s + SC_DA, s + SC_DO, s + SC_DW, gsm);
    gated_upper2(F, dkh, dG, s + SC_D, s + SC_DA, s + SC_DP, scale, s + SC_DW, s + SC_L, gsm);  // X2 + X4
    // dgamma: the state term plus sum_r khat e^{gamma-Gamma} dKt; then dlog alpha by a reverse running sum
    {
      // thread (channel k, half h of the rows): the half's share of dgamma and the total of its
      // dGamma (through shared memory, 2 x 2 x 128 floats), then the reverse running sum over its
      // half, the lower half starting from the upper half's total
      const int k = tid & (D - 1), h = tid >> 7;
      float pg = 0.f, tot = 0.f;
#pragma unroll 8
      for (int r = 32 * h; r < 32 * h + 32; ++r) {
        const int e = r * D + k;
        pg = fmaf(F.kh[e], s[SC_DKT + e], pg);
        tot += dG[e] + scale * F.qh[e] * dqh[e];
      }
      part[h * D + k] = pg;
      part[2 * D + h * D + k] = tot;
      __syncthreads();
      const float dgam = s[SC_DGAM + k] + part[k] + part[D + k];
      float run = h == 0 ? part[3 * D + k] : 0.f;
      for (int r0 = 32 * h + 16; r0 >= 32 * h; r0 -= 16) {
        float col[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int e = (r0 + r) * D + k;
          col[r] = dG[e] + scale * F.qh[e] * dqh[e];
        }
#pragma unroll
        for (int r = 15; r >= 0; --r) {
          run += col[r];
          dG[(r0 + r) * D + k] = run + dgam;
        }
      }
    }
    __syncthreads();
    // to the partial buffers: dqhat, dkhat, dlog alpha, dbeta
    float* pq = P.part;
    float* pk = P.part + (size_t)rows_total * D;
    float* pa = P.part + 2 * (size_t)rows_total * D;
    float* pb = P.part + 3 * (size_t)rows_total * D;
    ew<kB4>(ch.len * (D / 4),
              [&](int i) { return F4x4{scl4(ld4(dqh + 4 * i), scale), ld4(dkh + 4 * i), ld4(dG + 4 * i), {}}; },
              [&](int i, F4x4 v) {
                const int r = i >> 5, c4 = i & 31;
                const size_t o = ((size_t)(ch.t0 + r) * H + ch.h) * D + 4 * c4;
                st4(pq + o, v.a);
                st4(pk + o, v.b);
                st4(pa + o, v.c);
              });
    if (tid < ch.len) pb[(size_t)(ch.t0 + tid) * H + ch.h] = s[SC_DB + tid];
    __syncthreads();
  }
}

// Adds nothing up: applies the derivatives of the transforms to the per-token partials (dq and dk
// through the L2 norms, dg through the gate, dbeta through the sigmoid).  A CTA takes one head and
// a run of tokens (one warp per token at a time, a lane per 4 channels) and adds its sums of the
// gate-parameter gradients with one atomic per value.
__global__ void __launch_bounds__(256) bwd_finish_kernel(BwdParams P, int64_t tokens, int tokens_per_cta) {
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
  // a token per warp at a time, all of its loads issued before any store (the outputs may alias
  // nothing the compiler can prove, so it would not hoist a load above an earlier store)
  constexpr int kTok = 1;  // tokens per warp at a time (2 measured slower: 128 registers, fewer CTAs)
  for (int64_t t0 = t_begin + warp; t0 < t_end; t0 += 8 * kTok) {
    float4 a4[kTok], b4[kTok], c4[kTok], q4[kTok], k4[kTok], g4[kTok];
    float gb[kTok], bb[kTok];
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      const int64_t t = t0 + 8 * u;
      const size_t row = (size_t)(t < t_end ? t : t0) * H + h;
      const float* base = P.part + row * D + 4 * lane;
      a4[u] = *reinterpret_cast<const float4*>(base);
      b4[u] = *reinterpret_cast<const float4*>(base + (size_t)rows_total * D);
      c4[u] = *reinterpret_cast<const float4*>(base + 2 * (size_t)rows_total * D);
      gb[u] = P.part[3 * (size_t)rows_total * D + row];
      q4[u] = ld_bf16x4(p.q + row * D + 4 * lane);
      k4[u] = ld_bf16x4(p.k + row * D + 4 * lane);
      g4[u] = ld_bf16x4(p.g + row * D + 4 * lane);
      bb[u] = __bfloat162float(p.beta[row]);
    }
#pragma unroll
    for (int u = 0; u < kTok; ++u) {
      const int64_t t = t0 + 8 * u;
      if (t >= t_end) break;
      const size_t row = (size_t)t * H + h;
      // dq, dk: (dxhat - xhat (xhat . dxhat)) / n
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float4 x4 = which == 0 ? q4[u] : k4[u];
        const float4 g = which == 0 ? a4[u] : b4[u];
        const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, gx[4] = {g.x, g.y, g.z, g.w};
        float ss = xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float nrm = sqrtf(ss + kL2Eps);
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
      // dg through the gate (log alpha = lower_bound sigmoid(x), x = e^{A_log} (g + dt_bias)); the
      // sums for dt_bias and A_log
      const float gv[4] = {g4[u].x, g4[u].y, g4[u].z, g4[u].w}, ga[4] = {c4[u].x, c4[u].y, c4[u].z, c4[u].w};
      float dg[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float x = ea * (gv[j] + dts[j]);
        const float sg = sigmoid_acc(x);
        const float dx = ga[j] * p.lower_bound * sg * (1.f - sg);
        dg[j] = dx * ea;
        ddt[j] += dg[j];
        dA = fmaf(dx, x, dA);
      }
      st_bf16x4(P.dg + row * D + 4 * lane, dg[0], dg[1], dg[2], dg[3]);
      if (lane == 0) {
        const float b = sigmoid_acc(bb[u]);
        P.dbeta[row] = __float2bfloat16_rn(gb[u] * b * (1.f - b));
      }
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

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Workspace regions (byte offsets), all 256-aligned: the forward's split workspace (its header holds
// the status word), the checkpoints it writes, the chunk table, prep, dsp, dd, the partials, and the
// CTA scratch.
struct BwdLayout {
  size_t fwd, ckpt, out, table, prep, dsp, dd, part, scratch, total;
  int64_t chunk_cap;
};

constexpr int64_t kBwdMaxCtas = 296;  // persistent CTAs of the chunk-parallel kernels (bounds the scratch)
constexpr int kFinishTokens = 64;     // tokens per CTA of the finishing kernel

BwdLayout bwd_layout(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t t = total_tokens > 0 ? total_tokens : 0, n = num_seqs > 0 ? num_seqs : 0;
  const int64_t hh = num_heads > 0 ? num_heads : 0;
  BwdLayout L;
  L.chunk_cap = t / C + n;  // sum over sequences of ceil(len / 64)
  const int64_t slots = t / C + n + 1;
  size_t o = 0;
  L.fwd = o;
  o += align256(split_workspace_bytes(t, (int32_t)hh, (int32_t)n));
  L.ckpt = o;
  o += align256(checkpoint_bytes(t, (int32_t)hh, (int32_t)n));
  L.out = o;  // the recomputed forward's output (not used)
  o += align256((size_t)t * hh * D * sizeof(__nv_bfloat16));
  L.table = o;
  o += align256((size_t)(n + 1) * sizeof(int32_t));
  L.prep = o;
  o += align256((size_t)L.chunk_cap * hh * kPrepFloats * sizeof(float));
  L.dsp = o;
  o += align256((size_t)slots * hh * kStateElems * sizeof(float));
  L.dd = o;
  o += align256((size_t)L.chunk_cap * hh * kF * sizeof(float));
  L.part = o;
  o += align256((3 * (size_t)t * hh * D + (size_t)t * hh) * sizeof(float));
  L.scratch = o;  // the chunk-parallel kernels' CTAs, or one E buffer per unit for the state kernel
  const size_t sc = (size_t)kBwdMaxCtas * kScratchFloats, se = (size_t)(n * hh) * kF;
  o += align256((sc > se ? sc : se) * sizeof(float));
  L.total = o;
  return L;
}

}  // namespace

size_t bwd_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  return bwd_layout(total_tokens, num_heads, num_seqs).total;
}

cudaError_t launch_bwd(const FwdParams& f, const __nv_bfloat16* d_out, const float* d_final, __nv_bfloat16* dq,
                       __nv_bfloat16* dk, __nv_bfloat16* dv, __nv_bfloat16* dg, __nv_bfloat16* dbeta, float* dA_log,
                       float* ddt_bias, float* d_initial, const float* checkpoints, void* workspace,
                       cudaStream_t stream) {
  const int64_t units = (int64_t)f.num_seqs * f.num_heads;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(dA_log, 0, sizeof(float) * f.num_heads, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ddt_bias, 0, sizeof(float) * f.num_heads * kHeadDim, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, kWorkspaceHeader, stream);  // status word, counters
  if (e != cudaSuccess || units == 0) return e;
  const int64_t tokens = f.cu_seqlens ? f.seqlen : f.seqlen * f.num_seqs;
  const BwdLayout L = bwd_layout(tokens, f.num_heads, f.num_seqs);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdParams P;
  P.f = f;
  P.f.status = reinterpret_cast<uint32_t*>(ws + L.fwd);
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
  P.chunk_off = reinterpret_cast<int32_t*>(ws + L.table);
  P.prep = reinterpret_cast<float*>(ws + L.prep);
  P.dsp = reinterpret_cast<float*>(ws + L.dsp);
  P.dd = reinterpret_cast<float*>(ws + L.dd);
  P.part = reinterpret_cast<float*>(ws + L.part);
  P.scratch = reinterpret_cast<float*>(ws + L.scratch);
  if (checkpoints || tokens == 0) {
    P.ckpt = checkpoints;
  } else {
    // the forward, storing the chunk-start states (its outputs are not needed)
    float* ck = reinterpret_cast<float*>(ws + L.ckpt);
    FwdParams ff = P.f;
    ff.out = reinterpret_cast<__nv_bfloat16*>(ws + L.out);
    ff.final_state = nullptr;
    if ((e = launch_split(ff, ws + L.fwd, stream, ck)) != cudaSuccess) return e;
    P.ckpt = ck;
  }
  bwd_chunk_table_kernel<<<1, 1024, 0, stream>>>(P, const_cast<int32_t*>(P.chunk_off));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t items = L.chunk_cap * f.num_heads;  // an upper bound; items past the last chunk are skipped
  static bool attr_done[64] = {};
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if ((e = cudaFuncSetAttribute(bwd_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kChunkSmem)) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGradSmem)) !=
            cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(2 * sizeof(GemmSmem)))) != cudaSuccess)
      return e;
    // the rest of each SM's 256 KB as L1: shared memory for exactly two CTAs (one for the walk)
    auto carve = [](size_t bytes, int ctas) { return (int)((ctas * (bytes + 1024) * 100 + 232447) / 233472); };
    if ((e = cudaFuncSetAttribute(bwd_prep_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carve(kChunkSmem, 2))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_grad_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carve(kGradSmem, 2))) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_state_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carve(2 * sizeof(GemmSmem), 1))) != cudaSuccess)
      return e;
    attr_done[dev] = true;
  }
  int64_t grid = 2 * (int64_t)sms;
  if (grid > kBwdMaxCtas) grid = kBwdMaxCtas;
  if (grid > items) grid = items;
  if (tokens > 0) {
    bwd_prep_kernel<<<(unsigned)grid, kBwdThreads, kChunkSmem, stream>>>(P, items);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  bwd_state_kernel<<<(unsigned)units, 2 * kBwdThreads, 2 * sizeof(GemmSmem), stream>>>(P);  // also when every document is empty
  if ((e = cudaGetLastError()) != cudaSuccess || tokens == 0) return e;
  bwd_grad_kernel<<<(unsigned)grid, kBwdThreads, kGradSmem, stream>>>(P, items);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 fgrid((unsigned)((tokens + kFinishTokens - 1) / kFinishTokens), (unsigned)f.num_heads);
  bwd_finish_kernel<<<fgrid, 256, 0, stream>>>(P, tokens, kFinishTokens);
  return cudaGetLastError();
}

}  // namespace kda
