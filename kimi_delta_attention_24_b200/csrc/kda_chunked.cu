// Chunked KDA forward for sm_100a: one fused kernel, one CTA per (sequence, head) unit.
//
// Kimi Delta Attention (FlashKDA `fwd`, fla `chunk_kda`; vLLM PR #54859 report and "What CUDA
// Version Is Required to Use FlashKDA?", Usage Examples) is the gated delta rule
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t.
// The kernel walks the unit's tokens in chunks of C = 64 and uses the chunked (WY/UT) form.  With
// Gamma the in-chunk cumulative log-decay, Khat/Qhat the L2-normalised keys/queries,
//   A = strict_tril(diag(beta) (Khat e^Gamma)(Khat e^-Gamma)^T),  T = (I + A)^{-1},
//   P = scale * tril((Qhat e^Gamma)(Khat e^-Gamma)^T),  T_b = T diag(beta),
//   W = T_b (Khat e^Gamma),  U = T_b V,  Qtil = scale Qhat e^Gamma,  Ktil = Khat e^{Gamma_C - Gamma},
// each chunk does
//   Delta = U - W S,   O = Qtil S + P Delta = (Qtil - P W) S + P U,
//   S <- Diag(e^{Gamma_C}) S + Ktil^T Delta.
//
// Per chunk (everything on-chip; HBM sees the raw inputs once and the output once):
//   prologue  (CUDA cores) raw q, k, g rows straight from global memory into registers; L2 norms,
//             sigmoid(beta), safe gate alpha = exp(lower_bound * sigmoid(exp(A_log)(g + dt_bias)));
//             decays as running products of alpha inside each 16-row sub-block (exponent
//             referencing: every factor stays in [e^-80, e^80] for lower_bound >= -5); the bf16 MMA
//             operands, with the norms, beta and scale folded in.  v arrives by TMA.
//   MMA_AP    [LK; LQ] x R_I^T per 16-row sub-block I -> the gated K K^T and Q K^T blocks (TMEM).
//   assemble  A (fp32, shared memory) and P (bf16 operand).
//   solve     T = (I + A)^{-1}: the four 16x16 diagonal blocks by forward substitution, then the
//             off-diagonal blocks T_IJ = -T_II sum_K A_IK T_KJ, all in fp32; T_b as a bf16 hi+lo pair.
//   MMA_PT    P (T_hi + T_lo), read back as a hi+lo pair.
//   MMA_X     [T_b; P T_b] (hi + lo) x [Khat e^Gamma | V] -> [W | U; P W | P U] in TMEM.
//   WQ        [-W; Qtil - P W] written back to TMEM as the A operand of MMA1.
//   MMA1      accumulates [-W; Qtil - P W] x S onto [U; P U]  ->  [Delta; O].
//   ep1       Delta (bf16 hi+lo operand), O -> global bf16.
//   MMA2      Ktil^T (Delta_hi + Delta_lo); ep2: S = e^{Gamma_C} S + Ktil^T Delta (fp32 registers),
//             plus its bf16 copy (the B operand of the next MMA1).
// The hi+lo pairs matter when keys are nearly collinear: T then has entries close to -beta that
// cancel against the diagonal, and a chunk's Delta rows telescope, so a single bf16 rounding of
// T_b, P T_b or Delta would cost several percent of the state.  Ktil is built from the raw bf16 k
// (its 1/|k| is applied to Delta) so that equal keys round identically.
#include <cuda.h>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;          // chunk length
constexpr int D = kHeadDim;    // 128
constexpr int kThreads = 256;  // 8 warps
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (bytes from a 1024-aligned base).  "MN tile" = [2 blocks of 64 columns]
// [64 rows][128 B] with the 128-byte swizzle; "K tile" = [2 blocks of 64 K][rows][128 B].
constexpr uint32_t OFF_V = 0;            // v (TMA), MN-major B of MMA_X
constexpr uint32_t OFF_XK = 16384;       // Khat e^Gamma, MN-major B of MMA_X
constexpr uint32_t OFF_QB = 32768;       // Qtil (bf16), read when forming Qtil - P W
constexpr uint32_t OFF_KT = 49152;       // Ktil (raw k), MN-major A of MMA2
constexpr uint32_t OFF_SCR = 65536;      // scratch, 73728 bytes:
constexpr uint32_t OFF_LKQ = OFF_SCR;    //   [LK; LQ] K tile, 128 rows (prologue -> MMA_AP)
constexpr uint32_t OFF_R = OFF_SCR + 32768;  //   R_0..R_3 K tile, 160 rows (prologue -> MMA_AP)
constexpr uint32_t R_KBLK = 160 * 128;
constexpr uint32_t OFF_AS = OFF_SCR;             // A fp32 64 x 68 (assemble -> solve)
constexpr uint32_t OFF_TS = OFF_SCR + 17408;     // T fp32 64 x 68 (solve)
constexpr uint32_t OFF_YS = OFF_SCR + 17408 * 2; // solve temporaries, 3 x 16 x 16 fp32
constexpr uint32_t AS_LD = 68;
constexpr uint32_t OFF_TP = OFF_SCR + 40960;     // [T_hi; P -> (P T)_hi] 128 x 64, K tile
constexpr uint32_t OFF_TL = OFF_SCR + 57344;     // [T_lo; (P T)_lo]
constexpr uint32_t OFF_DL = OFF_SCR;             // Delta hi, MN tile (ep1 -> MMA2)
constexpr uint32_t OFF_DLLO = OFF_SCR + 16384;   // Delta lo
constexpr uint32_t OFF_S = OFF_SCR + 73728;      // S bf16, MN-major B of MMA1, 2 blocks x 128 rows
constexpr uint32_t OFF_SC = OFF_S + 32768;       // scalars
constexpr uint32_t SC_BETA = 0;                  // float[64]
constexpr uint32_t SC_IK = 256;                  // float[64] 1/|k_r| (0 for rows past the end)
constexpr uint32_t SC_GAM = 512;                 // float[128] e^{Gamma_C}
constexpr uint32_t SC_TOT = 1024;                // float[8][128] per-warp alpha products
constexpr uint32_t SC_BAR = 5120;                // 2 mbarriers
constexpr uint32_t SC_TMEM = 5136;
constexpr uint32_t SC_ABORT = 5140;
constexpr uint32_t SMEM_BYTES = OFF_SC + 5248;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;

// first row of R_I inside the R tile: 0, 16, 48, 96 (R_I holds 16 (I+1) rows)
__host__ __device__ constexpr uint32_t row_off(int I) { return 8u * I * (I + 1); }

// TMEM columns: AP products at row_off(I) (N = 16 (I+1)), then P T at 0..63, then
// [W PW] at 0..127 and [U PU] at 128..255; [-W; Qtil - PW] packed bf16 at 0..63; MMA1 and MMA2
// accumulate at 128..255.
constexpr uint32_t TM_WQ = 0;
constexpr uint32_t TM_UP = 128;
constexpr uint32_t kTmemCols = 256;

struct TensorMaps {
  CUtensorMap v;
};

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
__device__ __forceinline__ void bar_sync() { __syncthreads(); }

__global__ void __launch_bounds__(kThreads, 1)
    chunked_kernel(const __grid_constant__ TensorMaps maps, FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* sc_beta = reinterpret_cast<float*>(sm + OFF_SC + SC_BETA);
  float* sc_ik = reinterpret_cast<float*>(sm + OFF_SC + SC_IK);
  float* sc_gam = reinterpret_cast<float*>(sm + OFF_SC + SC_GAM);
  float* sc_tot = reinterpret_cast<float*>(sm + OFF_SC + SC_TOT);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + OFF_SC + SC_BAR);
  uint64_t* mma_bar = tma_bar + 1;
  uint32_t* sc_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SC + SC_TMEM);
  volatile int* sc_abort = reinterpret_cast<volatile int*>(sm + OFF_SC + SC_ABORT);
  float* As = reinterpret_cast<float*>(sm + OFF_AS);
  float* Ts = reinterpret_cast<float*>(sm + OFF_TS);
  float* Ys = reinterpret_cast<float*>(sm + OFF_YS);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, half = warp >> 2;
  const int H = p.num_heads;
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  int64_t bos, eos;
  seq_range(p, n, bos, eos);
  const int64_t seq_len = eos - bos;
  const int nchunks = (int)((seq_len + C - 1) / C);

  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    *sc_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.v);
  }
  if (warp == 0) {
    tmem_alloc(sc_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  bar_sync();
  tc_fence_after();
  const uint32_t tmem = *sc_tmem;
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;  // this warp's TMEM lane quarter

  // ---- state: thread owns row k = 32*quarter + lane, columns [64*half, 64*half + 64)
  const int srow = 32 * quarter + lane;
  const size_t soff = ((size_t)n * H + h) * (size_t)D * D;
  float S[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const int col = 64 * half + j;
    float s = 0.f;
    if (p.initial_state)
      s = p.state_transposed ? p.initial_state[soff + (size_t)col * D + srow]
                             : p.initial_state[soff + (size_t)srow * D + col];
    S[j] = s;
  }
  auto store_state_bf16 = [&]() {
    uint8_t* base = sm + OFF_S + half * (128 * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 w;
      w.x = pack_bf16(S[8 * c + 0], S[8 * c + 1]);
      w.y = pack_bf16(S[8 * c + 2], S[8 * c + 3]);
      w.z = pack_bf16(S[8 * c + 4], S[8 * c + 5]);
      w.w = pack_bf16(S[8 * c + 6], S[8 * c + 7]);
      *reinterpret_cast<uint4*>(base + sw128(srow, c)) = w;
    }
  };
  store_state_bf16();

  // prologue mapping: warp w owns chunk rows 8w..8w+7, lane owns channels 4*lane..4*lane+3
  const float gate_a = __expf(p.A_log[h]);
  const float4 dtb = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
  // exp(-a (g + dt)) = exp2(ga * g + gb)
  const float ga = -gate_a * kLog2e;
  const float gb[4] = {ga * dtb.x, ga * dtb.y, ga * dtb.z, ga * dtb.w};
  const float lb2 = p.lower_bound * kLog2e;
  const int kb = lane >> 4;                       // 64-channel block
  const uint32_t lane_chunk = (lane & 15) >> 1;   // 16-byte chunk within the 128-byte row
  const uint32_t lane_sub = (lane & 1) * 8;       // byte within the chunk
  const int blk = warp >> 1;                      // 16-row sub-block of this warp's rows
  const bool upper_half = warp & 1;               // rows 8..15 of the sub-block

  uint32_t tma_phase = 0, mma_phase = 0;
  if (tid == 0 && nchunks > 0) {
    mbar_arrive_expect_tx(tma_bar, 16384);
    tma_load_3d(sm + OFF_V, &maps.v, tma_bar, 0, h, (int)bos);
    tma_load_3d(sm + OFF_V + 8192, &maps.v, tma_bar, 64, h, (int)bos);
  }

  auto wait_all = [&](uint64_t* bar, uint32_t& phase) -> bool {
    const bool ok = mbar_wait(bar, phase, kWaitLimitNs);
    phase ^= 1u;
    if (!ok) {
      *sc_abort = 1;
      if (p.status) atomicOr(p.status, kStatusTimeout);
    }
    bar_sync();
    return *sc_abort == 0;
  };
  auto publish = [&]() {
    fence_proxy_async();
    tc_fence_before();
    bar_sync();
  };

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int len = (int)((eos - t0) < (int64_t)C ? (eos - t0) : (int64_t)C);

    // ================================================================ prologue
    {
      uint2 qr[8], kr[8];
      float al[8][4];
      float ssq[8], ssk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const bool valid = r < len;
        const size_t off = ((size_t)(t0 + r) * H + h) * D + 4 * lane;
        uint2 gr = make_uint2(0, 0);
        qr[i] = make_uint2(0, 0);
        kr[i] = make_uint2(0, 0);
        if (valid) {
          qr[i] = ldg_u2(p.q + off);
          kr[i] = ldg_u2(p.k + off);
          gr = ldg_u2(p.g + off);
        }
        const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        ssq[i] = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
        ssk[i] = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
        const float2 g01 = unpack_bf16(gr.x), g23 = unpack_bf16(gr.y);
        const float gv[4] = {g01.x, g01.y, g23.x, g23.y};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // alpha = 2^(lb*log2e * sigmoid(a (g + dt)))
          const float z = exp2f(fmaf(ga, gv[j], gb[j]));
          const float sig = __fdividef(1.0f, 1.0f + z);
          al[i][j] = valid ? exp2f(lb2 * sig) : 1.0f;
        }
      }
      // row sums of squares: transpose-reduce 16 values over the 32 lanes; lane l ends with the
      // total of value (l >> 1): q rows 0..7, then k rows 0..7
      float inv;
      {
        float v16[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v16[i] = ssq[i];
          v16[8 + i] = ssk[i];
        }
        const bool b4 = lane & 16;
        float w8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float send = b4 ? v16[j] : v16[j + 8];
          const float keep = b4 ? v16[j + 8] : v16[j];
          w8[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        const bool b3 = lane & 8;
        float w4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float send = b3 ? w8[j] : w8[j + 4];
          const float keep = b3 ? w8[j + 4] : w8[j];
          w4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const bool b2 = lane & 4;
        float w2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float send = b2 ? w4[j] : w4[j + 2];
          const float keep = b2 ? w4[j + 2] : w4[j];
          w2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
        const bool b1 = lane & 2;
        float w1 = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? w2[0] : w2[1], 2);
        w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
        inv = rsqrtf(w1 + kL2Eps);
      }
      // beta of row 8w + lane (lanes 0..7), broadcast to the warp
      float beta_l = 0.f;
      if (lane < 8) {
        const int r = 8 * warp + lane;
        if (r < len) beta_l = fast_sigmoid(__bfloat162float(p.beta[(size_t)(t0 + r) * H + h]));
        sc_beta[r] = beta_l;
      }
      float iq[8], ik[8], bt[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        iq[i] = __shfl_sync(0xffffffffu, inv, 2 * i) * p.scale;
        ik[i] = __shfl_sync(0xffffffffu, inv, 16 + 2 * i);
        bt[i] = __shfl_sync(0xffffffffu, beta_l, i);
      }
      if (lane < 8) {
        const int r = 8 * warp + lane;
        float v = ik[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) v = (lane == i) ? ik[i] : v;
        sc_ik[r] = (r < len) ? v : 0.f;
      }
      // running products of alpha over this warp's 8 rows (prefix in place) and their suffixes
      float suf[8][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        suf[7][j] = 1.f;
#pragma unroll
        for (int i = 6; i >= 0; --i) suf[i][j] = suf[i + 1][j] * al[i + 1][j];
#pragma unroll
        for (int i = 1; i < 8; ++i) al[i][j] *= al[i - 1][j];
      }
      reinterpret_cast<float4*>(sc_tot + warp * 128)[lane] = make_float4(al[7][0], al[7][1], al[7][2], al[7][3]);
      bar_sync();
      // sub-block totals b_J = e^{Gamma at the end of J - Gamma at its start}
      float bJ[4][4];
#pragma unroll
      for (int J = 0; J < 4; ++J) {
        const float4 t0v = reinterpret_cast<const float4*>(sc_tot + (2 * J) * 128)[lane];
        const float4 t1v = reinterpret_cast<const float4*>(sc_tot + (2 * J + 1) * 128)[lane];
        bJ[J][0] = t0v.x * t1v.x;
        bJ[J][1] = t0v.y * t1v.y;
        bJ[J][2] = t0v.z * t1v.z;
        bJ[J][3] = t0v.w * t1v.w;
      }
      const float4 partner = reinterpret_cast<const float4*>(sc_tot + (warp ^ 1) * 128)[lane];
      const float pt[4] = {partner.x, partner.y, partner.z, partner.w};
      // e_i = prod of alpha from the sub-block start to row i; f_i = prod after row i to its end
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (upper_half) al[i][j] *= pt[j];
          else suf[i][j] *= pt[j];
        }
      float pre[4], post[4], cI[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float a = 1.f, z = 1.f;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
          if (J < blk) a *= bJ[J][j];
          if (J > blk) z *= bJ[J][j];
        }
        pre[j] = a;
        post[j] = z;
        float m = 1.f;
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          cI[I][j] = (I == blk) ? 1.0f / bJ[blk][j] : m;
          if (I > blk) m *= bJ[I][j];
        }
      }
      if (warp == 0)
        reinterpret_cast<float4*>(sc_gam)[lane] =
            make_float4(bJ[0][0] * bJ[1][0] * bJ[2][0] * bJ[3][0], bJ[0][1] * bJ[1][1] * bJ[2][1] * bJ[3][1],
                        bJ[0][2] * bJ[1][2] * bJ[2][2] * bJ[3][2], bJ[0][3] * bJ[1][3] * bJ[2][3] * bJ[3][3]);
      // operands, one row at a time
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        const float qv[4] = {q01.x, q01.y, q23.x, q23.y};
        const float kv[4] = {k01.x, k01.y, k23.x, k23.y};
        float lk[4], lq[4], kf[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float kh = kv[j] * ik[i];
          lq[j] = qv[j] * iq[i] * al[i][j];   // scale * qhat * e
          lk[j] = kh * al[i][j];              // khat * e
          kf[j] = kh * suf[i][j];             // khat * f
        }
        const uint32_t offk = kb * 16384 + sw128(r, lane_chunk) + lane_sub;
        const uint32_t offq = kb * 16384 + sw128(64 + r, lane_chunk) + lane_sub;
        const uint32_t off64 = kb * 8192 + sw128(r, lane_chunk) + lane_sub;
        const float b = bt[i];
        *reinterpret_cast<uint2*>(sm + OFF_LKQ + offk) =
            make_uint2(pack_bf16(lk[0] * b, lk[1] * b), pack_bf16(lk[2] * b, lk[3] * b));
        *reinterpret_cast<uint2*>(sm + OFF_LKQ + offq) =
            make_uint2(pack_bf16(lq[0], lq[1]), pack_bf16(lq[2], lq[3]));
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          if (I < blk) continue;
          const uint32_t off = kb * R_KBLK + sw128(row_off(I) + r, lane_chunk) + lane_sub;
          *reinterpret_cast<uint2*>(sm + OFF_R + off) =
              make_uint2(pack_bf16(kf[0] * cI[I][0], kf[1] * cI[I][1]), pack_bf16(kf[2] * cI[I][2], kf[3] * cI[I][3]));
        }
        *reinterpret_cast<uint2*>(sm + OFF_XK + off64) =
            make_uint2(pack_bf16(lk[0] * pre[0], lk[1] * pre[1]), pack_bf16(lk[2] * pre[2], lk[3] * pre[3]));
        *reinterpret_cast<uint2*>(sm + OFF_QB + off64) =
            make_uint2(pack_bf16(lq[0] * pre[0], lq[1] * pre[1]), pack_bf16(lq[2] * pre[2], lq[3] * pre[3]));
        *reinterpret_cast<uint2*>(sm + OFF_KT + off64) =
            make_uint2(pack_bf16(kv[0] * suf[i][0] * post[0], kv[1] * suf[i][1] * post[1]),
                       pack_bf16(kv[2] * suf[i][2] * post[2], kv[3] * suf[i][3] * post[3]));
      }
    }
    publish();

    // ================================================================ MMA_AP
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int I = 0; I < 4; ++I) {
        const uint32_t idesc = idesc_bf16(128, 16 * (I + 1), false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = sdesc_sw128(sbase + OFF_LKQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(sbase + OFF_R + (ks >> 2) * R_KBLK + row_off(I) * 128 + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem + row_off(I), a, b, idesc, ks > 0);
        }
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();

    // ================================================================ assemble A and P
    {
      const int R = 32 * quarter + lane;  // accumulator row
      const bool qside = R >= 64;
      const int r = R & 63;
      const int Ib = r >> 4;
      const int q2 = quarter & 1;         // rows 32*q2 .. 32*q2+31 of this side: blocks 2 q2, 2 q2 + 1
      const bool skip = (half == 1) && (q2 == 0);  // s in [32, 64) lies above the diagonal there
      float d[32];
      if (!skip) {
        float d0[32], d1[32];
        tmem_ld32(tmem + lane_base + row_off(2 * q2) + 32 * half, d0);
        tmem_ld32(tmem + lane_base + row_off(2 * q2 + 1) + 32 * half, d1);
        const bool odd = Ib & 1;
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = odd ? d1[j] : d0[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = 0.f;
      }
      if (!qside) {
        float* dst = As + r * AS_LD + 32 * half;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int s = 32 * half + j;
          float4 o;
          o.x = (s + 0 < r) ? d[j + 0] : 0.f;
          o.y = (s + 1 < r) ? d[j + 1] : 0.f;
          o.z = (s + 2 < r) ? d[j + 2] : 0.f;
          o.w = (s + 3 < r) ? d[j + 3] : 0.f;
          *reinterpret_cast<float4*>(dst + j) = o;
        }
      } else {
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          float v8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int s = 32 * half + 8 * cch + u;
            v8[u] = (s <= r) ? d[8 * cch + u] : 0.f;
          }
          uint4 w;
          w.x = pack_bf16(v8[0], v8[1]);
          w.y = pack_bf16(v8[2], v8[3]);
          w.z = pack_bf16(v8[4], v8[5]);
          w.w = pack_bf16(v8[6], v8[7]);
          *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(64 + r, 4 * half + cch)) = w;
        }
      }
    }
    tc_fence_before();
    bar_sync();

    // ================================================================ solve T = (I + A)^{-1}
    // diagonal 16x16 blocks: warp I, lane j < 16 computes column j by forward substitution
    if (warp < 4 && lane < 16) {
      const int I = warp, j = lane;
      const float* a = As + (16 * I) * AS_LD + 16 * I;
      float x[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) x[m] = (m == j) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc = fmaf(a[i * AS_LD + m], x[m], acc);
        x[i] = (i > j) ? -acc : x[i];
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Ts[(16 * I + i) * AS_LD + 16 * I + j] = x[i];
    }
    bar_sync();
    // off-diagonal blocks by distance dd below the diagonal: T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ
#pragma unroll 1
    for (int dd = 1; dd < 4; ++dd) {
      const int nblk = 4 - dd;
      const int job = tid;                  // (block, row i, 4-column group)
      const bool active = job < nblk * 64;
      const int bI = dd + job / 64;         // block row I (J = I - dd)
      const int bJ = bI - dd;
      const int i = (job % 64) >> 2, cg = job & 3;
      if (active) {
        float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
        for (int K = bJ; K < bI; ++K) {
          const float* arow = As + (16 * bI + i) * AS_LD + 16 * K;
          const float* tcol = Ts + (16 * K) * AS_LD + 16 * bJ + 4 * cg;
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const float a = arow[m];
            const float4 t = *reinterpret_cast<const float4*>(tcol + m * AS_LD);
            y0 = fmaf(a, t.x, y0);
            y1 = fmaf(a, t.y, y1);
            y2 = fmaf(a, t.z, y2);
            y3 = fmaf(a, t.w, y3);
          }
        }
        *reinterpret_cast<float4*>(Ys + (job / 64) * 256 + i * 16 + 4 * cg) = make_float4(y0, y1, y2, y3);
      }
      bar_sync();
      if (active) {
        const float* trow = Ts + (16 * bI + i) * AS_LD + 16 * bI;
        const float* ycol = Ys + (job / 64) * 256 + 4 * cg;
        float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const float t = (m <= i) ? trow[m] : 0.f;
          const float4 y = *reinterpret_cast<const float4*>(ycol + m * 16);
          z0 = fmaf(t, y.x, z0);
          z1 = fmaf(t, y.y, z1);
          z2 = fmaf(t, y.z, z2);
          z3 = fmaf(t, y.w, z3);
        }
        *reinterpret_cast<float4*>(Ts + (16 * bI + i) * AS_LD + 16 * bJ + 4 * cg) = make_float4(-z0, -z1, -z2, -z3);
      }
      bar_sync();
    }
    // T_b = T diag(beta) as hi/lo bf16 into rows 0..63 of TP / TL (upper blocks are zero)
    {
      const int r = tid >> 2, c16 = tid & 3;   // row r, columns 16*c16 .. 16*c16+15
      const int I = r >> 4;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int c0 = 16 * c16 + 8 * hh;
        uint4 wh, wl;
        if (c16 > I) {
          wh = make_uint4(0, 0, 0, 0);
          wl = wh;
        } else {
          const float4 t0v = *reinterpret_cast<const float4*>(Ts + r * AS_LD + c0);
          const float4 t1v = *reinterpret_cast<const float4*>(Ts + r * AS_LD + c0 + 4);
          const float4 b0 = *reinterpret_cast<const float4*>(sc_beta + c0);
          const float4 b1 = *reinterpret_cast<const float4*>(sc_beta + c0 + 4);
          split2(t0v.x * b0.x, t0v.y * b0.y, wh.x, wl.x);
          split2(t0v.z * b0.z, t0v.w * b0.w, wh.y, wl.y);
          split2(t1v.x * b1.x, t1v.y * b1.y, wh.z, wl.z);
          split2(t1v.z * b1.z, t1v.w * b1.w, wh.w, wl.w);
        }
        *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(r, c0 >> 3)) = wh;
        *reinterpret_cast<uint4*>(sm + OFF_TL + sw128(r, c0 >> 3)) = wl;
      }
    }
    publish();

    // ================================================================ MMA_PT: [T_hi; P] x (T_hi + T_lo)
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + OFF_TP + (ks & 3) * 32, 16, 1024);
        const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem, a, b, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();
    if (quarter >= 2) {
      const int r = 32 * quarter + lane - 64;
      float d[32];
      tmem_ld32(tmem + lane_base + 32 * half, d);
#pragma unroll
      for (int cch = 0; cch < 4; ++cch) {
        uint4 wh, wl;
        split2(d[8 * cch + 0], d[8 * cch + 1], wh.x, wl.x);
        split2(d[8 * cch + 2], d[8 * cch + 3], wh.y, wl.y);
        split2(d[8 * cch + 4], d[8 * cch + 5], wh.z, wl.z);
        split2(d[8 * cch + 6], d[8 * cch + 7], wh.w, wl.w);
        *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(64 + r, 4 * half + cch)) = wh;
        *reinterpret_cast<uint4*>(sm + OFF_TL + sw128(64 + r, 4 * half + cch)) = wl;
      }
    }
    publish();

    // ================================================================ MMA_X: [T_b; P T_b] x [Xk | V]
    if (!wait_all(tma_bar, tma_phase)) break;   // v tile of this chunk
    if (len < C) {  // rows past the document end (another document's or zero-filled) -> 0
      for (int idx = tid; idx < 2 * (C - len) * 8; idx += kThreads) {
        const int blk2 = idx / ((C - len) * 8), rem = idx % ((C - len) * 8);
        const int r = len + rem / 8;
        *reinterpret_cast<uint4*>(sm + OFF_V + blk2 * 8192 + sw128(r, rem & 7)) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async();
      bar_sync();
    }
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 32, 16, 1024);
        const uint64_t bk = sdesc_sw128(sbase + OFF_XK + (ks & 3) * 2048, 8192, 1024);
        const uint64_t bv = sdesc_sw128(sbase + OFF_V + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem + TM_WQ, a, bk, idesc, ks > 0);
        umma_bf16(tmem + TM_UP, a, bv, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();
    // the v tile is free: fetch the next chunk's
    if (tid == 0 && c + 1 < nchunks) {
      mbar_arrive_expect_tx(tma_bar, 16384);
      tma_load_3d(sm + OFF_V, &maps.v, tma_bar, 0, h, (int)(t0 + C));
      tma_load_3d(sm + OFF_V + 8192, &maps.v, tma_bar, 64, h, (int)(t0 + C));
    }

    // ================================================================ [-W; Qtil - PW] -> TMEM (bf16)
    {
      const int R = 32 * quarter + lane;
      uint32_t packed[32];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + TM_WQ + 64 * half + 32 * part, d);
        if (R >= 64) {
          const int r = R - 64;
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            const uint4 qb = *reinterpret_cast<const uint4*>(sm + OFF_QB + half * 8192 + sw128(r, 4 * part + cch));
            const float2 a0 = unpack_bf16(qb.x), a1 = unpack_bf16(qb.y), a2 = unpack_bf16(qb.z),
                         a3 = unpack_bf16(qb.w);
            packed[16 * part + 4 * cch + 0] = pack_bf16(a0.x - d[8 * cch + 0], a0.y - d[8 * cch + 1]);
            packed[16 * part + 4 * cch + 1] = pack_bf16(a1.x - d[8 * cch + 2], a1.y - d[8 * cch + 3]);
            packed[16 * part + 4 * cch + 2] = pack_bf16(a2.x - d[8 * cch + 4], a2.y - d[8 * cch + 5]);
            packed[16 * part + 4 * cch + 3] = pack_bf16(a3.x - d[8 * cch + 6], a3.y - d[8 * cch + 7]);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) packed[16 * part + u] = pack_bf16(-d[2 * u], -d[2 * u + 1]);
        }
      }
      tc_fence_before();
      bar_sync();   // every thread has read [W PW] before any column 0..63 is overwritten
      tc_fence_after();
      tmem_st32(tmem + lane_base + TM_WQ + 32 * half, packed);
      tmem_wait_st();
    }
    publish();

    // ================================================================ MMA1: [U; PU] += [-W; Qtil - PW] x S
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t b = sdesc_sw128(sbase + OFF_S + ks * 2048, 16384, 1024);
        umma_bf16_tmem_a(tmem + TM_UP, tmem + TM_WQ + 8 * ks, b, idesc, 1);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();

    // ================================================================ ep1: Delta and O
    {
      const int R = 32 * quarter + lane;
      const int r = R & 63;
      const float ikr = sc_ik[r];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + TM_UP + 64 * half + 32 * part, d);
        if (R < 64) {
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            uint4 wh, wl;
            split2(d[8 * cch + 0] * ikr, d[8 * cch + 1] * ikr, wh.x, wl.x);
            split2(d[8 * cch + 2] * ikr, d[8 * cch + 3] * ikr, wh.y, wl.y);
            split2(d[8 * cch + 4] * ikr, d[8 * cch + 5] * ikr, wh.z, wl.z);
            split2(d[8 * cch + 6] * ikr, d[8 * cch + 7] * ikr, wh.w, wl.w);
            *reinterpret_cast<uint4*>(sm + OFF_DL + half * 8192 + sw128(r, 4 * part + cch)) = wh;
            *reinterpret_cast<uint4*>(sm + OFF_DLLO + half * 8192 + sw128(r, 4 * part + cch)) = wl;
          }
        } else if (r < len) {
          __nv_bfloat16* orow = p.out + ((size_t)(t0 + r) * H + h) * D + 64 * half + 32 * part;
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            uint4 w;
            w.x = pack_bf16(d[8 * cch + 0], d[8 * cch + 1]);
            w.y = pack_bf16(d[8 * cch + 2], d[8 * cch + 3]);
            w.z = pack_bf16(d[8 * cch + 4], d[8 * cch + 5]);
            w.w = pack_bf16(d[8 * cch + 6], d[8 * cch + 7]);
            reinterpret_cast<uint4*>(orow)[cch] = w;
          }
        }
      }
    }
    publish();

    // ================================================================ MMA2: Ktil^T x (Delta_hi + Delta_lo)
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, true, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + OFF_KT + (ks & 3) * 2048, 8192, 1024);
        const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_DL : OFF_DLLO) + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem + TM_UP, a, b, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();

    // ================================================================ ep2: state update
    {
      const float gam = sc_gam[srow];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + TM_UP + 64 * half + 32 * part, d);
#pragma unroll
        for (int j = 0; j < 32; ++j) S[32 * part + j] = fmaf(gam, S[32 * part + j], d[j]);
      }
      store_state_bf16();
    }
    publish();
  }

  // ---- final state
  if (p.final_state && *sc_abort == 0) {
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const int col = 64 * half + j;
      if (p.state_transposed) p.final_state[soff + (size_t)col * D + srow] = S[j];
      else p.final_state[soff + (size_t)srow * D + col] = S[j];
    }
  }
  tc_fence_before();
  bar_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// [tokens, H, 128] bf16 viewed as 3-D (channel, head, token); box 64 channels x 1 head x 64 tokens.
bool make_token_map(CUtensorMap* map, const void* base, int64_t tokens, int H) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)(tokens > 0 ? tokens : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)C};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunked(const FwdParams& p, cudaStream_t stream) {
  const int64_t units = (int64_t)p.num_seqs * p.num_heads;
  if (units == 0) return cudaSuccess;
  const int64_t tokens = p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs;
  TensorMaps maps;
  if (!make_token_map(&maps.v, p.v, tokens, p.num_heads)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(chunked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  chunked_kernel<<<(unsigned)units, kThreads, SMEM_ALLOC, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace kda
