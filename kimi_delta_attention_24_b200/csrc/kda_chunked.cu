// Chunked KDA forward for sm_100a: one fused kernel, one CTA per (sequence, head) unit.
//
// Kimi Delta Attention (FlashKDA `fwd`, fla `chunk_kda`; vLLM PR #54859 report and "What CUDA
// Version Is Required to Use FlashKDA?", Usage Examples) is the gated delta rule
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t.
// The kernel walks the unit's tokens in chunks of C = 64 and uses the chunked (WY/UT) form:
// with Gamma the in-chunk cumulative log-decay, A the strictly-lower gated key Gram matrix,
// T = (I + A)^{-1}, W = T diag(beta) (Khat * e^Gamma), U = T diag(beta) V,
// P = scale * tril_incl((Qhat * e^Gamma)(Khat * e^-Gamma)^T):
//     Delta = U - W S,   O = Qtil S + P Delta,   S <- Diag(e^{Gamma_C}) S + Ktil^T Delta,
// Qtil = scale * Qhat * e^Gamma, Ktil = Khat * e^{Gamma_C - Gamma}.  The output is rewritten as
// O = (Qtil - P W) S + P U so that the recurrence needs two MMAs per chunk.
//
// Per chunk (all on-chip; HBM sees the raw inputs once and the output once):
//   TMA       q, k, g, v tiles [64 tokens x 128] bf16, 128-byte swizzle, into shared memory.
//   prologue  (CUDA cores) L2 norms, sigmoid(beta), safe gate, block-relative Gamma, and the bf16
//             MMA operands with exponent referencing per 16-row sub-block (every factor within
//             [e^-80, e^80] for lower_bound >= -5).
//   MMA_AP    [LK; LQ] x R_I^T for the 4 sub-blocks -> gated K K^T and Q K^T blocks (TMEM).
//   assemble  A (fp32, shared) and P (bf16 operand).
//   solve     T = (I + A)^{-1} by fp32 forward substitution; T_beta = T diag(beta), kept as a
//             bf16 pair hi + lo (about 16 significant bits).
//   MMA_PT    P (T_hi + T_lo), read back as a hi + lo pair.
//   MMA_X     [T_beta; P T_beta] x [Khat e^Gamma | V] -> [W U; PW PU] (TMEM), hi and lo parts.
//   MMA1      [W; Qtil - PW] x S -> [W S; (Qtil - PW) S]
//   ep1       Delta = U - W S (bf16 hi + lo operands), O = (Qtil - PW) S + P U -> global bf16.
//   MMA2      Ktil^T (Delta_hi + Delta_lo); ep2: S = e^{Gamma_C} S + Ktil^T Delta (fp32 registers)
//             + bf16 copy.
// The hi + lo pairs matter when keys are nearly collinear: T then has entries close to -beta
// that cancel against the diagonal, and the chunk's Delta rows telescope, so single bf16
// rounding of T_beta, P T_beta or Delta would cost several percent of the state.
// The state stays in registers (fp32 master) and shared memory (bf16 MMA operand) for the
// whole sequence.
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

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_Q = 0;            // q tile -> Qb = scale/|q| * q * e^Gamma (bf16)
constexpr uint32_t OFF_K = 16384;        // k tile -> Ktil (MN-major A operand of MMA2)
constexpr uint32_t OFF_G = 32768;        // g tile -> Xk = khat * e^Gamma (MN-major B of MMA_X)
constexpr uint32_t OFF_V = 49152;        // v tile (MN-major B of MMA_X)
constexpr uint32_t OFF_U = 65536;        // union region (73728 bytes)
constexpr uint32_t OFF_LKQ = OFF_U;      //   [LK; LQ] K-major, 2 k-blocks x 128 rows
constexpr uint32_t OFF_R = OFF_U + 32768;  // R_0..R_3 K-major, 2 k-blocks x 160 rows
constexpr uint32_t R_KBLK = 160 * 128;
constexpr uint32_t OFF_AS = OFF_U;       //   A (fp32, 64 x 68)
constexpr uint32_t AS_LD = 68;
constexpr uint32_t OFF_WQ = OFF_U + 18432;   // [W; Qtil - PW] K-major, 2 k-blocks x 128 rows
constexpr uint32_t OFF_DL = OFF_U + 18432;   // Delta (hi), MN-major B, 2 n-blocks x 64 rows (after MMA1)
constexpr uint32_t OFF_DLLO = OFF_U + 34816; // Delta (lo)
constexpr uint32_t OFF_TL = OFF_U + 51200;   // [T_lo; (P T_beta)_lo] 128 x 64, K-major
constexpr uint32_t OFF_TP = OFF_U + 73728;   // [T_beta; P] (later [T_beta; P T_beta]) 128 x 64
constexpr uint32_t OFF_S = OFF_TP + 16384;   // S bf16, MN-major B, 2 n-blocks x 128 rows
constexpr uint32_t OFF_SC = OFF_S + 32768;   // scalars
constexpr uint32_t SC_BETA = 0;              // float[64]
constexpr uint32_t SC_IK = 256;              // float[64] 1/|k|
constexpr uint32_t SC_IQS = 512;             // float[64] scale/|q|
constexpr uint32_t SC_GAM = 768;             // float[128] e^{Gamma_C}
constexpr uint32_t SC_CARRY = 1280;          // float[4][128]
constexpr uint32_t SC_LEND = 3328;           // float[4][128]
constexpr uint32_t SC_BAR = 5376;            // 2 mbarriers
constexpr uint32_t SC_TMEM = 5392;
constexpr uint32_t SC_ABORT = 5396;
constexpr uint32_t SMEM_BYTES = OFF_SC + 5504;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;

// first row of R_I inside the R tile: 0, 16, 48, 96 (R_I holds 16 (I+1) rows)
__host__ __device__ constexpr uint32_t row_off(int I) { return 8u * I * (I + 1); }

// TMEM column map (512 allocated).
constexpr uint32_t TM_AP = 0;    // 4 x 64 (sub-block products), later P T_beta, later [W PW | U PU]
constexpr uint32_t TM_X = 0;
constexpr uint32_t TM_REC = 256; // MMA1 / MMA2 results
constexpr uint32_t kTmemCols = 512;

struct TensorMaps {
  CUtensorMap q, k, v, g;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u));
}
// Eight floats as a bf16 pair: hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void split_pack(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * u], x[2 * u + 1]);
    const float2 bf = __bfloat1622float2(b);
    const __nv_bfloat162 c = __floats2bfloat162_rn(x[2 * u] - bf.x, x[2 * u + 1] - bf.y);
    h[u] = *reinterpret_cast<const uint32_t*>(&b);
    l[u] = *reinterpret_cast<const uint32_t*>(&c);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}
__device__ __forceinline__ float fast_sigmoid(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

__device__ __forceinline__ void bar_sync() { __syncthreads(); }

__global__ void __launch_bounds__(kThreads, 1)
    chunked_kernel(const __grid_constant__ TensorMaps maps, FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  float* sc_beta = reinterpret_cast<float*>(sm + OFF_SC + SC_BETA);
  float* sc_ik = reinterpret_cast<float*>(sm + OFF_SC + SC_IK);
  float* sc_iqs = reinterpret_cast<float*>(sm + OFF_SC + SC_IQS);
  float* sc_gam = reinterpret_cast<float*>(sm + OFF_SC + SC_GAM);
  float* sc_carry = reinterpret_cast<float*>(sm + OFF_SC + SC_CARRY);
  float* sc_lend = reinterpret_cast<float*>(sm + OFF_SC + SC_LEND);
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(sm + OFF_SC + SC_BAR);
  uint64_t* mma_bar = tma_bar + 1;
  uint32_t* sc_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SC + SC_TMEM);
  volatile int* sc_abort = reinterpret_cast<volatile int*>(sm + OFF_SC + SC_ABORT);
  float* As = reinterpret_cast<float*>(sm + OFF_AS);

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
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.g);
  }
  if (warp == 0) {
    tmem_alloc(sc_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  bar_sync();
  tc_fence_after();
  const uint32_t tmem = *sc_tmem;

  // ---- initial state: thread owns row k = 32*quarter + lane, columns [64*half, 64*half + 64)
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

  // per-lane constants of the prologue mapping: warp w owns chunk rows 8w..8w+7, lane owns
  // channels 4*lane .. 4*lane+3
  const float gate_a = __expf(p.A_log[h]);
  const float4 dtb = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
  const int kb = lane >> 4;                       // 64-channel block
  const uint32_t lane_chunk = (lane & 15) >> 1;   // 16-byte chunk within the 128-byte row
  const uint32_t lane_sub = (lane & 1) * 8;       // byte within the chunk
  const int blk = warp >> 1;                      // sub-block of this warp's rows

  uint32_t tma_phase = 0, mma_phase = 0;
  auto issue_tma = [&](int64_t t0, bool qgv, bool kk) {
    const int c2 = (int)t0;
    for (int b = 0; b < 2; ++b) {
      if (qgv) {
        tma_load_3d(sm + OFF_Q + b * 8192, &maps.q, tma_bar, 64 * b, h, c2);
        tma_load_3d(sm + OFF_G + b * 8192, &maps.g, tma_bar, 64 * b, h, c2);
        tma_load_3d(sm + OFF_V + b * 8192, &maps.v, tma_bar, 64 * b, h, c2);
      }
      if (kk) tma_load_3d(sm + OFF_K + b * 8192, &maps.k, tma_bar, 64 * b, h, c2);
    }
  };
  if (tid == 0 && nchunks > 0) {
    mbar_arrive_expect_tx(tma_bar, 4 * 16384);
    issue_tma(bos, true, true);
  }

  // Waits on an mbarrier phase; on timeout records the device error.  Every thread then meets
  // at a barrier and reads the shared abort flag, so all threads leave the loop together.
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
  // Makes this thread's shared-memory writes and TMEM reads visible/ordered before an MMA issue.
  auto publish = [&]() {
    fence_proxy_async();
    tc_fence_before();
    bar_sync();
  };

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int len = (int)((eos - t0) < (int64_t)C ? (eos - t0) : (int64_t)C);
    if (!wait_all(tma_bar, tma_phase)) break;

    // ================================================================ prologue
    {
      // raw q, k (bf16) of this thread's 8 rows x 4 channels
      uint2 qr[8], kr[8];
      float la[8][4];
      float ssq[8], ssk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const uint32_t off = kb * 8192 + sw128(r, lane_chunk) + lane_sub;
        const bool valid = r < len;
        qr[i] = valid ? *reinterpret_cast<const uint2*>(sm + OFF_Q + off) : make_uint2(0, 0);
        kr[i] = valid ? *reinterpret_cast<const uint2*>(sm + OFF_K + off) : make_uint2(0, 0);
        const uint2 gr = *reinterpret_cast<const uint2*>(sm + OFF_G + off);
        const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        ssq[i] = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
        ssk[i] = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
        const float2 g01 = unpack_bf16(gr.x), g23 = unpack_bf16(gr.y);
        const float lb = p.lower_bound;
        la[i][0] = valid ? lb * fast_sigmoid(gate_a * (g01.x + dtb.x)) : 0.f;
        la[i][1] = valid ? lb * fast_sigmoid(gate_a * (g01.y + dtb.y)) : 0.f;
        la[i][2] = valid ? lb * fast_sigmoid(gate_a * (g23.x + dtb.z)) : 0.f;
        la[i][3] = valid ? lb * fast_sigmoid(gate_a * (g23.y + dtb.w)) : 0.f;
      }
      // row sums of squares: transpose-reduce 16 values over the 32 lanes
      float v16[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v16[i] = ssq[i];
        v16[8 + i] = ssk[i];
      }
      {
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
        // lane holds the total of index (lane >> 1): q rows 0..7, then k rows 0..7
        const float inv = rsqrtf(w1 + kL2Eps);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ssq[i] = __shfl_sync(0xffffffffu, inv, 2 * i);        // 1/|q_r|
          ssk[i] = __shfl_sync(0xffffffffu, inv, 16 + 2 * i);   // 1/|k_r|
        }
      }
      if (lane < 8) {
        const int r = 8 * warp + lane;
        float ik = ssk[0], iq = ssq[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
          if (lane == i) {
            ik = ssk[i];
            iq = ssq[i];
          }
        }
        const bool valid = r < len;
        sc_ik[r] = valid ? ik : 0.f;
        sc_iqs[r] = valid ? p.scale * iq : 0.f;
        const float rb = valid ? __bfloat162float(p.beta[(size_t)(t0 + r) * H + h]) : 0.f;
        sc_beta[r] = valid ? fast_sigmoid(rb) : 0.f;
      }
      // in-block cumulative log-decay (block = 16 rows = warps 2J, 2J+1)
#pragma unroll
      for (int i = 1; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) la[i][j] += la[i - 1][j];
      if ((warp & 1) == 0)
        reinterpret_cast<float4*>(sc_carry + blk * 128)[lane] = make_float4(la[7][0], la[7][1], la[7][2], la[7][3]);
      bar_sync();
      if (warp & 1) {
        const float4 cr = reinterpret_cast<const float4*>(sc_carry + blk * 128)[lane];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          la[i][0] += cr.x;
          la[i][1] += cr.y;
          la[i][2] += cr.z;
          la[i][3] += cr.w;
        }
        reinterpret_cast<float4*>(sc_lend + blk * 128)[lane] = make_float4(la[7][0], la[7][1], la[7][2], la[7][3]);
      }
      bar_sync();
      // b_J = e^{lambda_end(J)} for the 4 blocks, this lane's channels
      float bJ[4][4];
#pragma unroll
      for (int J = 0; J < 4; ++J) {
        const float4 le = reinterpret_cast<const float4*>(sc_lend + J * 128)[lane];
        bJ[J][0] = __expf(le.x);
        bJ[J][1] = __expf(le.y);
        bJ[J][2] = __expf(le.z);
        bJ[J][3] = __expf(le.w);
      }
      float lend[4];
      {
        const float4 le = reinterpret_cast<const float4*>(sc_lend + blk * 128)[lane];
        lend[0] = le.x; lend[1] = le.y; lend[2] = le.z; lend[3] = le.w;
      }
      float pre[4], post[4], rb[4], mid[4][4];
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
        rb[j] = 1.0f / bJ[blk][j];
        // mid[I][j] = prod_{J = blk+1}^{I-1} b_J  (for I > blk)
        float m = 1.f;
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          mid[I][j] = m;
          if (I > blk) m *= bJ[I][j];
        }
      }
      if (warp == 0) {
        float4 gm;
        gm.x = bJ[0][0] * bJ[1][0] * bJ[2][0] * bJ[3][0];
        gm.y = bJ[0][1] * bJ[1][1] * bJ[2][1] * bJ[3][1];
        gm.z = bJ[0][2] * bJ[1][2] * bJ[2][2] * bJ[3][2];
        gm.w = bJ[0][3] * bJ[1][3] * bJ[2][3] * bJ[3][3];
        reinterpret_cast<float4*>(sc_gam)[lane] = gm;
      }
      // operands, one row at a time
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 8 * warp + i;
        const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        const float qv[4] = {q01.x, q01.y, q23.x, q23.y};
        const float kv[4] = {k01.x, k01.y, k23.x, k23.y};
        float e[4], f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e[j] = __expf(la[i][j]);
          f[j] = __expf(lend[j] - la[i][j]);
        }
        const float iq = ssq[i] * p.scale, ik = ssk[i];
        const uint32_t off64 = kb * 8192 + sw128(r, lane_chunk) + lane_sub;     // 64-row tiles
        // LK (row r) and LQ (row 64 + r): K-major [2][128 rows][128 B]
        {
          const uint32_t offk = kb * 16384 + sw128(r, lane_chunk) + lane_sub;
          const uint32_t offq = kb * 16384 + sw128(64 + r, lane_chunk) + lane_sub;
          *reinterpret_cast<uint2*>(sm + OFF_LKQ + offk) =
              make_uint2(pack_bf16(kv[0] * e[0], kv[1] * e[1]), pack_bf16(kv[2] * e[2], kv[3] * e[3]));
          *reinterpret_cast<uint2*>(sm + OFF_LKQ + offq) =
              make_uint2(pack_bf16(qv[0] * e[0], qv[1] * e[1]), pack_bf16(qv[2] * e[2], qv[3] * e[3]));
        }
        // R_I rows for I >= blk
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          if (I < blk) continue;
          float fac[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) fac[j] = (I == blk) ? f[j] * rb[j] : f[j] * mid[I][j];
          const uint32_t row = row_off(I) + r;
          const uint32_t off = kb * R_KBLK + sw128(row, lane_chunk) + lane_sub;
          *reinterpret_cast<uint2*>(sm + OFF_R + off) =
              make_uint2(pack_bf16(kv[0] * fac[0], kv[1] * fac[1]), pack_bf16(kv[2] * fac[2], kv[3] * fac[3]));
        }
        // Xk = khat e^Gamma (in place of g), Qb = scale qhat e^Gamma (in place of q),
        // Ktil = k e^{Gamma_C - Gamma} (in place of k; 1/|k| is folded into Delta)
        *reinterpret_cast<uint2*>(sm + OFF_G + off64) =
            make_uint2(pack_bf16(kv[0] * e[0] * pre[0] * ik, kv[1] * e[1] * pre[1] * ik),
                       pack_bf16(kv[2] * e[2] * pre[2] * ik, kv[3] * e[3] * pre[3] * ik));
        *reinterpret_cast<uint2*>(sm + OFF_Q + off64) =
            make_uint2(pack_bf16(qv[0] * e[0] * pre[0] * iq, qv[1] * e[1] * pre[1] * iq),
                       pack_bf16(qv[2] * e[2] * pre[2] * iq, qv[3] * e[3] * pre[3] * iq));
        *reinterpret_cast<uint2*>(sm + OFF_K + off64) =
            make_uint2(pack_bf16(kv[0] * f[0] * post[0], kv[1] * f[1] * post[1]),
                       pack_bf16(kv[2] * f[2] * post[2], kv[3] * f[3] * post[3]));
        if (r >= len) *reinterpret_cast<uint2*>(sm + OFF_V + off64) = make_uint2(0, 0);
      }
    }
    publish();

    // ================================================================ MMA_AP
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int I = 0; I < 4; ++I) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = sdesc_sw128(sbase + OFF_LKQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(sbase + OFF_R + (ks >> 2) * R_KBLK + row_off(I) * 128 + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem + TM_AP + 64 * I, a, b, idesc, ks > 0);
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
      const int q2 = quarter & 1;         // rows 32*q2 .. 32*q2+31 of this side
      // s-range [32*half, 32*half+32) is entirely above the diagonal for rows < 32
      const bool skip = (half == 1) && (q2 == 0);
      float dsel[32];
      if (!skip) {
        float d0[32], d1[32];
        const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
        tmem_ld32(tmem + lane_addr + TM_AP + 64 * (2 * q2) + 32 * half, d0);
        tmem_ld32(tmem + lane_addr + TM_AP + 64 * (2 * q2 + 1) + 32 * half, d1);
        const bool odd = Ib & 1;
#pragma unroll
        for (int j = 0; j < 32; ++j) dsel[j] = odd ? d1[j] : d0[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) dsel[j] = 0.f;
      }
      if (!qside) {
        const float rowscale = sc_beta[r] * sc_ik[r];
        float* dst = As + r * AS_LD + 32 * half;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 o;
          const int s = 32 * half + j;
          o.x = (s + 0 < r) ? rowscale * sc_ik[s + 0] * dsel[j + 0] : 0.f;
          o.y = (s + 1 < r) ? rowscale * sc_ik[s + 1] * dsel[j + 1] : 0.f;
          o.z = (s + 2 < r) ? rowscale * sc_ik[s + 2] * dsel[j + 2] : 0.f;
          o.w = (s + 3 < r) ? rowscale * sc_ik[s + 3] * dsel[j + 3] : 0.f;
          *reinterpret_cast<float4*>(dst + j) = o;
        }
      } else {
        const float rowscale = sc_iqs[r];
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          float v8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 8 * cch + u;
            const int s = 32 * half + j;
            v8[u] = (s <= r) ? rowscale * sc_ik[s] * dsel[j] : 0.f;
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
    if (tid < 64) {
      const int j = tid;
      float x[C];
#pragma unroll
      for (int s = 0; s < C; ++s) x[s] = (s == j) ? 1.f : 0.f;
#pragma unroll
      for (int r = 1; r < C; ++r) {
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int s = 0; s < r; s += 4) {
          const float4 a = *reinterpret_cast<const float4*>(As + r * AS_LD + s);
          a0 = fmaf(a.x, x[s], a0);
          if (s + 1 < C) a1 = fmaf(a.y, x[s + 1], a1);
          if (s + 2 < C) a2 = fmaf(a.z, x[s + 2], a2);
          if (s + 3 < C) a3 = fmaf(a.w, x[s + 3], a3);
        }
        const float val = -((a0 + a1) + (a2 + a3));
        x[r] = (r > j) ? val : x[r];
      }
      const float bj = sc_beta[j];
      const uint32_t cbyte = (uint32_t)j * 2;
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t off = sw128(r, cbyte >> 4) + (cbyte & 15);
        const float tb = x[r] * bj;
        const __nv_bfloat16 hi = __float2bfloat16_rn(tb);
        *reinterpret_cast<__nv_bfloat16*>(sm + OFF_TP + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(sm + OFF_TL + off) = __float2bfloat16_rn(tb - __bfloat162float(hi));
      }
    }
    publish();

    // ================================================================ MMA_PT: [T_beta; P] x T_beta
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + OFF_TP + (ks & 3) * 32, 16, 1024);
        const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem + TM_AP, a, b, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();
    if (quarter >= 2) {
      const int r = 32 * quarter + lane - 64;
      float d[32];
      tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + TM_AP + 32 * half, d);
#pragma unroll
      for (int cch = 0; cch < 4; ++cch) {
        uint4 wh, wl;
        split_pack(&d[8 * cch], wh, wl);
        *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(64 + r, 4 * half + cch)) = wh;
        *reinterpret_cast<uint4*>(sm + OFF_TL + sw128(64 + r, 4 * half + cch)) = wl;
      }
    }
    publish();

    // ================================================================ MMA_X: [T_beta; P T_beta] x [Xk | V]
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 32, 16, 1024);
        const uint64_t bk = sdesc_sw128(sbase + OFF_G + (ks & 3) * 2048, 8192, 1024);
        const uint64_t bv = sdesc_sw128(sbase + OFF_V + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem + TM_X, a, bk, idesc, ks > 0);
        umma_bf16(tmem + TM_X + 128, a, bv, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();

    // ================================================================ [W; Qtil - PW] operand
    {
      const int R = 32 * quarter + lane;
      const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_addr + TM_X + 64 * half + 32 * part, d);
        if (R >= 64) {
          const int r = R - 64;
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            const uint32_t chunk = 4 * part + cch;  // within the 64-channel block `half`
            const uint4 qb = *reinterpret_cast<const uint4*>(sm + OFF_Q + half * 8192 + sw128(r, chunk));
            const float2 a0 = unpack_bf16(qb.x), a1 = unpack_bf16(qb.y), a2 = unpack_bf16(qb.z),
                         a3 = unpack_bf16(qb.w);
            d[8 * cch + 0] = a0.x - d[8 * cch + 0];
            d[8 * cch + 1] = a0.y - d[8 * cch + 1];
            d[8 * cch + 2] = a1.x - d[8 * cch + 2];
            d[8 * cch + 3] = a1.y - d[8 * cch + 3];
            d[8 * cch + 4] = a2.x - d[8 * cch + 4];
            d[8 * cch + 5] = a2.y - d[8 * cch + 5];
            d[8 * cch + 6] = a3.x - d[8 * cch + 6];
            d[8 * cch + 7] = a3.y - d[8 * cch + 7];
          }
        }
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          uint4 w;
          w.x = pack_bf16(d[8 * cch + 0], d[8 * cch + 1]);
          w.y = pack_bf16(d[8 * cch + 2], d[8 * cch + 3]);
          w.z = pack_bf16(d[8 * cch + 4], d[8 * cch + 5]);
          w.w = pack_bf16(d[8 * cch + 6], d[8 * cch + 7]);
          *reinterpret_cast<uint4*>(sm + OFF_WQ + half * 16384 + sw128(R, 4 * part + cch)) = w;
        }
      }
    }
    publish();

    // next chunk's q, g, v tiles may now be loaded (Qb read, Xk and V consumed by MMA_X)
    const bool has_next = (c + 1 < nchunks);
    if (tid == 0 && has_next) {
      mbar_arrive_expect_tx(tma_bar, 4 * 16384);
      issue_tma(t0 + C, true, false);
    }

    // ================================================================ MMA1: [W; Qtil - PW] x S
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + OFF_WQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
        const uint64_t b = sdesc_sw128(sbase + OFF_S + ks * 2048, 16384, 1024);
        umma_bf16(tmem + TM_REC, a, b, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();

    // ================================================================ ep1: Delta and O
    {
      const int R = 32 * quarter + lane;
      const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
      const int r = R & 63;
      const float ik = sc_ik[r];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float ws[32], uu[32];
        tmem_ld32(tmem + lane_addr + TM_REC + 64 * half + 32 * part, ws);
        tmem_ld32(tmem + lane_addr + TM_X + 128 + 64 * half + 32 * part, uu);
        if (R < 64) {
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            float dl[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) dl[u] = (uu[8 * cch + u] - ws[8 * cch + u]) * ik;
            uint4 wh, wl;
            split_pack(dl, wh, wl);
            *reinterpret_cast<uint4*>(sm + OFF_DL + half * 8192 + sw128(r, 4 * part + cch)) = wh;
            *reinterpret_cast<uint4*>(sm + OFF_DLLO + half * 8192 + sw128(r, 4 * part + cch)) = wl;
          }
        } else if (r < len) {
          __nv_bfloat16* orow = p.out + ((size_t)(t0 + r) * H + h) * D + 64 * half + 32 * part;
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            uint4 w;
            w.x = pack_bf16(ws[8 * cch + 0] + uu[8 * cch + 0], ws[8 * cch + 1] + uu[8 * cch + 1]);
            w.y = pack_bf16(ws[8 * cch + 2] + uu[8 * cch + 2], ws[8 * cch + 3] + uu[8 * cch + 3]);
            w.z = pack_bf16(ws[8 * cch + 4] + uu[8 * cch + 4], ws[8 * cch + 5] + uu[8 * cch + 5]);
            w.w = pack_bf16(ws[8 * cch + 6] + uu[8 * cch + 6], ws[8 * cch + 7] + uu[8 * cch + 7]);
            reinterpret_cast<uint4*>(orow)[cch] = w;
          }
        }
      }
    }
    publish();

    // ================================================================ MMA2: Ktil^T x Delta
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, true, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = sdesc_sw128(sbase + OFF_K + (ks & 3) * 2048, 8192, 1024);
        const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_DL : OFF_DLLO) + (ks & 3) * 2048, 8192, 1024);
        umma_bf16(tmem + TM_REC, a, b, idesc, ks > 0);
      }
      umma_commit(mma_bar);
    }
    if (!wait_all(mma_bar, mma_phase)) break;
    tc_fence_after();
    if (tid == 0 && has_next) issue_tma(t0 + C, false, true);

    // ================================================================ ep2: state update
    {
      const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
      const float gam = sc_gam[srow];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_addr + TM_REC + 64 * half + 32 * part, d);
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
  if (!make_token_map(&maps.q, p.q, tokens, p.num_heads) || !make_token_map(&maps.k, p.k, tokens, p.num_heads) ||
      !make_token_map(&maps.v, p.v, tokens, p.num_heads) || !make_token_map(&maps.g, p.g, tokens, p.num_heads))
    return cudaErrorInvalidValue;
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
