// Chunked KDA forward for sm_100a: one fused, warp-specialised kernel, one CTA per (sequence,
// head) unit.
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
// Roles (512 threads):
//   warp 0 (one thread)  issues every tcgen05 MMA, polling two dependency streams: the
//                        intra-chunk stream (AP, PT, Xk, Xv of chunk c+1) and the recurrence
//                        stream (MMA1, MMA2 of chunk c), so each runs as soon as its inputs exist.
//   warp 1 (one thread)  TMA loads of the q and k tiles (a single stage, refilled as soon as the
//                        intra warps have read it) and of the v tile.
//   warps 4..11 (intra)  per chunk:
//       prologue  raw q, k (shared memory), g (registers, prefetched one chunk ahead); L2 norms,
//                 sigmoid(beta), safe gate alpha = exp(lower_bound * sigmoid(exp(A_log)(g + dt_bias)));
//                 decays as running products of alpha inside each 16-row sub-block (exponent
//                 referencing: every factor stays in [e^-80, e^80] for lower_bound >= -5); the bf16
//                 MMA operands with the norms, beta and scale folded in.
//       assemble  A (fp32) and P (bf16) from the gated Gram blocks [LK; LQ] x R_I^T (MMA AP).
//       solve     T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution, off-diagonal
//                 blocks T_IJ = -T_II sum_K A_IK T_KJ, in fp32; T_b kept as a bf16 hi+lo pair.
//       PT        P (T_hi + T_lo) (MMA PT) read back as a hi+lo pair.
//       WQ        [-W; Qtil - P W] from [T_b; P T_b] x Khat e^Gamma (MMA Xk), written to TMEM as
//                 the A operand of MMA1.
//   warps 12..15 (rec)   MMA Xv writes [U; P U] into TMEM; MMA1 accumulates [-W; Qtil - PW] x S onto
//                 it, giving [Delta; O]; ep1 stores O and Delta (bf16 hi+lo); MMA2 accumulates
//                 Ktil^T Delta onto the fp32 state kept in TMEM (pre-scaled by e^{Gamma_C}); ep2
//                 refreshes the bf16 copy of S used as the B operand of the next MMA1.
// HBM sees the raw inputs once and the output once.  The hi+lo pairs matter when keys are nearly
// collinear: T then has entries close to -beta that cancel against the diagonal and a chunk's
// Delta rows telescope, so a single bf16 rounding of T_b, P T_b or Delta would cost several
// percent of the state.  Ktil is built from the raw bf16 k (its 1/|k| is applied to Delta) so that
// equal keys round identically.
//
// Every wait is bounded (kWaitLimitNs of wall time without progress): on expiry the kernel
// records KDA_ERR_DEVICE_TIMEOUT in the workspace status word, every role leaves its loop, and
// the tensor memory is released.
#include "kda_device.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;      // chunk length
constexpr int D = kHeadDim;    // 128
constexpr int kThreads = 512;  // 16 warps
constexpr int kIntraWarp0 = 4, kIntraThreads = 256;
constexpr int kRecWarp0 = 12, kRecThreads = 128;
constexpr uint32_t kBarIntra = 1, kBarRec = 2;

// Shared-memory map (bytes from a 1024-aligned base).  "MN tile" = [2 blocks of 64 columns]
// [64 rows][128 B] with the 128-byte swizzle; "K tile" = [2 blocks of 64 K][rows][128 B].
constexpr uint32_t OFF_RQ = 0;           // q tile (TMA)
constexpr uint32_t OFF_RK = 16384;       // k tile (TMA)
constexpr uint32_t OFF_XK = 32768;       // Khat e^Gamma, MN-major B of MMA Xk
constexpr uint32_t OFF_QB = 49152;       // Qtil (bf16), read when forming Qtil - P W
constexpr uint32_t OFF_KT = 65536;       // Ktil (raw k), MN-major A of MMA2
constexpr uint32_t OFF_DL = 81920;       // Delta hi, MN tile (ep1 -> MMA2)
constexpr uint32_t OFF_DLLO = 98304;     // Delta lo
constexpr uint32_t OFF_S = 114688;       // S bf16, MN-major B of MMA1, 2 blocks x 128 rows
constexpr uint32_t OFF_SCR = 147456;     // scratch, 73728 bytes:
constexpr uint32_t OFF_LKQ = OFF_SCR;            //   [LK; LQ] K tile, 128 rows (prologue -> AP)
constexpr uint32_t OFF_R = OFF_SCR + 32768;      //   R_0..R_3 K tile, 160 rows (prologue -> AP)
constexpr uint32_t R_KBLK = 160 * 128;
constexpr uint32_t OFF_TP = OFF_SCR;             //   [T_hi; P -> (P T)_hi] 128 x 64 K tile
constexpr uint32_t OFF_AS = OFF_SCR + 16384;     //   A fp32 64 x 68 (assemble -> solve)
constexpr uint32_t OFF_TL = OFF_SCR + 16384;     //   [T_lo; (P T)_lo] (after A is dead)
constexpr uint32_t OFF_TS = OFF_SCR + 33792;     //   T fp32 64 x 68
constexpr uint32_t OFF_YS = OFF_SCR + 51200;     //   solve temporaries 3 x 16 x 16 fp32
constexpr uint32_t OFF_V = OFF_SCR + 54272;      //   v tile (TMA, after AP), MN-major B of MMA Xv
constexpr uint32_t AS_LD = 68;
constexpr uint32_t OFF_SC = OFF_SCR + 73728;     // scalars
constexpr uint32_t SC_BETA = 0;                  // float[2][64]
constexpr uint32_t SC_IK = 512;                  // float[2][64] 1/|k_r| (0 past the end)
constexpr uint32_t SC_GAM = 1024;                // float[2][128] e^{Gamma_C}
constexpr uint32_t SC_TOT = 2048;                // float[8][128] per-warp alpha products
constexpr uint32_t SC_BAR = 6144;                // mbarriers
constexpr uint32_t SC_TMEM = 6400;
constexpr uint32_t SC_ABORT = 6404;
constexpr uint32_t SMEM_BYTES = OFF_SC + 6528;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// mbarrier indices
enum {
  B_RAW_FULL, B_RAW_EMPTY, B_V_FULL, B_OPS0, B_OPS1, B_KT, B_AP, B_TB, B_PT, B_TP, B_XK, B_XV, B_WQ,
  B_MMA1, B_DELTA, B_MMA2, B_S, B_COUNT
};


// TMEM columns: intra area 0..255 (AP products at row_off(I), P T at 0..63, [W PW] at 0..127,
// [-W; Qtil - PW] packed bf16 at 0..63); [U PU] -> [Delta O] at 256..383; fp32 state at 384..511.
constexpr uint32_t TM_UP = 256;
constexpr uint32_t TM_S = 384;
constexpr uint32_t kTmemCols = 512;

struct TensorMaps {
  CUtensorMap q, k, v;
};

struct Shared {
  uint8_t* sm;
  uint32_t sbase;
  uint64_t* bar;
  volatile int* abort;
  uint32_t tmem;
};

// Bounded wait on a phase; returns false once the abort flag is up (set here on time-out).
__device__ __forceinline__ bool wait_bar(const Shared& S_, int b, uint32_t parity, uint32_t* status) {
  uint64_t* bar = S_.bar + b;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63) == 0) {
      if (*S_.abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *S_.abort = 1;
        if (status) atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------------------ MMA issuer
__device__ void mma_issuer(const Shared& S_, const FwdParams& p, int nchunks) {
  const uint32_t sbase = S_.sbase, tmem = S_.tmem;
  uint64_t* bar = S_.bar;
  int ci = 0, ist = 0;  // intra stream: chunk, stage (0 AP, 1 PT, 2 Xk, 3 Xv)
  int cr = 0, rst = 0;  // recurrence stream: chunk, stage (0 MMA1, 1 MMA2)
  uint64_t last = globaltimer_ns();
  while (cr < nchunks) {
    if (*S_.abort) return;
    bool progressed = false;
    // ---- recurrence stream (priority)
    if (rst == 0) {
      if (ci > cr && mbar_test(bar + B_WQ, cr & 1) && mbar_test(bar + B_S, cr & 1)) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t b = sdesc_sw128(sbase + OFF_S + ks * 2048, 16384, 1024);
          umma_bf16_tmem_a(tmem + TM_UP, tmem + 8 * ks, b, idesc, 1);
        }
        umma_commit(bar + B_MMA1);
        rst = 1;
        progressed = true;
      }
    } else {
      if (mbar_test(bar + B_DELTA, cr & 1) && mbar_test(bar + B_KT, cr & 1)) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = sdesc_sw128(sbase + OFF_KT + (ks & 3) * 2048, 8192, 1024);
          const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_DL : OFF_DLLO) + (ks & 3) * 2048, 8192, 1024);
          umma_bf16(tmem + TM_S, a, b, idesc, 1);
        }
        umma_commit(bar + B_MMA2);
        rst = 0;
        ++cr;
        progressed = true;
      }
    }
    // ---- intra-chunk stream
    if (ci < nchunks) {
      if (ist == 0) {
        // AP(ci) overwrites the TMEM area that holds WQ(ci-1): MMA1(ci-1) must be issued first
        const bool wq_consumed = (ci == 0) || (cr > ci - 1) || (cr == ci - 1 && rst == 1);
        if (wq_consumed && mbar_test(bar + B_OPS0 + (ci & 1), (ci >> 1) & 1)) {
          tc_fence_after();
#pragma unroll
          for (int I = 0; I < 4; ++I) {
            const uint32_t idesc = idesc_bf16(128, 16 * (I + 1), false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint64_t a = sdesc_sw128(sbase + OFF_LKQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
              const uint64_t b =
                  sdesc_sw128(sbase + OFF_R + (ks >> 2) * R_KBLK + row_off(I) * 128 + (ks & 3) * 32, 16, 1024);
              umma_bf16(tmem + row_off(I), a, b, idesc, ks > 0);
            }
          }
          umma_commit(bar + B_AP);
          ist = 1;
          progressed = true;
        }
      } else if (ist == 1) {
        if (mbar_test(bar + B_TB, ci & 1)) {
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t a = sdesc_sw128(sbase + OFF_TP + (ks & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 2048, 8192, 1024);
            umma_bf16(tmem, a, b, idesc, ks > 0);
          }
          umma_commit(bar + B_PT);
          ist = 2;
          progressed = true;
        }
      } else if (ist == 2) {
        if (mbar_test(bar + B_TP, ci & 1)) {
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t a = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sbase + OFF_XK + (ks & 3) * 2048, 8192, 1024);
            umma_bf16(tmem, a, b, idesc, ks > 0);
          }
          umma_commit(bar + B_XK);
          ist = 3;
          progressed = true;
        }
      } else {
        // Xv(ci) writes [U PU] where [Delta O](ci-1) lives until ep1(ci-1) has read it
        const bool up_free = (ci == 0) || mbar_test(bar + B_DELTA, (ci - 1) & 1);
        if (up_free && mbar_test(bar + B_V_FULL, ci & 1)) {
          tc_fence_after();
          constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t a = sdesc_sw128(sbase + (ks < 4 ? OFF_TP : OFF_TL) + (ks & 3) * 32, 16, 1024);
            const uint64_t b = sdesc_sw128(sbase + OFF_V + (ks & 3) * 2048, 8192, 1024);
            umma_bf16(tmem + TM_UP, a, b, idesc, ks > 0);
          }
          umma_commit(bar + B_XV);
          ist = 0;
          ++ci;
          progressed = true;
        }
      }
    }
    if (progressed) {
      last = globaltimer_ns();
    } else {
      __nanosleep(64);
      if (globaltimer_ns() - last > kWaitLimitNs) {
        *S_.abort = 1;
        if (p.status) atomicOr(p.status, kStatusTimeout);
        return;
      }
    }
  }
}

// ------------------------------------------------------------------------------ TMA producer
__device__ void tma_producer(const Shared& S_, const TensorMaps& maps, const FwdParams& p, int h,
                             int64_t bos, int nchunks) {
  uint8_t* sm = S_.sm;
  uint64_t* bar = S_.bar;
  for (int c = 0; c < nchunks; ++c) {
    const int t0 = (int)(bos + (int64_t)c * C);
    if (c > 0 && !wait_bar(S_, B_RAW_EMPTY, (c - 1) & 1, p.status)) return;
    mbar_arrive_expect_tx(bar + B_RAW_FULL, 32768);
    tma_load_3d(sm + OFF_RQ, &maps.q, bar + B_RAW_FULL, 0, h, t0);
    tma_load_3d(sm + OFF_RQ + 8192, &maps.q, bar + B_RAW_FULL, 64, h, t0);
    tma_load_3d(sm + OFF_RK, &maps.k, bar + B_RAW_FULL, 0, h, t0);
    tma_load_3d(sm + OFF_RK + 8192, &maps.k, bar + B_RAW_FULL, 64, h, t0);
    // the v tile lands in the scratch once MMA AP has consumed the Gram operands
    if (!wait_bar(S_, B_AP, c & 1, p.status)) return;
    mbar_arrive_expect_tx(bar + B_V_FULL, 16384);
    tma_load_3d(sm + OFF_V, &maps.v, bar + B_V_FULL, 0, h, t0);
    tma_load_3d(sm + OFF_V + 8192, &maps.v, bar + B_V_FULL, 64, h, t0);
  }
}

// ------------------------------------------------------------------------------ intra warps
__device__ void intra_warps(const Shared& S_, const FwdParams& p, int h, int64_t bos, int64_t eos,
                            int nchunks, int itid) {
  uint8_t* sm = S_.sm;
  const uint32_t tmem = S_.tmem;
  const int H = p.num_heads;
  const int iw = itid >> 5, lane = itid & 31;
  const int quarter = iw & 3, ihalf = iw >> 2;       // TMEM lane quarter, column half
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  float* sc_beta = reinterpret_cast<float*>(sm + OFF_SC + SC_BETA);
  float* sc_ik = reinterpret_cast<float*>(sm + OFF_SC + SC_IK);
  float* sc_gam = reinterpret_cast<float*>(sm + OFF_SC + SC_GAM);
  float* sc_tot = reinterpret_cast<float*>(sm + OFF_SC + SC_TOT);
  float* As = reinterpret_cast<float*>(sm + OFF_AS);
  float* Ts = reinterpret_cast<float*>(sm + OFF_TS);
  float* Ys = reinterpret_cast<float*>(sm + OFF_YS);
  volatile int* abort_flag = S_.abort;
  auto sync = [&]() { named_bar(kBarIntra, kIntraThreads); };

  // prologue mapping: warp iw owns chunk rows 8 iw .. 8 iw + 7, lane owns channels 4 lane .. +3
  const float gate_a = __expf(p.A_log[h]);
  const float4 dtb = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
  const float ga = -gate_a * kLog2e;                 // exp(-a (g + dt)) = exp2(ga g + gb)
  const float gb[4] = {ga * dtb.x, ga * dtb.y, ga * dtb.z, ga * dtb.w};
  const float lb2 = p.lower_bound * kLog2e;
  const int kb = lane >> 4;
  const uint32_t lane_chunk = (lane & 15) >> 1;
  const uint32_t lane_sub = (lane & 1) * 8;
  const int blk = iw >> 1;
  const bool upper_half = iw & 1;

  uint2 gr[8];        // raw g of the chunk being prepared (loaded one chunk ahead)
  float beta_raw = 0.f;  // raw beta of row 8 iw + lane (lanes 0..7), loaded with g
  auto load_g = [&](int c) {
    const int64_t t0 = bos + (int64_t)c * C;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t t = t0 + 8 * iw + i;
      gr[i] = (c < nchunks && t < eos) ? ldg_u2(p.g + ((size_t)t * H + h) * D + 4 * lane) : make_uint2(0, 0);
    }
    const int64_t tb = t0 + 8 * iw + (lane & 7);
    beta_raw = (c < nchunks && tb < eos) ? __bfloat162float(p.beta[(size_t)tb * H + h]) : 0.f;
  };
  load_g(0);
  // shared-memory byte offset of this thread's 8 bytes of row 8 iw + i inside a 128-byte-row tile
  uint32_t xo[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) xo[i] = (uint32_t)((8 * iw + i) * 128) + (((lane_chunk ^ i) & 7u) << 4) + lane_sub;
  const uint32_t sbase = S_.sbase;
  const uint32_t a_rq = sbase + OFF_RQ + kb * 8192, a_rk = sbase + OFF_RK + kb * 8192;
  const uint32_t a_lk = sbase + OFF_LKQ + kb * 16384, a_lq = a_lk + 64 * 128;
  const uint32_t a_xk = sbase + OFF_XK + kb * 8192, a_qb = sbase + OFF_QB + kb * 8192, a_kt = sbase + OFF_KT + kb * 8192;
  const uint32_t a_r = sbase + OFF_R + kb * R_KBLK;

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int len = (int)((eos - t0) < (int64_t)C ? (eos - t0) : (int64_t)C);
    const int slot = c & 1;

    // ============================================================== prologue
    wait_bar(S_, B_RAW_FULL, c & 1, p.status);
    uint2 qr[8], kr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool valid = 8 * iw + i < len;
      qr[i] = valid ? lds64(a_rq + xo[i]) : make_uint2(0, 0);
      kr[i] = valid ? lds64(a_rk + xo[i]) : make_uint2(0, 0);
    }
    sync();
    if (*abort_flag) break;
    if (itid == 0) mbar_arrive(S_.bar + B_RAW_EMPTY);

    float a[8][4];  // alpha
    float ssq[8], ssk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 8 * iw + i;
      const bool valid = r < len;
      const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
      const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
      ssq[i] = q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y;
      ssk[i] = k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y;
      const float2 g01 = unpack_bf16(gr[i].x), g23 = unpack_bf16(gr[i].y);
      const float gv[4] = {g01.x, g01.y, g23.x, g23.y};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float sig = rcp_approx(1.0f + ex2_approx(fmaf(ga, gv[j], gb[j])));
        a[i][j] = valid ? ex2_approx(lb2 * sig) : 1.0f;
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
      for (int j = 0; j < 8; ++j)
        w8[j] = (b4 ? v16[j + 8] : v16[j]) + __shfl_xor_sync(0xffffffffu, b4 ? v16[j] : v16[j + 8], 16);
      const bool b3 = lane & 8;
      float w4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w4[j] = (b3 ? w8[j + 4] : w8[j]) + __shfl_xor_sync(0xffffffffu, b3 ? w8[j] : w8[j + 4], 8);
      const bool b2 = lane & 4;
      float w2[2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
        w2[j] = (b2 ? w4[j + 2] : w4[j]) + __shfl_xor_sync(0xffffffffu, b2 ? w4[j] : w4[j + 2], 4);
      const bool b1 = lane & 2;
      float w1 = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, b1 ? w2[0] : w2[1], 2);
      w1 += __shfl_xor_sync(0xffffffffu, w1, 1);
      inv = rsqrtf(w1 + kL2Eps);
    }
    const float beta_l = (lane < 8 && 8 * iw + lane < len) ? fast_sigmoid(beta_raw) : 0.f;
    float iqv[8], ikv[8], btv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      iqv[i] = __shfl_sync(0xffffffffu, inv, 2 * i) * p.scale;
      ikv[i] = __shfl_sync(0xffffffffu, inv, 16 + 2 * i);
      btv[i] = __shfl_sync(0xffffffffu, beta_l, i);
    }
    // per-warp alpha totals -> sub-block totals b_J
    float tot[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float t = a[0][j];
#pragma unroll
      for (int i = 1; i < 8; ++i) t *= a[i][j];
      tot[j] = t;
    }
    reinterpret_cast<float4*>(sc_tot + iw * 128)[lane] = make_float4(tot[0], tot[1], tot[2], tot[3]);
    sync();
    float pre[4], post[4], cI[4][4], gam[4], pt[4];
    {
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
      const float4 pv = reinterpret_cast<const float4*>(sc_tot + (iw ^ 1) * 128)[lane];
      pt[0] = pv.x; pt[1] = pv.y; pt[2] = pv.z; pt[3] = pv.w;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float pa = 1.f, z = 1.f;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
          if (J < blk) pa *= bJ[J][j];
          if (J > blk) z *= bJ[J][j];
        }
        pre[j] = pa;
        post[j] = z;
        gam[j] = bJ[0][j] * bJ[1][j] * bJ[2][j] * bJ[3][j];
        float m = 1.f;
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          cI[I][j] = (I == blk) ? 1.0f / bJ[blk][j] : m;
          if (I > blk) m *= bJ[I][j];
        }
      }
    }
    // the scratch and the scalar slot still serve the chunk two back / MMA Xv of the previous
    // chunk until MMA Xv has run (and, through it, ep1 of the chunk before)
    if (c > 0) wait_bar(S_, B_XV, (c - 1) & 1, p.status);
    sync();
    if (*abort_flag) break;
    {
      const float ikr = __shfl_sync(0xffffffffu, inv, 16 + 2 * (lane & 7));  // 1/|k| of row 8 iw + (lane & 7)
      if (lane < 8) {
        const int r = 8 * iw + lane;
        sc_beta[slot * 64 + r] = beta_l;
        sc_ik[slot * 64 + r] = (r < len) ? ikr : 0.f;
      }
    }
    if (iw == 0) reinterpret_cast<float4*>(sc_gam + slot * 128)[lane] = make_float4(gam[0], gam[1], gam[2], gam[3]);

    // pass 1, rows ascending: e_i = prod of alpha from the sub-block start to row i
    {
      float run[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) run[j] = upper_half ? pt[j] : 1.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 q01 = unpack_bf16(qr[i].x), q23 = unpack_bf16(qr[i].y);
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        const float qv[4] = {q01.x, q01.y, q23.x, q23.y};
        const float kv[4] = {k01.x, k01.y, k23.x, k23.y};
        float lk[4], lq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          run[j] *= a[i][j];
          lk[j] = kv[j] * (run[j] * ikv[i]);   // khat * e
          lq[j] = qv[j] * (run[j] * iqv[i]);   // scale * qhat * e
        }
        const float b = btv[i];
        sts64(a_lk + xo[i], bf16x2(lk[0] * b, lk[1] * b), bf16x2(lk[2] * b, lk[3] * b));
        sts64(a_lq + xo[i], bf16x2(lq[0], lq[1]), bf16x2(lq[2], lq[3]));
        sts64(a_xk + xo[i], bf16x2(lk[0] * pre[0], lk[1] * pre[1]), bf16x2(lk[2] * pre[2], lk[3] * pre[3]));
        sts64(a_qb + xo[i], bf16x2(lq[0] * pre[0], lq[1] * pre[1]), bf16x2(lq[2] * pre[2], lq[3] * pre[3]));
      }
    }
    // pass 2, rows descending: f_i = prod of alpha after row i to the sub-block end
    uint2 kt_pack[8];
    {
      float run[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) run[j] = upper_half ? 1.f : pt[j];
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
        const float kv[4] = {k01.x, k01.y, k23.x, k23.y};
        float kf[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) kf[j] = kv[j] * (run[j] * ikv[i]);   // khat * f
#pragma unroll
        for (int I = 0; I < 4; ++I) {
          if (I < blk) continue;
          sts64(a_r + row_off(I) * 128 + xo[i], bf16x2(kf[0] * cI[I][0], kf[1] * cI[I][1]),
                bf16x2(kf[2] * cI[I][2], kf[3] * cI[I][3]));
        }
        kt_pack[i] = make_uint2(bf16x2(kv[0] * (run[0] * post[0]), kv[1] * (run[1] * post[1])),
                                bf16x2(kv[2] * (run[2] * post[2]), kv[3] * (run[3] * post[3])));
#pragma unroll
        for (int j = 0; j < 4; ++j) run[j] *= a[i][j];
      }
    }
    load_g(c + 1);
    fence_proxy_async();
    sync();
    if (itid == 0) mbar_arrive(S_.bar + B_OPS0 + slot);
    // Ktil: the previous chunk's is read by MMA2 until it has run
    if (c > 0) wait_bar(S_, B_MMA2, (c - 1) & 1, p.status);
    sync();
    if (*abort_flag) break;
#pragma unroll
    for (int i = 0; i < 8; ++i) sts64(a_kt + xo[i], kt_pack[i].x, kt_pack[i].y);
    fence_proxy_async();
    sync();
    if (itid == 0) mbar_arrive(S_.bar + B_KT);

    // ============================================================== assemble A and P
    wait_bar(S_, B_AP, c & 1, p.status);
    sync();
    if (*abort_flag) break;
    tc_fence_after();
    {
      const int R = 32 * quarter + lane;
      const bool qside = R >= 64;
      const int r = R & 63;
      const int Ib = r >> 4;
      const int q2 = quarter & 1;
      const bool skip = (ihalf == 1) && (q2 == 0);
      float d[32];
      if (!skip) {
        float d0[32], d1[32];
        tmem_ld32(tmem + lane_base + row_off(2 * q2) + 32 * ihalf, d0);
        tmem_ld32(tmem + lane_base + row_off(2 * q2 + 1) + 32 * ihalf, d1);
        const bool odd = Ib & 1;
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = odd ? d1[j] : d0[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = 0.f;
      }
      if (!qside) {
        float* dst = As + r * AS_LD + 32 * ihalf;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int s = 32 * ihalf + j;
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
            const int s = 32 * ihalf + 8 * cch + u;
            v8[u] = (s <= r) ? d[8 * cch + u] : 0.f;
          }
          uint4 w;
          w.x = pack_bf16(v8[0], v8[1]);
          w.y = pack_bf16(v8[2], v8[3]);
          w.z = pack_bf16(v8[4], v8[5]);
          w.w = pack_bf16(v8[6], v8[7]);
          *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(64 + r, 4 * ihalf + cch)) = w;
        }
      }
    }
    tc_fence_before();
    sync();

    // ============================================================== solve T = (I + A)^{-1}
    if (iw < 4 && lane < 16) {
      const int I = iw, j = lane;
      const float* ab = As + (16 * I) * AS_LD + 16 * I;
      float x[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) x[m] = (m == j) ? 1.f : 0.f;
      // right-looking substitution: once x[m] is final, fold it into every later row
#pragma unroll
      for (int m = 0; m < 15; ++m) {
        const float xm = x[m];
#pragma unroll
        for (int i = m + 1; i < 16; ++i) x[i] = fmaf(-ab[i * AS_LD + m], xm, x[i]);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Ts[(16 * I + i) * AS_LD + 16 * I + j] = (i >= j) ? x[i] : 0.f;
    }
    sync();
    // off-diagonal blocks by distance dd below the diagonal, one warp per block:
    // T_IJ = -T_II (sum_{K=J}^{I-1} A_IK T_KJ), each 16x16x16 product on mma.sync m16n8k8 tf32
    // with both operands split hi + lo (three products), i.e. fp32-level accuracy
#pragma unroll 1
    for (int dd = 1; dd < 4; ++dd) {
      if (iw < 4 - dd) {
        const int bI = dd + iw, bJ2 = iw;
        const int g = lane >> 2, t = lane & 3;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        for (int K = bJ2; K < bI; ++K) {
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const float* ab = As + (16 * bI + g) * AS_LD + 16 * K + 8 * ks + t;
            uint32_t ah[4], al[4];
            tf32_split(ab[0], ah[0], al[0]);
            tf32_split(ab[8 * AS_LD], ah[1], al[1]);
            tf32_split(ab[4], ah[2], al[2]);
            tf32_split(ab[8 * AS_LD + 4], ah[3], al[3]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const float* tb = Ts + (16 * K + 8 * ks + t) * AS_LD + 16 * bJ2 + 8 * nt + g;
              uint32_t bh0, bl0, bh1, bl1;
              tf32_split(tb[0], bh0, bl0);
              tf32_split(tb[4 * AS_LD], bh1, bl1);
              mma_tf32(acc[nt], ah, bh0, bh1);
              mma_tf32(acc[nt], ah, bl0, bl1);
              mma_tf32(acc[nt], al, bh0, bh1);
            }
          }
        }
        float* ys = Ys + iw * 256;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          ys[g * 16 + 8 * nt + 2 * t] = acc[nt][0];
          ys[g * 16 + 8 * nt + 2 * t + 1] = acc[nt][1];
          ys[(g + 8) * 16 + 8 * nt + 2 * t] = acc[nt][2];
          ys[(g + 8) * 16 + 8 * nt + 2 * t + 1] = acc[nt][3];
        }
        __syncwarp();
        float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const float* tr = Ts + (16 * bI + g) * AS_LD + 16 * bI + 8 * ks + t;
          uint32_t ah[4], al[4];
          tf32_split(tr[0], ah[0], al[0]);
          tf32_split(tr[8 * AS_LD], ah[1], al[1]);
          tf32_split(tr[4], ah[2], al[2]);
          tf32_split(tr[8 * AS_LD + 4], ah[3], al[3]);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            uint32_t bh0, bl0, bh1, bl1;
            tf32_split(ys[(8 * ks + t) * 16 + 8 * nt + g], bh0, bl0);
            tf32_split(ys[(8 * ks + t + 4) * 16 + 8 * nt + g], bh1, bl1);
            mma_tf32(z[nt], ah, bh0, bh1);
            mma_tf32(z[nt], ah, bl0, bl1);
            mma_tf32(z[nt], al, bh0, bh1);
          }
        }
        float* to = Ts + (16 * bI) * AS_LD + 16 * bJ2;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          to[g * AS_LD + 8 * nt + 2 * t] = -z[nt][0];
          to[g * AS_LD + 8 * nt + 2 * t + 1] = -z[nt][1];
          to[(g + 8) * AS_LD + 8 * nt + 2 * t] = -z[nt][2];
          to[(g + 8) * AS_LD + 8 * nt + 2 * t + 1] = -z[nt][3];
        }
      }
      sync();
    }
    {
      const int r = itid >> 2, c16 = itid & 3;
      const int I = r >> 4;
      const float* sb = sc_beta + slot * 64;
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
          const float4 b0 = *reinterpret_cast<const float4*>(sb + c0);
          const float4 b1 = *reinterpret_cast<const float4*>(sb + c0 + 4);
          split2(t0v.x * b0.x, t0v.y * b0.y, wh.x, wl.x);
          split2(t0v.z * b0.z, t0v.w * b0.w, wh.y, wl.y);
          split2(t1v.x * b1.x, t1v.y * b1.y, wh.z, wl.z);
          split2(t1v.z * b1.z, t1v.w * b1.w, wh.w, wl.w);
        }
        *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(r, c0 >> 3)) = wh;
        *reinterpret_cast<uint4*>(sm + OFF_TL + sw128(r, c0 >> 3)) = wl;
      }
    }
    fence_proxy_async();
    sync();
    if (itid == 0) mbar_arrive(S_.bar + B_TB);

    // ============================================================== P T_b
    wait_bar(S_, B_PT, c & 1, p.status);
    if (len < C) wait_bar(S_, B_V_FULL, c & 1, p.status);
    sync();
    if (*abort_flag) break;
    tc_fence_after();
    if (quarter >= 2) {
      const int r = 32 * quarter + lane - 64;
      float d[32];
      tmem_ld32(tmem + lane_base + 32 * ihalf, d);
#pragma unroll
      for (int cch = 0; cch < 4; ++cch) {
        uint4 wh, wl;
        split2(d[8 * cch + 0], d[8 * cch + 1], wh.x, wl.x);
        split2(d[8 * cch + 2], d[8 * cch + 3], wh.y, wl.y);
        split2(d[8 * cch + 4], d[8 * cch + 5], wh.z, wl.z);
        split2(d[8 * cch + 6], d[8 * cch + 7], wh.w, wl.w);
        *reinterpret_cast<uint4*>(sm + OFF_TP + sw128(64 + r, 4 * ihalf + cch)) = wh;
        *reinterpret_cast<uint4*>(sm + OFF_TL + sw128(64 + r, 4 * ihalf + cch)) = wl;
      }
    }
    if (len < C) {
      // rows of the v tile past the document end (another document's, or zero-filled) -> 0
      for (int idx = itid; idx < 2 * (C - len) * 8; idx += kIntraThreads) {
        const int blk2 = idx / ((C - len) * 8), rem = idx % ((C - len) * 8);
        *reinterpret_cast<uint4*>(sm + OFF_V + blk2 * 8192 + sw128(len + rem / 8, rem & 7)) = make_uint4(0, 0, 0, 0);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    sync();
    if (itid == 0) mbar_arrive(S_.bar + B_TP);

    // ============================================================== [-W; Qtil - PW] -> TMEM
    wait_bar(S_, B_XK, c & 1, p.status);
    sync();
    if (*abort_flag) break;
    tc_fence_after();
    {
      const int R = 32 * quarter + lane;
      uint32_t packed[32];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + 64 * ihalf + 32 * part, d);
        if (R >= 64) {
          const int r = R - 64;
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            const uint4 qb = *reinterpret_cast<const uint4*>(sm + OFF_QB + ihalf * 8192 + sw128(r, 4 * part + cch));
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
      sync();  // every [W PW] column read before any is overwritten
      tc_fence_after();
      tmem_st32(tmem + lane_base + 32 * ihalf, packed);
      tmem_wait_st();
    }
    tc_fence_before();
    sync();
    if (itid == 0) mbar_arrive(S_.bar + B_WQ);
  }
}

// ------------------------------------------------------------------------------ recurrence warps
__device__ void rec_warps(const Shared& S_, const FwdParams& p, int n, int h, int64_t bos, int64_t eos,
                          int nchunks, int rtid) {
  uint8_t* sm = S_.sm;
  const uint32_t tmem = S_.tmem;
  const int H = p.num_heads;
  const int quarter = rtid >> 5, lane = rtid & 31;
  const int R = 32 * quarter + lane;  // TMEM lane: state row k, or chunk row (Delta / O)
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  const float* sc_ik = reinterpret_cast<const float*>(sm + OFF_SC + SC_IK);
  const float* sc_gam = reinterpret_cast<const float*>(sm + OFF_SC + SC_GAM);
  const size_t soff = ((size_t)n * H + h) * (size_t)D * D;

  auto store_row_bf16 = [&](int part, const float (&v)[32]) {
    // columns 32 part .. 32 part + 31 of row R of the bf16 state (MN tile of 128 rows)
    uint8_t* base = sm + OFF_S + (part >> 1) * (128 * 128);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 w;
      w.x = pack_bf16(v[8 * c + 0], v[8 * c + 1]);
      w.y = pack_bf16(v[8 * c + 2], v[8 * c + 3]);
      w.z = pack_bf16(v[8 * c + 4], v[8 * c + 5]);
      w.w = pack_bf16(v[8 * c + 6], v[8 * c + 7]);
      *reinterpret_cast<uint4*>(base + sw128(R, 4 * (part & 1) + c)) = w;
    }
  };
  auto store_final = [&](int part, const float (&v)[32]) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int col = 32 * part + j;
      if (p.state_transposed) p.final_state[soff + (size_t)col * D + R] = v[j];
      else p.final_state[soff + (size_t)R * D + col] = v[j];
    }
  };

  // initial state: bf16 copy for MMA1(0); fp32 copy pre-scaled by e^{Gamma_C}(0) for MMA2(0)
  {
    bool ok = true;
    if (nchunks > 0) ok = wait_bar(S_, B_OPS0, 0, p.status);
    const float gam = (nchunks > 0 && ok) ? sc_gam[R] : 1.f;
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = 32 * part + j;
        float s = 0.f;
        if (p.initial_state)
          s = p.state_transposed ? p.initial_state[soff + (size_t)col * D + R]
                                 : p.initial_state[soff + (size_t)R * D + col];
        v[j] = s;
      }
      if (nchunks == 0) {
        if (p.final_state) store_final(part, v);
        continue;
      }
      store_row_bf16(part, v);
      uint32_t u[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(gam * v[j]);
      tmem_st32(tmem + lane_base + TM_S + 32 * part, u);
    }
    if (nchunks == 0) return;
    tmem_wait_st();
    fence_proxy_async();
    tc_fence_before();
    named_bar(kBarRec, kRecThreads);
    if (*S_.abort) return;
    if (rtid == 0) mbar_arrive(S_.bar + B_S);
  }

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int len = (int)((eos - t0) < (int64_t)C ? (eos - t0) : (int64_t)C);
    const int slot = c & 1;
    // ============================================================== ep1: Delta and O
    // the scalar slot of this chunk (1/|k|) is acquired from the intra warps' own barrier
    wait_bar(S_, B_OPS0 + slot, (c >> 1) & 1, p.status);
    wait_bar(S_, B_MMA1, c & 1, p.status);
    named_bar(kBarRec, kRecThreads);
    if (*S_.abort) break;
    tc_fence_after();
    {
      const int r = R & 63;
      const float ikr = sc_ik[slot * 64 + r];
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + TM_UP + 32 * part, d);
        if (R < 64) {
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            uint4 wh, wl;
            split2(d[8 * cch + 0] * ikr, d[8 * cch + 1] * ikr, wh.x, wl.x);
            split2(d[8 * cch + 2] * ikr, d[8 * cch + 3] * ikr, wh.y, wl.y);
            split2(d[8 * cch + 4] * ikr, d[8 * cch + 5] * ikr, wh.z, wl.z);
            split2(d[8 * cch + 6] * ikr, d[8 * cch + 7] * ikr, wh.w, wl.w);
            const uint32_t off = (part >> 1) * 8192 + sw128(r, 4 * (part & 1) + cch);
            *reinterpret_cast<uint4*>(sm + OFF_DL + off) = wh;
            *reinterpret_cast<uint4*>(sm + OFF_DLLO + off) = wl;
          }
        } else if (r < len) {
          __nv_bfloat16* orow = p.out + ((size_t)(t0 + r) * H + h) * D + 32 * part;
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
    fence_proxy_async();
    tc_fence_before();
    named_bar(kBarRec, kRecThreads);
    if (rtid == 0) mbar_arrive(S_.bar + B_DELTA);

    // ============================================================== ep2: state
    wait_bar(S_, B_MMA2, c & 1, p.status);
    const bool last = (c + 1 == nchunks);
    if (!last) wait_bar(S_, B_OPS0 + ((c + 1) & 1), ((c + 1) >> 1) & 1, p.status);
    named_bar(kBarRec, kRecThreads);
    if (*S_.abort) break;
    tc_fence_after();
    {
      const float gam = last ? 1.f : sc_gam[((c + 1) & 1) * 128 + R];
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {
        float v[32];
        tmem_ld32(tmem + lane_base + TM_S + 32 * part, v);
        if (last) {
          if (p.final_state) store_final(part, v);
        } else {
          store_row_bf16(part, v);
          uint32_t u[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(gam * v[j]);
          tmem_st32(tmem + lane_base + TM_S + 32 * part, u);
        }
      }
      if (!last) tmem_wait_st();
    }
    if (last) break;
    fence_proxy_async();
    tc_fence_before();
    named_bar(kBarRec, kRecThreads);
    if (rtid == 0) mbar_arrive(S_.bar + B_S);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    chunked_kernel(const __grid_constant__ TensorMaps maps, FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared S_;
  S_.sm = sm;
  S_.sbase = smem_u32(sm);
  S_.bar = reinterpret_cast<uint64_t*>(sm + OFF_SC + SC_BAR);
  S_.abort = reinterpret_cast<volatile int*>(sm + OFF_SC + SC_ABORT);
  uint32_t* sc_tmem = reinterpret_cast<uint32_t*>(sm + OFF_SC + SC_TMEM);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = p.num_heads;
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  int64_t bos, eos;
  seq_range(p, n, bos, eos);
  if (tid == 0 && h == 0 && p.status && !seq_entries_ok(p, n)) atomicOr(p.status, kStatusBadSeqlens);
  // offsets out of order: every document is empty (as in the split path), so no two units can
  // write the same output rows
  if (!cta_seqlens_ok(p)) eos = bos;
  const int nchunks = (int)((eos - bos + C - 1) / C);

  if (tid == 0) {
    for (int b = 0; b < B_COUNT; ++b) mbar_init(S_.bar + b, 1);
    *S_.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
  }
  if (warp == 0) {
    tmem_alloc(sc_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  S_.tmem = *sc_tmem;

  // register budget per warpgroup: control 56, intra 168, recurrence 96 (4*56 + 8*168 + 4*96 warps-worth
  // of 32-thread rows = 62464 <= 65536)
  if (warp < kIntraWarp0) {
    setmaxnreg_dec<56>();
    if (warp == 0) {
      if (lane == 0) mma_issuer(S_, p, nchunks);
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) tma_producer(S_, maps, p, h, bos, nchunks);
      __syncwarp();
    }
  } else if (warp < kRecWarp0) {
    setmaxnreg_inc<168>();
    intra_warps(S_, p, h, bos, eos, nchunks, tid - 32 * kIntraWarp0);
  } else {
    setmaxnreg_dec<96>();
    rec_warps(S_, p, n, h, bos, eos, nchunks, tid - 32 * kRecWarp0);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(S_.tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------ host side

}  // namespace

cudaError_t launch_chunked(const FwdParams& p, cudaStream_t stream) {
  const int64_t units = (int64_t)p.num_seqs * p.num_heads;
  if (units == 0) return cudaSuccess;
  const int64_t tokens = p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs;
  TensorMaps maps;
  if (!make_token_map(&maps.q, p.q, tokens, p.num_heads) || !make_token_map(&maps.k, p.k, tokens, p.num_heads) ||
      !make_token_map(&maps.v, p.v, tokens, p.num_heads))
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  cudaError_t e = set_smem_once(chunked_kernel, SMEM_ALLOC, attr_set);
  if (e != cudaSuccess) return e;
  chunked_kernel<<<(unsigned)units, kThreads, SMEM_ALLOC, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace kda
