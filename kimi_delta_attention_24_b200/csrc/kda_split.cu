// Chunked KDA forward for sm_100a, split into a chunk-parallel intra-chunk kernel and a
// per-(sequence, head) recurrence kernel.
//
// Kimi Delta Attention (FlashKDA `fwd`, fla `chunk_kda`; vLLM PR #54859 report and "What CUDA
// Version Is Required to Use FlashKDA?", Usage Examples) is the gated delta rule
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = scale S_t^T q_t,
// evaluated in chunks of C = 64 tokens in the WY/UT form.  With Gamma the in-chunk cumulative
// log-decay and Khat/Qhat the L2-normalised keys/queries:
//   A = strict_tril(diag(beta) (Khat e^Gamma)(Khat e^-Gamma)^T),  T = (I + A)^{-1},  T_b = T diag(beta),
//   P = scale tril((Qhat e^Gamma)(Khat e^-Gamma)^T),  W = T_b (Khat e^Gamma),  U = T_b V,
//   Qtil = scale Qhat e^Gamma,  Ktil = Khat e^{Gamma_C - Gamma},
// and per chunk
//   Delta = U - W S,   O = Qtil S + P Delta = (Qtil - P W) S + P U,   S <- Diag(e^{Gamma_C}) S + Ktil^T Delta.
//
// Everything that does not involve S is independent across chunks, so it runs chunk-parallel over
// every SM (intra_kernel, persistent, two CTAs per SM): the gate, the norms, the decays, the Gram
// products, the solve and the products with T_b.  It leaves one "item" per (chunk, head) in the
// workspace, stored as the byte image of the shared-memory tiles the recurrence feeds its MMAs:
//   [-W; Qtil - P W]   (B of MMA1, K-major)          [T_b; P T_b] hi and lo   (B of MMA Xv, K-major)
//   Ktil (raw k scaled by the decays; B of MMA2)     1/|k_r| per row, e^{Gamma_C} per channel.
// rec_kernel then walks each (sequence, head) chunk by chunk with the state transposed (S^T) and
// every state-side operand in tensor memory (its own comment below gives the steps).
// The hi+lo pairs matter when keys are nearly collinear (T then has entries near -beta that cancel
// against the diagonal, and a chunk's Delta rows telescope), and Ktil is built from the raw bf16 k
// with 1/|k| applied to Delta, so that equal keys round identically.
//
// Launches, on one stream: chunk_table_kernel (chunk offsets, item counters), then intra and rec
// over global chunks [0, g_cut), then intra and rec over [g_cut, end).  Each launch after the first
// intra carries the programmatic-serialization attribute: when the recurrence (one CTA and one SM
// per (sequence, head)) leaves SMs free, the second intra launch fills them while the first
// recurrence runs.  g_cut = end (one stage) when there are at least as many units as SMs.
//
// Every wait is bounded (kWaitLimitNs of wall time): on expiry the kernel records
// KDA_ERR_DEVICE_TIMEOUT in the workspace status word and the affected work is skipped.
#include <type_traits>
#include "kda_device.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;
constexpr int D = kHeadDim;

// ------------------------------------------------------------------------- item image (workspace)
constexpr uint32_t IT_WQ = 0;          // [-W; Qtil - P W] bf16: 2 K-blocks x [128 rows][128 B], SW128
constexpr uint32_t IT_TP = 32768;      // [T_b; P T_b] hi: [128 rows][128 B], SW128 (K = 64 tokens)
constexpr uint32_t IT_TL = 49152;      // [T_b; P T_b] lo
constexpr uint32_t IT_KT = 65536;      // Ktil: 2 channel blocks x [64 tokens][128 B], SW128
constexpr uint32_t IT_IK = 81920;      // float[64] 1/|k_r| (0 past the end of the sequence)
constexpr uint32_t IT_GAM = 82176;     // float[128] e^{Gamma_C}
constexpr uint32_t IT_SC_BYTES = 768;  // IT_IK .. IT_GAM + 512
constexpr uint32_t ITEM_BYTES = 82944;

struct SplitArgs {
  FwdParams p;
  const int32_t* chunk_off;  // [N + 1] first global chunk of each sequence
  uint8_t* items;            // ITEM_BYTES per (global chunk, head), chunk-major
  int64_t item_begin, item_end;  // intra_kernel: items [item_begin, item_end) (item = chunk * H + head)
  int64_t g0, g1;                // rec_kernel: global chunks [g0, g1) (g1 = INT64_MAX: to the end)
  float* boundary;               // [H][128 * 128] S^T of the one sequence cut between two launches
  unsigned long long* queue;     // intra_kernel: item counter (zeroed by chunk_table_kernel)
  // rec_kernel map mode (the segment map S_out = M S_in + B of each unit): a grid of 2 N H CTAs;
  // CTA u < N H computes B (v as given, zero initial state), CTA N H + u computes M (v = 0, identity
  // initial state); each writes its final state [k][v] to map_B / map_M and no output.
  int map_mode;
  float* map_M;                  // [N, H, 128, 128]
  float* map_B;                  // [N, H, 128, 128]
  float* ckpt;                   // checkpoint mode: [T / 64 + N + 1 slots][H][128 v][128 k] chunk-start states
};

constexpr int kQueues = 2;  // item counters in the workspace header, one per intra launch

// ------------------------------------------------------------------------- chunk table
// chunk_off[n] = sum over m < n of ceil(len_m / C); one block of 1024 threads.  A cu_seqlens that
// does not tile the T tokens in order gives every sequence zero chunks (so no later kernel reads a
// token or writes an output) and raises kStatusBadSeqlens; the final states are then the initial ones.
__global__ void __launch_bounds__(1024) chunk_table_kernel(FwdParams p, int32_t* chunk_off,
                                                           unsigned long long* queues) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    chunk_off[0] = 0;
    for (int i = 0; i < kQueues; ++i) queues[i] = 0;
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
      const int64_t len = eos > bos ? eos - bos : 0;
      cnt = (int32_t)((len + C - 1) / C);
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
      warp_tot[lane] = w;  // inclusive
    }
    __syncthreads();
    const int32_t incl = carry + x + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (n < p.num_seqs) chunk_off[n + 1] = incl;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
}

// Sequence of global chunk gc: the largest n with chunk_off[n] <= gc (skips empty sequences).
__device__ __forceinline__ int seq_of_chunk(const int32_t* co, int nseq, int64_t gc) {
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)co[mid] <= gc) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// ========================================================================= intra-chunk kernel
// 256 threads, two CTAs per SM.  Shared-memory map (bytes from a 1024-aligned base); "MN tile" =
// 2 blocks of 64 columns x [64 rows][128 B] with the 128-byte swizzle, "K tile" = 2 blocks of 64 K
// x [rows][128 B].
constexpr int kIntraThreads = 256;
constexpr uint32_t I_RQ = 0;        // q tile (TMA); becomes XK row by row in pass 1
constexpr uint32_t I_RK = 16384;    // k tile (TMA); becomes QB once k sits in registers
constexpr uint32_t I_XK = 0;        // -Khat e^Gamma (pre-scaled to the chunk start), MN tile, B of MMA Xk
constexpr uint32_t I_QB = 16384;    // Qtil, MN tile, B of the MMA that seeds [0; Qtil]
constexpr uint32_t I_LKQ = 32768;   // [LK; LQ] K tile, 128 rows (A of MMA AP)
constexpr uint32_t I_R = 65536;     // R_1..R_3 K tile, 144 rows (B of MMA AP)
constexpr uint32_t kRRows = 144;
constexpr uint32_t I_RKBLK = kRRows * 128;
constexpr uint32_t I_TP = 32768;    // after MMA AP: [T_b hi; P -> (P T_b) hi], 128 rows x 64
constexpr uint32_t I_TL = 49152;    //               [T_b lo; (P T_b) lo]
constexpr uint32_t I_AS = 65536;    //               A fp32 64 x 68 (then, over AS and TS, the
                                    //               [-W; Qtil - P W] image for the bulk copy)
constexpr uint32_t I_TS = 82944;    //               T fp32 64 x 68
constexpr uint32_t I_YS = 100352;   //               solve temporaries 8 x 16 x 8 fp32
constexpr uint32_t AS_LD = 68;
constexpr uint32_t I_SC = 106496;   // scalars
constexpr uint32_t I_TOT = I_SC;            // float[8][128] per-warp alpha products
constexpr uint32_t I_BETA = I_SC + 4096;    // float[64]
constexpr uint32_t I_BAR = I_SC + 4352;     // 3 mbarriers
constexpr uint32_t I_TMEM = I_SC + 4376;    // allocated TMEM address
constexpr uint32_t I_ABORT = I_SC + 4380;
constexpr uint32_t I_SMEM = I_SC + 4480;
constexpr uint32_t I_ALLOC = I_SMEM + 1024;
static_assert(I_YS + 4096 <= I_SC, "intra shared-memory map");
static_assert(2 * (I_ALLOC + 1024) <= 233472, "two intra CTAs per SM");
constexpr uint32_t kIntraTmemCols = 256;
constexpr uint32_t kIdCol = 192;  // [0; I_64] as bf16 (32 columns), A of the MMA that seeds [0; Qtil]
// Row of the R tile where the right operand of row block I starts.  Row block I >= 1 refers its
// Gram entries to the decays at its own start, so R_I holds rows 0 .. 16 I + 15 of Khat scaled to
// that reference; row block 0 refers to the start of block 1 (its left factors then lie in
// [1, e^{80}], its right ones in [e^{-80}, 1]) and shares R_1.
__host__ __device__ constexpr uint32_t r_seg(int I) { return I <= 1 ? 0u : 8u * I * (I + 1) - 16u; }
static_assert(r_seg(3) + 64 == kRRows, "R tile rows");

struct IntraMaps {
  CUtensorMap q, k, g;
};

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }
__device__ __forceinline__ uint32_t bf16x2_of(float2 v) { return bf16x2(v.x, v.y); }

// Persistent: every CTA takes items [item_begin, item_end) in chunk-major order (item = global
// chunk * H + head) from a shared counter, pulling its next item's q, k and g tiles into L2 while
// it works on the current one and loading the next q, k tiles as soon as MMA Xk has freed them.
// Per item (8 warps; warp iw owns rows 8 iw .. + 7 in the element-wise phases):
//   prologue  norms, sigmoid(beta), the gate, per-warp decay products (q read, k kept in registers)
//   pass 1    [LK; LQ] (Gram left operand), XK = -Khat e^Gamma and QB = Qtil (q read again)
//   pass 2    R_1..R_3 (Gram right operand, one decay reference per row block) and Ktil (to the item)
//   MMA AP    [LK; LQ] R^T (N = 144) -> assembly of A (fp32) and P (bf16)
//   solve     diagonal 16 x 16 blocks by substitution (warps 0 and 5, which assembled them), then
//             the off-diagonal blocks column by column on 3xTF32 mma.sync, warp-local levels
//   T_b       hi + lo split; MMA PT: P T_b (hi + lo), read back as a hi + lo pair
//   MMA Xk    [0; I] Qtil + [T_b; P T_b] (-XK) = [-W; Qtil - P W] in one accumulator -> bf16 image
// kGatePre: g holds fp32 log alpha (the safe gate is not applied; values are clamped to
// [lower_bound, 0], the range the exponent referencing relies on).  The other input flags (no q/k
// L2 norm, fp32 beta) are uniform run-time branches.
template <bool kGatePre>
__global__ void __launch_bounds__(kIntraThreads, 2)
    intra_kernel(const __grid_constant__ IntraMaps maps, const SplitArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const FwdParams& p = args.p;
  const int H = p.num_heads;
  const int32_t* co = args.chunk_off;

  const int itid = threadIdx.x;
  const int iw = itid >> 5, lane = itid & 31;
  const uint32_t sbase = smem_u32(sm);
  // [0] q/k tiles landed, [1] MMA done, [2] final drain
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + I_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + I_ABORT);
  float* sc_tot = reinterpret_cast<float*>(sm + I_TOT);
  float* sc_beta = reinterpret_cast<float*>(sm + I_BETA);
  float* As = reinterpret_cast<float*>(sm + I_AS);
  float* Ts = reinterpret_cast<float*>(sm + I_TS);
  float* Ys = reinterpret_cast<float*>(sm + I_YS);
  auto sync = [&]() { __syncthreads(); };

  if (itid == 0) {
    mbar_init(bar + 0, 1);
    mbar_init(bar + 1, 1);
    mbar_init(bar + 2, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.g);
  }
  if (iw == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(sm + I_TMEM), kIntraTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + I_TMEM);
  // A = [0; I_64] (128 x 64 bf16, two per column, low half first) in columns kIdCol .. + 31, which
  // no accumulator reaches (the Gram product uses columns 0 .. 159)
  if (iw < 4) {
    const int r = 32 * iw + lane - 64;  // identity row, or negative in the zero half
    uint32_t u[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) u[c] = (r >= 0 && (r >> 1) == c) ? ((r & 1) ? 0x3F800000u : 0x3F80u) : 0u;
    tmem_st32(tmem + ((uint32_t)(32 * iw) << 16) + kIdCol, u);
    tmem_wait_st();
  }
  tc_fence_before();
  sync();
  tc_fence_after();

  // one thread waits on the mbarrier, the others in the CTA barrier; the answer (abort?) is uniform
  uint32_t raw_par = 0, mma_par = 0;
  bool raw_pending = false;  // thread 0: a q/k load is armed and has not been seen to land
  auto cta_wait = [&](int b, uint32_t& par) -> bool {
    if (itid == 0 && bounded_wait(bar + b, par, abort_flag, p.status) && b == 0) raw_pending = false;
    par ^= 1;
    return __syncthreads_or(*abort_flag) != 0;
  };
  struct Loc {
    int h, len;
    int64_t t0, gc;
  };
  auto locate = [&](int64_t gc, int h) {
    Loc L;
    L.gc = gc;
    L.h = h;
    const int n = seq_of_chunk(co, p.num_seqs, gc);
    int64_t bos, eos;
    seq_range(p, n, bos, eos);
    L.t0 = bos + (gc - co[n]) * C;
    L.len = (int)((eos - L.t0) < (int64_t)C ? (eos - L.t0) : (int64_t)C);
    return L;
  };
  const int64_t total_gc = co[p.num_seqs];

  // prologue mapping: warp iw owns chunk rows 8 iw .. 8 iw + 7, lane owns channels 4 lane .. +3
  const int kb = lane >> 4;
  const uint32_t lane_chunk = (lane & 15) >> 1;
  const uint32_t lane_sub = (lane & 1) * 8;
  const int blk = iw >> 1;
  const bool upper_half = iw & 1;
  const int quarter = iw & 3, ihalf = iw >> 2;  // TMEM lane quarter, column half
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  const float lb2 = p.lower_bound * kLog2e;
  // shared-memory byte offset of this thread's 8 bytes of row 8 iw + i inside a 128-byte-row tile
  const uint32_t xo_base = (uint32_t)(iw * 1024) + lane_sub, xo_l = lane_chunk << 4;
  auto xo = [&](int i) { return xo_base + (uint32_t)(i * 128) + (xo_l ^ (uint32_t)(i << 4)); };
  const uint32_t a_rq = sbase + I_RQ + kb * 8192, a_rk = sbase + I_RK + kb * 8192;
  const uint32_t a_lk = sbase + I_LKQ + kb * 16384, a_lq = a_lk + 64 * 128;
  const uint32_t a_xk = sbase + I_XK + kb * 8192, a_qb = sbase + I_QB + kb * 8192;
  const uint32_t a_r = sbase + I_R + kb * I_RKBLK;
  // matrix descriptors of the MMA operand tiles (thread 0 issues; k-steps are offsets)
  const uint64_t d_lkq = sdesc_sw128(sbase + I_LKQ, 16, 1024);   // K-major, 128 rows
  const uint64_t d_r = sdesc_sw128(sbase + I_R, 16, 1024);       // K-major, 144 rows
  const uint64_t d_tpk = sdesc_sw128(sbase + I_TP, 16, 1024);    // [T; P] / [T; PT] as K-major A
  const uint64_t d_tlk = sdesc_sw128(sbase + I_TL, 16, 1024);
  const uint64_t d_tpm = sdesc_sw128(sbase + I_TP, 8192, 1024);  // T_b hi / lo as MN-major B
  const uint64_t d_tlm = sdesc_sw128(sbase + I_TL, 8192, 1024);
  const uint64_t d_xk = sdesc_sw128(sbase + I_XK, 8192, 1024);   // MN-major B
  const uint64_t d_qb = sdesc_sw128(sbase + I_QB, 8192, 1024);   // MN-major B

  // Items (gc * H + h, chunk-major) come from a counter, so that a CTA that starts late (on an SM
  // freed by another kernel) takes fewer.  Thread 32 takes the next item while the current one runs,
  // locates it (sequence, first token, length) and publishes both in s_item / s_loc[j & 1]
  // (double-buffered: read after the item's last barrier).
  __shared__ int64_t s_item[2];
  __shared__ Loc s_loc[2];
  const int64_t item_end = args.item_end < total_gc * H ? args.item_end : total_gc * H;
  if (itid == 0) {
    const int64_t it = args.item_begin + (int64_t)atomicAdd(args.queue, 1ull);
    s_item[1] = it;
    if (it < item_end) {
      const int64_t gc = it / H;
      s_loc[1] = locate(gc, (int)(it - gc * H));
    }
  }
  __syncthreads();
  // thread 0: the q and k tiles of an item (issued for the next item as soon as MMA Xk of the
  // current one has read XK / QB, the tiles they land in)
  auto load_qk = [&](const Loc& N) {
    raw_pending = true;
    mbar_arrive_expect_tx(bar + 0, 32768);
    tma_load_3d(sm + I_RQ, &maps.q, bar + 0, 0, N.h, (int)N.t0);
    tma_load_3d(sm + I_RQ + 8192, &maps.q, bar + 0, 64, N.h, (int)N.t0);
    tma_load_3d(sm + I_RK, &maps.k, bar + 0, 0, N.h, (int)N.t0);
    tma_load_3d(sm + I_RK + 8192, &maps.k, bar + 0, 64, N.h, (int)N.t0);
  };
  int64_t cur_it = s_item[1];
  if (itid == 0 && cur_it < item_end) load_qk(s_loc[1]);
  for (uint32_t j = 0; cur_it < item_end; ++j) {
    const Loc L = s_loc[(j + 1) & 1];
    const int h = L.h, len = L.len;
    const int64_t t0 = L.t0;
    uint8_t* item = args.items + ((size_t)L.gc * H + h) * ITEM_BYTES;
    int64_t nxt = 0;
    if (itid == 32) nxt = args.item_begin + (int64_t)atomicAdd(args.queue, 1ull);

    float2 ga2, gb2[2];
    uint2 gr[8];
    float4 gf[kGatePre ? 8 : 1];
    if constexpr (!kGatePre) {
      const float gate_a = __expf(p.A_log[h]);
      const float4 dtb = reinterpret_cast<const float4*>(p.dt_bias + (size_t)h * D)[lane];
      const float ga = -gate_a * kLog2e;  // exp(-a (g + dt)) = exp2(ga g + gb)
      ga2 = splat2(ga);
      gb2[0] = make_float2(ga * dtb.x, ga * dtb.y);
      gb2[1] = make_float2(ga * dtb.z, ga * dtb.w);
      const __nv_bfloat16* gp = p.g + ((size_t)(t0 + 8 * iw) * H + h) * D + 4 * lane;
      const uint32_t row_stride = (uint32_t)H * D;  // elements between consecutive tokens
#pragma unroll
      for (int i = 0; i < 8; ++i) gr[i] = (8 * iw + i < len) ? ldg_u2(gp + i * row_stride) : make_uint2(0, 0);
    } else {
      const float4* gp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.g) +
                                                         ((size_t)(t0 + 8 * iw) * H + h) * D) + lane;
      const uint32_t row_stride = (uint32_t)H * (D / 4);  // float4s between consecutive tokens
#pragma unroll
      for (int i = 0; i < 8; ++i)
        gf[i] = (8 * iw + i < len) ? __ldg(gp + i * row_stride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float beta_raw = 0.f;
    if (8 * iw + (lane & 7) < len) {
      const size_t bi = (size_t)(t0 + 8 * iw) * H + h + (uint32_t)(lane & 7) * (uint32_t)H;
      beta_raw = (p.flags & kFlagBetaPrecomputed) ? reinterpret_cast<const float*>(p.beta)[bi]
                                                  : __bfloat162float(p.beta[bi]);
    }

    // ================================================================ prologue
    if (cta_wait(0, raw_par)) break;
    if (itid == 32) {
      // the counter's answer has had the q / k load's time to arrive; warm L2 for the next item
      s_item[j & 1] = nxt;
      if (nxt < item_end) {
        const int64_t ngc = nxt / H;
        const Loc N = locate(ngc, (int)(nxt - ngc * H));
        s_loc[j & 1] = N;
        tma_prefetch_3d(&maps.q, 0, N.h, (int)N.t0);
        tma_prefetch_3d(&maps.q, 64, N.h, (int)N.t0);
        tma_prefetch_3d(&maps.k, 0, N.h, (int)N.t0);
        tma_prefetch_3d(&maps.k, 64, N.h, (int)N.t0);
        tma_prefetch_3d(&maps.g, 0, N.h, (int)N.t0);
        tma_prefetch_3d(&maps.g, 64, N.h, (int)N.t0);
      }
    }
    // k stays in registers (its tile becomes QB in pass 1); q is read again in pass 1, from the
    // same 8 bytes that its XK value then overwrites
    uint2 kr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) kr[i] = (8 * iw + i < len) ? lds64(a_rk + xo(i)) : make_uint2(0, 0);
    float2 a2[8][2];  // alpha of channels (4 lane, +1), (4 lane + 2, +3)
    float ssq[8], ssk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool valid = 8 * iw + i < len;
      const uint2 qri = valid ? lds64(a_rq + xo(i)) : make_uint2(0, 0);
      const float2 q01 = unpack_bf16(qri.x), q23 = unpack_bf16(qri.y);
      const float2 k01 = unpack_bf16(kr[i].x), k23 = unpack_bf16(kr[i].y);
      const float2 sq = fma2(q23, q23, mul2(q01, q01)), sk = fma2(k23, k23, mul2(k01, k01));
      ssq[i] = sq.x + sq.y;
      ssk[i] = sk.x + sk.y;
      if constexpr (!kGatePre) {
        const float2 gv[2] = {unpack_bf16(gr[i].x), unpack_bf16(gr[i].y)};
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const float2 x = fma2(ga2, gv[m], gb2[m]);
          const float2 d = fma2(make_float2(ex2_approx(x.x), ex2_approx(x.y)), splat2(1.f), splat2(1.f));
          const float2 y = mul2(splat2(lb2), make_float2(rcp_approx(d.x), rcp_approx(d.y)));
          a2[i][m] = valid ? make_float2(ex2_approx(y.x), ex2_approx(y.y)) : make_float2(1.f, 1.f);
        }
      } else {
        // log alpha clamped to [lower_bound, 0], then alpha = 2^(log2 e * log alpha)
        const float lg[4] = {gf[i].x, gf[i].y, gf[i].z, gf[i].w};
        float al[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) al[c] = ex2_approx(fminf(fmaxf(lg[c], p.lower_bound), 0.f) * kLog2e);
        a2[i][0] = valid ? make_float2(al[0], al[1]) : make_float2(1.f, 1.f);
        a2[i][1] = valid ? make_float2(al[2], al[3]) : make_float2(1.f, 1.f);
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
      inv = (p.flags & kFlagNoQkL2Norm) ? 1.f : rsqrtf(w1 + kL2Eps);
    }
    const float beta_l = (lane < 8 && 8 * iw + lane < len)
                             ? ((p.flags & kFlagBetaPrecomputed) ? beta_raw : fast_sigmoid(beta_raw))
                             : 0.f;
    const float inv_s = inv * (lane < 16 ? p.scale : 1.f);  // scale folded into 1/|q|
    {
      const float ikr = __shfl_sync(0xffffffffu, inv, 16 + 2 * (lane & 7));  // 1/|k| of row 8 iw + (lane & 7)
      if (lane < 8) {
        const int r = 8 * iw + lane;
        sc_beta[r] = beta_l;
        reinterpret_cast<float*>(item + IT_IK)[r] = (r < len) ? ikr : 0.f;
      }
    }
    // per-warp alpha totals -> sub-block totals b_J
    {
      float2 t[2] = {a2[0][0], a2[0][1]};
#pragma unroll
      for (int i = 1; i < 8; ++i) {
        t[0] = mul2(t[0], a2[i][0]);
        t[1] = mul2(t[1], a2[i][1]);
      }
      reinterpret_cast<float4*>(sc_tot + iw * 128)[lane] = make_float4(t[0].x, t[0].y, t[1].x, t[1].y);
    }
    // the previous item's bulk copies have read TP / TL / AS, which the passes overwrite
    if (itid == 0) bulk_wait_read<0>();
    sync();  // also: every thread holds its k rows, so the k tile may be overwritten
    // sub-block totals b_J = prod of alpha over rows 16 J .. 16 J + 15 (channels 4 lane .. + 3)
    auto load_bJ = [&](float2 (&bJ)[4][2]) {
#pragma unroll
      for (int J = 0; J < 4; ++J) {
        const float4 t0v = reinterpret_cast<const float4*>(sc_tot + (2 * J) * 128)[lane];
        const float4 t1v = reinterpret_cast<const float4*>(sc_tot + (2 * J + 1) * 128)[lane];
        bJ[J][0] = mul2(make_float2(t0v.x, t0v.y), make_float2(t1v.x, t1v.y));
        bJ[J][1] = mul2(make_float2(t0v.z, t0v.w), make_float2(t1v.z, t1v.w));
      }
    };
    float2 pre[2], pt[2];
    {
      float2 bJ[4][2];
      load_bJ(bJ);
      const float4 pv = reinterpret_cast<const float4*>(sc_tot + (iw ^ 1) * 128)[lane];
      pt[0] = make_float2(pv.x, pv.y);
      pt[1] = make_float2(pv.z, pv.w);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        float2 pa = make_float2(1.f, 1.f);
#pragma unroll
        for (int J = 0; J < 4; ++J)
          if (J < blk) pa = mul2(pa, bJ[J][m]);
        pre[m] = pa;
      }
      if (iw == 0) {
        const float2 g0 = mul2(mul2(bJ[0][0], bJ[1][0]), mul2(bJ[2][0], bJ[3][0]));
        const float2 g1 = mul2(mul2(bJ[0][1], bJ[1][1]), mul2(bJ[2][1], bJ[3][1]));
        reinterpret_cast<float4*>(item + IT_GAM)[lane] = make_float4(g0.x, g0.y, g1.x, g1.y);
      }
    }

    // pass 1, rows ascending: e_i = prod of alpha from the sub-block start to row i.  Rows of
    // sub-block J >= 1 refer to its start, rows of sub-block 0 to the start of sub-block 1 (e_i / b_0);
    // XK = -Khat e^Gamma and QB = Qtil refer to the chunk start, where pre takes them.  XK is
    // written negated, so that MMA Xk subtracts [W; P W] from the [0; Qtil] it starts from
    {
      float2 run[2];
#pragma unroll
      for (int m = 0; m < 2; ++m) run[m] = upper_half ? pt[m] : make_float2(1.f, 1.f);
      if (blk == 0) {
        const float4 t0v = reinterpret_cast<const float4*>(sc_tot)[lane];
        const float4 t1v = reinterpret_cast<const float4*>(sc_tot + 128)[lane];
        const float2 b0[2] = {mul2(make_float2(t0v.x, t0v.y), make_float2(t1v.x, t1v.y)),
                              mul2(make_float2(t0v.z, t0v.w), make_float2(t1v.z, t1v.w))};
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          run[m] = mul2(run[m], make_float2(1.0f / b0[m].x, 1.0f / b0[m].y));
          pre[m] = b0[m];
        }
      }
      const float2 npre[2] = {make_float2(-pre[0].x, -pre[0].y), make_float2(-pre[1].x, -pre[1].y)};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint2 qri = (8 * iw + i < len) ? lds64(a_rq + xo(i)) : make_uint2(0, 0);
        const float2 qv[2] = {unpack_bf16(qri.x), unpack_bf16(qri.y)};
        const float2 kv[2] = {unpack_bf16(kr[i].x), unpack_bf16(kr[i].y)};
        const float2 iq = splat2(__shfl_sync(0xffffffffu, inv_s, 2 * i));
        const float2 ik = splat2(__shfl_sync(0xffffffffu, inv_s, 16 + 2 * i));
        const float2 b = splat2(__shfl_sync(0xffffffffu, beta_l, i));
        float2 lk[2], lq[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          run[m] = mul2(run[m], a2[i][m]);
          lk[m] = mul2(kv[m], mul2(run[m], ik));  // khat * e
          lq[m] = mul2(qv[m], mul2(run[m], iq));  // scale * qhat * e
        }
        sts64(a_lk + xo(i), bf16x2_of(mul2(lk[0], b)), bf16x2_of(mul2(lk[1], b)));
        sts64(a_lq + xo(i), bf16x2_of(lq[0]), bf16x2_of(lq[1]));
        sts64(a_xk + xo(i), bf16x2_of(mul2(lk[0], npre[0])), bf16x2_of(mul2(lk[1], npre[1])));
        sts64(a_qb + xo(i), bf16x2_of(mul2(lq[0], pre[0])), bf16x2_of(mul2(lq[1], pre[1])));
      }
    }
    // pass 2, rows descending: f_i = prod of alpha after row i to the sub-block end; Ktil goes
    // straight to the item (same swizzled image as a shared-memory MN tile).  Specialised on the
    // warp's row block B, which writes R_max(B,1) .. R_3
    {
      float2 bJ[4][2];
      load_bJ(bJ);
      uint8_t* kt_dst = item + IT_KT + kb * 8192;
      auto pass2 = [&](auto nb) {
        constexpr int B = decltype(nb)::value;
        constexpr int I0 = B < 1 ? 1 : B;
        float2 post[2], cI[4][2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          float2 z = make_float2(1.f, 1.f);
#pragma unroll
          for (int J = B + 1; J < 4; ++J) z = mul2(z, bJ[J][m]);
          post[m] = z;
          if (B >= 1) cI[B][m] = make_float2(1.0f / bJ[B][m].x, 1.0f / bJ[B][m].y);
          float2 mm = make_float2(1.f, 1.f);
#pragma unroll
          for (int I = B + 1; I < 4; ++I) {
            cI[I][m] = mm;
            mm = mul2(mm, bJ[I][m]);
          }
        }
        float2 run[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) run[m] = upper_half ? make_float2(1.f, 1.f) : pt[m];
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          const float2 kv[2] = {unpack_bf16(kr[i].x), unpack_bf16(kr[i].y)};
          const float2 ik = splat2(__shfl_sync(0xffffffffu, inv_s, 16 + 2 * i));
          float2 kr_f[2], kf[2];
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            kr_f[m] = mul2(kv[m], run[m]);  // raw k * f, shared by R (normalised) and Ktil
            kf[m] = mul2(kr_f[m], ik);      // khat * f
          }
#pragma unroll
          for (int I = I0; I < 4; ++I)
            sts64(a_r + r_seg(I) * 128 + xo(i), bf16x2_of(mul2(kf[0], cI[I][0])), bf16x2_of(mul2(kf[1], cI[I][1])));
          *reinterpret_cast<uint2*>(kt_dst + xo(i)) =
              make_uint2(bf16x2_of(mul2(kr_f[0], post[0])), bf16x2_of(mul2(kr_f[1], post[1])));
#pragma unroll
          for (int m = 0; m < 2; ++m) run[m] = mul2(run[m], a2[i][m]);
        }
      };
      switch (blk) {
        case 0: pass2(std::integral_constant<int, 0>()); break;
        case 1: pass2(std::integral_constant<int, 1>()); break;
        case 2: pass2(std::integral_constant<int, 2>()); break;
        default: pass2(std::integral_constant<int, 3>()); break;
      }
    }
    fence_proxy_async();
    if (__syncthreads_or(*abort_flag)) break;

    // ================================================================ MMA AP: [LK; LQ] x R_I^T
    if (itid == 0) {
      tc_fence_after();
      // the right operands R_1..R_3 are consecutive rows of one tile: a single N = 144 product
      constexpr uint32_t idesc = idesc_bf16(128, kRRows, false, false);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = sdesc_add(d_lkq, (ks >> 2) * 16384 + (ks & 3) * 32);
        const uint64_t bd = sdesc_add(d_r, (ks >> 2) * I_RKBLK + (ks & 3) * 32);
        umma_bf16(tmem, ad, bd, idesc, ks > 0);
      }
      umma_commit(bar + 1);
    }
    if (cta_wait(1, mma_par)) break;
    tc_fence_after();

    // ================================================================ assemble A (fp32) and P (bf16)
    {
      const int R = 32 * quarter + lane;
      const bool qside = R >= 64;
      const int r = R & 63;
      const int Ib = r >> 4;
      const int q2 = quarter & 1;
      const bool skip = (ihalf == 1) && (q2 == 0);
      float d[32];
      if (!skip && q2 == 0) {
        tmem_ld32(tmem + lane_base + 32 * ihalf, d);  // row blocks 0 and 1 share R_1
      } else if (!skip) {
        float d0[32], d1[32];
        tmem_ld32(tmem + lane_base + r_seg(2) + 32 * ihalf, d0);
        tmem_ld32(tmem + lane_base + r_seg(3) + 32 * ihalf, d1);
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
          *reinterpret_cast<uint4*>(sm + I_TP + sw128(64 + r, 4 * ihalf + cch)) = w;
        }
      }
    }

    // ================================================================ solve T = (I + A)^{-1}
    // The diagonal blocks of A are rows / columns 0..31 of warp 0's share of the assembly and
    // 32..63 of warp 5's: those two warps solve them at once, 16 lanes (one column each) per block.
    if (iw == 0 || iw == 5) {
      __syncwarp();
      const int I = (iw == 0 ? 0 : 2) + (lane >> 4), j = lane & 15;
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
    // off-diagonal blocks by distance dd below the diagonal: T_IJ = -T_II (sum_{K=J}^{I-1} A_IK T_KJ),
    // each 16x16x16 product on mma.sync m16n8k8 tf32 with both operands split hi + lo (three
    // products, fp32-level accuracy).  Warp w takes block column J = w / 2 and its 8 columns
    // nt = w % 2 all the way down: every T_KJ it reads in those columns it wrote itself, and the
    // diagonal blocks are final, so the levels need no barrier across warps.  The three partial
    // products accumulate separately so their chains stay short.
#pragma unroll 1
    for (int dd = 1; dd < 4; ++dd) {
      const int bJ2 = iw >> 1, nt = iw & 1, bI = bJ2 + dd;
      if (bI < 4) {
        const int g = lane >> 2, t = lane & 3;
        float hh[4] = {0.f, 0.f, 0.f, 0.f}, hl[4] = {0.f, 0.f, 0.f, 0.f}, lh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 3; ++kk) {
          if (kk < dd) {
            const int K = bJ2 + kk;
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const float* ab = As + (16 * bI + g) * AS_LD + 16 * K + 8 * ks + t;
              const float* tb = Ts + (16 * K + 8 * ks + t) * AS_LD + 16 * bJ2 + 8 * nt + g;
              const float a0 = ab[0], a1 = ab[8 * AS_LD], a2v = ab[4], a3 = ab[8 * AS_LD + 4];
              const float b0 = tb[0], b1 = tb[4 * AS_LD];
              uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
              tf32_split(a0, ah[0], al[0]);
              tf32_split(a1, ah[1], al[1]);
              tf32_split(a2v, ah[2], al[2]);
              tf32_split(a3, ah[3], al[3]);
              tf32_split(b0, bh0, bl0);
              tf32_split(b1, bh1, bl1);
              mma_tf32(hh, ah, bh0, bh1);
              mma_tf32(hl, ah, bl0, bl1);
              mma_tf32(lh, al, bh0, bh1);
            }
          }
        }
        // Y (16 x 8) through shared memory, then Z = T_II Y
        float* ys = Ys + iw * 128;
        ys[g * 8 + 2 * t] = hh[0] + (hl[0] + lh[0]);
        ys[g * 8 + 2 * t + 1] = hh[1] + (hl[1] + lh[1]);
        ys[(g + 8) * 8 + 2 * t] = hh[2] + (hl[2] + lh[2]);
        ys[(g + 8) * 8 + 2 * t + 1] = hh[3] + (hl[3] + lh[3]);
        __syncwarp();
        float zh[4] = {0.f, 0.f, 0.f, 0.f}, zm[4] = {0.f, 0.f, 0.f, 0.f}, zl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const float* tr = Ts + (16 * bI + g) * AS_LD + 16 * bI + 8 * ks + t;
          const float a0 = tr[0], a1 = tr[8 * AS_LD], a2v = tr[4], a3 = tr[8 * AS_LD + 4];
          const float b0 = ys[(8 * ks + t) * 8 + g], b1 = ys[(8 * ks + t + 4) * 8 + g];
          uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
          tf32_split(a0, ah[0], al[0]);
          tf32_split(a1, ah[1], al[1]);
          tf32_split(a2v, ah[2], al[2]);
          tf32_split(a3, ah[3], al[3]);
          tf32_split(b0, bh0, bl0);
          tf32_split(b1, bh1, bl1);
          mma_tf32(zh, ah, bh0, bh1);
          mma_tf32(zm, ah, bl0, bl1);
          mma_tf32(zl, al, bh0, bh1);
        }
        float* to = Ts + (16 * bI) * AS_LD + 16 * bJ2 + 8 * nt;
        to[g * AS_LD + 2 * t] = -(zh[0] + (zm[0] + zl[0]));
        to[g * AS_LD + 2 * t + 1] = -(zh[1] + (zm[1] + zl[1]));
        to[(g + 8) * AS_LD + 2 * t] = -(zh[2] + (zm[2] + zl[2]));
        to[(g + 8) * AS_LD + 2 * t + 1] = -(zh[3] + (zm[3] + zl[3]));
      }
      __syncwarp();
    }
    sync();
    // T_b = T diag(beta) as a bf16 hi + lo pair, rows 0..63 of TP / TL (a warp takes 32 rows of one
    // 16-column band, so its 16-byte reads of T hit distinct banks)
    {
      const int r = itid & 63, c16 = itid >> 6;
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
        *reinterpret_cast<uint4*>(sm + I_TP + sw128(r, c0 >> 3)) = wh;
        *reinterpret_cast<uint4*>(sm + I_TL + sw128(r, c0 >> 3)) = wl;
      }
    }
    fence_proxy_async();
    sync();

    // ================================================================ MMA PT: P (T_hi + T_lo)
    if (itid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = sdesc_add(d_tpk, (ks & 3) * 32);
        const uint64_t bd = sdesc_add(ks < 4 ? d_tpm : d_tlm, (ks & 3) * 2048);
        umma_bf16(tmem, ad, bd, idesc, ks > 0);
      }
      umma_commit(bar + 1);
    }
    if (cta_wait(1, mma_par)) break;
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
        *reinterpret_cast<uint4*>(sm + I_TP + sw128(64 + r, 4 * ihalf + cch)) = wh;
        *reinterpret_cast<uint4*>(sm + I_TL + sw128(64 + r, 4 * ihalf + cch)) = wl;
      }
    }
    fence_proxy_async();
    tc_fence_before();
    sync();

    // ================================================================ MMA Xk: [0; Qtil] - [T_b; P T_b] x Khat e^Gamma
    if (itid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, true);  // B MN-major (A K-major or in TMEM)
      // [0; I_64] x Qtil seeds the accumulator with [0; Qtil] ...
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_bf16_tmem_a(tmem, tmem + kIdCol + 8 * ks, sdesc_add(d_qb, ks * 2048), idesc, ks > 0);
      // ... and [T_b; P T_b] (hi + lo) x (-Khat e^Gamma) completes [-W; Qtil - P W]
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = sdesc_add(ks < 4 ? d_tpk : d_tlk, (ks & 3) * 32);
        const uint64_t bd = sdesc_add(d_xk, (ks & 3) * 2048);
        umma_bf16(tmem, ad, bd, idesc, 1);
      }
      umma_commit(bar + 1);
      // [T_b; P T_b] hi and lo are final: copy both tiles to the item while the MMA runs
      bulk_store(item + IT_TP, sm + I_TP, 32768);
      bulk_commit();
    }
    if (cta_wait(1, mma_par)) break;
    tc_fence_after();
    if (itid == 0 && s_item[j & 1] < item_end) load_qk(s_loc[j & 1]);

    // ================================================================ [-W; Qtil - P W] -> item
    {
      // staged in the (now dead) A / T scratch as the item's byte image, then one bulk copy
      const int R = 32 * quarter + lane;
      uint8_t* dst = sm + I_AS + ihalf * 16384 + R * 128;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float d[32];
        tmem_ld32(tmem + lane_base + 64 * ihalf + 32 * part, d);
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          uint4 w;
          w.x = pack_bf16(d[8 * cch + 0], d[8 * cch + 1]);
          w.y = pack_bf16(d[8 * cch + 2], d[8 * cch + 3]);
          w.z = pack_bf16(d[8 * cch + 4], d[8 * cch + 5]);
          w.w = pack_bf16(d[8 * cch + 6], d[8 * cch + 7]);
          *reinterpret_cast<uint4*>(dst + ((((uint32_t)(4 * part + cch) ^ (uint32_t)R) & 7u) << 4)) = w;
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();  // this item's tensor-memory reads, before the next item's MMAs
    sync();
    if (itid == 0) {
      bulk_store(item + IT_WQ, sm + I_AS, 32768);
      bulk_commit();
    }
    // no barrier here: the next item's TMA only overwrites XK / QB (read by MMA Xk, which has
    // completed), and thread 0 lets the bulk copies finish reading TP / TL / AS before the barrier
    // that precedes the next item's passes (which overwrite them)
    cur_it = s_item[j & 1];
  }
  // no item left for this CTA: a kernel launched after this one as a programmatic dependent may
  // start its CTAs
  griddep_launch_dependents();

  tc_fence_before();
  sync();
  if (itid == 0) {
    // after an abort, copies or MMAs may still be in flight: let them land before leaving
    if (*abort_flag) {
      if (raw_pending) mbar_wait(bar + 0, raw_par ^ 1, kWaitLimitNs);
      umma_commit(bar + 2);
      mbar_wait(bar + 2, 0, kWaitLimitNs);
    }
    bulk_wait_all();
  }
  sync();
  if (iw == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kIntraTmemCols);
  }
  // when launched as a programmatic dependent of a recurrence launch, completion of this grid
  // implies completion of that one (the next recurrence launch reads its boundary states)
  if (itid == 0) griddep_wait();
}

// ========================================================================= recurrence kernel
// One CTA per (sequence, head).  The state is carried transposed, S^T (lane = v, column = k), so
// that every state-side MMA operand lives in tensor memory and the epilogues on the per-chunk
// critical path never touch shared memory:
//   MMA Xv   [U^T | (P U)^T]   = V^T [T_b; P T_b]^T           (A = V tile, MN-major; B = TP / TL images)
//   MMA1     [Delta^T | O^T]  += S^T_bf16 [-W; Qtil - P W]^T  (A = S^T in TMEM; B = WQ image, K-major)
//   ep1      Delta^T / |k| -> bf16 hi + lo into TMEM (A of MMA2); O^T -> staging tile -> TMA store
//   MMA2     S^T_tmem += Delta^T (hi + lo) Ktil                (A in TMEM; B = Ktil image, MN-major)
//   ep2      S^T -> bf16 into TMEM (A of the next MMA1); S^T_tmem <- S^T Diag(e^{Gamma_C} of the next chunk).
// 640 threads: warp 0 issues the MMAs, warp 1 loads (and zeroes the v rows past a sequence's end),
// warps 4..19 run the epilogues; warp w reads TMEM lanes 32 (w % 4) .. + 31 and columns
// 32 cb .. + 31, cb = (w - 4) / 4 (ep1: cb 0, 1 hold Delta^T, cb 2, 3 hold O^T).  MMA Xv of the next
// chunk goes into the other accumulator buffer in two halves that fill the tensor pipe while ep1
// and ep2 run.
constexpr int kRecThreads = 640;
constexpr int kEpiThreads = 512;
constexpr uint32_t kBarEpi = 1, kBarOut = 3, kBarOutGo = 4;
constexpr uint32_t kEpiWarps = kEpiThreads / 32, kDeltaWarps = kEpiWarps / 2;
constexpr uint32_t R_TPV = 0;         // 2 stages x [TP 16K][TL 16K][V 16K]
constexpr uint32_t R_TPV_STAGE = 49152;
constexpr uint32_t R_WQ = 98304;      // 2 stages x 32K
constexpr uint32_t R_KT = 163840;     // 2 stages x 16K
constexpr uint32_t R_OST = 196608;    // 2 x 16K: O staging tile (same layout as the TMA box of `out`)
constexpr uint32_t R_SC = 229376;     // 2 stages x 768: 1/|k| and e^{Gamma_C}
constexpr uint32_t R_BAR = R_SC + 2 * IT_SC_BYTES;
constexpr uint32_t R_TMEM = R_BAR + 8 * 24;
constexpr uint32_t R_ABORT = R_TMEM + 4;
constexpr uint32_t R_SMEM = R_BAR + 256;
constexpr uint32_t R_ALLOC = R_SMEM + 1024;
static_assert(R_ALLOC <= 232448, "recurrence shared-memory budget");
constexpr uint32_t TM_ACC = 0;   // 2 buffers x 128 columns: [U^T | (PU)^T] -> [Delta^T | O^T] of chunk c in buffer c % 2
constexpr uint32_t TM_ST = 256;  // fp32 S^T (lane = v, column = k)
constexpr uint32_t TM_SB = 384;  // S^T as bf16 pairs (A of MMA1), 64 columns
constexpr uint32_t TM_DH = 448;  // Delta^T hi as bf16 pairs (A of MMA2), 32 columns
constexpr uint32_t TM_DL = 480;  // Delta^T lo
constexpr uint32_t kRecTmemCols = 512;

enum {
  RB_TPV_FULL = 0,   // 2 stages
  RB_TPV_EMPTY = 2,  // 2 stages; count 2: the commit after MMA Xv, and the Delta warps after ep1
  RB_WQ_FULL = 4,
  RB_WQ_EMPTY = 6,
  RB_KT_FULL = 8,
  RB_KT_EMPTY = 10,
  RB_VZ = 12,        // tail rows of the v tile zeroed
  RB_MMA1 = 13,
  RB_DELTA = 14,
  RB_MMA2 = 15,
  RB_S = 16,         // bf16 S^T written (A of the next MMA1)
  RB_ST = 17,        // fp32 S^T rescaled by the next chunk's decay (accumulator of the next MMA2)
  RB_FINAL = 18,
  RB_COUNT = 19
};

struct RecMaps {
  CUtensorMap v, out;
};

// kMode: kModeFwd, the forward; kModeMap, map mode (see SplitArgs); kModeCkpt, the forward that also
// stores each chunk's starting state (S^T, fp32) in args.ckpt for the backward.  Compiled
// separately, so that the forward's code is unchanged.
constexpr int kModeFwd = 0, kModeMap = 1, kModeCkpt = 2;
template <int kMode>
__global__ void __launch_bounds__(kRecThreads, 1)
    rec_kernel(const __grid_constant__ RecMaps maps, const SplitArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const FwdParams& p = args.p;
  const int H = p.num_heads;
  const int units = p.num_seqs * H;
  constexpr bool kMap = kMode == kModeMap;
  const bool map_part_M = kMap && (int)blockIdx.x >= units;  // map mode: this CTA computes M
  const int ub = kMap ? (int)blockIdx.x % units : (int)blockIdx.x;
  const int n = ub / H, h = ub % H;
  int64_t bos, eos;
  seq_range(p, n, bos, eos);
  const int64_t ck_slot0 = bos / C + n;  // checkpoint mode: the sequence's first checkpoint slot
  // launched as a programmatic dependent: let the next launch place its CTAs beside this grid's,
  // then wait until the items this launch reads are complete
  // This launch walks the sequence's chunks that fall in global chunks [g0, g1); a sequence cut at
  // g0 or g1 takes or leaves its state in args.boundary (S^T, [v][k]).
  griddep_launch_dependents();
  griddep_wait();
  const int64_t co_n = args.chunk_off[n], co_n1 = args.chunk_off[n + 1];
  const int64_t first = co_n > args.g0 ? co_n : args.g0, lastx = co_n1 < args.g1 ? co_n1 : args.g1;
  const bool empty_seq = (co_n == co_n1);
  if (empty_seq ? !(co_n >= args.g0 && co_n < args.g1) : (first >= lastx)) return;  // nothing here
  const int c_begin = empty_seq ? 0 : (int)(first - co_n), c_end = empty_seq ? 0 : (int)(lastx - co_n);
  const bool state_in_user = (c_begin == 0), state_out_user = (c_end == (int)(co_n1 - co_n));
  bos += (int64_t)c_begin * C;
  const int nch = c_end - c_begin;
  const int64_t item0 = co_n + c_begin;
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + R_BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + R_ABORT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto chunk_len = [&](int c) -> int {
    const int64_t rem = eos - (bos + (int64_t)c * C);
    return (int)(rem < (int64_t)C ? rem : (int64_t)C);
  };
  auto item_ptr = [&](int c) -> const uint8_t* {
    return args.items + ((size_t)(item0 + c) * H + h) * ITEM_BYTES;
  };
  auto wait = [&](int b, uint32_t parity) { return bounded_wait(bar + b, parity, abort_flag, p.status); };
  auto spin = [&](int b, uint32_t parity) { return bounded_spin(bar + b, parity, abort_flag, p.status); };

  if (tid == 0) {
    for (int b = 0; b < RB_COUNT; ++b) {
      uint32_t count = 1;
      if (b == RB_TPV_EMPTY || b == RB_TPV_EMPTY + 1) count = 1 + kDeltaWarps;  // the Xv commit, each Delta warp
      if (b == RB_DELTA) count = kDeltaWarps;
      if (b == RB_S) count = kEpiWarps;
      mbar_init(bar + b, count);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.out);
  }
  if (warp == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(sm + R_TMEM), kRecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + R_TMEM);

  if (warp == 1) {
    // ------------------------------------------------------------ loader (lane 0 issues; the
    // whole warp zeroes the v rows past the end of the sequence in the last chunk)
    int armed[3][2] = {{-1, -1}, {-1, -1}, {-1, -1}};  // last chunk armed per (TPV, WQ, KT) stage
    if (map_part_M) {
      // M of the segment map: v = 0.  Both stages' v tiles are zeroed once, before the first copy
      // into either stage is armed, and never loaded
      for (int idx = lane; idx < 2 * 16384 / 16; idx += 32) {
        const int st = idx / 1024, off = (idx % 1024) * 16;
        *reinterpret_cast<uint4*>(sm + R_TPV + st * R_TPV_STAGE + 32768 + off) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async();
      __syncwarp();
    }
    for (int c = 0; c < nch; ++c) {
      const int s = c & 1;
      const uint32_t par = ((c >> 1) - 1) & 1;
      const uint8_t* it = item_ptr(c);
      int ok = 1;
      if (lane == 0) {
        if (c >= 2 && !wait(RB_TPV_EMPTY + s, par)) ok = 0;
        if (ok) {
          armed[0][s] = c;
          mbar_arrive_expect_tx(bar + RB_TPV_FULL + s, 32768 + (map_part_M ? 0 : 16384) + IT_SC_BYTES);
          bulk_load(sm + R_TPV + s * R_TPV_STAGE, it + IT_TP, 16384, bar + RB_TPV_FULL + s);
          bulk_load(sm + R_TPV + s * R_TPV_STAGE + 16384, it + IT_TL, 16384, bar + RB_TPV_FULL + s);
          bulk_load(sm + R_SC + s * IT_SC_BYTES, it + IT_IK, IT_SC_BYTES, bar + RB_TPV_FULL + s);
          if (!map_part_M) {
            const int t0 = (int)(bos + (int64_t)c * C);
            tma_load_3d(sm + R_TPV + s * R_TPV_STAGE + 32768, &maps.v, bar + RB_TPV_FULL + s, 0, h, t0);
            tma_load_3d(sm + R_TPV + s * R_TPV_STAGE + 40960, &maps.v, bar + RB_TPV_FULL + s, 64, h, t0);
          }
        }
        if (ok && c >= 2 && !wait(RB_WQ_EMPTY + s, par)) ok = 0;
        if (ok) {
          armed[1][s] = c;
          mbar_arrive_expect_tx(bar + RB_WQ_FULL + s, 32768);
          bulk_load(sm + R_WQ + s * 32768, it + IT_WQ, 16384, bar + RB_WQ_FULL + s);
          bulk_load(sm + R_WQ + s * 32768 + 16384, it + IT_WQ + 16384, 16384, bar + RB_WQ_FULL + s);
        }
        if (ok && c >= 2 && !wait(RB_KT_EMPTY + s, par)) ok = 0;
        if (ok) {
          armed[2][s] = c;
          mbar_arrive_expect_tx(bar + RB_KT_FULL + s, 16384);
          bulk_load(sm + R_KT + s * 16384, it + IT_KT, 16384, bar + RB_KT_FULL + s);
        }
        if (ok && chunk_len(c) < C && !wait(RB_TPV_FULL + s, (c >> 1) & 1)) ok = 0;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int len = chunk_len(c);
      if (len < C) {
        // rows of the v tile past the sequence end (another sequence's, or zero-filled) -> 0
        uint8_t* vt = sm + R_TPV + s * R_TPV_STAGE + 32768;
        for (int idx = lane; idx < 2 * (C - len) * 8; idx += 32) {
          const int b2 = idx / ((C - len) * 8), rem = idx % ((C - len) * 8);
          *reinterpret_cast<uint4*>(vt + b2 * 8192 + sw128(len + rem / 8, rem & 7)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + RB_VZ);
      }
    }
    // leave no copy in flight: wait for the last armed phase of every stage
    if (lane == 0)
      for (int kind = 0; kind < 3; ++kind)
        for (int s = 0; s < 2; ++s)
          if (armed[kind][s] >= 0)
            mbar_wait(bar + (kind == 0 ? RB_TPV_FULL : kind == 1 ? RB_WQ_FULL : RB_KT_FULL) + s,
                      (armed[kind][s] >> 1) & 1, kWaitLimitNs);
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nch > 0) {
      constexpr uint32_t idesc_xv = idesc_bf16(128, 128, true, false);   // A MN-major (V), B K-major
      constexpr uint32_t idesc_1 = idesc_bf16(128, 128, false, false);   // A in TMEM, B K-major
      constexpr uint32_t idesc_2 = idesc_bf16(128, 128, false, true);    // A in TMEM, B MN-major
      // matrix descriptors of stage 0; stage 1 and the k-steps are constant offsets (one thread
      // issues every MMA, so its per-MMA work is kept to an add)
      const uint64_t dv0 = sdesc_sw128(sbase + R_TPV + 32768, 8192, 1024);  // V tile: MN-major A
      const uint64_t dtp0 = sdesc_sw128(sbase + R_TPV, 16, 1024);           // TP / TL: K-major B
      const uint64_t dwq0 = sdesc_sw128(sbase + R_WQ, 16, 1024);            // WQ: K-major B
      const uint64_t dkt0 = sdesc_sw128(sbase + R_KT, 8192, 1024);          // Ktil: MN-major B
      // half `part` of MMA Xv into accumulator buffer c % 2: V^T [T_b; P T_b]_{hi / lo}^T
      auto issue_xv = [&](int c, int part) -> bool {
        const int s = c & 1;
        if (part == 0) {
          if (!wait(RB_TPV_FULL + s, (c >> 1) & 1)) return false;
          if (chunk_len(c) < C && !wait(RB_VZ, 0)) return false;
          // the buffer held [Delta^T | O^T] of chunk c - 2, read by ep1(c - 2): ep2(c - 2) followed
          // it on every epilogue warp before S(c - 1) arrived, and MMA1(c - 1) waited for S(c - 1)
          tc_fence_after();
        }
        const uint64_t dv = dv0 + (uint32_t)s * (R_TPV_STAGE >> 4);
        const uint64_t dtp = dtp0 + (uint32_t)s * (R_TPV_STAGE >> 4) + (uint32_t)part * (16384 >> 4);
        const uint32_t acc = tmem + TM_ACC + 128 * (c & 1);
        umma_bf16(acc, dv, dtp, idesc_xv, part);
        umma_bf16(acc, dv + (2048 >> 4), dtp + 2, idesc_xv, 1);
        umma_bf16(acc, dv + (4096 >> 4), dtp + 4, idesc_xv, 1);
        umma_bf16(acc, dv + (6144 >> 4), dtp + 6, idesc_xv, 1);
        if (part == 1) umma_commit(bar + RB_TPV_EMPTY + s);
        return true;
      };
      bool ok = issue_xv(0, 0) && issue_xv(0, 1);
      for (int c = 0; ok && c < nch; ++c) {
        const int s = c & 1;
        const uint32_t par = (c >> 1) & 1;
        // MMA1: [Delta^T | O^T] += S^T [-W; Qtil - P W]^T
        if (!wait(RB_WQ_FULL + s, par) || !spin(RB_S, c & 1)) break;
        tc_fence_after();
        {
          const uint64_t dwq = dwq0 + (uint32_t)s * (32768 >> 4);
          const uint32_t acc = tmem + TM_ACC + 128 * (c & 1), sb = tmem + TM_SB;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_bf16_tmem_a(acc, sb + 8 * ks, dwq + (ks >> 2) * (16384 >> 4) + (ks & 3) * 2, idesc_1, 1);
        }
        umma_commit(bar + RB_MMA1);
        umma_commit(bar + RB_WQ_EMPTY + s);
        if (c + 1 < nch && !issue_xv(c + 1, 0)) break;
        // MMA2: S^T += Delta^T (hi + lo) Ktil
        if (!wait(RB_KT_FULL + s, par) || !spin(RB_DELTA, c & 1) || !spin(RB_ST, c & 1)) break;
        tc_fence_after();
        {
          const uint64_t dkt = dkt0 + (uint32_t)s * (16384 >> 4);
          const uint32_t st = tmem + TM_ST, dh = tmem + TM_DH, dl = tmem + TM_DL;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_bf16_tmem_a(st, (ks < 4 ? dh : dl) + 8 * (ks & 3), dkt + (ks & 3) * (2048 >> 4), idesc_2, 1);
        }
        umma_commit(bar + RB_MMA2);
        umma_commit(bar + RB_KT_EMPTY + s);
        if (c + 1 < nch) ok = issue_xv(c + 1, 1);
      }
      // every MMA issued has completed before the tensor memory is released
      umma_commit(bar + RB_FINAL);
      mbar_wait(bar + RB_FINAL, 0, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue warps
    const int et = tid - 128;
    const int quarter = warp & 3, cb = (warp - 4) >> 2;
    const int v = 32 * quarter + lane;  // TMEM lane: the state / output column v
    const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
    const uint32_t col0 = 32 * cb;      // this thread's 32 columns (k for the state; tokens in ep1)
    // a barrier of all epilogue warps whose answer (has any role aborted?) is the same for all
    auto epi_sync_abort = [&]() { return named_bar_or(kBarEpi, kEpiThreads, *abort_flag != 0); };
    const float* sc_ik = reinterpret_cast<const float*>(sm + R_SC);
    const float* sc_gam = reinterpret_cast<const float*>(sm + R_SC + (IT_GAM - IT_IK));
    const bool out_issuer = (cb == 2 && quarter == 0 && lane == 0);  // first thread of the O warps (warp 12)

    // state columns: S^T[v][k] = S[k][v], k = col0 + j.  A sequence cut between two launches hands
    // its state over in args.boundary (S^T, slot h); each thread stores only what it loaded itself
    const size_t soff = ((size_t)n * H + h) * (size_t)D * D;
    float* const bnd = args.boundary + (size_t)h * D * D;
    const float* st_in = state_in_user ? (p.initial_state ? p.initial_state + soff : nullptr) : bnd;
    float* st_out = state_out_user ? (p.final_state ? p.final_state + soff : nullptr) : bnd;
    bool in_t = state_in_user ? p.state_transposed != 0 : true;
    bool out_t = state_out_user ? p.state_transposed != 0 : true;
    if (kMap) {  // one stage: B from a zero state, M from the identity; both stored [k][v]
      st_in = nullptr;
      st_out = (map_part_M ? args.map_M : args.map_B) + soff;
      in_t = out_t = false;
    }
    auto load_state = [&](float (&x)[32]) {
      if (map_part_M) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = (col0 + j == (uint32_t)v) ? 1.f : 0.f;
      } else if (!st_in) {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = 0.f;
      } else if (in_t) {
        const float4* src = reinterpret_cast<const float4*>(st_in + (size_t)v * D + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 t = src[j];
          x[4 * j] = t.x;
          x[4 * j + 1] = t.y;
          x[4 * j + 2] = t.z;
          x[4 * j + 3] = t.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = st_in[(size_t)(col0 + j) * D + v];
      }
    };
    auto store_final = [&](const float (&x)[32]) {
      if (!st_out) return;
      if (out_t) {
        float4* dst = reinterpret_cast<float4*>(st_out + (size_t)v * D + col0);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) st_out[(size_t)(col0 + j) * D + v] = x[j];
      }
    };
    // bf16 copy (A of MMA1)
    auto store_state_bf16 = [&](const float (&x)[32]) {
      uint32_t b[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) b[j] = pack_bf16(x[2 * j], x[2 * j + 1]);
      tmem_st16(tmem + lane_base + TM_SB + col0 / 2, b);
      tmem_wait_st();
    };
    // fp32 copy scaled column-wise by gam (the next chunk's decay): the accumulator of the next MMA2
    auto store_state_scaled = [&](const float (&x)[32], const float* gam) {
      uint32_t u[32];
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 g = *reinterpret_cast<const float4*>(gam + col0 + j);
        u[j] = __float_as_uint(g.x * x[j]);
        u[j + 1] = __float_as_uint(g.y * x[j + 1]);
        u[j + 2] = __float_as_uint(g.z * x[j + 2]);
        u[j + 3] = __float_as_uint(g.w * x[j + 3]);
      }
      tmem_st32(tmem + lane_base + TM_ST + col0, u);
      tmem_wait_st();
    };

    // checkpoint mode: S^T at the start of this sequence's chunk c (slot per (chunk, head), [v][k])
    auto store_ckpt = [&](const float (&x)[32], int c) {
      float4* dst = reinterpret_cast<float4*>(args.ckpt + ((size_t)(ck_slot0 + c) * H + h) * (size_t)D * D +
                                              (size_t)v * D + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
    };
    if (nch == 0) {
      float x[32];
      load_state(x);
      store_final(x);
    } else {
      // initial state: bf16 copy for MMA1(0); fp32 copy scaled by e^{Gamma_C}(0) for MMA2(0)
      wait(RB_TPV_FULL, 0);
      {
        float x[32];
        load_state(x);
        if constexpr (kMode == kModeCkpt) store_ckpt(x, c_begin);
        store_state_bf16(x);
        store_state_scaled(x, sc_gam);
      }
      tc_fence_before();
      named_bar(kBarEpi, kEpiThreads);
      if (lane == 0) mbar_arrive(bar + RB_S);
      if (et == 0) mbar_arrive(bar + RB_ST);

      for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        const int len = chunk_len(c);
        const int64_t t0 = bos + (int64_t)c * C;
        const uint32_t acc = tmem + lane_base + TM_ACC + 128 * (c & 1);
        // ---------------------------------------------------- ep1: Delta^T (columns 0..63), O^T (64..127)
        // no barrier of all epilogue warps on the critical path: a failed wait raises the abort flag,
        // the warp carries on (its results are then discarded) and every warp leaves the loop
        // together at the barrier that closes ep2
        if (cb < 2) wait(RB_TPV_FULL + s, (c >> 1) & 1);  // 1/|k| of this chunk
        wait(RB_MMA1, c & 1);
        tc_fence_after();
        if (cb < 2) {
          float d[32];
          tmem_ld32(acc + col0, d);
          const float* ik = sc_ik + s * (IT_SC_BYTES / 4) + col0;  // 1/|k_t| of tokens col0 .. + 31
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 f = *reinterpret_cast<const float4*>(ik + j);
            split2(d[j] * f.x, d[j + 1] * f.y, hi[j / 2], lo[j / 2]);
            split2(d[j + 2] * f.z, d[j + 3] * f.w, hi[j / 2 + 1], lo[j / 2 + 1]);
          }
          tmem_st16(tmem + lane_base + TM_DH + col0 / 2, hi);
          tmem_st16(tmem + lane_base + TM_DL + col0 / 2, lo);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar + RB_DELTA);
            mbar_arrive(bar + RB_TPV_EMPTY + s);
          }
          named_bar_arrive(kBarOutGo, kEpiThreads);  // the O warps start once Delta^T is out
        } else if (kMap) {
          named_bar(kBarOutGo, kEpiThreads);  // no output in map mode
        } else {
          named_bar(kBarOutGo, kEpiThreads);
          float d[32];
          tmem_ld32(acc + col0, d);  // O^T of tokens tb .. tb + 31
          const int tb = (int)col0 - 64;
          if (len == C) {
            // staging tile [2 blocks of 64 v][64 tokens][128 B], 128-byte swizzle (the TMA box layout)
            uint8_t* ost = sm + R_OST + (c & 1) * 16384 + (v >> 6) * 8192;
            if (out_issuer) bulk_wait_read<1>();  // the store of chunk c - 2 has read this buffer
            named_bar(kBarOut, kEpiThreads / 2);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = tb + j;
              *reinterpret_cast<__nv_bfloat16*>(ost + sw128(t, (v & 63) >> 3) + (v & 7) * 2) = __float2bfloat16_rn(d[j]);
            }
            fence_proxy_async();
            named_bar(kBarOut, kEpiThreads / 2);
            if (out_issuer) {
              const uint8_t* base = sm + R_OST + (c & 1) * 16384;
              tma_store_3d(&maps.out, base, 0, h, (int)t0);
              tma_store_3d(&maps.out, base + 8192, 64, h, (int)t0);
              bulk_commit();
            }
          } else {
            // the last chunk of a sequence: only rows below len belong to it
            for (int j = 0; j < 32; ++j) {
              const int t = tb + j;
              if (t < len) p.out[((size_t)(t0 + t) * H + h) * D + v] = __float2bfloat16_rn(d[j]);
            }
          }
          tc_fence_before();
        }
        // ---------------------------------------------------- ep2: state
        const bool last = (c + 1 == nch);
        wait(RB_MMA2, c & 1);
        if (!last) wait(RB_TPV_FULL + ((c + 1) & 1), ((c + 1) >> 1) & 1);
        tc_fence_after();
        float x[32];
        tmem_ld32(tmem + lane_base + TM_ST + col0, x);
        if (last) {
          store_final(x);
          break;
        }
        store_state_bf16(x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + RB_S);
        if constexpr (kMode == kModeCkpt) store_ckpt(x, c_begin + c + 1);
        // off the critical path (MMA1 of the next chunk runs meanwhile): the rescaled fp32 state,
        // then the one barrier of all epilogue warps per chunk, which also decides (for all of them)
        // whether to stop; it keeps ep1 of the next chunk after every warp's reads of this stage
        store_state_scaled(x, sc_gam + ((c + 1) & 1) * (IT_SC_BYTES / 4));
        tc_fence_before();
        if (epi_sync_abort()) break;
        if (et == 0) mbar_arrive(bar + RB_ST);
      }
      if (out_issuer) bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kRecTmemCols);
  }
}

bool g_intra_attr[2][64] = {};
bool g_rec_attr[3][64] = {};

}  // namespace

namespace {

constexpr size_t kQueueOffset = 128;  // two item counters inside the workspace header
size_t table_bytes(int64_t n) { return ((size_t)(n + 1) * sizeof(int32_t) + 1023) / 1024 * 1024; }

// Upper bound on the global chunks of N sequences holding T tokens in total.
int64_t chunk_bound(int64_t tokens, int64_t n) { return (tokens + (int64_t)(C - 1) * n) / C; }

// First global chunk of the second stage, or max_chunks when the call runs in one stage.
// Two stages when the recurrence leaves SMs free (fewer units than SMs): the recurrence over the
// first g_cut global chunks runs, one SM per unit, while the intra launch of the remaining chunks
// already fills the other SMs, and all of them once that recurrence is done.  The second stage's
// share f is sized so that its intra work about fits on the free SMs during the first recurrence:
// f / (1 - f) = 2 (SMs - units) t_chunk / (H t_item), with t_chunk / t_item the ratio of one
// recurrence chunk to one intra item on one CTA; the constant 2 t_chunk / t_item is set by a sweep
// (flat optimum from 0.40 to 0.60 on the 96-head prefill; 0.45).
int64_t stage_cut(int64_t max_chunks, int64_t units, int heads, int sms) {
  if (units >= sms || heads <= 0) return max_chunks;
  const double x = 0.45 * (double)(sms - units) / (double)heads;
  const int64_t g_cut = max_chunks - (int64_t)((double)max_chunks * x / (1.0 + x));
  return (g_cut <= 0 || g_cut >= max_chunks) ? max_chunks : g_cut;
}

}  // namespace

size_t checkpoint_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t t = total_tokens > 0 ? total_tokens : 0, n = num_seqs > 0 ? num_seqs : 0;
  const int64_t hh = num_heads > 0 ? num_heads : 0;
  return (size_t)(t / C + n + 1) * (size_t)hh * D * D * sizeof(float);
}

size_t split_workspace_bytes(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t n = num_seqs > 0 ? num_seqs : 0;
  const int64_t t = total_tokens > 0 ? total_tokens : 0;
  const int64_t hh = num_heads > 0 ? num_heads : 0;
  const int64_t max_chunks = chunk_bound(t, n);
  return kWorkspaceHeader + table_bytes(n) + (size_t)max_chunks * (size_t)hh * ITEM_BYTES +
         (size_t)hh * D * D * sizeof(float);
}

cudaError_t launch_split(const FwdParams& p, void* workspace, cudaStream_t stream, float* ckpt) {
  const int64_t units = (int64_t)p.num_seqs * p.num_heads;
  if (units == 0) return cudaSuccess;
  const int64_t tokens = p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs;
  const int64_t max_chunks = chunk_bound(tokens, p.num_seqs);
  const int64_t items = max_chunks * p.num_heads;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SplitArgs args{};
  args.p = p;
  args.chunk_off = reinterpret_cast<int32_t*>(ws + kWorkspaceHeader);
  args.items = ws + kWorkspaceHeader + table_bytes(p.num_seqs);
  args.boundary = reinterpret_cast<float*>(args.items + (size_t)items * ITEM_BYTES);

  IntraMaps im;
  RecMaps rm;
  const bool gate_pre = (p.flags & kFlagGatePrecomputed) != 0;
  if (!make_token_map(&im.q, p.q, tokens, p.num_heads) || !make_token_map(&im.k, p.k, tokens, p.num_heads) ||
      !(gate_pre ? make_token_map_f32(&im.g, p.g, tokens, p.num_heads)
                 : make_token_map(&im.g, p.g, tokens, p.num_heads)) ||
      !make_token_map(&rm.v, p.v, tokens, p.num_heads) || !make_token_map(&rm.out, p.out, tokens, p.num_heads))
    return cudaErrorInvalidValue;
  auto intra_fn = gate_pre ? intra_kernel<true> : intra_kernel<false>;
  cudaError_t e = set_smem_once(intra_fn, I_ALLOC, g_intra_attr[gate_pre ? 1 : 0]);
  if (e != cudaSuccess) return e;
  auto rec_fn = ckpt ? rec_kernel<kModeCkpt> : rec_kernel<kModeFwd>;
  e = set_smem_once(rec_fn, R_ALLOC, g_rec_attr[ckpt ? 2 : 0]);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;

  unsigned long long* queues = reinterpret_cast<unsigned long long*>(ws + kQueueOffset);
  // a launch with the programmatic-serialization attribute may start its CTAs once every CTA of
  // the previous launch in the stream has signalled or exited; the kernels wait (griddepcontrol)
  // for what they read
  auto launch = [&](auto kernel, int64_t grid, int threads, uint32_t smem, bool dependent, auto maps,
                    const SplitArgs& a) -> cudaError_t {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, maps, a);
  };
  auto intra = [&](int64_t b, int64_t en, int q, bool dependent) -> cudaError_t {
    if (en <= b) return cudaSuccess;
    SplitArgs a = args;
    a.item_begin = b;
    a.item_end = en;
    a.queue = queues + q;
    const int64_t grid = en - b < 2 * (int64_t)sms ? en - b : 2 * (int64_t)sms;
    return launch(intra_fn, grid, kIntraThreads, I_ALLOC, dependent, im, a);
  };
  auto rec = [&](int64_t g0, int64_t g1) -> cudaError_t {
    SplitArgs a = args;
    a.g0 = g0;
    a.g1 = g1;
    a.ckpt = ckpt;
    return launch(rec_fn, units, kRecThreads, R_ALLOC, true, rm, a);
  };

  chunk_table_kernel<<<1, 1024, 0, stream>>>(p, const_cast<int32_t*>(args.chunk_off), queues);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // only the sequence holding chunk g_cut is cut; it hands its state over in args.boundary
  const int64_t g_cut = stage_cut(max_chunks, units, p.num_heads, sms);
  if (g_cut >= max_chunks) {
    if ((e = intra(0, items, 0, false)) != cudaSuccess) return e;
    return rec(0, INT64_MAX);
  }
  if ((e = intra(0, g_cut * p.num_heads, 0, false)) != cudaSuccess) return e;
  if ((e = rec(0, g_cut)) != cudaSuccess) return e;
  if ((e = intra(g_cut * p.num_heads, items, 1, true)) != cudaSuccess) return e;
  return rec(g_cut, INT64_MAX);
}

// The segment map of every (sequence, head) unit: chunk table, the intra-chunk kernel over every
// item (once: the items do not depend on v or on the state), then one recurrence launch of 2 N H
// CTAs in map mode (B from v and a zero state, M from v = 0 and the identity), as a programmatic
// dependent of the intra launch.
cudaError_t launch_segment_map(const FwdParams& p, void* workspace, float* map_M, float* map_B,
                               cudaStream_t stream) {
  const int64_t units = (int64_t)p.num_seqs * p.num_heads;
  if (units == 0) return cudaSuccess;
  const int64_t tokens = p.cu_seqlens ? p.seqlen : p.seqlen * p.num_seqs;
  const int64_t max_chunks = chunk_bound(tokens, p.num_seqs);
  const int64_t items = max_chunks * p.num_heads;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SplitArgs args{};
  args.p = p;
  args.chunk_off = reinterpret_cast<int32_t*>(ws + kWorkspaceHeader);
  args.items = ws + kWorkspaceHeader + table_bytes(p.num_seqs);
  args.boundary = reinterpret_cast<float*>(args.items + (size_t)items * ITEM_BYTES);
  IntraMaps im;
  RecMaps rm;
  const bool gate_pre = (p.flags & kFlagGatePrecomputed) != 0;
  if (!make_token_map(&im.q, p.q, tokens, p.num_heads) || !make_token_map(&im.k, p.k, tokens, p.num_heads) ||
      !(gate_pre ? make_token_map_f32(&im.g, p.g, tokens, p.num_heads)
                 : make_token_map(&im.g, p.g, tokens, p.num_heads)) ||
      !make_token_map(&rm.v, p.v, tokens, p.num_heads) || !make_token_map(&rm.out, p.v, tokens, p.num_heads))
    return cudaErrorInvalidValue;  // (no output in map mode: the out map is never used)
  auto intra_fn = gate_pre ? intra_kernel<true> : intra_kernel<false>;
  cudaError_t e = set_smem_once(intra_fn, I_ALLOC, g_intra_attr[gate_pre ? 1 : 0]);
  if (e != cudaSuccess) return e;
  e = set_smem_once(rec_kernel<kModeMap>, R_ALLOC, g_rec_attr[1]);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  unsigned long long* queues = reinterpret_cast<unsigned long long*>(ws + kQueueOffset);
  chunk_table_kernel<<<1, 1024, 0, stream>>>(p, const_cast<int32_t*>(args.chunk_off), queues);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (items > 0) {
    SplitArgs a = args;
    a.item_begin = 0;
    a.item_end = items;
    a.queue = queues;
    const int64_t grid = items < 2 * (int64_t)sms ? items : 2 * (int64_t)sms;
    intra_fn<<<(unsigned)grid, kIntraThreads, I_ALLOC, stream>>>(im, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  SplitArgs a = args;
  a.g0 = 0;
  a.g1 = INT64_MAX;
  a.map_mode = 1;
  a.map_M = map_M;
  a.map_B = map_B;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * units));
  cfg.blockDim = dim3((unsigned)kRecThreads);
  cfg.dynamicSmemBytes = R_ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rec_kernel<kModeMap>, rm, a);
}

int split_launch_count(int64_t total_tokens, int32_t num_heads, int32_t num_seqs) {
  const int64_t units = (int64_t)(num_seqs > 0 ? num_seqs : 0) * (num_heads > 0 ? num_heads : 0);
  if (units == 0) return 0;
  const int sms = sm_count();
  if (sms <= 0) return -1;
  const int64_t max_chunks = chunk_bound(total_tokens > 0 ? total_tokens : 0, num_seqs);
  if (stage_cut(max_chunks, units, num_heads, sms) < max_chunks) return 5;
  return max_chunks > 0 ? 3 : 2;
}

}  // namespace kda
