// Fused quantized attention mainloop for sm_100a ("H3 Performance Roadmap",
// Phase 4: Dense Sage-Compatible Attention; numerical checkpoints of "Phase 2B
// Aligned Numerical Prototype", Exactness).
//
// One CTA owns two 128-row Q tiles (A and B) of one (b, h) and streams all
// 128-key K/V tiles past both, so every K/V tile crosses L2 -> shared memory
// once per 256 query rows.  Warp roles (512 threads, four warpgroups):
//   WG0  warp 0   TMA producer of the Q tiles and the K tiles (2-stage ring).
//        warp 2   TMA producer of the V^T tiles (3-stage ring).
//        warp 1   tensor-memory allocator and QK issuer (one thread):
//                 S(x) = Q(x) K^T  tcgen05.mma kind::f16 on the INT8 words held
//                 as BF16 (exact) with FP32 accumulation: every product and
//                 partial sum is an integer below 2^24, so S equals the INT32
//                 scores.  QK(x, j+1) is issued as soon as softmax x has loaded
//                 S(x, j), so the next scores are ready before they are needed.
//        warp 3   PV issuer (one thread):
//                 O(x) += P(x) V   tcgen05.mma kind::f8f6f4 (E4M3 operands from
//                 shared memory, F32 accumulate).
//                 A tcgen05.mma issue blocks for about its execution time, so
//                 the two products have their own issuing threads and neither
//                 waits behind the other's dependencies.
//   WG1  softmax of Q tile A, WG2 softmax of Q tile B; thread = one Q row, over
//        every key tile in order.  Each warpgroup owns the running max and row
//        sum of its rows.  Their exp2 passes (bound by the MUFU unit) start in
//        turn A(j) B(j) A(j+1) ...; a warpgroup hands the turn over part-way
//        through its pass (kTurnHandoverKey), so the end of one pass overlaps the
//        start of the next and the MUFU unit stays busy through the stalls of
//        either instruction stream.  Everything else a warpgroup does for a key
//        tile (score load, row max, probability store) runs while the other
//        warpgroup has the MUFU unit and holds no MUFU work of its own: the
//        rescale factor alpha = 2^(m_old - m_new) is the first exp2 of the pass,
//        and the correction warpgroup reads it instead of computing it.  What
//        bounds a key tile is the instruction stream of the two softmax
//        warpgroups on each SM sub-partition, so the pass forms the exp2
//        arguments next to each exp2 (kFoldArg), converts four probabilities per
//        instruction (kCvtX4), and the ragged last key tile runs a separate
//        masked copy after the loop, which keeps the loop's unrolled code (and its
//        instruction-cache footprint) to one copy.
//   WG3  O correction of both tiles (rescale by alpha when the running max
//        moves) and the epilogue (final reciprocal, BF16 store).
// Tensor memory (512 columns allocated): S(A) [0,128) S(B) [128,256)
// O(A) [256,384) O(B) [384,512).  The softmax frees S(x) as soon as it has
// read the scores.  Its E4M3 probabilities (128 x 128 bytes) go to shared
// memory in the 128-byte-swizzled K-major layout the PV MMA reads, once PV of
// the previous key tile has consumed the buffer.
//
// Every wait is bounded: after the limit the waiter records
// H3ATTN_ERR_TIMEOUT in the workspace status word, raises a CTA-wide abort
// flag, drains the asynchronous work it issued and leaves; the tensor memory
// is freed.  The barrier protocol is listed beside AttnSmem.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "exp2_poly.h"
#include "h3attn_internal.h"
#include "sm100_ptx.cuh"

namespace h3 {
namespace {

constexpr int kStagesK = 2;  // K ring (BF16 tiles, 32 KB each), shared by both Q tiles
constexpr int kStagesV = 3;  // V ring (E4M3 tiles, 16 KB each)
constexpr int kThreads = 512;
constexpr uint32_t kTileBytes = 128 * 128;          // one 128 x 128-byte swizzled tile
constexpr uint32_t kQKTileBytes = 2 * kTileBytes;   // a BF16 128 x 128 tile: two 64-column halves
__device__ __forceinline__ uint32_t col_s(int x) { return 128u * (uint32_t)x; }        // S(A), S(B)
__device__ __forceinline__ uint32_t col_o(int x) { return 256u + 128u * (uint32_t)x; } // O(A), O(B)
// Key (of 128) after which a softmax warpgroup hands the MUFU turn to the other.
#ifndef H3ATTN_TURN_HANDOVER_KEY
#define H3ATTN_TURN_HANDOVER_KEY 64
#endif
constexpr int kTurnHandoverKey = H3ATTN_TURN_HANDOVER_KEY;
// Key of the exp2 pass at which the barriers the rest of the tile (and the next one)
// depends on are tested without blocking: a blocking test of an already-completed
// phase still costs the barrier round trip on the chain between two passes, which
// these tests instead overlap with the pass.
constexpr int kMidPassKey = 96;
// 1: the exp2 arguments u = s*f - mq are formed inside the exp2 pass, next to each
// exp2; 0: in place before the pass (pre_turn).  Either gives the same bits.
#ifndef H3ATTN_FOLD_ARG
#define H3ATTN_FOLD_ARG 1
#endif
constexpr bool kFoldArg = H3ATTN_FOLD_ARG != 0;
// 1: four probabilities per conversion instruction (cvt_e4m3x4_half_up) instead of two
// per instruction and a byte pack.
#ifndef H3ATTN_CVT_X4
#define H3ATTN_CVT_X4 1
#endif
constexpr bool kCvtX4 = H3ATTN_CVT_X4 != 0;
static_assert(kTurnHandoverKey >= 0 && kTurnHandoverKey <= 128 && kTurnHandoverKey % 4 == 0, "handover key");
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, 128);
constexpr uint64_t kWaitLimitNs = kDefaultWaitLimitNs;
// setmaxnreg split (registers per thread): control, correction, softmax warpgroups.
constexpr int kRegsControl = 64, kRegsCorrection = 56, kRegsSoftmax = 192;
constexpr int64_t kRegSplitTotal = 128 * (kRegsControl + kRegsCorrection + 2 * kRegsSoftmax);
static_assert(kRegSplitTotal <= 65536, "register split exceeds the SM register file");
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s

// Barrier protocol, per Q tile x and key tile j (phase j of each barrier unless
// noted).  Each waiter is shown the back-edge that keeps its producer from
// completing a later phase before the wait has been satisfied:
//   s_full[x]   QK(x,j) done -> softmax x.   QK(x,j+1) needs s_free[x](j).
//   s_free[x]   softmax x read S(x,j) -> QK issuer.  softmax x reaches the next
//               arrival only after s_full[x](j+1), which needs this wait.
//   a_full[x][j%2]  alpha of tile j -> correction.  softmax x publishes alpha
//               of tile j+2 only after pv_done[x](j) (P buffer free for tile
//               j+1), i.e. after the correction's o_ready[x](j), which follows
//               its read of alpha(j).
//   o_ready[x]  correction -> PV issuer.  The correction waits pv_done[x](j-1)
//               before arriving for tile j, so phase j-1 has been consumed.
//   p_full[x]   P(x,j) in shared memory -> PV issuer.  softmax x writes P(x,j+1)
//               only after pv_done[x](j), i.e. after PV(x,j) was issued.
//   pv_done[x]  PV(x,j) done -> softmax x (P buffer free) and correction (O
//               final up to tile j).  PV(x,j+1) needs p_full[x](j+1) and
//               o_ready[x](j+1), which both follow these waits.
//   tok[A]      A's exp2 pass of tile j past the handover key -> softmax B
//               (waits phase j).  A's pass of j+1 needs tok[B](j), which B
//               arrives after this wait.
//   tok[B]      B's exp2 pass of tile j past the handover key -> softmax A
//               (waits phase j before its pass of j+1).  B's pass of j+1 needs
//               tok[A](j+1), after it.
struct __align__(1024) AttnSmem {
  uint8_t q[2][2][kTileBytes];         // [Q tile][half] BF16 Q tiles: key dims [0,64) and [64,128)
  uint8_t k[kStagesK][2][kTileBytes];  // BF16 K tiles, same split
  uint8_t v[kStagesV][kTileBytes];     // E4M3 V^T tiles
  uint8_t p[2][kTileBytes];            // [Q tile] E4M3 probabilities, SW128 K-major (A operand of PV)
  uint64_t q_full;
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], o_ready[2];
  uint64_t a_full[2][2];
  uint64_t tok[2];    // [Q tile] softmax x passed the handover key of its exp2 pass of key tile j
  uint64_t o_full;    // MMA -> epilogue: the last PV completed
  uint64_t d_full;    // softmax (both warpgroups) -> epilogue: row sums published
  uint64_t drain[2];  // QK issuer, PV issuer: all own MMAs completed
  uint32_t tmem_base;
  int abort;
  float sv[kD];
  float arow[2][2][kTile];  // [Q tile][key tile % 2][row]: alpha of that tile
  float dsum[2][kTile];     // [Q tile][row]: sum of 448*p relative to the final max
};
static_assert(sizeof(AttnSmem) + 1024 <= 227 * 1024, "shared memory per CTA");

// Wait-site identifiers recorded in the status detail word.
enum : int {
  kSiteProdKEmpty = 1, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaP, kSiteMmaO, kSiteMmaV, kSiteMmaS,
  kSiteSoftS, kSiteSoftTok, kSiteSoftPV, kSiteCorrA, kSiteCorrPV, kSiteEpi
};

__device__ void record_failure(DevStatus* st, int code, int site, volatile int* abort) {
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->detail = site;
    st->block = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
  }
  *abort = 1;
  __threadfence_block();
}

__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, int quarter, uint32_t col) {
  return base + ((uint32_t)(32 * quarter) << 16) + col;
}

constexpr float kMagicF = 12582912.0f;  // 1.5 * 2^23: float + magic rounds to an integer
constexpr float kLog2_448 = 8.80735492205760410749f;
// Key pairs, out of every 8, whose exp2 runs on the FMA pipe instead of MUFU.
#ifndef H3ATTN_FMA_EXP2_PAIRS_OF_8
#define H3ATTN_FMA_EXP2_PAIRS_OF_8 0
#endif
constexpr int kFmaExp2PairsOf8 = H3ATTN_FMA_EXP2_PAIRS_OF_8;
// Packed FP32-pair partial sums of each row's probabilities (4: partial k holds the pairs
// (2i, 2i+1) with i = k mod 4; 8: i = k mod 8).
#ifndef H3ATTN_SUM_ACC
#define H3ATTN_SUM_ACC 4
#endif
constexpr int kSumAcc = H3ATTN_SUM_ACC;
static_assert(kSumAcc == 4 || kSumAcc == 8, "row-sum partials");

// Maximum of the 64 FP32 scores s[OFF, OFF + 64) of one 64-key half (integer-valued:
// the exact INT32 dot products); with kMasked, keys e >= valid (counted from the
// half's first key; keys past Tkv) are ignored.  The maximum is exact in any order; it
// is taken as a balanced tree of 3-input maxima (64 -> 22 -> 8 -> 4 -> 2 -> 1), the
// mask applied where each score is used so that no masked copy is kept.
template <bool kMasked, int OFF>
__device__ __forceinline__ float rowmax64(const uint32_t (&s)[128], int valid) {
  const auto v = [&](int e) {
    const float a = __uint_as_float(s[OFF + e]);
    return kMasked && e >= valid ? -INFINITY : a;
  };
  float l1[22], l2[8];
#pragma unroll
  for (int k = 0; k < 21; ++k) l1[k] = fmax3(v(3 * k), v(3 * k + 1), v(3 * k + 2));
  l1[21] = v(63);
#pragma unroll
  for (int k = 0; k < 7; ++k) l2[k] = fmax3(l1[3 * k], l1[3 * k + 1], l1[3 * k + 2]);
  l2[7] = l1[21];
  const float a = fmax3(l2[0], l2[1], l2[2]), b = fmax3(l2[3], l2[4], l2[5]);
  return fmaxf(fmax3(a, b, l2[6]), l2[7]);
}

// 2^u for a pair of arguments on the FMA pipe instead of the MUFU unit
// (Cody-Waite range reduction and the polynomial of exp2_poly.h): n = rint(u)
// through the 1.5*2^23 magic number, r = u - n exactly, 2^r by Horner in
// packed FP32, then 2^n added into the exponent field.  u is clamped to
// >= -125 so that the result stays normal (below that 2^u is < 2^-125 and
// rounds to the E4M3 zero like the hardware exp2 does).
__device__ __forceinline__ void exp2_fma_pair(uint64_t u, float& q0, float& q1) {
  float u0, u1;
  f2_unpack(u, u0, u1);
  const uint64_t uc = f2_pack(fmaxf(u0, -125.0f), fmaxf(u1, -125.0f));
  const uint64_t y = f2_add(uc, f2_pack(kMagicF, kMagicF));   // 1.5*2^23 + n
  const uint64_t n = f2_add(y, f2_pack(-kMagicF, -kMagicF));  // n
  const uint64_t r = f2_fma(n, f2_pack(-1.0f, -1.0f), uc);    // u - n
  uint64_t pp = f2_fma(f2_pack(kExp2C5, kExp2C5), r, f2_pack(kExp2C4, kExp2C4));
  pp = f2_fma(pp, r, f2_pack(kExp2C3, kExp2C3));
  pp = f2_fma(pp, r, f2_pack(kExp2C2, kExp2C2));
  pp = f2_fma(pp, r, f2_pack(kExp2C1, kExp2C1));
  pp = f2_fma(pp, r, f2_pack(kExp2C0, kExp2C0));
  float p0, p1, y0, y1;
  f2_unpack(pp, p0, p1);
  f2_unpack(y, y0, y1);
  // bits(y) << 23 == n << 23 (mod 2^32): the magic number's low 9 bits are zero
  q0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(y0) << 23));
  q1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(y1) << 23));
}

// Softmax arithmetic of one row (128 keys, one per register), in two parts so that
// only MUFU work needs the MUFU turn:
//   pre_turn   in place, before the turn: u = s*f - mq (FP32 FMA; mq = m - log2(448),
//              so 2^u = 448 * 2^(t - m)), and for kFmaExp2PairsOf8 of every 8 key
//              pairs already q = 2^u by the FMA-pipe polynomial (exp2_fma_pair);
//   probs128   in the turn: q = 2^u on MUFU for the other pairs, FP32 partial sums of q
//              into acc2 and the E4M3 words of q into w (4 keys per word); with
//              kMasked, keys >= valid give 0.  The sums and conversions of every pair
//              fill the MUFU latency.  Every exp2 stays after the turn's wait: with
//              kFoldArg through its arguments (mq, f0 and f1 are redefined after the
//              wait), which leaves the compiler free to interleave the exp2s with the
//              other work of the pass; without it, as a volatile instruction.  At key
//              kTurnHandoverKey it arrives on tok, the
//              other warpgroup's turn; at key kMidPassKey it runs mid_pass (the
//              early barrier tests of the tile).
__device__ __forceinline__ void pre_turn(uint32_t (&x)[128], float f0, float f1, float mq) {
  const uint64_t ff0 = f2_pack(f0, f0), ff1 = f2_pack(f1, f1);
  const uint64_t negm = f2_pack(-mq, -mq);
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const uint64_t u = f2_fma(f2_pack(__uint_as_float(x[i]), __uint_as_float(x[i + 1])), i < 64 ? ff0 : ff1, negm);
    float q0, q1;
    if (((i >> 1) & 7) < kFmaExp2PairsOf8)
      exp2_fma_pair(u, q0, q1);
    else
      f2_unpack(u, q0, q1);
    x[i] = __float_as_uint(q0);
    x[i + 1] = __float_as_uint(q1);
  }
  // every value exists here: none of this work is left for the turn
#pragma unroll
  for (int i = 0; i < 128; ++i) asm volatile("" : "+r"(x[i]));
}

template <bool kMasked, typename MidPass>
__device__ __forceinline__ void probs128(const uint32_t (&x)[128], int valid, float f0, float f1, float mq,
                                         uint64_t (&acc2)[kSumAcc], uint32_t (&w)[32], uint64_t* tok,
                                         const MidPass& mid_pass) {
  const uint64_t ff0 = f2_pack(f0, f0), ff1 = f2_pack(f1, f1);
  const uint64_t negm = f2_pack(-mq, -mq);
#pragma unroll
  for (int e = 0; e < 128; e += 4) {
    if (e == kTurnHandoverKey) mbar_arrive(tok);
    if (e == kMidPassKey) mid_pass();
    uint32_t half[2];
    float qq[4];
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      const int i = e + 2 * hp;
      float q0 = __uint_as_float(x[i]), q1 = __uint_as_float(x[i + 1]);
      const bool fma_pair = ((i >> 1) & 7) < kFmaExp2PairsOf8;
      if (kFoldArg) {  // u = s*f - mq here instead of in pre_turn (same FMA, same rounding)
        const uint64_t u = f2_fma(f2_pack(q0, q1), i < 64 ? ff0 : ff1, negm);
        if (fma_pair)
          exp2_fma_pair(u, q0, q1);
        else
          f2_unpack(u, q0, q1);
      }
      if (!fma_pair) {
        if (kFoldArg) {  // ordered after the turn through its arguments (mq, f0, f1)
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(q0) : "f"(q0));
          asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(q1) : "f"(q1));
        } else {         // arguments formed before the turn: the exp2 itself stays after it
          asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(q0) : "f"(q0));
          asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(q1) : "f"(q1));
        }
      }
      if (kMasked) {
        if (i >= valid) q0 = 0.0f;
        if (i + 1 >= valid) q1 = 0.0f;
      }
      acc2[(i >> 1) & (kSumAcc - 1)] = f2_add(acc2[(i >> 1) & (kSumAcc - 1)], f2_pack(q0, q1));
      if (kCvtX4) {
        qq[2 * hp] = q0;
        qq[2 * hp + 1] = q1;
      } else {
        half[hp] = cvt_e4m3x2(q0, q1);
      }
    }
    w[e >> 2] = kCvtX4 ? cvt_e4m3x4_half_up(qq[0], qq[1], qq[2], qq[3]) : half[0] | (half[1] << 16);
  }
  if (kTurnHandoverKey == 128) mbar_arrive(tok);
}

// End of every role: all 512 threads meet, then warp 1 frees the tensor memory.
__device__ __forceinline__ void attn_teardown(uint32_t tmem, bool owner) {
  tc_fence_before();
  __syncthreads();
  if (owner) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Timeline trace (debug export only): clock64() of per-key-tile events of one CTA,
// trace[(event * 2 + slot) * nkv + j]; slot = Q tile (0 = A, 1 = B) of the pair.
enum : int {
  kEvSReady = 0,   // softmax warp: scores of key tile j ready (after the wait)
  kEvAPub = 1,     // softmax warp: alpha of tile j published to the correction
  kEvPDone = 2,    // softmax warp: probabilities stored, MMA issuer signalled
  kEvQK = 3,       // MMA issuer: QK of key tile j issued
  kEvPV = 4,       // MMA issuer: PV of key tile j issued
  kEvCorr = 5,     // correction warp: O rescaled (or left alone), MMA issuer signalled
  kEvKFull = 6,    // MMA issuer: K tile j landed in shared memory (slot 0)
  kEvProbs = 7,    // softmax warp: probabilities and their E4M3 words computed (end of the pass)
  kEvPVDone = 8,   // MMA issuer: PV of key tile j issued and committed
  kEvSFree = 9,    // MMA issuer: scores of key tile j-1 released (QK of tile j may start)
  kEvLd = 10,      // softmax warp: scores in registers (score buffer released)
  kEvMax = 11,     // softmax warp: row maximum known
  kEvPFree = 12,   // softmax warp: probability buffer free (PV of tile j-1 completed)
  kEvPVP = 13,     // MMA issuer: probabilities of key tile j observed (p_full)
  kEvPVO = 14,     // MMA issuer: O ready for key tile j observed (o_ready)
  kEvTurn = 15,    // softmax warp: MUFU turn taken (start of the pass)
  kNumEvents = 16
};
static_assert(kNumEvents == kTraceEvents, "trace buffer layout");

// Failure-path test hook: with kWithholdOReady the correction warpgroup never
// arrives on o_ready, so the PV issuer's first wait runs out after
// wait_limit_ns; it records H3ATTN_ERR_TIMEOUT (site kSiteMmaO) and raises the
// abort flag, and every other role leaves through its drain path.
constexpr int kWithholdNone = 0, kWithholdOReady = 1;

struct AttnParams {
  const float* sq;   // [B,H,Tq_pad/32]
  const float* sk;   // [B,H,Tkv_pad/64]
  const float* sv;   // [B,H,128]
  __nv_bfloat16* out;
  int64_t out_sb, out_st, out_sh;
  int H, Tq, Tkv;
  int64_t Tq_pad, Tkv_pad;
  float c_log2;      // float(softmax_scale * log2(e))
  DevStatus* status;
  uint64_t* trace;   // timeline trace buffer (traced instantiation only)
  int trace_block;   // linear block index that records the trace
  uint64_t wait_limit_ns;  // bound of every barrier wait
  int withhold;      // test hook: kWithholdOReady makes the correction skip its o_ready arrivals
};

template <bool kTrace>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2, quarter = warp & 3;
  const int64_t h = blockIdx.y, b = blockIdx.z, bh = b * p.H + h;
  const int qt0 = 2 * blockIdx.x;  // Q tiles qt0 (A) and qt0 + 1 (B)
  const int nqt = (int)(p.Tq_pad / kTile);
  const int nkv = (p.Tkv + kTile - 1) / kTile;
  volatile int* abort = &sm.abort;
  const bool tracing =
      kTrace && (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) == p.trace_block;
  auto trace = [&](int ev, int slot, int j) {
    if (kTrace && tracing) p.trace[(int64_t)(ev * 2 + slot) * nkv + j] = clock_now();
  };

  // ------------------------------------------------------------ set-up ----
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.s_free[x], kTile);
      mbar_init(&sm.p_full[x], kTile);
      mbar_init(&sm.pv_done[x], 1);
      mbar_init(&sm.o_ready[x], kTile);
      mbar_init(&sm.a_full[x][0], kTile);
      mbar_init(&sm.a_full[x][1], kTile);
      mbar_init(&sm.tok[x], kTile);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.d_full, 2 * kTile);
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4) {
    for (int c = lane; c < kD; c += 32) sm.sv[c] = p.sv[bh * kD + c];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Register split of the 512 x 128 launch budget: control warpgroup 64,
  // correction warpgroup 56, each softmax warpgroup 192:
  // 128*64 + 128*56 + 256*192 = 64512 <= 65536.  The host checks that the
  // kernel was built with 128 registers per thread before launching.
  if (wg == 0) {
    regs_dealloc<kRegsControl>();
    if (warp == 0) {
      // ---------------------------------------------- TMA producer: Q, K ----
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        // Rows of Q tile B past this head's padded length (an odd tile count)
        // are read from the next head or zero-filled; they are never stored.
        mbar_arrive_expect_tx(&sm.q_full, 2 * kQKTileBytes);
        for (int x = 0; x < 2; ++x) {
          const int qrow = (int)(bh * p.Tq_pad + (int64_t)(qt0 + x) * kTile);
          tma_load_2d(sm.q[x][0], &tm_q, &sm.q_full, 0, qrow);
          tma_load_2d(sm.q[x][1], &tm_q, &sm.q_full, 64, qrow);
        }
        const int krow = (int)(bh * p.Tkv_pad);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % kStagesK;
          if (!mbar_wait(&sm.k_empty[s], ((uint32_t)(j / kStagesK) & 1u) ^ 1u, abort, p.wait_limit_ns)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteProdKEmpty, abort);
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[s], kQKTileBytes);
          tma_load_2d(sm.k[s][0], &tm_k, &sm.k_full[s], 0, krow + j * kTile);
          tma_load_2d(sm.k[s][1], &tm_k, &sm.k_full[s], 64, krow + j * kTile);
          issued = j + 1;
        }
        if (*abort) {
          // let every copy this thread started land before the CTA can exit
          mbar_wait(&sm.q_full, 0, nullptr, kDrainLimitNs);
          for (int j = (issued > kStagesK ? issued - kStagesK : 0); j < issued; ++j)
            mbar_wait(&sm.k_full[j % kStagesK], (uint32_t)(j / kStagesK) & 1u, nullptr, kDrainLimitNs);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ------------------------------------------------- TMA producer: V ----
      if (lane == 0) {
        tma_prefetch_desc(&tm_v);
        const int vrow = (int)(bh * kD);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % kStagesV;
          if (!mbar_wait(&sm.v_empty[s], ((uint32_t)(j / kStagesV) & 1u) ^ 1u, abort, p.wait_limit_ns)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteProdVEmpty, abort);
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
          tma_load_2d(sm.v[s], &tm_v, &sm.v_full[s], j * kTile, vrow);
          issued = j + 1;
        }
        if (*abort) {
          for (int j = (issued > kStagesV ? issued - kStagesV : 0); j < issued; ++j)
            mbar_wait(&sm.v_full[j % kStagesV], (uint32_t)(j / kStagesV) & 1u, nullptr, kDrainLimitNs);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------ QK issuer ----
      if (lane == 0) {
        bool ok = mbar_wait(&sm.q_full, 0, abort, p.wait_limit_ns);
        if (!ok) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaQ, abort);
        tc_fence_after();
        for (int j = 0; ok && j < nkv; ++j) {
          const int s = j % kStagesK;
          if (!mbar_wait(&sm.k_full[s], (uint32_t)(j / kStagesK) & 1u, abort, p.wait_limit_ns)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaK, abort);
            ok = false;
            break;
          }
          trace(kEvKFull, 0, j);
          for (int x = 0; x < 2; ++x) {
            if (j >= 1) {
              // S(x) is free once the softmax of Q tile x has read key tile j-1
              if (!mbar_wait(&sm.s_free[x], (uint32_t)(j - 1) & 1u, abort, p.wait_limit_ns)) {
                record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaS, abort);
                ok = false;
                break;
              }
              trace(kEvSFree, x, j);
            }
            tc_fence_after();
            // 8 MMAs of K = 16: BF16 key dims [16kk, 16kk+16) = bytes 32*(kk%4) of half kk/4
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q[x][kk >> 2])) + 2 * (kk & 3);
              const uint64_t dk = sdesc_k_sw128(smem_u32(sm.k[s][kk >> 2])) + 2 * (kk & 3);
              mma_bf16_ss(tmem + col_s(x), dq, dk, kIdescQK, kk > 0);
            }
            mma_commit(&sm.s_full[x]);
            trace(kEvQK, x, j);
          }
          if (!ok) break;
          mma_commit(&sm.k_empty[s]);
        }
        // wait until every MMA this thread issued has completed
        mma_commit(&sm.drain[0]);
        mbar_wait(&sm.drain[0], 0, nullptr, ok ? p.wait_limit_ns : kDrainLimitNs);
      }
      __syncwarp();
    } else if (warp == 3) {
      // ------------------------------------------------ PV issuer ----
      if (lane == 0) {
        bool ok = true;
        for (int j = 0; ok && j < nkv; ++j) {
          const int s = j % kStagesV;
          if (!mbar_wait(&sm.v_full[s], (uint32_t)(j / kStagesV) & 1u, abort, p.wait_limit_ns)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaV, abort);
            ok = false;
            break;
          }
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.v[s]));
          for (int x = 0; x < 2; ++x) {
            if (!mbar_wait(&sm.p_full[x], (uint32_t)j & 1u, abort, p.wait_limit_ns)) {
              record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaP, abort);
              ok = false;
              break;
            }
            trace(kEvPVP, x, j);
            if (!mbar_wait(&sm.o_ready[x], (uint32_t)j & 1u, abort, p.wait_limit_ns)) {
              record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaO, abort);
              ok = false;
              break;
            }
            trace(kEvPVO, x, j);
            tc_fence_after();
            trace(kEvPV, x, j);
            const uint64_t dp = sdesc_k_sw128(smem_u32(sm.p[x]));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f8_ss(tmem + col_o(x), dp + 2 * kk, dv + 2 * kk, kIdescPV, j > 0 || kk > 0);
            mma_commit(&sm.pv_done[x]);
            trace(kEvPVDone, x, j);
          }
          if (!ok) break;
          mma_commit(&sm.v_empty[s]);
        }
        if (ok) mma_commit(&sm.o_full);
        mma_commit(&sm.drain[1]);
        mbar_wait(&sm.drain[1], 0, nullptr, ok ? p.wait_limit_ns : kDrainLimitNs);
      }
      __syncwarp();
    }
    attn_teardown(tmem, warp == 1);
    return;
  }

  const int row = 32 * quarter + lane;
  if (wg == 3) {
    // -------------------------------------------- correction + epilogue ----
    regs_dealloc<kRegsCorrection>();
    bool ok = true;
    for (int j = 0; ok && j < nkv; ++j) {
      for (int x = 0; x < 2; ++x) {
        ok = mbar_wait(&sm.a_full[x][j & 1], (uint32_t)(j >> 1) & 1u, abort, p.wait_limit_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteCorrA, abort);
          break;
        }
        const float alpha = sm.arow[x][j & 1][row];
        if (j > 0) {
          // O(x) holds the sum over key tiles < j once PV(x, j-1) has completed;
          // the wait also retires the previous phase of o_ready[x].
          ok = mbar_wait(&sm.pv_done[x], (uint32_t)(j - 1) & 1u, abort, p.wait_limit_ns);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (!ok) {
            if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteCorrPV, abort);
            break;
          }
          if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
            tc_fence_after();
            const uint32_t tO = tmem_lane_addr(tmem, quarter, col_o(x));
            const uint64_t aa = f2_pack(alpha, alpha);
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * ch, o);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float lo, hi;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), aa), lo, hi);
                o[e] = __float_as_uint(lo);
                o[e + 1] = __float_as_uint(hi);
              }
              tmem_st32(tO + 32 * ch, o);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        if (p.withhold != kWithholdOReady) mbar_arrive(&sm.o_ready[x]);
        if (quarter == 0 && lane == 0) trace(kEvCorr, x, j);
      }
    }
    if (ok) {
      ok = mbar_wait(&sm.d_full, 0, abort, p.wait_limit_ns) && mbar_wait(&sm.o_full, 0, abort, p.wait_limit_ns);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok && lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteEpi, abort);
    }
    if (ok) {
      tc_fence_after();
      for (int x = 0; x < 2; ++x) {
        // d = sum over key tiles of 448*p relative to the final max
        const float r = __frcp_rn(sm.dsum[x][row]);
        const int64_t grow = (int64_t)(qt0 + x) * kTile + row;
        const uint32_t tO = tmem_lane_addr(tmem, quarter, col_o(x));
        __nv_bfloat16* orow = p.out + b * p.out_sb + grow * p.out_st + h * p.out_sh;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * ch, o);
          if (grow < p.Tq) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t w[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int c0 = 32 * ch + e + 2 * u;
                const float y0 = __fmul_rn(__fmul_rn(__uint_as_float(o[e + 2 * u]), r), sm.sv[c0]);
                const float y1 = __fmul_rn(__fmul_rn(__uint_as_float(o[e + 2 * u + 1]), r), sm.sv[c0 + 1]);
                const __nv_bfloat162 pr2 = __floats2bfloat162_rn(y0, y1);
                w[u] = *reinterpret_cast<const uint32_t*>(&pr2);
              }
              *reinterpret_cast<uint4*>(orow + 32 * ch + e) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
    attn_teardown(tmem, false);
    return;
  }

  // -------------------------------------------------------- softmax ----
  regs_alloc<kRegsSoftmax>();
  const int x = wg - 1;  // this warpgroup owns Q tile x of the pair, over all key tiles
  {
    // a Q tile past the padded length (odd tile count) reuses the last tile's scale
    const int qts = min(qt0 + x, nqt - 1);
    const float sqi = p.sq[bh * (p.Tq_pad / kQGroup) + (int64_t)qts * (kTile / kQGroup) + quarter];
    const float* skh = p.sk + bh * (p.Tkv_pad / kKGroup);
    const uint32_t tS = tmem_lane_addr(tmem, quarter, col_s(x));
    // this row of the swizzled probability tile: 16-byte chunk c at c ^ (row % 8)
    const uint32_t prow = smem_u32(sm.p[x]) + (uint32_t)row * 128u;
    float m_w = -INFINITY, d_w = 0.0f;  // running max after the previous key tile, its row sum
    float sk0 = __ldg(skh), sk1 = __ldg(skh + 1);
    // One key tile; false when a wait gave up (the failure is recorded).  Only the
    // last tile can have keys past Tkv: it runs the masked instantiation after the
    // loop, so the loop body holds one copy of the unrolled code.
    // Outcomes of the early (non-blocking) barrier tests, carried to where each barrier
    // is needed; a test that found its phase incomplete falls back to the blocking wait.
    bool s_seen = false;    // scores of this tile's key tile already seen complete
    bool tok_seen = false;  // this tile's MUFU turn already seen granted
    const auto tile = [&](const int j, auto masked) -> bool {
      constexpr bool kMasked = decltype(masked)::value;
      bool ok = true;
      const float f0 = __fmul_rn(__fmul_rn(sqi, sk0), p.c_log2);
      const float f1 = __fmul_rn(__fmul_rn(sqi, sk1), p.c_log2);
      if (j + 1 < nkv) {  // the next tile's K scales, a tile ahead of their use
        sk0 = ldg_f32_issued_here(skh + 2 * (j + 1));
        sk1 = ldg_f32_issued_here(skh + 2 * (j + 1) + 1);
      }
      if (!s_seen) {
        ok = mbar_wait(&sm.s_full[x], (uint32_t)j & 1u, abort, p.wait_limit_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftS, abort);
          return false;
        }
      }
      tc_fence_after();
      const bool tr = kTrace && tracing && quarter == 0 && lane == 0;
      if (tr) trace(kEvSReady, x, j);
      const int valid = kMasked ? p.Tkv - j * kTile : kTile;
      // scores: keys [0,64) loaded and waited for, keys [64,128) in flight while the
      // first half's maximum is taken
      uint32_t xs[128];
      tmem_ld64_wait_at<0>(tS, xs);
      tmem_ld64_async_at<64>(tS + 64u, xs);
      const float xm0 = kMasked && valid < 64 ? rowmax64<true, 0>(xs, valid) : rowmax64<false, 0>(xs, valid);
      tmem_wait_ld_at<64>(xs);
      tc_fence_before();
      mbar_arrive(&sm.s_free[x]);  // QK of the next key tile may overwrite S(x)
      if (tr) trace(kEvLd, x, j);
      const float xm1 =
          kMasked ? rowmax64<true, 64>(xs, valid - 64) : rowmax64<false, 64>(xs, valid - 64);
      const float t0m = __fmul_rn(xm0, f0);                           // valid >= 1: half 0 has a key
      const float t1m = valid > 64 ? __fmul_rn(xm1, f1) : -INFINITY;
      const float m_j = fmaxf(m_w, fmaxf(t0m, t1m));
      if (tr) {
        asm volatile("" ::"f"(m_j));  // the maximum exists before the stamp is taken
        trace(kEvMax, x, j);
      }
      uint32_t pw[32];
      uint64_t acc2[kSumAcc];
#pragma unroll
      for (int i = 0; i < kSumAcc; ++i) acc2[i] = 0ull;
      const float mq = __fsub_rn(m_j, kLog2_448);
      if (!kFoldArg) pre_turn(xs, f0, f1, mq);
      // MUFU turn: the exp2 passes start in turn A(0) B(0) A(1) B(1) ..., each
      // after the other warpgroup's pass has reached its handover key, so that
      // a pass has the MUFU unit (nearly) to itself while the other warpgroup
      // does the rest of its tile.
      if ((x == 1 || j >= 1) && !tok_seen) {
        const int jt = x == 1 ? j : j - 1;  // A waits for B's pass of j-1, B for A's pass of j
        ok = mbar_wait(&sm.tok[1 - x], (uint32_t)jt & 1u, abort, p.wait_limit_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftTok, abort);
          return false;
        }
      }
      if (tr) trace(kEvTurn, x, j);
      // The exp2 instructions are not volatile, so that the compiler can interleave them
      // with the sums and conversions of earlier keys; their arguments come from copies
      // of mq, f0 and f1 that this empty volatile statement redefines after the turn's
      // wait, which keeps every exp2 of the pass after the wait.
      float mq_t = mq, f0_t = f0, f1_t = f1;
      asm volatile("" : "+f"(mq_t), "+f"(f0_t), "+f"(f1_t));
      // the rescale factor of this tile, on MUFU inside the turn (2^-inf = 0 on the first tile)
      float alpha;
      asm volatile("ex2.approx.f32 %0, %1;" : "=f"(alpha) : "f"(__fsub_rn(m_w, m_j)));
      // mid-pass: test the probability buffer (PV of tile j-1) and the next tile's scores
      bool p_seen = j == 0;
      s_seen = false;
      const auto mid_pass = [&]() {
        if (j >= 1) p_seen = mbar_test(&sm.pv_done[x], (uint32_t)(j - 1) & 1u);
        if (j + 1 < nkv) s_seen = mbar_test(&sm.s_full[x], (uint32_t)(j + 1) & 1u);
      };
      probs128<kMasked>(xs, valid, f0_t, f1_t, mq_t, acc2, pw, &sm.tok[x], mid_pass);
      if (tr) trace(kEvProbs, x, j);
      sm.arow[x][j & 1][row] = alpha;
      mbar_arrive(&sm.a_full[x][j & 1]);
      if (tr) trace(kEvAPub, x, j);
      if (!p_seen) {
        // the probability buffer still feeds PV(x, j-1) until that MMA has completed
        ok = mbar_wait(&sm.pv_done[x], (uint32_t)(j - 1) & 1u, abort, p.wait_limit_ns);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftPV, abort);
          return false;
        }
        if (tr) trace(kEvPFree, x, j);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + ((uint32_t)(c ^ (row & 7)) << 4)),
                     "r"(pw[4 * c]), "r"(pw[4 * c + 1]), "r"(pw[4 * c + 2]), "r"(pw[4 * c + 3])
                     : "memory");
      fence_proxy_async_smem();
      mbar_arrive(&sm.p_full[x]);
      if (tr) trace(kEvPDone, x, j);
      // the next tile's MUFU turn, tested now so that its round trip overlaps the row sum
      tok_seen = false;
      if (j + 1 < nkv) {
        const int jt = x == 1 ? j + 1 : j;
        tok_seen = mbar_test(&sm.tok[1 - x], (uint32_t)jt & 1u);
      }
      float a[2 * kSumAcc];
#pragma unroll
      for (int i = 0; i < kSumAcc; ++i) f2_unpack(acc2[i], a[2 * i], a[2 * i + 1]);
      if (kSumAcc == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = a[i] + a[i + 8];
      }
      const float es = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
      d_w = __fadd_rn(__fmul_rn(d_w, alpha), es);
      m_w = m_j;
      return true;
    };
    const int full_tiles = p.Tkv % kTile == 0 ? nkv : nkv - 1;  // tiles whose 128 keys are all valid
    bool ok = true;
    for (int j = 0; ok && j < full_tiles; ++j) ok = tile(j, std::false_type{});
    if (ok && full_tiles < nkv) ok = tile(nkv - 1, std::true_type{});
    if (ok) {
      sm.dsum[x][row] = d_w;
      mbar_arrive(&sm.d_full);
    }
  }
  attn_teardown(tmem, false);
}

// ------------------------------------------------------- debug QK tile ----
// One CTA of 128 threads computes the QK^T tile of (b, h, qt, kt) with the
// same TMA + tcgen05 path as the attention kernel and writes it to global
// memory as INT32 (the FP32 scores are exact integers).
struct __align__(1024) DebugSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[2][kTileBytes];
  uint64_t full, done;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int qrow,
                    int krow, int32_t* __restrict__ out, DevStatus* status) {
  extern __shared__ uint8_t smem_raw[];
  DebugSmem& sm = *reinterpret_cast<DebugSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm.abort;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&sm.full, 2 * kQKTileBytes);
    tma_load_2d(sm.q[0], &tm_q, &sm.full, 0, qrow);
    tma_load_2d(sm.q[1], &tm_q, &sm.full, 64, qrow);
    tma_load_2d(sm.k[0], &tm_k, &sm.full, 0, krow);
    tma_load_2d(sm.k[1], &tm_k, &sm.full, 64, krow);
    if (mbar_wait(&sm.full, 0, nullptr, kWaitLimitNs)) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q[kk >> 2])) + 2 * (kk & 3);
        const uint64_t dk = sdesc_k_sw128(smem_u32(sm.k[kk >> 2])) + 2 * (kk & 3);
        mma_bf16_ss(tmem, dq, dk, kIdescQK, kk > 0);
      }
      mma_commit(&sm.done);
    } else {
      record_failure(status, H3ATTN_ERR_TIMEOUT, kSiteMmaK, abort);
    }
  }
  __syncwarp();
  bool ok = mbar_wait(&sm.done, 0, abort, kWaitLimitNs);
  ok = __all_sync(0xFFFFFFFFu, ok);
  if (ok) {
    tc_fence_after();
    const int row = 32 * warp + lane;
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t a[32];
      tmem_ld32(tmem_lane_addr(tmem, warp, 32 * ch), a);
      tmem_wait_ld();
      // the FP32 scores are integers below 2^24: exact INT32 values
      for (int e = 0; e < 32; ++e) out[row * 128 + 32 * ch + e] = __float2int_rn(__uint_as_float(a[e]));
    }
  } else if (lane == 0) {
    record_failure(status, H3ATTN_ERR_TIMEOUT, kSiteSoftS, abort);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------ host side ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2D tensor [rows, inner] (inner in elements) with a row pitch in bytes; boxes of
// 128 rows x 128 bytes, 128-byte swizzle.  8-bit data (UINT8) or BF16.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch, bool bf16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {bf16 ? 64u : 128u, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base),
            dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kAttnSmemBytes = sizeof(AttnSmem) + 1024;
constexpr size_t kDebugSmemBytes = sizeof(DebugSmem) + 1024;

cudaError_t ensure_attrs() {
  static ContextSet done;  // contexts whose attributes are set
  if (done.contains(current_context_id())) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_sm100_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(debug_qk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDebugSmemBytes);
  if (e != cudaSuccess) return e;
  // The warpgroup register split (setmaxnreg) needs the full launch budget.
  cudaFuncAttributes fa;
  for (int traced = 0; traced < 2; ++traced) {
    e = cudaFuncGetAttributes(&fa, traced ? (const void*)attn_sm100_kernel<true> : (const void*)attn_sm100_kernel<false>);
    if (e != cudaSuccess) return e;
    if ((int64_t)fa.numRegs * kThreads < kRegSplitTotal) return cudaErrorInvalidConfiguration;
  }
  done.add(current_context_id());  // the calls above made the device's primary context current if none was
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attention(const char* ws, const Shape& s, const Layout& L, float c_log2,
                             const h3attn_bf16_out& out, cudaStream_t st, h3attn_status* why, uint64_t* trace,
                             int trace_block, uint64_t wait_limit_ns, bool withhold_o_ready) {
  *why = H3ATTN_OK;
  cudaError_t e = ensure_attrs();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  const uint64_t BH = (uint64_t)s.B * s.H;
  if (!make_tmap(&tq, ws + L.off[H3ATTN_WS_Q8], kD, BH * s.Tq_pad, 2 * kD, true) ||
      !make_tmap(&tk, ws + L.off[H3ATTN_WS_K8], kD, BH * s.Tkv_pad, 2 * kD, true) ||
      !make_tmap(&tv, ws + L.off[H3ATTN_WS_V8T], s.Tkv_pad, BH * kD, s.Tkv_pad)) {
    *why = H3ATTN_ERR_CUDA;
    return cudaErrorInvalidValue;
  }
  AttnParams p;
  p.sq = reinterpret_cast<const float*>(ws + L.off[H3ATTN_WS_SQ]);
  p.sk = reinterpret_cast<const float*>(ws + L.off[H3ATTN_WS_SK]);
  p.sv = reinterpret_cast<const float*>(ws + L.off[H3ATTN_WS_SV]);
  p.out = static_cast<__nv_bfloat16*>(out.data);
  p.out_sb = out.stride_b;
  p.out_st = out.stride_t;
  p.out_sh = out.stride_h;
  p.H = s.H;
  p.Tq = s.Tq;
  p.Tkv = s.Tkv;
  p.Tq_pad = s.Tq_pad;
  p.Tkv_pad = s.Tkv_pad;
  p.c_log2 = c_log2;
  p.status = reinterpret_cast<DevStatus*>(const_cast<char*>(ws) + L.off[H3ATTN_WS_STATUS]);
  p.trace = trace;
  p.trace_block = trace_block;
  p.wait_limit_ns = wait_limit_ns;
  p.withhold = withhold_o_ready ? kWithholdOReady : kWithholdNone;
  dim3 grid((unsigned)((s.Tq_pad / kTile + 1) / 2), (unsigned)s.H, (unsigned)s.B);
  if (trace != nullptr)
    attn_sm100_kernel<true><<<grid, kThreads, kAttnSmemBytes, st>>>(tq, tk, tv, p);
  else
    attn_sm100_kernel<false><<<grid, kThreads, kAttnSmemBytes, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_debug_qk(const char* ws, const Shape& s, const Layout& L, int b, int h, int qt, int kt,
                            int32_t* out, cudaStream_t st, h3attn_status* why) {
  *why = H3ATTN_OK;
  cudaError_t e = ensure_attrs();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk;
  const uint64_t BH = (uint64_t)s.B * s.H;
  if (!make_tmap(&tq, ws + L.off[H3ATTN_WS_Q8], kD, BH * s.Tq_pad, 2 * kD, true) ||
      !make_tmap(&tk, ws + L.off[H3ATTN_WS_K8], kD, BH * s.Tkv_pad, 2 * kD, true)) {
    *why = H3ATTN_ERR_CUDA;
    return cudaErrorInvalidValue;
  }
  const int64_t bh = (int64_t)b * s.H + h;
  const int qrow = (int)(bh * s.Tq_pad + (int64_t)qt * kTile);
  const int krow = (int)(bh * s.Tkv_pad + (int64_t)kt * kTile);
  auto* status = reinterpret_cast<DevStatus*>(const_cast<char*>(ws) + L.off[H3ATTN_WS_STATUS]);
  debug_qk_kernel<<<1, 128, kDebugSmemBytes, st>>>(tq, tk, qrow, krow, out, status);
  return cudaGetLastError();
}

}  // namespace h3
