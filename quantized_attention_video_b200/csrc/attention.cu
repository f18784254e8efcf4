// Fused quantized attention mainloop for sm_100a ("H3 Performance Roadmap",
// Phase 4: Dense Sage-Compatible Attention; numerical checkpoints of "Phase 2B
// Aligned Numerical Prototype", Exactness).
//
// One CTA owns one 128-row Q tile of one (b, h) and streams all 128-key K/V
// tiles past it.  Warp roles (512 threads, four warpgroups):
//   WG0  warp 0   TMA producer of the Q tile and the K tiles (3-stage ring).
//        warp 2   TMA producer of the V^T tiles (4-stage ring), so K tiles
//                 run ahead of V tiles by as much as the rings allow.
//        warp 1   tensor-memory allocator and QK issuer (one thread):
//                 S = Q K^T  tcgen05.mma kind::f16 on the INT8 words held as
//                 BF16 (exact) with FP32 accumulation: every product and partial
//                 sum is an integer below 2^24, so S equals the INT32 scores.
//        warp 3   PV issuer (one thread):
//                 O += P V   tcgen05.mma kind::f8f6f4 (E4M3, A = P read from
//                 tensor memory, F32 accumulate).
//                 A tcgen05.mma issue blocks for about its execution time, so
//                 the two products have their own issuing threads and neither
//                 waits behind the other's dependencies.  Their MMAs touch
//                 disjoint tensor memory; every true dependency is a barrier.
//   WG1  softmax of the even key tiles (scores in S0)  } thread = one Q row.
//   WG2  softmax of the odd key tiles (scores in S1)   } The running row max
//        is handed from the warpgroup of tile j to that of tile j+1, so one
//        warpgroup's max/exchange phase overlaps the other's exp2 phase.
//   WG3  O correction (rescale by alpha when the running max moves) and the
//        epilogue (final reciprocal, BF16 store).
// Tensor memory (512 columns allocated): S0 [0,128) S1 [128,256) O [256,384)
// P0 [384,416) P1 [416,448).  FP32 scores of key tile j go to S(j%2) and its E4M3
// probabilities (128 x 128 bytes = 32 columns) to P(j%2).  The softmax frees
// S(j%2) as soon as it has read the scores, so QK(j+2) runs on the tensor
// cores while the softmax of tile j is still computing; it writes P(j%2)
// only after PV(j-2) has consumed the previous contents.
//
// Every hand-off whose producer could otherwise run two phases ahead of its
// consumer uses two barriers (indexed by key tile parity).  Every wait is
// bounded: after the limit the waiter records H3ATTN_ERR_TIMEOUT in the
// workspace status word, raises a CTA-wide abort flag, drains the
// asynchronous work it issued and leaves; the tensor memory is freed.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>
#include <mutex>

#include "exp2_poly.h"
#include "h3attn_internal.h"
#include "sm100_ptx.cuh"

namespace h3 {
namespace {

constexpr int kStagesK = 3;  // K ring (BF16 tiles, 32 KB each)
constexpr int kStagesV = 4;  // V ring (E4M3 tiles, 16 KB each)
constexpr int kThreads = 512;
constexpr uint32_t kTileBytes = 128 * 128;          // one 128 x 128-byte swizzled tile
constexpr uint32_t kQKTileBytes = 2 * kTileBytes;   // a BF16 128 x 128 tile: two 64-column halves
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 416;
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, 128);
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// setmaxnreg split (registers per thread): control, correction, softmax warpgroups.
constexpr int kRegsControl = 64, kRegsCorrection = 56, kRegsSoftmax = 192;
constexpr int64_t kRegSplitTotal = 128 * (kRegsControl + kRegsCorrection + 2 * kRegsSoftmax);
static_assert(kRegSplitTotal <= 65536, "register split exceeds the SM register file");
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s

struct __align__(1024) AttnSmem {
  uint8_t q[2][kTileBytes];            // BF16 Q tile: key dims [0,64) and [64,128)
  uint8_t k[kStagesK][2][kTileBytes];  // BF16 K tiles, same split
  uint8_t v[kStagesV][kTileBytes];     // E4M3 V^T tiles
  uint64_t q_full;
  uint64_t k_full[kStagesK], k_empty[kStagesK];
  uint64_t v_full[kStagesV], v_empty[kStagesV];
  uint64_t s_full[2];   // MMA -> softmax: scores of key tile j in S(j%2)
  uint64_t s_free[2];   // softmax -> MMA: scores of key tile j read, S(j%2) may be overwritten
  uint64_t p_full[2];   // softmax -> MMA: P of key tile j in P(j%2)
  uint64_t m_full[4];   // softmax of tile j -> softmax of tile j+1 and correction: running max in mrow[j%4]
  uint64_t o_ready[2];  // correction -> MMA: O rescaled for key tile j
  uint64_t pv_done[2];  // MMA -> correction, softmax: PV of key tile j completed (P(j%2) free)
  uint64_t o_full;      // MMA -> epilogue: the last PV completed
  uint64_t d_full;      // softmax (both warpgroups) -> epilogue: partial row sums published
  uint64_t drain[2];  // QK issuer, PV issuer: all own MMAs completed
  uint32_t tmem_base;
  int abort;
  float sv[kD];
  float mrow[4][kTile];   // [key tile % 4][row]: running max after that tile (log2 domain)
  float dsum[2][kTile];   // [warpgroup][row]: sum of 448*p over its tiles, relative to mlast
  float mlast[2][kTile];  // [warpgroup][row]: running max at its last tile
};

// Wait-site identifiers recorded in the status detail word.
enum : int {
  kSiteProdKEmpty = 1, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaP, kSiteMmaO, kSiteMmaV, kSiteMmaS,
  kSiteSoftS, kSiteSoftM, kSiteSoftPV, kSiteCorrM, kSiteCorrPV, kSiteEpi
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
#define H3ATTN_FMA_EXP2_PAIRS_OF_8 2
#endif
constexpr int kFmaExp2PairsOf8 = H3ATTN_FMA_EXP2_PAIRS_OF_8;

// Row maxima of the two 64-key halves (one K scale each) of the 128 FP32
// scores of a row (integer-valued: the exact INT32 dot products), with 3-input
// max; with kMasked, columns >= valid (keys past Tkv) are ignored.
template <bool kMasked>
__device__ __forceinline__ void rowmax128(const uint32_t (&s)[128], int valid, float& xm0, float& xm1) {
  float m[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m[c] = -INFINITY;
#pragma unroll
  for (int e = 0; e < 128; e += 2) {
    const int c = ((e >> 1) & 3) + (e >= 64 ? 4 : 0);
    float a = __uint_as_float(s[e]), b = __uint_as_float(s[e + 1]);
    if (kMasked) {
      if (e >= valid) a = -INFINITY;
      if (e + 1 >= valid) b = -INFINITY;
    }
    m[c] = fmax3(m[c], a, b);
  }
  xm0 = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
  xm1 = fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7]));
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

__device__ __forceinline__ float exp2_fma(float u) {
  float q0, q1;
  exp2_fma_pair(f2_pack(u, u), q0, q1);
  return q0;
}

// Scaled probabilities of the 128 keys of a row: q = 2^(acc*f - mq) with
// mq = m - log2(448), i.e. q = 448 * 2^(t - m); FP32 partial sums of q
// into acc2 and the E4M3 words of q into w (4 keys per word).  kFmaExp2PairsOf8
// key pairs in every eight take their exp2 from the FMA pipe (exp2_fma_pair),
// the rest from MUFU, to balance the two units.
template <bool kMasked>
__device__ __forceinline__ void probs128(const uint32_t (&x)[128], int valid, float f0, float f1, float mq,
                                         uint64_t (&acc2)[4], uint32_t (&w)[32]) {
  const uint64_t ff0 = f2_pack(f0, f0), ff1 = f2_pack(f1, f1);
  const uint64_t negm = f2_pack(-mq, -mq);
#pragma unroll
  for (int e = 0; e < 128; e += 4) {
    uint32_t half[2];
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      const int i = e + 2 * hp;
      const uint64_t a = f2_pack(__uint_as_float(x[i]), __uint_as_float(x[i + 1]));
      const uint64_t u = f2_fma(a, i < 64 ? ff0 : ff1, negm);
      float q0, q1;
      if (((i >> 1) & 7) < kFmaExp2PairsOf8) {
        exp2_fma_pair(u, q0, q1);
      } else {
        float u0, u1;
        f2_unpack(u, u0, u1);
        q0 = ex2_ftz(u0);
        q1 = ex2_ftz(u1);
      }
      if (kMasked) {
        if (i >= valid) q0 = 0.0f;
        if (i + 1 >= valid) q1 = 0.0f;
      }
      acc2[(i >> 1) & 3] = f2_add(acc2[(i >> 1) & 3], f2_pack(q0, q1));
      half[hp] = cvt_e4m3x2(q0, q1);
    }
    w[e >> 2] = half[0] | (half[1] << 16);
  }
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
// trace[(event * 2 + slot) * nkv + j]; slot = key half for the softmax events, 0 otherwise.
enum : int {
  kEvSReady = 0,   // softmax warp: scores of key tile j ready (after the wait)
  kEvAlpha = 1,    // softmax warp: row maximum exchanged, alpha known
  kEvPDone = 2,    // softmax warp: probabilities stored, MMA issuer signalled
  kEvQK = 3,       // MMA issuer: QK of key tile j issued
  kEvPV = 4,       // MMA issuer: P and O ready, PV of key tile j issued
  kEvCorr = 5,     // correction warp: O rescaled (or skipped), MMA issuer signalled
  kEvKFull = 6,    // MMA issuer: K tile j landed in shared memory
  kEvProbs = 7,    // softmax warp: probabilities and their E4M3 words computed (before the P store)
  kEvPVDone = 8,   // MMA issuer: PV of key tile j issued and committed
  kEvSFree = 9,    // MMA issuer: scores of key tile j released by the softmax (QK(j+2) may start)
  kEvLd = 10,      // softmax warp: scores in registers
  kEvMax = 11,     // softmax warp: own row maxima known (before the running-max hand-off)
  kEvMWait = 12,   // softmax warp: running max of tile j-1 received
  kEvPVP = 13,     // MMA issuer: probabilities of key tile j observed (p_full)
  kEvPVO = 14,     // MMA issuer: O ready for key tile j observed (o_ready)
  kEvPDoneLast = 15,  // softmax warp of the last row quarter: probabilities handed over
  kNumEvents = 16
};
static_assert(kNumEvents == kTraceEvents, "trace buffer layout");

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
  const int qt = blockIdx.x;  // Q tile index
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], kTile);
      mbar_init(&sm.pv_done[i], 1);
      mbar_init(&sm.p_full[i], kTile);
      mbar_init(&sm.m_full[i], kTile);
      mbar_init(&sm.m_full[i + 2], kTile);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sm.o_ready[i], kTile);
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
        const int qrow = (int)(bh * p.Tq_pad + (int64_t)qt * kTile);
        mbar_arrive_expect_tx(&sm.q_full, kQKTileBytes);
        tma_load_2d(sm.q[0], &tm_q, &sm.q_full, 0, qrow);
        tma_load_2d(sm.q[1], &tm_q, &sm.q_full, 64, qrow);
        const int krow = (int)(bh * p.Tkv_pad);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % kStagesK;
          if (!mbar_wait(&sm.k_empty[s], ((uint32_t)(j / kStagesK) & 1u) ^ 1u, abort, kWaitLimitNs)) {
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
          if (!mbar_wait(&sm.v_empty[s], ((uint32_t)(j / kStagesV) & 1u) ^ 1u, abort, kWaitLimitNs)) {
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
        bool ok = mbar_wait(&sm.q_full, 0, abort, kWaitLimitNs);
        if (!ok) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaQ, abort);
        tc_fence_after();
        for (int j = 0; ok && j < nkv; ++j) {
          const int s = j % kStagesK;
          if (j >= 2) {
            // S(j%2) is free once the softmax of tile j-2 has read its scores
            if (!mbar_wait(&sm.s_free[j & 1], (uint32_t)((j - 2) >> 1) & 1u, abort, kWaitLimitNs)) {
              record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaS, abort);
              ok = false;
              break;
            }
            tc_fence_after();
            trace(kEvSFree, 0, j - 2);
          }
          if (!mbar_wait(&sm.k_full[s], (uint32_t)(j / kStagesK) & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaK, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          trace(kEvKFull, 0, j);
          const uint32_t s_col = (j & 1) ? kColS1 : kColS0;
          // 8 MMAs of K = 16: BF16 key dims [16kk, 16kk+16) = bytes 32*(kk%4) of half kk/4
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q[kk >> 2])) + 2 * (kk & 3);
            const uint64_t dk = sdesc_k_sw128(smem_u32(sm.k[s][kk >> 2])) + 2 * (kk & 3);
            mma_bf16_ss(tmem + s_col, dq, dk, kIdescQK, kk > 0);
          }
          mma_commit(&sm.s_full[j & 1]);
          mma_commit(&sm.k_empty[s]);
          trace(kEvQK, 0, j);
        }
        // wait until every MMA this thread issued has completed
        mma_commit(&sm.drain[0]);
        mbar_wait(&sm.drain[0], 0, nullptr, ok ? kWaitLimitNs : kDrainLimitNs);
      }
      __syncwarp();
    } else if (warp == 3) {
      // ------------------------------------------------ PV issuer ----
      if (lane == 0) {
        bool ok = true;
        for (int j = 0; ok && j < nkv; ++j) {
          const int s = j % kStagesV;
          if (!mbar_wait(&sm.p_full[j & 1], (uint32_t)(j >> 1) & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaP, abort);
            ok = false;
            break;
          }
          trace(kEvPVP, 0, j);
          if (!mbar_wait(&sm.o_ready[j & 1], (uint32_t)(j >> 1) & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaO, abort);
            ok = false;
            break;
          }
          trace(kEvPVO, 0, j);
          if (!mbar_wait(&sm.v_full[s], (uint32_t)(j / kStagesV) & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaV, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          trace(kEvPV, 0, j);
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.v[s]));
          const uint32_t p_col = (j & 1) ? kColP1 : kColP0;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts(tmem + kColO, tmem + p_col + 8 * kk, dv + 2 * kk, kIdescPV, j > 0 || kk > 0);
          mma_commit(&sm.pv_done[j & 1]);
          mma_commit(&sm.v_empty[s]);
          trace(kEvPVDone, 0, j);
        }
        if (ok) mma_commit(&sm.o_full);
        mma_commit(&sm.drain[1]);
        mbar_wait(&sm.drain[1], 0, nullptr, ok ? kWaitLimitNs : kDrainLimitNs);
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
    const uint32_t tO = tmem_lane_addr(tmem, quarter, kColO);
    bool ok = true;
    float m_prev = -INFINITY;  // running max after key tile j-1
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait(&sm.m_full[j & 3], (uint32_t)(j >> 2) & 1u, abort, kWaitLimitNs);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteCorrM, abort);
        break;
      }
      const float m_j = sm.mrow[j & 3][row];
      const float alpha = ex2_approx(__fsub_rn(m_prev, m_j));
      m_prev = m_j;
      if (j > 0) {
        // A warp whose rows all kept their maximum leaves O alone: PV(j) may follow
        // PV(j-1) in the tensor pipe directly.  It still waits for PV(j-2), which
        // consumed the previous phase of o_ready[j%2], so that this warpgroup never
        // runs two phases ahead of the PV issuer.  A warp that rescales needs O to
        // hold the sum over key tiles < j, i.e. PV(j-1) completed.
        const bool rescale = __any_sync(0xFFFFFFFFu, alpha != 1.0f);
        const int jw = rescale ? j - 1 : j - 2;
        if (jw >= 0) {
          ok = mbar_wait(&sm.pv_done[jw & 1], (uint32_t)(jw >> 1) & 1u, abort, kWaitLimitNs);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (!ok) {
            if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteCorrPV, abort);
            break;
          }
        }
        if (rescale) {
          tc_fence_after();
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
      mbar_arrive(&sm.o_ready[j & 1]);
      if (quarter == 0 && lane == 0) trace(kEvCorr, 0, j);
    }
    if (ok) {
      ok = mbar_wait(&sm.d_full, 0, abort, kWaitLimitNs) && mbar_wait(&sm.o_full, 0, abort, kWaitLimitNs);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok && lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteEpi, abort);
    }
    if (ok) {
      tc_fence_after();
      // d = sum over tiles of 448*p relative to the final max, from the two warpgroups
      const float m0 = sm.mlast[0][row], m1 = sm.mlast[1][row];
      const float mf = fmaxf(m0, m1);
      const float d = __fadd_rn(__fmul_rn(sm.dsum[0][row], ex2_approx(__fsub_rn(m0, mf))),
                                __fmul_rn(sm.dsum[1][row], ex2_approx(__fsub_rn(m1, mf))));
      const float r = __frcp_rn(d);
      const int64_t grow = (int64_t)qt * kTile + row;
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
    attn_teardown(tmem, false);
    return;
  }

  // -------------------------------------------------------- softmax ----
  regs_alloc<kRegsSoftmax>();
  const int par = wg - 1;  // this warpgroup owns key tiles j with j % 2 == par (scores in S(par))
  {
    const float sqi = p.sq[bh * (p.Tq_pad / kQGroup) + (int64_t)qt * (kTile / kQGroup) + quarter];
    const float* skh = p.sk + bh * (p.Tkv_pad / kKGroup);
    const uint32_t tS = tmem_lane_addr(tmem, quarter, par ? kColS1 : kColS0);
    const uint32_t tP = tmem_lane_addr(tmem, quarter, par ? kColP1 : kColP0);
    float m_w = -INFINITY, d_w = 0.0f;  // running max at this warpgroup's previous tile, its sum
    float sk0 = 0.0f, sk1 = 0.0f;
    if (par < nkv) {
      sk0 = __ldg(skh + 2 * par);
      sk1 = __ldg(skh + 2 * par + 1);
    }
    bool ok = true;
    for (int j = par; j < nkv; j += 2) {
      const float f0 = __fmul_rn(__fmul_rn(sqi, sk0), p.c_log2);
      const float f1 = __fmul_rn(__fmul_rn(sqi, sk1), p.c_log2);
      if (j + 2 < nkv) {
        sk0 = __ldg(skh + 2 * (j + 2));
        sk1 = __ldg(skh + 2 * (j + 2) + 1);
      }
      ok = mbar_wait(&sm.s_full[par], (uint32_t)(j >> 1) & 1u, abort, kWaitLimitNs);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftS, abort);
        break;
      }
      tc_fence_after();
      const bool tr = kTrace && tracing && quarter == 0 && lane == 0;
      if (tr) trace(kEvSReady, par, j);
      const int valid = min(kTile, p.Tkv - j * kTile);
      uint32_t x[128];
      tmem_ld64x2(tS, x);
      tc_fence_before();
      mbar_arrive(&sm.s_free[par]);
      if (tr) trace(kEvLd, par, j);
      float xm0, xm1;
      if (valid < kTile)
        rowmax128<true>(x, valid, xm0, xm1);
      else
        rowmax128<false>(x, valid, xm0, xm1);
      const float t0m = __fmul_rn(xm0, f0);  // valid >= 1: half 0 has a key
      const float t1m = valid > 64 ? __fmul_rn(xm1, f1) : -INFINITY;
      if (tr) {
        asm volatile("" ::"f"(t0m), "f"(t1m));  // the maxima exist before the stamp is taken
        trace(kEvMax, par, j);
      }
      // running max after tile j-1, from the other warpgroup
      float m_prev = -INFINITY;
      if (j > 0) {
        ok = mbar_wait(&sm.m_full[(j - 1) & 3], (uint32_t)((j - 1) >> 2) & 1u, abort, kWaitLimitNs);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftM, abort);
          break;
        }
        m_prev = sm.mrow[(j - 1) & 3][row];
      }
      if (tr) trace(kEvMWait, par, j);
      const float m_j = fmaxf(m_prev, fmaxf(t0m, t1m));
      sm.mrow[j & 3][row] = m_j;
      mbar_arrive(&sm.m_full[j & 3]);
      if (tr) trace(kEvAlpha, par, j);
      uint32_t pw[32];
      uint64_t acc2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc2[i] = 0ull;
      const float mq = __fsub_rn(m_j, kLog2_448);
      if (valid < kTile)
        probs128<true>(x, valid, f0, f1, mq, acc2, pw);
      else
        probs128<false>(x, valid, f0, f1, mq, acc2, pw);
      if (tr) trace(kEvProbs, par, j);
      if (j >= 2) {
        // P(j%2) still feeds PV(j-2) until that MMA has completed
        ok = mbar_wait(&sm.pv_done[par], (uint32_t)((j - 2) >> 1) & 1u, abort, kWaitLimitNs);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftPV, abort);
          break;
        }
        tc_fence_after();
      }
      tmem_st32(tP, pw);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[par]);
      if (tr) trace(kEvPDone, par, j);
      if (kTrace && tracing && quarter == 3 && lane == 0) trace(kEvPDoneLast, par, j);
      float a[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(acc2[i], a[2 * i], a[2 * i + 1]);
      const float es = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
      d_w = __fadd_rn(__fmul_rn(d_w, exp2_fma(__fsub_rn(m_w, m_j))), es);
      m_w = m_j;
    }
    if (ok) {
      sm.dsum[par][row] = d_w;
      sm.mlast[par][row] = m_w;
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
  static int done_mask = 0;  // one bit per device ordinal < 32
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 32 && (done_mask >> dev) & 1) return cudaSuccess;
  e = cudaFuncSetAttribute(attn_sm100_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmemBytes);
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
  if (dev < 32) done_mask |= 1 << dev;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attention(const char* ws, const Shape& s, const Layout& L, float c_log2,
                             const h3attn_bf16_out& out, cudaStream_t st, h3attn_status* why, uint64_t* trace,
                             int trace_block) {
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
  dim3 grid((unsigned)(s.Tq_pad / kTile), (unsigned)s.H, (unsigned)s.B);
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
