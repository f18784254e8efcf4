// Fused quantized attention mainloop for sm_100a ("H3 Performance Roadmap",
// Phase 4: Dense Sage-Compatible Attention; numerical checkpoints of "Phase 2B
// Aligned Numerical Prototype", Exactness).
//
// One CTA owns two 128-row Q tiles (A and B) of one (b, h) and streams all
// 128-key K/V tiles past them.  Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K and V^T tiles into a
//               3-stage shared-memory ring (separate K and V barriers).
//   warp 1      tensor-memory allocator and single-thread MMA issuer:
//               S = Q K^T  with tcgen05.mma kind::i8 (INT8 x INT8 -> S32),
//               O += P V   with tcgen05.mma kind::f8f6f4 (E4M3, A = P read
//               from tensor memory, F32 accumulate).
//   warps 2-3   stage the per-channel output scales, then idle.
//   warps 4-7   softmax + correction + epilogue for Q tile A,
//   warps 8-11  the same for Q tile B.  Thread = one Q row (= one TMEM lane).
// Tensor memory (512 columns): S_A [0,128) S_B [128,256) O_A [256,384)
// O_B [384,512).  P (128 x 128 E4M3 = 32 columns) overwrites the first 32
// columns of its S after the scores were read.  MMAs issued by one thread run
// in order, so S of tile j+1 is written only after P of tile j was consumed.
// The MMA order per key tile j keeps the tensor pipe busy while one softmax
// warpgroup works: QK_A(j), PV_B(j-1), QK_B(j), PV_A(j).
//
// Every wait is bounded: after the limit the waiter records H3ATTN_ERR_TIMEOUT
// in the workspace status word, raises a CTA-wide abort flag, drains the
// asynchronous work it issued and leaves; the tensor memory is freed.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>
#include <mutex>

#include "h3attn_internal.h"
#include "sm100_ptx.cuh"

namespace h3 {
namespace {

constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr uint32_t kTileBytes = 128 * 128;
constexpr uint32_t kColSA = 0, kColSB = 128, kColOA = 256, kColOB = 384;
constexpr uint32_t kIdescQK = idesc_i8_s32(128, 128);
constexpr uint32_t kIdescPV = idesc_e4m3_f32(128, 128);
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
// setmaxnreg split (registers per thread): control, correction, softmax warpgroups.
constexpr int kRegsControl = 56, kRegsCorrection = 96, kRegsSoftmax = 176;
constexpr int64_t kRegSplitTotal = 128 * (kRegsControl + kRegsCorrection + 2 * kRegsSoftmax);
static_assert(kRegSplitTotal <= 65536, "register split exceeds the SM register file");
constexpr uint64_t kDrainLimitNs = 200000000ull;  // 0.2 s

struct __align__(1024) AttnSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t a_full[2];   // softmax -> correction: alpha of the key tile published (one phase per tile)
  uint64_t o_ready[2];  // correction -> MMA issuer: O rescaled for the key tile
  uint64_t d_full[2];   // softmax -> correction: final row sum d published (one phase)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float svs[kD];
  float alpha[2][kTile];
  float dsum[2][kTile];
};

// Wait-site identifiers recorded in the status detail word.
enum : int {
  kSiteProdKEmpty = 1, kSiteProdVEmpty, kSiteMmaQ, kSiteMmaK, kSiteMmaPA, kSiteMmaPB, kSiteMmaV,
  kSiteSoftS, kSiteSoftO, kSiteMmaO, kSiteCorrA, kSiteCorrS, kSiteEpiO
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

constexpr uint32_t kMagic = 0x4B400000u;  // bit pattern of 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;     // 1.5 * 2^23

// Maximum of 64 INT32 scores of one row (tile columns col0 ..); with kMasked,
// columns >= valid (keys past Tkv) are ignored.  Eight independent chains.
template <bool kMasked, int kCol0>
__device__ __forceinline__ int rowmax64(const uint32_t (&s)[128], int valid) {
  int m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = INT_MIN;
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    int v = (int)s[kCol0 + e];
    if (kMasked && kCol0 + e >= valid) v = INT_MIN;
    m[e & 7] = max(m[e & 7], v);
  }
  return max(max(max(m[0], m[1]), max(m[2], m[3])), max(max(m[4], m[5]), max(m[6], m[7])));
}

// Probabilities of 64 scores of one row: t = float(acc) * f (float(acc) exact
// through the 1.5*2^23 magic number, |acc| < 2^22), p = 2^(t - m) in FP32,
// FP32 partial sums of p into acc2, E4M3 words of 448*p into w[0..15] (4 per word).
template <bool kMasked, int kCol0>
__device__ __forceinline__ void probs64(const uint32_t (&s)[128], int valid, float f, float m,
                                        uint64_t (&acc2)[4], uint32_t (&w)[32]) {
  const uint64_t negC = f2_pack(-kMagicF, -kMagicF);
  const uint64_t ff = f2_pack(f, f);
  const uint64_t negm = f2_pack(-m, -m);
  const uint64_t c448 = f2_pack(448.0f, 448.0f);
#pragma unroll
  for (int e = 0; e < 64; e += 4) {
    uint32_t half[2];
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      const int i = kCol0 + e + 2 * hp;
      const uint64_t x = f2_pack(__uint_as_float(s[i] + kMagic), __uint_as_float(s[i + 1] + kMagic));
      const uint64_t u = f2_add(f2_mul(f2_add(x, negC), ff), negm);
      float u0, u1;
      f2_unpack(u, u0, u1);
      float p0 = ex2_ftz(u0), p1 = ex2_ftz(u1);
      if (kMasked) {
        if (i >= valid) p0 = 0.0f;
        if (i + 1 >= valid) p1 = 0.0f;
      }
      const uint64_t pp = f2_pack(p0, p1);
      acc2[(i >> 1) & 3] = f2_add(acc2[(i >> 1) & 3], pp);
      float q0, q1;
      f2_unpack(f2_mul(pp, c448), q0, q1);
      half[hp] = cvt_e4m3x2(q0, q1);
    }
    w[(kCol0 + e) >> 2] = half[0] | (half[1] << 16);
  }
}

// One key tile of the online softmax for the row this thread owns: reads the
// INT32 scores from tensor memory (tS), updates the running max m; publishes
// alpha = 2^(m_old - m_new) to the correction warpgroup as soon as it is known
// (alpha_slot, a_bar), then writes the 32 E4M3 probability words over the first
// 32 score columns, hands them to the MMA issuer (p_bar) and updates the sum d.
template <bool kMasked>
__device__ __forceinline__ void softmax_tile(uint32_t tS, float f0, float f1, int valid, float& m, float& dsum,
                                             float* alpha_slot, uint64_t* a_bar, uint64_t* p_bar) {
  uint32_t pw[32];
  uint64_t acc2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc2[i] = 0ull;
  float m_new, alpha;
  {
    uint32_t sc[128];
    tmem_ld64x2(tS, sc);
    const int mi0 = rowmax64<kMasked, 0>(sc, valid);
    const int mi1 = rowmax64<kMasked, 64>(sc, valid);
    const float t0m = mi0 == INT_MIN ? -INFINITY : __fmul_rn(__int2float_rn(mi0), f0);
    const float t1m = mi1 == INT_MIN ? -INFINITY : __fmul_rn(__int2float_rn(mi1), f1);
    m_new = fmaxf(m, fmaxf(t0m, t1m));
    alpha = ex2_approx(__fsub_rn(m, m_new));
    *alpha_slot = alpha;
    mbar_arrive(a_bar);
    probs64<kMasked, 0>(sc, valid, f0, m_new, acc2, pw);
    probs64<kMasked, 64>(sc, valid, f1, m_new, acc2, pw);
  }
  tmem_st32(tS, pw);
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(p_bar);
  float a[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) f2_unpack(acc2[i], a[2 * i], a[2 * i + 1]);
  const float es = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  dsum = __fadd_rn(__fmul_rn(dsum, alpha), es);
  m = m_new;
}

// End of every role: all 384 threads meet, then warp 1 frees the tensor memory.
__device__ __forceinline__ void attn_teardown(uint32_t tmem, bool owner) {
  tc_fence_before();
  __syncthreads();
  if (owner) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

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
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2, quarter = warp & 3;
  const int64_t h = blockIdx.y, b = blockIdx.z, bh = b * p.H + h;
  const int qt0 = 2 * blockIdx.x;                       // Q tile index of tile A
  const bool has_b = (int64_t)(qt0 + 1) * kTile < p.Tq;  // tile B holds at least one row
  const int ntiles = has_b ? 2 : 1;
  const int nkv = (p.Tkv + kTile - 1) / kTile;
  volatile int* abort = &sm.abort;

  // ------------------------------------------------------------ set-up ----
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], kTile);
      mbar_init(&sm.o_full[t], 1);
      mbar_init(&sm.a_full[t], kTile);
      mbar_init(&sm.o_ready[t], kTile);
      mbar_init(&sm.d_full[t], kTile);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 2 || warp == 3) {
    for (int c = threadIdx.x - 64; c < kD; c += 64) sm.svs[c] = __fdiv_rn(p.sv[bh * kD + c], 448.0f);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Register split of the 512 x 128 launch budget: control warpgroup 56,
  // correction warpgroup 96, each softmax warpgroup 176:
  // 128*56 + 128*96 + 256*176 = 64512 <= 65536.  The host checks that the
  // kernel was built with 128 registers per thread before launching.
  if (wg == 0) {
    regs_dealloc<kRegsControl>();
    if (warp == 0) {
      // ---------------------------------------------------- TMA producer ----
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        const int qrow = (int)(bh * p.Tq_pad + (int64_t)qt0 * kTile);
        mbar_arrive_expect_tx(&sm.q_full, has_b ? 2 * kTileBytes : kTileBytes);
        tma_load_2d(sm.q[0], &tm_q, &sm.q_full, 0, qrow);
        if (has_b) tma_load_2d(sm.q[1], &tm_q, &sm.q_full, 0, qrow + kTile);
        const int krow = (int)(bh * p.Tkv_pad);
        const int vrow = (int)(bh * kD);
        int issued_k = 0, issued_v = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % kStages;
          const uint32_t ph = (uint32_t)(j / kStages) & 1u;
          if (!mbar_wait(&sm.k_empty[s], ph ^ 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteProdKEmpty, abort);
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[s], kTileBytes);
          tma_load_2d(sm.k[s], &tm_k, &sm.k_full[s], 0, krow + j * kTile);
          issued_k = j + 1;
          if (!mbar_wait(&sm.v_empty[s], ph ^ 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteProdVEmpty, abort);
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[s], kTileBytes);
          tma_load_2d(sm.v[s], &tm_v, &sm.v_full[s], j * kTile, vrow);
          issued_v = j + 1;
        }
        if (*abort) {
          // let every copy this thread started land before the CTA can exit
          mbar_wait(&sm.q_full, 0, nullptr, kDrainLimitNs);
          for (int j = (issued_k > kStages ? issued_k - kStages : 0); j < issued_k; ++j)
            mbar_wait(&sm.k_full[j % kStages], (uint32_t)(j / kStages) & 1u, nullptr, kDrainLimitNs);
          for (int j = (issued_v > kStages ? issued_v - kStages : 0); j < issued_v; ++j)
            mbar_wait(&sm.v_full[j % kStages], (uint32_t)(j / kStages) & 1u, nullptr, kDrainLimitNs);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------ MMA issuer ----
      if (lane == 0) {
        bool ok = mbar_wait(&sm.q_full, 0, abort, kWaitLimitNs);
        if (!ok) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaQ, abort);
        tc_fence_after();
        const uint64_t dq0 = sdesc_k_sw128(smem_u32(sm.q[0]));
        const uint64_t dq1 = sdesc_k_sw128(smem_u32(sm.q[1]));
        // PV of tile t for key tile jj once its P and its rescaled O are ready
        auto pv = [&](int t, int jj) -> bool {
          if (!mbar_wait(&sm.p_full[t], (uint32_t)jj & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, t ? kSiteMmaPB : kSiteMmaPA, abort);
            return false;
          }
          if (!mbar_wait(&sm.o_ready[t], (uint32_t)jj & 1u, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaO, abort);
            return false;
          }
          tc_fence_after();
          const uint64_t dv = sdesc_k_sw128(smem_u32(sm.v[jj % kStages]));
          const uint32_t o_col = t ? kColOB : kColOA, s_col = t ? kColSB : kColSA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ts(tmem + o_col, tmem + s_col + 8 * kk, dv + 2 * kk, kIdescPV, jj > 0 || kk > 0);
          return true;
        };
        for (int j = 0; ok && j < nkv; ++j) {
          const int s = j % kStages;
          const uint32_t ph = (uint32_t)(j / kStages) & 1u;
          if (!mbar_wait(&sm.k_full[s], ph, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaK, abort);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = sdesc_k_sw128(smem_u32(sm.k[s]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_i8_ss(tmem + kColSA, dq0 + 2 * kk, dk + 2 * kk, kIdescQK, kk > 0);
          mma_commit(&sm.s_full[0]);
          if (has_b) {
            if (j > 0) {
              if (!(ok = pv(1, j - 1))) break;
              mma_commit(&sm.v_empty[(j - 1) % kStages]);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_i8_ss(tmem + kColSB, dq1 + 2 * kk, dk + 2 * kk, kIdescQK, kk > 0);
            mma_commit(&sm.s_full[1]);
          }
          mma_commit(&sm.k_empty[s]);
          if (!mbar_wait(&sm.v_full[s], ph, abort, kWaitLimitNs)) {
            record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteMmaV, abort);
            ok = false;
            break;
          }
          if (!(ok = pv(0, j))) break;
          if (!has_b) mma_commit(&sm.v_empty[s]);
          if (j == nkv - 1) mma_commit(&sm.o_full[0]);
        }
        if (ok && has_b) {
          if ((ok = pv(1, nkv - 1))) {
            mma_commit(&sm.v_empty[(nkv - 1) % kStages]);
            mma_commit(&sm.o_full[1]);
          }
        }
        // wait until every MMA this thread issued has completed
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, ok ? kWaitLimitNs : kDrainLimitNs);
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
      for (int t = 0; t < ntiles; ++t) {
        ok = mbar_wait(&sm.a_full[t], (uint32_t)j & 1u, abort, kWaitLimitNs) &&
             mbar_wait(&sm.s_full[t], (uint32_t)j & 1u, abort, kWaitLimitNs);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) {
          if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteCorrA, abort);
          break;
        }
        tc_fence_after();
        const float alpha = sm.alpha[t][row];
        // O holds the sum over key tiles < j and the PV of tile j-1 has completed
        if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
          const uint32_t tO = tmem_lane_addr(tmem, quarter, t ? kColOB : kColOA);
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
        tc_fence_before();
        mbar_arrive(&sm.o_ready[t]);
      }
    }
    for (int t = 0; ok && t < ntiles; ++t) {
      ok = mbar_wait(&sm.d_full[t], 0, abort, kWaitLimitNs) && mbar_wait(&sm.o_full[t], 0, abort, kWaitLimitNs);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteEpiO, abort);
        break;
      }
      tc_fence_after();
      const float r = __frcp_rn(sm.dsum[t][row]);
      const int64_t grow = (int64_t)(qt0 + t) * kTile + row;
      const uint32_t tO = tmem_lane_addr(tmem, quarter, t ? kColOB : kColOA);
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
              const float y0 = __fmul_rn(__fmul_rn(__uint_as_float(o[e + 2 * u]), r), sm.svs[c0]);
              const float y1 = __fmul_rn(__fmul_rn(__uint_as_float(o[e + 2 * u + 1]), r), sm.svs[c0 + 1]);
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
  const int t = wg - 1;  // 0 = tile A, 1 = tile B
  if (t < ntiles) {
    const int qt = qt0 + t;
    const float sqi = p.sq[bh * (p.Tq_pad / kQGroup) + (int64_t)qt * (kTile / kQGroup) + quarter];
    const float* skh = p.sk + bh * (p.Tkv_pad / kKGroup);
    const uint32_t tS = tmem_lane_addr(tmem, quarter, t ? kColSB : kColSA);
    float m = -INFINITY, dsum = 0.0f;
    float sk0 = __ldg(skh + 0), sk1 = __ldg(skh + 1);
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const float f0 = __fmul_rn(__fmul_rn(sqi, sk0), p.c_log2);
      const float f1 = __fmul_rn(__fmul_rn(sqi, sk1), p.c_log2);
      if (j + 1 < nkv) {
        sk0 = __ldg(skh + 2 * (j + 1));
        sk1 = __ldg(skh + 2 * (j + 1) + 1);
      }
      ok = mbar_wait(&sm.s_full[t], (uint32_t)j & 1u, abort, kWaitLimitNs);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) {
        if (lane == 0) record_failure(p.status, H3ATTN_ERR_TIMEOUT, kSiteSoftS, abort);
        break;
      }
      tc_fence_after();
      const int valid = min(kTile, p.Tkv - j * kTile);
      if (valid < kTile)
        softmax_tile<true>(tS, f0, f1, valid, m, dsum, &sm.alpha[t][row], &sm.a_full[t], &sm.p_full[t]);
      else
        softmax_tile<false>(tS, f0, f1, valid, m, dsum, &sm.alpha[t][row], &sm.a_full[t], &sm.p_full[t]);
    }
    if (ok) {
      sm.dsum[t][row] = dsum;
      mbar_arrive(&sm.d_full[t]);
    }
  }
  attn_teardown(tmem, false);
}

// ------------------------------------------------------- debug QK tile ----
// One CTA of 128 threads computes the INT32 QK^T tile of (b, h, qt, kt) with
// the same TMA + tcgen05 kind::i8 path and writes it to global memory.
struct __align__(1024) DebugSmem {
  uint8_t q[kTileBytes];
  uint8_t k[kTileBytes];
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
    mbar_arrive_expect_tx(&sm.full, 2 * kTileBytes);
    tma_load_2d(sm.q, &tm_q, &sm.full, 0, qrow);
    tma_load_2d(sm.k, &tm_k, &sm.full, 0, krow);
    if (mbar_wait(&sm.full, 0, nullptr, kWaitLimitNs)) {
      tc_fence_after();
      const uint64_t dq = sdesc_k_sw128(smem_u32(sm.q)), dk = sdesc_k_sw128(smem_u32(sm.k));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_i8_ss(tmem, dq + 2 * kk, dk + 2 * kk, kIdescQK, kk > 0);
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
      for (int e = 0; e < 32; ++e) out[row * 128 + 32 * ch + e] = (int32_t)a[e];
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

// 2D byte tensor [rows, inner] with a row pitch; 128 x 128-byte boxes, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
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
  e = cudaFuncSetAttribute(attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(debug_qk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDebugSmemBytes);
  if (e != cudaSuccess) return e;
  // The warpgroup register split (setmaxnreg) needs the full launch budget.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_sm100_kernel);
  if (e != cudaSuccess) return e;
  if ((int64_t)fa.numRegs * kThreads < kRegSplitTotal) return cudaErrorInvalidConfiguration;
  if (dev < 32) done_mask |= 1 << dev;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attention(const char* ws, const Shape& s, const Layout& L, float c_log2,
                             const h3attn_bf16_out& out, cudaStream_t st, h3attn_status* why) {
  *why = H3ATTN_OK;
  cudaError_t e = ensure_attrs();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  const uint64_t BH = (uint64_t)s.B * s.H;
  if (!make_tmap(&tq, ws + L.off[H3ATTN_WS_Q8], kD, BH * s.Tq_pad, kD) ||
      !make_tmap(&tk, ws + L.off[H3ATTN_WS_K8], kD, BH * s.Tkv_pad, kD) ||
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
  const unsigned pairs = (unsigned)((s.Tq_pad / kTile + 1) / 2);
  dim3 grid(pairs, (unsigned)s.H, (unsigned)s.B);
  attn_sm100_kernel<<<grid, kThreads, kAttnSmemBytes, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_debug_qk(const char* ws, const Shape& s, const Layout& L, int b, int h, int qt, int kt,
                            int32_t* out, cudaStream_t st, h3attn_status* why) {
  *why = H3ATTN_OK;
  cudaError_t e = ensure_attrs();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk;
  const uint64_t BH = (uint64_t)s.B * s.H;
  if (!make_tmap(&tq, ws + L.off[H3ATTN_WS_Q8], kD, BH * s.Tq_pad, kD) ||
      !make_tmap(&tk, ws + L.off[H3ATTN_WS_K8], kD, BH * s.Tkv_pad, kD)) {
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
