// Preparation kernels of the quantized attention ("H3 Performance Roadmap",
// the Sage2 decomposition: K smoothing, Q/K INT8 quantization, V transpose and
// FP8 quantization; Phase 4 item 2: keep the per-warp INT8 Q/K and FP8 V policy).
//
//   stats_kernel    : one pass over K and V. Per (b, h, 64-token chunk, channel):
//                     FP64 sum of K in token order, FP32 absmax of V.  One block
//                     per 128-token slab; the slab is staged in shared memory with
//                     every load in flight before the in-order sums start.
//   finalize_kernel : per (b, h, channel): K mean = (sum of chunk sums in chunk
//                     order) / Tkv, rounded to FP32; V absmax and scale amax/448.
//                     The chunk sums pass through shared memory in 256-chunk
//                     passes, so that one warp's in-order sum never waits on a
//                     global load.
//   quantize_kernel : one pass over Q, K, V in 128-token slabs. INT8 Q per
//                     32-token group, INT8 (K - mean) per 64-token group, FP8 E4M3
//                     V per channel written transposed (channel-major), zero
//                     padding up to the 128-token tile multiple.  The INT8 Q/K
//                     words are stored as BF16 values (every integer in [-127, 127]
//                     is exact in BF16) so that the attention kernel can take QK^T
//                     on the BF16 tensor-core path with FP32 scores that equal the
//                     INT32 dot products exactly.
//
// All loads are 16-byte vectors of 8 BF16 channels; 16 threads cover one
// 128-channel row, so a warp reads two contiguous 256-byte rows per load.
//
// With the Q/K RMSNorm + RoPE preparation ("H3 Performance Roadmap", Component 2
// item 1: Q/K normalization and RoPE where the attention consumes Q and K), each
// Q and K row passes through norm_rope_row once, in registers, so the
// quantization sees the same BF16 values a separate norm_rope_kernel pass would
// have written.  norm_rope_kernel writes the transformed Q straight into the
// Q-word area of the workspace; the statistics pass transforms K (it needs it for
// the K means) and leaves it in the K-word area; the quantize pass reads both from
// there and overwrites them with the words.  Q, K and V are read raw once, and K
// is never written or re-read outside the workspace.
#include <cuda_bf16.h>

#include <mutex>

#include "h3attn_internal.h"
#include "sm100_ptx.cuh"

namespace h3 {
namespace {

// Sequences of at most this many 128-token slabs take the one-launch preparation.
constexpr int64_t kSmallSlabs = 4;

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// ------------------------------------------------------- Q/K norm + RoPE ----
// Two FP32 values rounded to the nearest BF16 (ties to even) and packed, lo in the low half.
__device__ __forceinline__ uint32_t bf16_pair(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// a, b replaced by their values rounded to the nearest BF16.
__device__ __forceinline__ void bf16_round2(float& a, float& b) {
  const uint32_t u = bf16_pair(a, b);
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xFFFF0000u);
}

// The half-warp of this thread (the 16 lanes that share one row).
__device__ __forceinline__ unsigned half_warp_mask() { return 0xFFFFu << (threadIdx.x & 16); }

// Per-head RMSNorm and rotary embedding of 128-channel rows.  The 16 lanes of a
// half-warp (lane & 15 = c16) hold channels [8 c16, 8 c16 + 8) of a row as one
// 16-byte word each and get them back transformed:
//   ss  = sum of x^2 in FP32: each lane adds its 8 squares in channel order, then
//         the 16 slice sums are added pairwise over lane distances 8, 4, 2, 1
//         (slice s with s + 8, those pairs with the pairs 4 apart, ...);
//   r   = 1 / sqrt(ss / 128 + eps), each FP32 step correctly rounded;
//   z_c = bf16(bf16(x_c r) * gamma_c);
//   (z_2i, z_2i+1) rotated by (cos_i, sin_i), every product and sum rounded to
//   FP32 separately (no FMA), then to BF16.
// Every product that feeds a sum uses the __fmul_rn / __fadd_rn intrinsics, which
// the compiler never contracts into a fused multiply-add (packed FP32-pair
// arithmetic gave fused results for the rotation in a measured build).  Each sum
// of the tree is computed by the lanes of its two operands with the operands
// swapped; addition commutes, so they get the same bits.

// This lane's 8 squares, in channel order.
__device__ __forceinline__ float slice_ss(const float (&x)[8]) {
  float part = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) part = __fadd_rn(part, __fmul_rn(x[e], x[e]));
  return part;
}

// 1 / sqrt(ss / 128 + eps).
__device__ __forceinline__ float rms_rcp(float ss, float eps) {
  const float ms = __fmul_rn(ss, 1.0f / kD);  // exact scaling: the same value as ss / 128
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
}

// n, z and the rotation of this lane's channels given r; g holds gamma of them, c
// and sn cos/sin of pairs [4 c16, 4 c16 + 4).
__device__ __forceinline__ uint4 norm_rope_apply(const float (&x)[8], float r, const float (&g)[8], float4 c,
                                                 float4 sn) {
  const uint64_t rr = f2_pack(r, r);
  const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float a, b;
    f2_unpack(f2_mul(f2_pack(x[2 * i], x[2 * i + 1]), rr), a, b);
    bf16_round2(a, b);  // n
    f2_unpack(f2_mul(f2_pack(a, b), f2_pack(g[2 * i], g[2 * i + 1])), a, b);
    bf16_round2(a, b);  // z
    // (a c - b s, b c + a s): products rounded, then one rounded sum each
    o[i] = bf16_pair(__fsub_rn(__fmul_rn(a, cc[i]), __fmul_rn(b, ss[i])),
                     __fadd_rn(__fmul_rn(b, cc[i]), __fmul_rn(a, ss[i])));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// One row per half-warp (`mask`): cs, sn point at cos/sin of pairs [4 c16, 4 c16 + 4)
// of the row's token (16-byte aligned).
__device__ __forceinline__ uint4 norm_rope_row(uint4 w, const float (&g)[8], const float* cs, const float* sn,
                                               float eps, unsigned mask) {
  const float4 c = __ldg(reinterpret_cast<const float4*>(cs));
  const float4 s = __ldg(reinterpret_cast<const float4*>(sn));
  float x[8];
  unpack8(w, x);
  float part = slice_ss(x);
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(mask, part, o));
  return norm_rope_apply(x, rms_rcp(part, eps), g, c, s);
}

// gamma of channels [8 c16, 8 c16 + 8)
__device__ __forceinline__ void load_gamma8(const float* gamma, int c16, float (&g)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(gamma + 8 * c16));
  const float4 b = __ldg(reinterpret_cast<const float4*>(gamma + 8 * c16 + 4));
  g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
  g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
}


// All three kernels take the same arguments.
struct PrepParams {
  const uint16_t* q;
  int64_t qsb, qst, qsh;
  const uint16_t* k;
  int64_t ksb, kst, ksh;
  const uint16_t* v;
  int64_t vsb, vst, vsh;
  int H, Tq, Tkv;
  int64_t Tq_pad, Tkv_pad, nchunk;
  double* ksum;  // [B, H, nchunk, 128] FP64 K chunk sums
  float* vmax;   // [B, H, nchunk, 128] V chunk absmax; chunk row 0 ends as the channel absmax
  float* km;
  float* sv;
  uint16_t* q8;
  float* sq;
  uint16_t* k8;
  float* sk;
  uint8_t* v8t;
  DevStatus* status;
  // Q/K RMSNorm + RoPE (kNormRope instantiations only): gamma [128], cos/sin [T, 64]
  const float* gamma_q;
  const float* gamma_k;
  const float* cos_q;
  const float* sin_q;
  const float* cos_k;
  const float* sin_k;
  float eps;
};

// ------------------------------------------------------------------ stats ----
// Statistics of slab `slab` (128 tokens = chunks 2 slab, 2 slab + 1) of (b, h), by a
// block of kStatsThreads threads.  Thread (c16 = tid & 15, r0 = tid >> 4) loads channels
// [8*c16, 8*c16+8) of slab rows r0 + 16 i (i < 8; rows of chunk i / 4): sixteen 16-byte
// loads in flight per thread.  K goes to shared memory (ks), where thread (chunk,
// channel) then adds its chunk's tokens in token order in FP64; the V absmax is reduced
// from the registers (a max is exact in any order) through vred.  Writes the chunk sums
// and maxima to the ksum / vmax scratch.  Contains one block barrier.
constexpr int kStatsThreads = 256;
typedef float VRed[kTile / kChunk][kD];  // [chunk][channel], one per warp

template <bool kNormRope>
__device__ __forceinline__ void stats_slab(const PrepParams& p, int64_t slab, int64_t h, int64_t b, uint16_t* ks,
                                           VRed* vred) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, r0 = tid >> 4;
  const int64_t bh = b * p.H + h, t0 = slab * kTile;
  const uint16_t* kp = p.k + b * p.ksb + h * p.ksh + c16 * 8;
  const uint16_t* vp = p.v + b * p.vsb + h * p.vsh + c16 * 8;
  uint4 kr[8], vr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + r0 + 16 * i;
    const bool in = t < p.Tkv;
    kr[i] = in ? ldg16(kp + t * p.kst) : make_uint4(0u, 0u, 0u, 0u);
    vr[i] = in ? ldg16(vp + t * p.vst) : make_uint4(0u, 0u, 0u, 0u);
  }
  if (kNormRope) {
    // the slab's K rows, transformed; also left in the K-word area for the quantize pass
    float g[8];
    load_gamma8(p.gamma_k, c16, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t t = t0 + r0 + 16 * i;
      if (t < p.Tkv) {  // the same for the 16 lanes of the row
        kr[i] = norm_rope_row(kr[i], g, p.cos_k + t * (kD / 2) + 4 * c16, p.sin_k + t * (kD / 2) + 4 * c16, p.eps,
                              half_warp_mask());
        *reinterpret_cast<uint4*>(p.k8 + (bh * p.Tkv_pad + t) * kD + c16 * 8) = kr[i];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4*>(ks + (r0 + 16 * i) * kD + c16 * 8) = kr[i];
  float vm[2][8];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) vm[c][e] = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float x[8];
    unpack8(vr[i], x);
#pragma unroll
    for (int e = 0; e < 8; ++e) vm[i >> 2][e] = fmaxf(vm[i >> 2][e], fabsf(x[e]));
  }
  // lanes l and l ^ 16 hold the same channels (slab rows 2w and 2w + 1 of each 16)
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) vm[c][e] = fmaxf(vm[c][e], __shfl_xor_sync(0xFFFFFFFFu, vm[c][e], 16));
  if (lane < 16) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int e = 0; e < 8; ++e) vred[warp][c][c16 * 8 + e] = vm[c][e];
  }
  __syncthreads();
  const int ck = tid >> 7, ch = tid & (kD - 1);
  const int64_t chunk = slab * (kTile / kChunk) + ck;
  if (chunk >= p.nchunk) return;
  const int n = (int)min((int64_t)kChunk, p.Tkv - chunk * kChunk);
  const uint16_t* col = ks + ck * kChunk * kD + ch;
  double acc = 0.0;
#pragma unroll 16
  for (int r = 0; r < n; ++r) acc = __dadd_rn(acc, (double)__uint_as_float((uint32_t)col[r * kD] << 16));
  float m = 0.0f;
#pragma unroll
  for (int w = 0; w < kStatsThreads / 32; ++w) m = fmaxf(m, vred[w][ck][ch]);
  const int64_t unit = bh * p.nchunk + chunk;
  p.ksum[unit * kD + ch] = acc;
  p.vmax[unit * kD + ch] = m;
}

// Slab blockIdx.x of (b = blockIdx.z, h = blockIdx.y).
template <bool kNormRope>
__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const PrepParams p) {
  __shared__ __align__(16) uint16_t ks[kTile * kD];  // [row][channel] BF16
  __shared__ VRed vred[kStatsThreads / 32];
  stats_slab<kNormRope>(p, blockIdx.x, blockIdx.y, blockIdx.z, ks, vred);
}

// --------------------------------------------------------------- finalize ----
// Channel c of (b, h): K mean = (sum of the chunk sums in chunk order) / Tkv, rounded
// to FP32; V absmax over all keys (left in chunk row 0 of the V-absmax scratch) and the
// V scale amax/448.
__device__ __forceinline__ void finalize_channel(const PrepParams& p, int64_t bh, int c) {
  const double* kp = p.ksum + bh * p.nchunk * kD + c;
  float* vp = p.vmax + bh * p.nchunk * kD + c;
  double s = 0.0;
  float m = 0.0f;
  // the sum stays sequential in chunk order; unrolling lets the loads run ahead of it
#pragma unroll 16
  for (int64_t ch = 0; ch < p.nchunk; ++ch) {
    s = __dadd_rn(s, kp[ch * kD]);
    m = fmaxf(m, vp[ch * kD]);
  }
  p.km[bh * kD + c] = __double2float_rn(__ddiv_rn(s, (double)p.Tkv));
  p.sv[bh * kD + c] = __fdiv_rn(m, 448.0f);
  vp[0] = m;
}

// Initialises the workspace status block of a new workspace (marker words absent).  An
// initialised block is left alone, so a failure recorded by an earlier call on this
// workspace survives until h3attn_check_status reads and clears it.
__device__ __forceinline__ void init_status(const PrepParams& p) {
  DevStatus* st = p.status;
  if (st->marker[0] != kStatusMarker0 || st->marker[1] != kStatusMarker1) {
    st->code = 0;
    st->detail = 0;
    st->block = 0;
    st->marker[0] = kStatusMarker0;
    st->marker[1] = kStatusMarker1;
  }
}

// Block (b*H + h = blockIdx.x, channels [32*blockIdx.y, 32*blockIdx.y + 32)); lane =
// channel.  Pass q stages the chunk sums of chunks [256q, 256q + 256) in shared memory
// (warp w loads 16 chunk rows, all in flight); warp 0 adds them in chunk order while
// every warp's loads of pass q + 1 are in flight.  The same sum, mean, absmax and
// scale as finalize_channel.
constexpr int kFinThreads = 512;
constexpr int kFinRowsPerWarp = 16;
constexpr int kFinRows = kFinThreads / 32 * kFinRowsPerWarp;
constexpr size_t kFinSmemBytes = 2 * (size_t)kFinRows * 32 * sizeof(double);

__global__ void __launch_bounds__(kFinThreads) finalize_kernel(const PrepParams p) {
  extern __shared__ __align__(16) double fin[];  // [2][kFinRows][32]
  __shared__ float vred[kFinThreads / 32][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = blockIdx.x;
  const int c = blockIdx.y * 32 + lane;
  if (bh == 0 && blockIdx.y == 0 && tid == 0) init_status(p);
  const double* kp = p.ksum + bh * p.nchunk * kD + c;
  float* vp = p.vmax + bh * p.nchunk * kD + c;
  const int64_t npass = (p.nchunk + kFinRows - 1) / kFinRows;
  double kr[kFinRowsPerWarp];
  float vr[kFinRowsPerWarp];
  float m = 0.0f;
  const auto load = [&](int64_t q) {
#pragma unroll
    for (int i = 0; i < kFinRowsPerWarp; ++i) {
      const int64_t ch = q * kFinRows + warp * kFinRowsPerWarp + i;
      const bool in = ch < p.nchunk;
      kr[i] = in ? kp[ch * kD] : 0.0;
      vr[i] = in ? vp[ch * kD] : 0.0f;
    }
  };
  const auto store = [&](int64_t q) {
    double* dst = fin + ((q & 1) * kFinRows + warp * kFinRowsPerWarp) * 32 + lane;
#pragma unroll
    for (int i = 0; i < kFinRowsPerWarp; ++i) {
      dst[i * 32] = kr[i];
      m = fmaxf(m, vr[i]);
    }
  };
  load(0);
  store(0);
  __syncthreads();
  double s = 0.0;
  for (int64_t q = 0; q < npass; ++q) {
    if (q + 1 < npass) load(q + 1);
    if (warp == 0) {
      const int n = (int)min((int64_t)kFinRows, p.nchunk - q * kFinRows);
      const double* row = fin + (q & 1) * kFinRows * 32 + lane;
#pragma unroll 16
      for (int r = 0; r < n; ++r) s = __dadd_rn(s, row[r * 32]);
    }
    // buffer (q + 1) & 1 was last read by warp 0 in pass q - 1, before the barrier
    if (q + 1 < npass) store(q + 1);
    __syncthreads();
  }
  vred[warp][lane] = m;
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int w = 1; w < kFinThreads / 32; ++w) m = fmaxf(m, vred[w][lane]);
  p.km[bh * kD + c] = __double2float_rn(__ddiv_rn(s, (double)p.Tkv));
  p.sv[bh * kD + c] = __fdiv_rn(m, 448.0f);
  vp[0] = m;
}

// --------------------------------------------------------------- quantize ----
__device__ __forceinline__ int q_i8(float x, float inv) {
  int r = __float2int_rn(__fmul_rn(x, inv));
  return max(-127, min(127, r));
}

// BF16 bit pattern of a small integer (|v| <= 127: exact).
__device__ __forceinline__ uint32_t bf16_of_int(int v) { return __float_as_uint(__int2float_rn(v)) >> 16; }

// Eight quantized values of one row slice as BF16 words, one 16-byte store.
__device__ __forceinline__ void store_words(uint16_t* dst, const float (&x)[8], float inv) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e)
    w[e] = bf16_of_int(q_i8(x[2 * e], inv)) | (bf16_of_int(q_i8(x[2 * e + 1], inv)) << 16);
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
  return x;
}

// Thread (c16 = tid & 15, rq = tid >> 4) owns channels [8*c16, 8*c16+8) of the
// 8 consecutive slab rows [8*rq, 8*rq+8).  Warp w covers slab rows [16w, 16w+16).
// The Q and K row loads are issued before either is used and the V loads right
// after the Q pass, so that a block keeps 64 KB in flight through its passes; the
// raw BF16 words stay in registers until each tensor's pass unpacks them.
__device__ __forceinline__ void load_rows(uint4 (&raw)[8], const uint16_t* p, int64_t st, int64_t t0, int rq,
                                          int T) {
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int64_t t = t0 + 8 * rq + r;
    raw[r] = t < T ? ldg16(p + t * st) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// load_rows from a dense [T_pad, 128] row block written earlier (by another kernel,
// or by this block before a barrier): loads cached in L2 only, never the
// non-coherent read-only path.
__device__ __forceinline__ void load_rows_cg(uint4 (&raw)[8], const uint16_t* p, int64_t t0, int rq, int T) {
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int64_t t = t0 + 8 * rq + r;
    raw[r] = t < T ? __ldcg(reinterpret_cast<const uint4*>(p + t * kD)) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Slab `slab` (128 tokens) of (b, h).  red, gmax and vt are the block's shared scratch.
template <bool kNormRope>
__device__ __forceinline__ void quantize_slab(const PrepParams& p, int64_t slab, int64_t h, int64_t b, float* red,
                                              float* gmax, uint8_t* vt) {
  const uint16_t* __restrict__ q = p.q;
  const uint16_t* __restrict__ k = p.k;
  const uint16_t* __restrict__ v = p.v;
  const int64_t qsb = p.qsb, qst = p.qst, qsh = p.qsh, ksb = p.ksb, kst = p.kst, ksh = p.ksh;
  const int64_t vsb = p.vsb, vst = p.vst, vsh = p.vsh;
  const int H = p.H, Tq = p.Tq, Tkv = p.Tkv;
  const int64_t Tq_pad = p.Tq_pad, Tkv_pad = p.Tkv_pad, nchunk = p.nchunk;
  const float* __restrict__ km = p.km;
  const float* __restrict__ vmax = p.vmax;
  uint16_t* __restrict__ q8 = p.q8;
  float* __restrict__ sq = p.sq;
  uint16_t* __restrict__ k8 = p.k8;
  float* __restrict__ sk = p.sk;
  uint8_t* __restrict__ v8t = p.v8t;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rq = tid >> 4;
  const int64_t t0 = slab * kTile;
  const int64_t bh = b * H + h;
  const bool has_q = t0 < Tq_pad, has_kv = t0 < Tkv_pad;

  // padding rows (t >= T) load as zero words (BF16 +0)
  uint4 rq8[8], rk8[8], rv8[8];
  if (kNormRope) {
    // Q and K rows already transformed by the statistics pass, in this slab's word areas
    load_rows_cg(rq8, p.q8 + bh * Tq_pad * kD + c16 * 8, t0, rq, has_q ? Tq : 0);
    load_rows_cg(rk8, p.k8 + bh * Tkv_pad * kD + c16 * 8, t0, rq, has_kv ? Tkv : 0);
  } else {
    load_rows(rq8, q + b * qsb + h * qsh + c16 * 8, qst, t0, rq, has_q ? Tq : 0);
    load_rows(rk8, k + b * ksb + h * ksh + c16 * 8, kst, t0, rq, has_kv ? Tkv : 0);
  }

  // ---------------------------------------------------------------- Q ----
  if (has_q) {
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float x[8];
      unpack8(rq8[r], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (tid < 4) {
      const float a = fmaxf(red[2 * tid], red[2 * tid + 1]);
      gmax[tid] = a;
      sq[bh * (Tq_pad / kQGroup) + t0 / kQGroup + tid] = __fdiv_rn(a, 127.0f);
    }
    __syncthreads();
    const float a = gmax[rq >> 2];
    const float inv = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float x[8];
      unpack8(rq8[r], x);
      store_words(q8 + (bh * Tq_pad + t0 + 8 * rq + r) * kD + c16 * 8, x, inv);
    }
    __syncthreads();
  }

  if (!has_kv) return;
  load_rows(rv8, v + b * vsb + h * vsh + c16 * 8, vst, t0, rq, Tkv);
  // ---------------------------------------------------------------- K ----
  {
    float kmv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) kmv[e] = km[bh * kD + c16 * 8 + e];
    // smoothed values of valid rows; padding rows stay exactly 0
    const auto smooth = [&](int r, float (&x)[8]) {
      unpack8(rk8[r], x);
      if (t0 + 8 * rq + r < Tkv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], kmv[e]);
      }
    };
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float x[8];
      smooth(r, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (tid < 2) {
      const float a = fmaxf(fmaxf(red[4 * tid], red[4 * tid + 1]), fmaxf(red[4 * tid + 2], red[4 * tid + 3]));
      gmax[tid] = a;
      sk[bh * (Tkv_pad / kKGroup) + t0 / kKGroup + tid] = __fdiv_rn(a, 127.0f);
    }
    __syncthreads();
    const float a = gmax[rq >> 3];
    const float inv = a > 0.0f ? __fdiv_rn(127.0f, a) : 0.0f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float x[8];
      smooth(r, x);
      store_words(k8 + (bh * Tkv_pad + t0 + 8 * rq + r) * kD + c16 * 8, x, inv);
    }
  }
  // ---------------------------------------------------------------- V ----
  {
    float inv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = vmax[bh * nchunk * kD + c16 * 8 + e];
      inv[e] = a > 0.0f ? __fdiv_rn(448.0f, a) : 0.0f;
    }
    // byte r of lo[e] / hi[e]: channel e of row r / r + 4 (E4M3)
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) lo[e] = hi[e] = 0u;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float x[8];
      unpack8(rv8[r], x);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const uint32_t p = cvt_e4m3x2(__fmul_rn(x[e], inv[e]), __fmul_rn(x[e + 1], inv[e + 1]));
        const int sh = 8 * (r & 3);
        if (r < 4) {
          lo[e] |= (p & 0xFFu) << sh;
          lo[e + 1] |= (p >> 8) << sh;
        } else {
          hi[e] |= (p & 0xFFu) << sh;
          hi[e + 1] |= (p >> 8) << sh;
        }
      }
    }
    // rows [8rq, 8rq+8) of channel c are bytes [8rq, 8rq+8) of smem row c; the
    // 16-byte chunk index is XORed with (c >> 3) & 7 to spread banks.
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = c16 * 8 + e;
      const int chunk = (rq >> 1) ^ ((c >> 3) & 7);
      *reinterpret_cast<uint2*>(vt + c * kTile + chunk * 16 + (rq & 1) * 8) = make_uint2(lo[e], hi[e]);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int vec = tid + 256 * j;
      const int c = vec >> 3, part = vec & 7;
      const int chunk = part ^ ((c >> 3) & 7);
      const uint4 val = *reinterpret_cast<const uint4*>(vt + c * kTile + chunk * 16);
      *reinterpret_cast<uint4*>(v8t + (bh * kD + c) * Tkv_pad + t0 + part * 16) = val;
    }
  }
}


// Slab blockIdx.x of (b = blockIdx.z, h = blockIdx.y).
template <bool kNormRope>
__global__ void __launch_bounds__(256, 2) quantize_kernel(const PrepParams p) {
  __shared__ float red[8];
  __shared__ float gmax[4];
  __shared__ __align__(16) uint8_t vt[kD * kTile];  // [channel][token], 16-byte chunks XOR-swizzled
  quantize_slab<kNormRope>(p, blockIdx.x, blockIdx.y, blockIdx.z, red, gmax, vt);
}

// Short sequences: the whole preparation of (b, h) = blockIdx.x in one block and one
// launch (statistics, their ordered reduction, then every slab), the same arithmetic
// as the three-kernel path.  Every stage's global writes are read by other threads of
// the block only after a block barrier.
template <bool kNormRope>
__global__ void __launch_bounds__(kStatsThreads, 1) prep_small_kernel(const PrepParams p) {
  __shared__ float red[8];
  __shared__ float gmax[4];
  // the statistics' staged K and V maxima, then (after a barrier) the V transpose tile
  __shared__ __align__(16) uint8_t scratch[kTile * kD * 2 + sizeof(VRed) * (kStatsThreads / 32)];
  uint16_t* ks = reinterpret_cast<uint16_t*>(scratch);
  VRed* vred = reinterpret_cast<VRed*>(scratch + kTile * kD * 2);
  uint8_t* vt = scratch;
  const int64_t bh = blockIdx.x;
  if (bh == 0 && threadIdx.x == 0) init_status(p);
  if (kNormRope) {
    // Q rows transformed into the Q-word area (half-warp = one row), K rows by stats_slab
    const int c16 = threadIdx.x & 15;
    float g[8];
    load_gamma8(p.gamma_q, c16, g);
    const uint16_t* qp = p.q + (bh / p.H) * p.qsb + (bh % p.H) * p.qsh + c16 * 8;
    for (int64_t t = threadIdx.x >> 4; t < p.Tq; t += blockDim.x >> 4)
      *reinterpret_cast<uint4*>(p.q8 + (bh * p.Tq_pad + t) * kD + c16 * 8) =
          norm_rope_row(ldg16(qp + t * p.qst), g, p.cos_q + t * (kD / 2) + 4 * c16, p.sin_q + t * (kD / 2) + 4 * c16,
                        p.eps, half_warp_mask());
  }
  for (int64_t slab = 0; slab < p.Tkv_pad / kTile; ++slab) {
    stats_slab<kNormRope>(p, slab, bh % p.H, bh / p.H, ks, vred);
    __syncthreads();  // ks and vred are rewritten by the next slab
  }
  if (threadIdx.x < kD) finalize_channel(p, bh, threadIdx.x);
  __syncthreads();
  const int64_t slabs = (p.Tq_pad > p.Tkv_pad ? p.Tq_pad : p.Tkv_pad) / kTile;
  for (int64_t slab = 0; slab < slabs; ++slab) quantize_slab<kNormRope>(p, slab, bh % p.H, bh / p.H, red, gmax, vt);
}

// Separate Q/K RMSNorm + RoPE pass (BF16 in, BF16 out) over the (b, t, h) rows of the
// [B, T, H, 128] view x: each half-warp takes kNormRopeRows consecutive rows, loads
// them all before transforming any, and writes them to the same rows of out.  out
// may be x itself (each lane reads its 16 bytes of a row before writing them).  The
// fused preparation also runs it on Q with out = the Q-word area of the workspace.
constexpr int kNormRopeRows = 4;

__global__ void __launch_bounds__(256) norm_rope_kernel(const uint16_t* x, int64_t xsb, int64_t xst, int64_t xsh,
                                                        uint16_t* out, int64_t osb, int64_t ost, int64_t osh, int T,
                                                        int H, int64_t nrows, const float* gamma, const float* cosv,
                                                        const float* sinv, float eps) {
  const int64_t row0 = ((int64_t)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4)) * kNormRopeRows;
  const int c16 = threadIdx.x & 15;
  float g[8];
  load_gamma8(gamma, c16, g);
  // (b, t, h) of the first row, then stepped row by row (h fastest)
  int64_t h = row0 % H, t = (row0 / H) % T, b = row0 / H / T;
  uint4 w[kNormRopeRows];
  int64_t oo[kNormRopeRows], tt[kNormRopeRows];
#pragma unroll
  for (int j = 0; j < kNormRopeRows; ++j) {
    oo[j] = b * osb + t * ost + h * osh + c16 * 8;
    tt[j] = t;
    w[j] = row0 + j < nrows ? ldg16(x + b * xsb + t * xst + h * xsh + c16 * 8) : make_uint4(0u, 0u, 0u, 0u);
    if (++h == H) {
      h = 0;
      if (++t == T) {
        t = 0;
        ++b;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kNormRopeRows; ++j) {
    if (row0 + j >= nrows) break;  // uniform over the half-warp
    *reinterpret_cast<uint4*>(out + oo[j]) = norm_rope_row(w[j], g, cosv + tt[j] * (kD / 2) + 4 * c16,
                                                           sinv + tt[j] * (kD / 2) + 4 * c16, eps, half_warp_mask());
  }
}

// The finalize kernel's shared memory is above the default 48 KB limit (set once per context).
cudaError_t ensure_prep_attrs() {
  static ContextSet done;  // contexts whose attribute is set
  if (done.contains(current_context_id())) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFinSmemBytes);
  if (e != cudaSuccess) return e;
  done.add(current_context_id());
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_quantize(const h3attn_bf16_view& q, const h3attn_bf16_view& k, const h3attn_bf16_view& v,
                            const Shape& s, const Layout& L, char* ws, cudaStream_t st,
                            const h3attn_qk_norm_rope* nr) {
  PrepParams p;
  p.q = static_cast<const uint16_t*>(q.data);
  p.qsb = q.stride_b; p.qst = q.stride_t; p.qsh = q.stride_h;
  p.k = static_cast<const uint16_t*>(k.data);
  p.ksb = k.stride_b; p.kst = k.stride_t; p.ksh = k.stride_h;
  p.v = static_cast<const uint16_t*>(v.data);
  p.vsb = v.stride_b; p.vst = v.stride_t; p.vsh = v.stride_h;
  p.H = s.H; p.Tq = s.Tq; p.Tkv = s.Tkv;
  p.Tq_pad = s.Tq_pad; p.Tkv_pad = s.Tkv_pad; p.nchunk = s.nchunk;
  p.ksum = reinterpret_cast<double*>(ws + L.off[H3ATTN_WS_KSUM]);
  p.vmax = reinterpret_cast<float*>(ws + L.off[H3ATTN_WS_VMAX]);
  p.km = reinterpret_cast<float*>(ws + L.off[H3ATTN_WS_KM]);
  p.sv = reinterpret_cast<float*>(ws + L.off[H3ATTN_WS_SV]);
  p.q8 = reinterpret_cast<uint16_t*>(ws + L.off[H3ATTN_WS_Q8]);
  p.sq = reinterpret_cast<float*>(ws + L.off[H3ATTN_WS_SQ]);
  p.k8 = reinterpret_cast<uint16_t*>(ws + L.off[H3ATTN_WS_K8]);
  p.sk = reinterpret_cast<float*>(ws + L.off[H3ATTN_WS_SK]);
  p.v8t = reinterpret_cast<uint8_t*>(ws + L.off[H3ATTN_WS_V8T]);
  p.status = reinterpret_cast<DevStatus*>(ws + L.off[H3ATTN_WS_STATUS]);
  p.gamma_q = nr ? nr->gamma_q : nullptr;
  p.gamma_k = nr ? nr->gamma_k : nullptr;
  p.cos_q = nr ? nr->cos_q : nullptr;
  p.sin_q = nr ? nr->sin_q : nullptr;
  p.cos_k = nr ? nr->cos_k : nullptr;
  p.sin_k = nr ? nr->sin_k : nullptr;
  p.eps = nr ? nr->eps : 0.0f;
  const int64_t slabs = (s.Tq_pad > s.Tkv_pad ? s.Tq_pad : s.Tkv_pad) / kTile;
  if (slabs <= kSmallSlabs) {
    // few tokens per head: one launch, one block per (b, h)
    if (nr)
      prep_small_kernel<true><<<(unsigned)((int64_t)s.B * s.H), 256, 0, st>>>(p);
    else
      prep_small_kernel<false><<<(unsigned)((int64_t)s.B * s.H), 256, 0, st>>>(p);
    return cudaGetLastError();
  }
  const cudaError_t e = ensure_prep_attrs();
  if (e != cudaSuccess) return e;
  if (nr) {
    // Q rows transformed by the separate-pass kernel straight into the Q-word area
    // ([B, H, Tq_pad, 128]), where the quantize pass reads them
    const h3attn_bf16_out qa = {p.q8, (int64_t)s.H * s.Tq_pad * kD, kD, s.Tq_pad * kD};
    const cudaError_t e2 = launch_norm_rope(q, s.B, s.Tq, s.H, nr->gamma_q, nr->cos_q, nr->sin_q, nr->eps, qa, st);
    if (e2 != cudaSuccess) return e2;
  }
  const dim3 sgrid((unsigned)(s.Tkv_pad / kTile), (unsigned)s.H, (unsigned)s.B);
  if (nr)
    stats_kernel<true><<<sgrid, kStatsThreads, 0, st>>>(p);
  else
    stats_kernel<false><<<sgrid, kStatsThreads, 0, st>>>(p);
  finalize_kernel<<<dim3((unsigned)(s.B * s.H), kD / 32), kFinThreads, kFinSmemBytes, st>>>(p);
  dim3 grid((unsigned)slabs, (unsigned)s.H, (unsigned)s.B);
  if (nr)
    quantize_kernel<true><<<grid, 256, 0, st>>>(p);
  else
    quantize_kernel<false><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_norm_rope(const h3attn_bf16_view& x, int B, int T, int H, const float* gamma, const float* cosv,
                             const float* sinv, float eps, const h3attn_bf16_out& out, cudaStream_t st) {
  const int64_t nrows = (int64_t)B * T * H;
  const int64_t per_block = 16 * kNormRopeRows;
  const int64_t blocks = (nrows + per_block - 1) / per_block;
  norm_rope_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const uint16_t*>(x.data), x.stride_b, x.stride_t, x.stride_h, static_cast<uint16_t*>(out.data),
      out.stride_b, out.stride_t, out.stride_h, T, H, nrows, gamma, cosv, sinv, eps);
  return cudaGetLastError();
}

}  // namespace h3
