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
};

// ------------------------------------------------------------------ stats ----
// One (unit, sub) pair: unit = (b*H + h)*nchunk + chunk, sub = 8-channel slice.
__device__ __forceinline__ void stats_unit(const PrepParams& p, int64_t unit, int sub) {
  const int64_t chunk = unit % p.nchunk, bh = unit / p.nchunk;
  const int64_t h = bh % p.H, b = bh / p.H;
  const int t0 = (int)(chunk * kChunk);
  const int t1 = min(p.Tkv, t0 + kChunk);
  const uint16_t* kp = p.k + b * p.ksb + h * p.ksh + sub * 8;
  const uint16_t* vp = p.v + b * p.vsb + h * p.vsh + sub * 8;
  double acc[8];
  float vm[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { acc[e] = 0.0; vm[e] = 0.0f; }
#pragma unroll 4
  for (int t = t0; t < t1; ++t) {
    float kf[8], vf[8];
    unpack8(ldg16(kp + (int64_t)t * p.kst), kf);
    unpack8(ldg16(vp + (int64_t)t * p.vst), vf);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[e] = __dadd_rn(acc[e], (double)kf[e]);
      vm[e] = fmaxf(vm[e], fabsf(vf[e]));
    }
  }
  double* ko = p.ksum + unit * kD + sub * 8;
  float* vo = p.vmax + unit * kD + sub * 8;
#pragma unroll
  for (int e = 0; e < 8; ++e) { ko[e] = acc[e]; vo[e] = vm[e]; }
}

// Slab blockIdx.x (128 tokens = chunks 2x, 2x + 1) of (b = blockIdx.z, h = blockIdx.y).
// Thread (c16 = tid & 15, r0 = tid >> 4) loads channels [8*c16, 8*c16+8) of slab rows
// r0 + 16 i (i < 8; rows of chunk i / 4): sixteen 16-byte loads in flight per thread.
// K goes to shared memory, where thread (chunk, channel) then adds its chunk's tokens
// in token order; the V absmax is reduced from the registers (a max is exact in any
// order).  The same sums and maxima as stats_unit.
constexpr int kStatsThreads = 256;

__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const PrepParams p) {
  __shared__ __align__(16) uint16_t ks[kTile * kD];                 // [row][channel] BF16
  __shared__ float vred[kStatsThreads / 32][kTile / kChunk][kD];  // [warp][chunk][channel]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, r0 = tid >> 4;
  const int64_t slab = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
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

// Clears the workspace status word, so each quantize call starts clean.
__device__ __forceinline__ void clear_status(const PrepParams& p) {
  p.status->code = 0;
  p.status->detail = 0;
  p.status->block = 0;
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
  if (bh == 0 && blockIdx.y == 0 && tid == 0) clear_status(p);
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

// Slab `slab` (128 tokens) of (b, h).  red, gmax and vt are the block's shared scratch.
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
  load_rows(rq8, q + b * qsb + h * qsh + c16 * 8, qst, t0, rq, has_q ? Tq : 0);
  load_rows(rk8, k + b * ksb + h * ksh + c16 * 8, kst, t0, rq, has_kv ? Tkv : 0);

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
__global__ void __launch_bounds__(256, 2) quantize_kernel(const PrepParams p) {
  __shared__ float red[8];
  __shared__ float gmax[4];
  __shared__ __align__(16) uint8_t vt[kD * kTile];  // [channel][token], 16-byte chunks XOR-swizzled
  quantize_slab(p, blockIdx.x, blockIdx.y, blockIdx.z, red, gmax, vt);
}

// Short sequences: the whole preparation of (b, h) = blockIdx.x in one block and one
// launch (statistics, their ordered reduction, then every slab), the same arithmetic
// as the three-kernel path.  Every stage's global writes are read by other threads of
// the block only after a block barrier.
__global__ void __launch_bounds__(256, 1) prep_small_kernel(const PrepParams p) {
  __shared__ float red[8];
  __shared__ float gmax[4];
  __shared__ __align__(16) uint8_t vt[kD * kTile];
  const int64_t bh = blockIdx.x;
  if (bh == 0 && threadIdx.x == 0) clear_status(p);
  for (int64_t c = threadIdx.x >> 4; c < p.nchunk; c += blockDim.x >> 4)
    stats_unit(p, bh * p.nchunk + c, (int)(threadIdx.x & 15));
  __syncthreads();
  if (threadIdx.x < kD) finalize_channel(p, bh, threadIdx.x);
  __syncthreads();
  const int64_t slabs = (p.Tq_pad > p.Tkv_pad ? p.Tq_pad : p.Tkv_pad) / kTile;
  for (int64_t slab = 0; slab < slabs; ++slab) quantize_slab(p, slab, bh % p.H, bh / p.H, red, gmax, vt);
}

// The finalize kernel's shared memory is above the default 48 KB limit (set once per device).
cudaError_t ensure_prep_attrs() {
  static int done_mask = 0;  // one bit per device ordinal < 32
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 32 && (done_mask >> dev) & 1) return cudaSuccess;
  e = cudaFuncSetAttribute(finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFinSmemBytes);
  if (e != cudaSuccess) return e;
  if (dev < 32) done_mask |= 1 << dev;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_quantize(const h3attn_bf16_view& q, const h3attn_bf16_view& k, const h3attn_bf16_view& v,
                            const Shape& s, const Layout& L, char* ws, cudaStream_t st) {
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
  const int64_t slabs = (s.Tq_pad > s.Tkv_pad ? s.Tq_pad : s.Tkv_pad) / kTile;
  if (slabs <= kSmallSlabs) {
    // few tokens per head: one launch, one block per (b, h)
    prep_small_kernel<<<(unsigned)((int64_t)s.B * s.H), 256, 0, st>>>(p);
    return cudaGetLastError();
  }
  const cudaError_t e = ensure_prep_attrs();
  if (e != cudaSuccess) return e;
  stats_kernel<<<dim3((unsigned)(s.Tkv_pad / kTile), (unsigned)s.H, (unsigned)s.B), kStatsThreads, 0, st>>>(p);
  finalize_kernel<<<dim3((unsigned)(s.B * s.H), kD / 32), kFinThreads, kFinSmemBytes, st>>>(p);
  dim3 grid((unsigned)slabs, (unsigned)s.H, (unsigned)s.B);
  quantize_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace h3
