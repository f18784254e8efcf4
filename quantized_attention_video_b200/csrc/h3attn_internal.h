// Internal definitions shared by the host API and the kernels of libh3attn.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/h3attn.h"

namespace h3 {

constexpr int kD = H3ATTN_HEAD_DIM;     // head dimension (fixed)
constexpr int kTile = H3ATTN_TILE;      // Q rows / keys per attention tile
constexpr int kQGroup = H3ATTN_Q_GROUP; // Q tokens per scale
constexpr int kKGroup = H3ATTN_K_GROUP; // K tokens per scale
constexpr int kChunk = 64;              // tokens per K-mean / V-absmax partial

struct Shape {
  int B, Tq, Tkv, H;
  int64_t Tq_pad, Tkv_pad;  // multiples of kTile
  int64_t nchunk;           // ceil(Tkv / kChunk)
};

struct Layout {
  int64_t off[H3ATTN_WS_NFIELDS];
};

inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

inline Shape make_shape(int B, int Tq, int Tkv, int H) {
  Shape s;
  s.B = B; s.Tq = Tq; s.Tkv = Tkv; s.H = H;
  s.Tq_pad = round_up(Tq, kTile);
  s.Tkv_pad = round_up(Tkv, kTile);
  s.nchunk = (Tkv + kChunk - 1) / kChunk;
  return s;
}

inline Layout make_layout(const Shape& s) {
  const int64_t BH = (int64_t)s.B * s.H;
  int64_t sz[H3ATTN_WS_NFIELDS] = {};
  sz[H3ATTN_WS_STATUS] = 256;
  sz[H3ATTN_WS_Q8] = BH * s.Tq_pad * kD * 2;   // INT8 words held as equal BF16 values
  sz[H3ATTN_WS_K8] = BH * s.Tkv_pad * kD * 2;
  sz[H3ATTN_WS_V8T] = BH * kD * s.Tkv_pad;
  sz[H3ATTN_WS_SQ] = BH * (s.Tq_pad / kQGroup) * 4;
  sz[H3ATTN_WS_SK] = BH * (s.Tkv_pad / kKGroup) * 4;
  sz[H3ATTN_WS_KM] = BH * kD * 4;
  sz[H3ATTN_WS_SV] = BH * kD * 4;
  sz[H3ATTN_WS_KSUM] = BH * s.nchunk * kD * 8;
  sz[H3ATTN_WS_VMAX] = BH * s.nchunk * kD * 4;
  Layout L;
  int64_t o = 0;
  for (int f = 0; f < H3ATTN_WS_END; ++f) {
    L.off[f] = o;
    o = round_up(o + sz[f], 1024);
  }
  L.off[H3ATTN_WS_END] = o;
  return L;
}

// A strided BF16 view's pointer and strides (elements): non-null, 16-byte aligned
// data, non-negative strides that are multiples of 8 elements (16-byte vectors).
inline h3attn_status check_strides(const void* data, int64_t sb, int64_t st, int64_t sh) {
  if (data == nullptr) return H3ATTN_ERR_INVALID_ARG;
  if (sb < 0 || st < 0 || sh < 0) return H3ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(data) % 16 != 0) return H3ATTN_ERR_ALIGNMENT;
  if (sb % 8 != 0 || st % 8 != 0 || sh % 8 != 0) return H3ATTN_ERR_ALIGNMENT;
  return H3ATTN_OK;
}

// Device-side status words at the start of the workspace.  The status is sticky: a
// quantize pass initialises the block only when its two marker words are missing (a
// new workspace), and h3attn_check_status clears the code but keeps the marker, so a
// failure recorded by any call stays until h3attn_check_status reads and clears it.
constexpr uint32_t kStatusMarker0 = 0x68336174u, kStatusMarker1 = 0x74737453u;
struct DevStatus {
  int code;    // h3attn_status of the first failure, 0 if none
  int detail;  // which wait expired (kernel-defined id)
  int block;   // linear block index that recorded it
  uint32_t marker[2];  // kStatusMarker0, kStatusMarker1 once initialised
  int pad[59];
};
static_assert(sizeof(DevStatus) == 256, "status block size");

// Kernel launchers (defined in quantize.cu / attention.cu).
// nr != nullptr: Q and K rows pass through the RMSNorm + RoPE transform as they are loaded.
cudaError_t launch_quantize(const h3attn_bf16_view& q, const h3attn_bf16_view& k, const h3attn_bf16_view& v,
                            const Shape& s, const Layout& L, char* ws, cudaStream_t st,
                            const h3attn_qk_norm_rope* nr = nullptr);
// The separate RMSNorm + RoPE pass over a [B, T, H, 128] view.
cudaError_t launch_norm_rope(const h3attn_bf16_view& x, int B, int T, int H, const float* gamma, const float* cosv,
                             const float* sinv, float eps, const h3attn_bf16_out& out, cudaStream_t st);

// The attention grid: one CTA per pair of 128-row Q tiles of one (b, h).
inline int64_t attention_ctas(const Shape& s) { return ((s.Tq_pad / kTile + 1) / 2) * (int64_t)s.H * s.B; }

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // bound of every barrier wait: 2 s
cudaError_t launch_attention(const char* ws, const Shape& s, const Layout& L, float c_log2,
                             const h3attn_bf16_out& out, cudaStream_t st, h3attn_status* why,
                             uint64_t* trace = nullptr, int trace_block = -1,
                             uint64_t wait_limit_ns = kDefaultWaitLimitNs, bool withhold_o_ready = false);
constexpr int kTraceEvents = 16;  // events per (tile slot, key tile) in the timeline trace

// Kernel attributes (cudaFuncSetAttribute) belong to a CUDA context, so a record of the
// contexts whose attributes are set must name contexts, not device ordinals: after a
// cudaDeviceReset, or with another context made current on the same device, the
// attributes have to be set again.  current_context_id() is the driver's id of the
// context current on this thread (unique for the life of the process; cuCtxGetId), or
// 0 when there is none or the driver cannot tell, in which case nothing is recorded.
uint64_t current_context_id();

// A thread-safe record of the contexts that have been set up.
class ContextSet {
 public:
  bool contains(uint64_t id);
  void add(uint64_t id);  // ignores id 0

 private:
  uint64_t ids_[64] = {};
  int n_ = 0;
  int next_ = 0;
};
cudaError_t launch_debug_qk(const char* ws, const Shape& s, const Layout& L, int b, int h, int qt, int kt,
                            int32_t* out, cudaStream_t st, h3attn_status* why);

}  // namespace h3
