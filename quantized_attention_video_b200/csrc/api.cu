// C ABI of libh3attn.so: argument validation, workspace layout, launches.
// Every check that needs no GPU runs before the first CUDA call, so a bad
// argument is reported without touching the device.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "h3attn_internal.h"

using namespace h3;

uint64_t h3::current_context_id() {
  typedef int (*GetCurrentFn)(void**);
  typedef int (*GetIdFn)(void*, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != 0 || ctx == nullptr || get_id(ctx, &id) != 0) return 0;
  return (uint64_t)id;
}

namespace {
std::mutex g_context_set_mu;
}  // namespace

bool h3::ContextSet::contains(uint64_t id) {
  if (id == 0) return false;
  std::lock_guard<std::mutex> lk(g_context_set_mu);
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == id) return true;
  return false;
}

void h3::ContextSet::add(uint64_t id) {
  if (id == 0) return;
  std::lock_guard<std::mutex> lk(g_context_set_mu);
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == id) return;
  ids_[next_] = id;  // beyond 64 contexts the oldest record is dropped (its attributes are then set again)
  next_ = (next_ + 1) % 64;
  if (n_ < 64) ++n_;
}

namespace {

constexpr double kLog2e = 1.44269504088896340736;

h3attn_status check_sizes(int B, int Tq, int Tkv, int H, int D) {
  if (D != kD) return H3ATTN_ERR_UNSUPPORTED;
  if (B < 1 || Tq < 1 || Tkv < 1 || H < 1) return H3ATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return H3ATTN_ERR_INVALID_ARG;  // grid y / z limits
  const Shape s = make_shape(B, Tq, Tkv, H);
  const int64_t BH = (int64_t)B * H;
  // tensor-map row coordinates are signed 32-bit
  if (BH * s.Tq_pad >= ((int64_t)1 << 31) || BH * s.Tkv_pad >= ((int64_t)1 << 31) ||
      BH * kD >= ((int64_t)1 << 31))
    return H3ATTN_ERR_INVALID_ARG;
  return H3ATTN_OK;
}

h3attn_status check_view(const h3attn_bf16_view* v) {
  if (v == nullptr) return H3ATTN_ERR_INVALID_ARG;
  return check_strides(v->data, v->stride_b, v->stride_t, v->stride_h);
}

h3attn_status check_out(const h3attn_bf16_out* o) {
  if (o == nullptr) return H3ATTN_ERR_INVALID_ARG;
  return check_strides(o->data, o->stride_b, o->stride_t, o->stride_h);
}

// An FP32 parameter table (gamma, cos, sin): non-null, 16-byte aligned (float4 loads).
h3attn_status check_table(const float* t) {
  if (t == nullptr) return H3ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t) % 16 != 0) return H3ATTN_ERR_ALIGNMENT;
  return H3ATTN_OK;
}

h3attn_status check_ws(const void* ws, size_t bytes, const Layout& L) {
  if (ws == nullptr) return H3ATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return H3ATTN_ERR_WORKSPACE;
  if (bytes < (size_t)L.off[H3ATTN_WS_END]) return H3ATTN_ERR_WORKSPACE;
  return H3ATTN_OK;
}

// The current device must be compute capability 10.0 (sm_100a code only).
h3attn_status check_device() {
  static std::mutex mu;
  static int known[64] = {};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return H3ATTN_ERR_CUDA;
  if (dev < 0 || dev >= 64) return H3ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (known[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return H3ATTN_ERR_CUDA;
    known[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return known[dev] == 1 ? H3ATTN_OK : H3ATTN_ERR_UNSUPPORTED;
}

#define H3_TRY(expr)                         \
  do {                                       \
    const h3attn_status st_ = (expr);        \
    if (st_ != H3ATTN_OK) return st_;        \
  } while (0)

}  // namespace

extern "C" {

size_t h3attn_workspace_bytes(int B, int Tq, int Tkv, int H, int D) {
  if (check_sizes(B, Tq, Tkv, H, D) != H3ATTN_OK) return 0;
  return (size_t)make_layout(make_shape(B, Tq, Tkv, H)).off[H3ATTN_WS_END];
}

h3attn_status h3attn_workspace_layout(int B, int Tq, int Tkv, int H, int D, int64_t offsets[H3ATTN_WS_NFIELDS]) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  if (offsets == nullptr) return H3ATTN_ERR_INVALID_ARG;
  const Layout L = make_layout(make_shape(B, Tq, Tkv, H));
  for (int f = 0; f < H3ATTN_WS_NFIELDS; ++f) offsets[f] = L.off[f];
  return H3ATTN_OK;
}

h3attn_status h3attn_quantize_qkv(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                                  int B, int Tq, int Tkv, int H, int D, void* ws, size_t ws_bytes, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_view(q));
  H3_TRY(check_view(k));
  H3_TRY(check_view(v));
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  H3_TRY(check_ws(ws, ws_bytes, L));
  H3_TRY(check_device());
  if (launch_quantize(*q, *k, *v, s, L, static_cast<char*>(ws), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_attend(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H, int D,
                            float softmax_scale, const h3attn_bf16_out* out, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_out(out));
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return H3ATTN_ERR_INVALID_ARG;
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  H3_TRY(check_ws(ws, ws_bytes, L));
  H3_TRY(check_device());
  const float c_log2 = (float)((double)softmax_scale * kLog2e);
  h3attn_status why = H3ATTN_OK;
  if (launch_attention(static_cast<const char*>(ws), s, L, c_log2, *out, static_cast<cudaStream_t>(stream), &why) !=
      cudaSuccess)
    return why != H3ATTN_OK ? why : H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_forward_ex(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                                int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                const h3attn_bf16_out* out, void* ws, size_t ws_bytes, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_out(out));
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return H3ATTN_ERR_INVALID_ARG;
  H3_TRY(h3attn_quantize_qkv(q, k, v, B, Tq, Tkv, H, D, ws, ws_bytes, stream));
  return h3attn_attend(ws, ws_bytes, B, Tq, Tkv, H, D, softmax_scale, out, stream);
}

h3attn_status h3attn_forward(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                             int B, int T, int H, int D, float softmax_scale, const h3attn_bf16_out* out, void* ws,
                             size_t ws_bytes, void* stream) {
  return h3attn_forward_ex(q, k, v, B, T, T, H, D, softmax_scale, out, ws, ws_bytes, stream);
}

h3attn_status h3attn_quantize_qkv_norm_rope(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                            const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                            const h3attn_qk_norm_rope* nr, void* ws, size_t ws_bytes,
                                            void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_view(q));
  H3_TRY(check_view(k));
  H3_TRY(check_view(v));
  if (nr == nullptr) return H3ATTN_ERR_INVALID_ARG;
  for (const float* t : {nr->gamma_q, nr->gamma_k, nr->cos_q, nr->sin_q, nr->cos_k, nr->sin_k})
    H3_TRY(check_table(t));
  if (!(nr->eps > 0.0f) || !std::isfinite(nr->eps)) return H3ATTN_ERR_INVALID_ARG;
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  H3_TRY(check_ws(ws, ws_bytes, L));
  H3_TRY(check_device());
  if (launch_quantize(*q, *k, *v, s, L, static_cast<char*>(ws), static_cast<cudaStream_t>(stream), nr) !=
      cudaSuccess)
    return H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_forward_norm_rope(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                       const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                       float softmax_scale, const h3attn_qk_norm_rope* nr,
                                       const h3attn_bf16_out* out, void* ws, size_t ws_bytes, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_out(out));
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return H3ATTN_ERR_INVALID_ARG;
  H3_TRY(h3attn_quantize_qkv_norm_rope(q, k, v, B, Tq, Tkv, H, D, nr, ws, ws_bytes, stream));
  return h3attn_attend(ws, ws_bytes, B, Tq, Tkv, H, D, softmax_scale, out, stream);
}

h3attn_status h3attn_norm_rope(const h3attn_bf16_view* x, int B, int T, int H, int D, const float* gamma,
                               const float* cos_tab, const float* sin_tab, float eps,
                               const h3attn_bf16_out* out, void* stream) {
  H3_TRY(check_sizes(B, T, T, H, D));
  H3_TRY(check_view(x));
  H3_TRY(check_out(out));
  for (const float* t : {gamma, cos_tab, sin_tab}) H3_TRY(check_table(t));
  if (!(eps > 0.0f) || !std::isfinite(eps)) return H3ATTN_ERR_INVALID_ARG;
  H3_TRY(check_device());
  if (launch_norm_rope(*x, B, T, H, gamma, cos_tab, sin_tab, eps, *out, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_check_status(void* ws, void* stream) {
  if (ws == nullptr || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return H3ATTN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return H3ATTN_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return H3ATTN_ERR_CUDA;
  // clear the code, detail and block words and leave the block initialised (marker
  // set), so that the next quantize pass keeps, rather than re-initialises, whatever a
  // later call records
  const uint32_t fresh[5] = {0u, 0u, 0u, kStatusMarker0, kStatusMarker1};
  if (cudaMemcpy(ws, fresh, sizeof(fresh), cudaMemcpyHostToDevice) != cudaSuccess) return H3ATTN_ERR_CUDA;
  if (code < 0 || code > H3ATTN_ERR_TIMEOUT) return H3ATTN_ERR_CUDA;
  return static_cast<h3attn_status>(code);
}

h3attn_status h3attn_debug_qk_scores(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H, int D, int b,
                                     int h, int qt, int kt, int32_t* out_dev, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  H3_TRY(check_ws(ws, ws_bytes, L));
  if (out_dev == nullptr) return H3ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out_dev) % 16 != 0) return H3ATTN_ERR_ALIGNMENT;
  if (b < 0 || b >= B || h < 0 || h >= H || qt < 0 || qt >= s.Tq_pad / kTile || kt < 0 || kt >= s.Tkv_pad / kTile)
    return H3ATTN_ERR_INVALID_ARG;
  H3_TRY(check_device());
  h3attn_status why = H3ATTN_OK;
  if (launch_debug_qk(static_cast<const char*>(ws), s, L, b, h, qt, kt, out_dev, static_cast<cudaStream_t>(stream),
                      &why) != cudaSuccess)
    return why != H3ATTN_OK ? why : H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_debug_attend_timeout(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H, int D,
                                          float softmax_scale, const h3attn_bf16_out* out,
                                          uint64_t wait_limit_ns, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_out(out));
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return H3ATTN_ERR_INVALID_ARG;
  if (wait_limit_ns < 1000000ull || wait_limit_ns > kDefaultWaitLimitNs) return H3ATTN_ERR_INVALID_ARG;
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  H3_TRY(check_ws(ws, ws_bytes, L));
  H3_TRY(check_device());
  const float c_log2 = (float)((double)softmax_scale * kLog2e);
  h3attn_status why = H3ATTN_OK;
  if (launch_attention(static_cast<const char*>(ws), s, L, c_log2, *out, static_cast<cudaStream_t>(stream), &why,
                       nullptr, -1, wait_limit_ns, true) != cudaSuccess)
    return why != H3ATTN_OK ? why : H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

h3attn_status h3attn_debug_attend_trace(const void* ws, size_t ws_bytes, int B, int Tq, int Tkv, int H, int D,
                                        float softmax_scale, const h3attn_bf16_out* out, int trace_block,
                                        uint64_t* trace_dev, void* stream) {
  H3_TRY(check_sizes(B, Tq, Tkv, H, D));
  H3_TRY(check_out(out));
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale)) return H3ATTN_ERR_INVALID_ARG;
  if (trace_dev == nullptr) return H3ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(trace_dev) % 8 != 0) return H3ATTN_ERR_ALIGNMENT;
  const Shape s = make_shape(B, Tq, Tkv, H);
  const Layout L = make_layout(s);
  const int64_t ctas = attention_ctas(s);
  if (trace_block < 0 || trace_block >= ctas) return H3ATTN_ERR_INVALID_ARG;
  H3_TRY(check_ws(ws, ws_bytes, L));
  H3_TRY(check_device());
  const float c_log2 = (float)((double)softmax_scale * kLog2e);
  h3attn_status why = H3ATTN_OK;
  if (launch_attention(static_cast<const char*>(ws), s, L, c_log2, *out, static_cast<cudaStream_t>(stream), &why,
                       trace_dev, trace_block) != cudaSuccess)
    return why != H3ATTN_OK ? why : H3ATTN_ERR_CUDA;
  return H3ATTN_OK;
}

const char* h3attn_status_string(h3attn_status s) {
  switch (s) {
    case H3ATTN_OK: return "ok";
    case H3ATTN_ERR_INVALID_ARG: return "invalid argument";
    case H3ATTN_ERR_UNSUPPORTED: return "unsupported (head dim must be 128; device must be sm_100)";
    case H3ATTN_ERR_ALIGNMENT: return "misaligned pointer or stride (16-byte data, strides multiple of 8)";
    case H3ATTN_ERR_WORKSPACE: return "workspace null, not 256-byte aligned, or too small";
    case H3ATTN_ERR_CUDA: return "CUDA error";
    case H3ATTN_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int h3attn_version(void) { return H3ATTN_VERSION; }

}  // extern "C"
