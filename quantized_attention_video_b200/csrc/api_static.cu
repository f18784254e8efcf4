// h3attn_forward_static: the forward pass for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a device workspace. Examples: a host
// application that owns the device allocator and gives this library no route
// to request memory through a C interface, or a runtime whose rules forbid
// device allocation after start-up. This entry point takes only the inputs and
// the output. The workspace (quantized Q/K/V, scales and the reduction scratch)
// lives in one file-scope device array of H3ATTN_STATIC_WS_BYTES. Every GPU that
// loads this library holds that array until the process exits.
//
// Behaviour:
//   - The first call on a device, with that device current, looks up the
//     array's device address with cudaGetSymbolAddress and caches it for that
//     device. That first call should come before any stream capture.
//   - Host code cannot pass the array's name to a kernel: on the host the name
//     is only a stand-in, not a device address. The looked-up address is passed
//     instead.
//   - No cudaMalloc, cudaFree or other allocating routine is ever called.
//   - Shapes whose workspace exceeds the array are rejected with
//     H3ATTN_ERR_WORKSPACE before anything is enqueued.
//   - Every call shares the array, and it keeps the previous call's contents.
//     Calls whose work overlaps on the GPU (for example on two streams) race
//     on it; the caller must order them.
//   - What must start at zero is rewritten by every call: the quantize pass
//     clears the status word and writes the zero padding.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/h3attn.h"

namespace {

__device__ __align__(256) unsigned char g_static_ws[H3ATTN_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws for the current device (looked up once per device).
h3attn_status static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return H3ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return H3ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ws_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || ptr == nullptr) return H3ATTN_ERR_CUDA;
    g_ws_ptr[dev] = ptr;
  }
  *out = g_ws_ptr[dev];
  return H3ATTN_OK;
}

}  // namespace

extern "C" h3attn_status h3attn_forward_static(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                               const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                               float softmax_scale, const h3attn_bf16_out* out, void* stream) {
  const size_t need = h3attn_workspace_bytes(B, Tq, Tkv, H, D);
  if (need == 0) return D != H3ATTN_HEAD_DIM ? H3ATTN_ERR_UNSUPPORTED : H3ATTN_ERR_INVALID_ARG;
  if (need > (size_t)H3ATTN_STATIC_WS_BYTES) return H3ATTN_ERR_WORKSPACE;
  void* ws = nullptr;
  const h3attn_status st = static_workspace(&ws);
  if (st != H3ATTN_OK) return st;
  return h3attn_forward_ex(q, k, v, B, Tq, Tkv, H, D, softmax_scale, out, ws, (size_t)H3ATTN_STATIC_WS_BYTES,
                           stream);
}
