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
//   - Every call looks up the array's device address for the current device and
//     context with cudaGetSymbolAddress (a host-side query) and checks the result.
//     The first call on a device also makes the runtime load this library's device
//     code there, so that first call should come before any stream capture.
//     Looking the address up on every call, rather than caching it, means that a
//     device reset or a different current context never gets a stale address.
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
//     writes the zero padding of every field it uses.  The status block at the
//     start of the array is zero when the library loads; the first quantize pass
//     initialises it, and from then on it keeps the first device-side failure of
//     any call until h3attn_static_check_status reads and clears it.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/h3attn.h"

namespace {

__device__ __align__(256) unsigned char g_static_ws[H3ATTN_STATIC_WS_BYTES];

// Device address of g_static_ws for the current device and context.
h3attn_status static_workspace(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_ws) != cudaSuccess || ptr == nullptr) return H3ATTN_ERR_CUDA;
  *out = ptr;
  return H3ATTN_OK;
}

// Rejects shapes whose workspace does not fit the array.
h3attn_status static_fit(int B, int Tq, int Tkv, int H, int D) {
  const size_t need = h3attn_workspace_bytes(B, Tq, Tkv, H, D);
  if (need == 0) return D != H3ATTN_HEAD_DIM ? H3ATTN_ERR_UNSUPPORTED : H3ATTN_ERR_INVALID_ARG;
  if (need > (size_t)H3ATTN_STATIC_WS_BYTES) return H3ATTN_ERR_WORKSPACE;
  return H3ATTN_OK;
}

}  // namespace

extern "C" {

size_t h3attn_static_workspace_bytes(void) { return (size_t)H3ATTN_STATIC_WS_BYTES; }

h3attn_status h3attn_forward_static(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                                    int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                    const h3attn_bf16_out* out, void* stream) {
  const h3attn_status fit = static_fit(B, Tq, Tkv, H, D);
  if (fit != H3ATTN_OK) return fit;
  void* ws = nullptr;
  const h3attn_status st = static_workspace(&ws);
  if (st != H3ATTN_OK) return st;
  return h3attn_forward_ex(q, k, v, B, Tq, Tkv, H, D, softmax_scale, out, ws, (size_t)H3ATTN_STATIC_WS_BYTES,
                           stream);
}

h3attn_status h3attn_static_check_status(void* stream) {
  void* ws = nullptr;
  const h3attn_status st = static_workspace(&ws);
  if (st != H3ATTN_OK) return st;
  return h3attn_check_status(ws, stream);
}

h3attn_status h3attn_debug_static_attend_timeout(int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                                 const h3attn_bf16_out* out, uint64_t wait_limit_ns,
                                                 void* stream) {
  const h3attn_status fit = static_fit(B, Tq, Tkv, H, D);
  if (fit != H3ATTN_OK) return fit;
  void* ws = nullptr;
  const h3attn_status st = static_workspace(&ws);
  if (st != H3ATTN_OK) return st;
  return h3attn_debug_attend_timeout(ws, (size_t)H3ATTN_STATIC_WS_BYTES, B, Tq, Tkv, H, D, softmax_scale, out,
                                     wait_limit_ns, stream);
}

}  // extern "C"
