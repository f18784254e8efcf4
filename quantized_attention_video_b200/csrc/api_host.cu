// h3attn_forward_host: the forward pass from and to host memory, pipelined by head
// groups so that host<->device copies overlap the kernels.
//
// Heads are independent problems (K smoothing, every scale and the attention are per
// (b, h)), so running the forward pass on groups of heads gives the same bytes as one
// call on all heads.  Group g is uploaded on one stream, computed on the caller's
// stream and downloaded on a third; two device slots (staging + workspace) let the
// upload of group g+1 and the download of group g-1 run while group g computes.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "h3attn_internal.h"

using namespace h3;

namespace {

constexpr size_t kRowBytes = (size_t)kD * 2;  // one head of one token, BF16

size_t align1k(size_t x) { return (x + 1023) & ~size_t(1023); }

// Byte offsets of one slot's pieces: staged Q, K, V and output ([B, T, g, D],
// compact), then the workspace of a g-head call.
struct Slot {
  size_t q, k, v, o, ws, ws_bytes, bytes;
};

bool make_slot(int B, int Tq, int Tkv, int g, Slot* s) {
  const size_t wsb = h3attn_workspace_bytes(B, Tq, Tkv, g, kD);
  if (wsb == 0) return false;
  const size_t qb = align1k((size_t)B * Tq * g * kRowBytes), kvb = align1k((size_t)B * Tkv * g * kRowBytes);
  s->q = 0;
  s->k = s->q + qb;
  s->v = s->k + kvb;
  s->o = s->v + kvb;
  s->ws = s->o + qb;
  s->ws_bytes = align1k(wsb);
  s->bytes = s->ws + s->ws_bytes;
  return true;
}

// Heads [h0, h0 + gn) of a strided [B, T, H, D] host view <-> compact [B, T, gn, D]
// device staging.  One 2D copy per batch item when the heads of a token are adjacent,
// else one per (batch item, head).
cudaError_t copy_heads(char* dev, const char* host, int64_t sb, int64_t st, int64_t sh, int B, int T, int h0,
                       int gn, bool to_device, cudaStream_t s) {
  const size_t dpitch = (size_t)gn * kRowBytes, hpitch = (size_t)st * 2;
  for (int b = 0; b < B; ++b) {
    char* d = dev + (size_t)b * T * dpitch;
    const char* h = host + 2 * ((size_t)b * sb + (size_t)h0 * sh);
    const int pieces = sh == kD ? 1 : gn;
    const size_t width = sh == kD ? dpitch : kRowBytes;
    for (int p = 0; p < pieces; ++p) {
      char* dp = d + (size_t)p * kRowBytes;
      char* hp = const_cast<char*>(h) + 2 * (size_t)p * sh;
      const cudaError_t e = to_device
          ? cudaMemcpy2DAsync(dp, dpitch, hp, hpitch, width, (size_t)T, cudaMemcpyHostToDevice, s)
          : cudaMemcpy2DAsync(hp, hpitch, dp, dpitch, width, (size_t)T, cudaMemcpyDeviceToHost, s);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

// The head groups of a call: heads_per_group each, except that with more than
// 2 * heads_per_group heads the first and the last group take heads_per_group / 2 (at
// least 1).  Only the first group's upload and the last group's download are not
// overlapped by kernels, so halving those two groups shortens the call.
int group_starts(int H, int g, int* starts) {  // starts[0 .. n] with starts[n] = H; returns n
  int n = 0, h = 0;
  const int half = g / 2 > 0 ? g / 2 : 1;
  const bool halved_ends = g >= 2 && H > 2 * g;
  if (halved_ends) {
    starts[n++] = 0;
    h = half;
  }
  const int end = halved_ends ? H - half : H;
  while (h < end) {
    starts[n++] = h;
    h += std::min(g, end - h);
  }
  if (halved_ends) starts[n++] = end;
  starts[n] = H;
  return n;
}

}  // namespace

extern "C" {

int h3attn_forward_host_groups(int H, int heads_per_group, int* group_start) {
  if (H < 1 || heads_per_group < 1 || heads_per_group > H) return 0;
  int tmp[4097];
  if (H > 4096) return 0;
  const int n = group_starts(H, heads_per_group, tmp);
  if (group_start != nullptr)
    for (int i = 0; i <= n; ++i) group_start[i] = tmp[i];
  return n;
}

size_t h3attn_forward_host_bytes(int B, int Tq, int Tkv, int H, int D, int heads_per_group) {
  if (h3attn_workspace_bytes(B, Tq, Tkv, H, D) == 0) return 0;
  if (heads_per_group < 1 || heads_per_group > H) return 0;
  Slot s;
  if (!make_slot(B, Tq, Tkv, heads_per_group, &s)) return 0;
  return 2 * s.bytes;
}

}  // extern "C"

namespace {

// The pipeline of h3attn_forward_host.  fail_group >= 0 (test hook): that group's
// attention runs through h3attn_debug_attend_timeout with waits bounded by
// wait_limit_ns, so it records a device-side timeout in its slot's status word.
h3attn_status forward_host_impl(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                                int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                const h3attn_bf16_out* out, int heads_per_group, void* dev_buf, size_t dev_bytes,
                                void* stream, int fail_group, uint64_t wait_limit_ns) {
  const size_t need = h3attn_forward_host_bytes(B, Tq, Tkv, H, D, heads_per_group);
  if (need == 0) return D != kD ? H3ATTN_ERR_UNSUPPORTED : H3ATTN_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return H3ATTN_ERR_INVALID_ARG;
  for (const h3attn_bf16_view* hv : {q, k, v}) {
    const h3attn_status st = check_strides(hv->data, hv->stride_b, hv->stride_t, hv->stride_h);
    if (st != H3ATTN_OK) return st;
  }
  {
    const h3attn_status st = check_strides(out->data, out->stride_b, out->stride_t, out->stride_h);
    if (st != H3ATTN_OK) return st;
  }
  if (!(softmax_scale > 0.0f) || !(softmax_scale < INFINITY)) return H3ATTN_ERR_INVALID_ARG;
  if (dev_buf == nullptr || reinterpret_cast<uintptr_t>(dev_buf) % 1024 != 0 || dev_bytes < need)
    return H3ATTN_ERR_WORKSPACE;

  const int g = heads_per_group;
  if (H > 4096) return H3ATTN_ERR_INVALID_ARG;
  int starts[4097];
  const int ngroups = group_starts(H, g, starts);
  Slot sl{};
  if (!make_slot(B, Tq, Tkv, g, &sl)) return H3ATTN_ERR_INVALID_ARG;
  char* base = static_cast<char*>(dev_buf);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // Per-call copy streams and events: no state survives the call (the runtime
  // releases them once their pending work has completed).
  cudaStream_t up = nullptr, dn = nullptr;
  cudaEvent_t ev[8] = {};
  const auto release = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
    if (up) cudaStreamDestroy(up);
    if (dn) cudaStreamDestroy(dn);
  };
  if (cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&dn, cudaStreamNonBlocking) != cudaSuccess) {
    release();
    return H3ATTN_ERR_CUDA;
  }
  for (cudaEvent_t& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      release();
      return H3ATTN_ERR_CUDA;
    }
  cudaEvent_t& ev_start = ev[0];
  cudaEvent_t* ev_up = ev + 1;    // [slot] inputs staged
  cudaEvent_t* ev_comp = ev + 3;  // [slot] forward pass done (inputs free, output ready)
  cudaEvent_t* ev_dn = ev + 5;    // [slot] output downloaded (output staging free)
  cudaEvent_t& ev_end = ev[7];

  h3attn_status result = H3ATTN_OK;
  bool ok = cudaEventRecord(ev_start, cs) == cudaSuccess && cudaStreamWaitEvent(up, ev_start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(dn, ev_start, 0) == cudaSuccess;
  for (int gi = 0; ok && gi < ngroups; ++gi) {
    const int slot = gi & 1, h0 = starts[gi], gn = starts[gi + 1] - starts[gi];
    char* sb = base + (size_t)slot * sl.bytes;
    // upload: the slot's inputs are free once the forward pass of group gi-2 is done
    if (gi >= 2) ok = ok && cudaStreamWaitEvent(up, ev_comp[slot], 0) == cudaSuccess;
    ok = ok && copy_heads(sb + sl.q, static_cast<const char*>(q->data), q->stride_b, q->stride_t, q->stride_h, B,
                          Tq, h0, gn, true, up) == cudaSuccess;
    ok = ok && copy_heads(sb + sl.k, static_cast<const char*>(k->data), k->stride_b, k->stride_t, k->stride_h, B,
                          Tkv, h0, gn, true, up) == cudaSuccess;
    ok = ok && copy_heads(sb + sl.v, static_cast<const char*>(v->data), v->stride_b, v->stride_t, v->stride_h, B,
                          Tkv, h0, gn, true, up) == cudaSuccess;
    ok = ok && cudaEventRecord(ev_up[slot], up) == cudaSuccess;
    // forward pass on the caller's stream: inputs staged, output staging downloaded
    ok = ok && cudaStreamWaitEvent(cs, ev_up[slot], 0) == cudaSuccess;
    if (gi >= 2) ok = ok && cudaStreamWaitEvent(cs, ev_dn[slot], 0) == cudaSuccess;
    if (!ok) break;
    const int64_t tq = (int64_t)gn * kD, tk = (int64_t)gn * kD;
    const h3attn_bf16_view dq = {sb + sl.q, (int64_t)Tq * tq, tq, kD};
    const h3attn_bf16_view dk = {sb + sl.k, (int64_t)Tkv * tk, tk, kD};
    const h3attn_bf16_view dv = {sb + sl.v, (int64_t)Tkv * tk, tk, kD};
    const h3attn_bf16_out dout = {sb + sl.o, (int64_t)Tq * tq, tq, kD};
    if (gi == fail_group) {
      result = h3attn_quantize_qkv(&dq, &dk, &dv, B, Tq, Tkv, gn, D, sb + sl.ws, sl.ws_bytes, cs);
      if (result == H3ATTN_OK)
        result = h3attn_debug_attend_timeout(sb + sl.ws, sl.ws_bytes, B, Tq, Tkv, gn, D, softmax_scale, &dout,
                                             wait_limit_ns, cs);
    } else {
      result = h3attn_forward_ex(&dq, &dk, &dv, B, Tq, Tkv, gn, D, softmax_scale, &dout, sb + sl.ws, sl.ws_bytes,
                                 cs);
    }
    if (result != H3ATTN_OK) break;
    ok = cudaEventRecord(ev_comp[slot], cs) == cudaSuccess;
    // download
    ok = ok && cudaStreamWaitEvent(dn, ev_comp[slot], 0) == cudaSuccess;
    ok = ok && copy_heads(sb + sl.o, static_cast<const char*>(out->data), out->stride_b, out->stride_t,
                          out->stride_h, B, Tq, h0, gn, false, dn) == cudaSuccess;
    ok = ok && cudaEventRecord(ev_dn[slot], dn) == cudaSuccess;
  }
  // the caller's stream covers every copy of this call (also after a failure)
  const bool joined = cudaEventRecord(ev_end, dn) == cudaSuccess && cudaStreamWaitEvent(cs, ev_end, 0) == cudaSuccess &&
                      cudaEventRecord(ev_end, up) == cudaSuccess && cudaStreamWaitEvent(cs, ev_end, 0) == cudaSuccess;
  release();
  if (result != H3ATTN_OK) return result;
  return ok && joined ? H3ATTN_OK : H3ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

h3attn_status h3attn_forward_host(const h3attn_bf16_view* q, const h3attn_bf16_view* k, const h3attn_bf16_view* v,
                                  int B, int Tq, int Tkv, int H, int D, float softmax_scale,
                                  const h3attn_bf16_out* out, int heads_per_group, void* dev_buf,
                                  size_t dev_bytes, void* stream) {
  return forward_host_impl(q, k, v, B, Tq, Tkv, H, D, softmax_scale, out, heads_per_group, dev_buf, dev_bytes,
                           stream, -1, 0);
}

h3attn_status h3attn_debug_forward_host_timeout(const h3attn_bf16_view* q, const h3attn_bf16_view* k,
                                                const h3attn_bf16_view* v, int B, int Tq, int Tkv, int H, int D,
                                                float softmax_scale, const h3attn_bf16_out* out,
                                                int heads_per_group, void* dev_buf, size_t dev_bytes,
                                                int fail_group, uint64_t wait_limit_ns, void* stream) {
  if (fail_group < 0 || fail_group >= h3attn_forward_host_groups(H, heads_per_group, nullptr))
    return H3ATTN_ERR_INVALID_ARG;
  return forward_host_impl(q, k, v, B, Tq, Tkv, H, D, softmax_scale, out, heads_per_group, dev_buf, dev_bytes,
                           stream, fail_group, wait_limit_ns);
}

h3attn_status h3attn_forward_host_check_status(void* dev_buf, int B, int Tq, int Tkv, int H, int D,
                                               int heads_per_group, void* stream) {
  if (h3attn_forward_host_bytes(B, Tq, Tkv, H, D, heads_per_group) == 0) return H3ATTN_ERR_INVALID_ARG;
  if (dev_buf == nullptr || reinterpret_cast<uintptr_t>(dev_buf) % 1024 != 0) return H3ATTN_ERR_WORKSPACE;
  Slot sl{};
  if (!make_slot(B, Tq, Tkv, heads_per_group, &sl)) return H3ATTN_ERR_INVALID_ARG;
  h3attn_status first = H3ATTN_OK;
  const int used = h3attn_forward_host_groups(H, heads_per_group, nullptr) >= 2 ? 2 : 1;  // an unused slot holds no status
  for (int slot = 0; slot < used; ++slot) {
    const h3attn_status st = h3attn_check_status(static_cast<char*>(dev_buf) + slot * sl.bytes + sl.ws, stream);
    if (first == H3ATTN_OK) first = st;
  }
  return first;
}

}  // extern "C"
