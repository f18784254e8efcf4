/* A plain C caller of libh3attn.so: no Python, no PyTorch.  It reads one BF16 Q/K/V
 * problem from a file, runs h3attn_forward_ex on device buffers it allocates itself,
 * checks the device status and writes the BF16 output.  tests/test_c_abi.py builds it
 * (CPU) and runs it against the Python binding's result on the same inputs (GPU).
 *
 * Input file: int32 B, Tq, Tkv, H; float softmax_scale; then Q [B,Tq,H,128], K and V
 * [B,Tkv,H,128] as BF16 bit patterns, dense.  Output file: the [B,Tq,H,128] BF16 result.
 * Exit status 0 on success, 1 on an I/O or CUDA error, 2 + the h3attn status otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "h3attn.h"

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n; }

/* One forward pass of the problem in host[] (Q, K, V dense) into out_host[]: allocates the
 * device buffers, uploads, runs, checks the device status, downloads and frees. */
static int run_once(const uint16_t* host, int B, int Tq, int Tkv, int H, float scale, uint16_t* out_host) {
  const int D = H3ATTN_HEAD_DIM;
  const size_t nq = (size_t)B * Tq * H * D, nkv = (size_t)B * Tkv * H * D;
  const size_t ws_bytes = h3attn_workspace_bytes(B, Tq, Tkv, H, D);
  if (ws_bytes == 0) return 2 + H3ATTN_ERR_INVALID_ARG;
  void *dq, *dk, *dv, *dout, *ws;
  if (cudaMalloc(&dq, 2 * nq) != cudaSuccess || cudaMalloc(&dk, 2 * nkv) != cudaSuccess ||
      cudaMalloc(&dv, 2 * nkv) != cudaSuccess || cudaMalloc(&dout, 2 * nq) != cudaSuccess ||
      cudaMalloc(&ws, ws_bytes) != cudaSuccess)
    return 1;
  if (cudaMemcpy(dq, host, 2 * nq, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dk, host + nq, 2 * nkv, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dv, host + nq + nkv, 2 * nkv, cudaMemcpyHostToDevice) != cudaSuccess)
    return 1;

  /* dense [B, T, H, 128] views: strides in elements */
  const h3attn_bf16_view q = {dq, (int64_t)Tq * H * D, (int64_t)H * D, D};
  const h3attn_bf16_view k = {dk, (int64_t)Tkv * H * D, (int64_t)H * D, D};
  const h3attn_bf16_view v = {dv, (int64_t)Tkv * H * D, (int64_t)H * D, D};
  const h3attn_bf16_out out = {dout, (int64_t)Tq * H * D, (int64_t)H * D, D};
  h3attn_status st = h3attn_forward_ex(&q, &k, &v, B, Tq, Tkv, H, D, scale, &out, ws, ws_bytes, NULL);
  if (st != H3ATTN_OK) {
    fprintf(stderr, "h3attn_forward_ex: %s\n", h3attn_status_string(st));
    return 2 + st;
  }
  st = h3attn_check_status(ws, NULL); /* synchronises the stream */
  if (st != H3ATTN_OK) {
    fprintf(stderr, "device status: %s\n", h3attn_status_string(st));
    return 2 + st;
  }
  if (cudaMemcpy(out_host, dout, 2 * nq, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  cudaFree(dq);
  cudaFree(dk);
  cudaFree(dv);
  cudaFree(dout);
  cudaFree(ws);
  return 0;
}

/* With a third argument "reset": after the first pass the program resets the device (which
 * destroys its context and every allocation in it) and runs the pass again in the new
 * context; the two outputs must be equal.  The library sets its kernels' shared-memory
 * attributes once per context, so this checks that it notices the new context. */
int main(int argc, char** argv) {
  if (argc != 3 && !(argc == 4 && strcmp(argv[3], "reset") == 0)) {
    fprintf(stderr, "usage: %s input.bin output.bin [reset]\n", argv[0]);
    return 1;
  }
  FILE* in = fopen(argv[1], "rb");
  if (!in) return 1;
  int32_t dims[4];
  float scale;
  if (!read_all(in, dims, sizeof dims) || !read_all(in, &scale, sizeof scale)) return 1;
  const int B = dims[0], Tq = dims[1], Tkv = dims[2], H = dims[3], D = H3ATTN_HEAD_DIM;
  const size_t nq = (size_t)B * Tq * H * D, nkv = (size_t)B * Tkv * H * D;
  uint16_t* host = (uint16_t*)malloc(2 * (nq + 2 * nkv));
  uint16_t* result = (uint16_t*)malloc(2 * nq);
  if (!host || !result || !read_all(in, host, 2 * (nq + 2 * nkv))) return 1;
  fclose(in);

  int rc = run_once(host, B, Tq, Tkv, H, scale, result);
  if (rc != 0) return rc;
  if (argc == 4) {
    uint16_t* again = (uint16_t*)malloc(2 * nq);
    if (!again) return 1;
    if (cudaDeviceReset() != cudaSuccess) return 1;
    rc = run_once(host, B, Tq, Tkv, H, scale, again);
    if (rc != 0) return rc;
    if (memcmp(again, result, 2 * nq) != 0) {
      fprintf(stderr, "the output after the device reset differs\n");
      return 1;
    }
    free(again);
  }
  FILE* o = fopen(argv[2], "wb");
  if (!o || fwrite(result, 2, nq, o) != nq) return 1;
  fclose(o);
  free(host);
  free(result);
  printf("ok: B=%d Tq=%d Tkv=%d H=%d, library version %d%s\n", B, Tq, Tkv, H, h3attn_version(),
         argc == 4 ? ", again after a device reset" : "");
  return 0;
}
