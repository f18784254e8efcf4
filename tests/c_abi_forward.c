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

#include <cuda_runtime.h>

#include "h3attn.h"

static int read_all(FILE* f, void* p, size_t n) { return fread(p, 1, n, f) == n; }

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s input.bin output.bin\n", argv[0]);
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
  if (!host || !read_all(in, host, 2 * (nq + 2 * nkv))) return 1;
  fclose(in);

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
  if (cudaMemcpy(host, dout, 2 * nq, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  FILE* o = fopen(argv[2], "wb");
  if (!o || fwrite(host, 2, nq, o) != nq) return 1;
  fclose(o);
  cudaFree(dq);
  cudaFree(dk);
  cudaFree(dv);
  cudaFree(dout);
  cudaFree(ws);
  free(host);
  printf("ok: B=%d Tq=%d Tkv=%d H=%d, library version %d\n", B, Tq, Tkv, H, h3attn_version());
  return 0;
}
