/*
 * A plain C caller of the layer, through include/moe.h alone (no Python, no
 * C++): reads bf16 inputs from files, runs moe_layer_fwd on the GPU, writes
 * y, top_experts and routing weights back to files.
 *
 *   layer_fwd N H E K F in_dir out_dir
 *     in_dir:  x.bin [N,H] W_r.bin [H,E] W1.bin [E,H,F] W3.bin [E,H,F] W2.bin [E,F,H] (bf16)
 *     out_dir: y.bin [N,H] bf16, top.bin [N,K] int32, weights.bin [N,K] float32
 * Exit status 0 on success; a message on stderr otherwise.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe.h"

static int fail(const char* what, int code) {
  fprintf(stderr, "layer_fwd: %s failed (%d)\n", what, code);
  return 1;
}

static void* load_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  FILE* f = fopen(path, "rb");
  if (!f) return NULL;
  void* buf = malloc(bytes);
  size_t got = buf ? fread(buf, 1, bytes, f) : 0;
  fclose(f);
  if (got != bytes) {
    free(buf);
    return NULL;
  }
  return buf;
}

static int save_file(const char* dir, const char* name, const void* buf, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof(path), "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f) return 1;
  size_t put = fwrite(buf, 1, bytes, f);
  fclose(f);
  return put == bytes ? 0 : 1;
}

static void* to_device(const void* host, size_t bytes) {
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess) return NULL;
  if (cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
  return d;
}

int main(int argc, char** argv) {
  if (argc != 8) {
    fprintf(stderr, "usage: layer_fwd N H E K F in_dir out_dir\n");
    return 2;
  }
  const int32_t N = atoi(argv[1]), H = atoi(argv[2]), E = atoi(argv[3]), K = atoi(argv[4]), F = atoi(argv[5]);
  const char* in_dir = argv[6];
  const char* out_dir = argv[7];
  const size_t b = 2; /* bf16 */
  const size_t sx = (size_t)N * H * b, swr = (size_t)H * E * b, sw13 = (size_t)E * H * F * b,
               sw2 = (size_t)E * F * H * b;
  void* hx = load_file(in_dir, "x.bin", sx);
  void* hwr = load_file(in_dir, "W_r.bin", swr);
  void* hw1 = load_file(in_dir, "W1.bin", sw13);
  void* hw3 = load_file(in_dir, "W3.bin", sw13);
  void* hw2 = load_file(in_dir, "W2.bin", sw2);
  if (!hx || !hwr || !hw1 || !hw3 || !hw2) return fail("reading the inputs", 0);

  void* x = to_device(hx, sx);
  void* W_r = to_device(hwr, swr);
  void* W1 = to_device(hw1, sw13);
  void* W3 = to_device(hw3, sw13);
  void* W2 = to_device(hw2, sw2);
  void *y = NULL, *top = NULL, *w = NULL, *idx = NULL, *bins = NULL, *pbins = NULL, *ws = NULL;
  const size_t ws_bytes = moe_workspace_size(N, H, E, K, F, MOE_BF16, 0);
  if (ws_bytes == 0) return fail("moe_workspace_size", 0);
  if (!x || !W_r || !W1 || !W3 || !W2 || cudaMalloc(&y, sx) != cudaSuccess ||
      cudaMalloc(&top, (size_t)N * K * 4) != cudaSuccess || cudaMalloc(&w, (size_t)N * K * 4) != cudaSuccess ||
      cudaMalloc(&idx, (size_t)N * K * 4) != cudaSuccess || cudaMalloc(&bins, (size_t)E * 4) != cudaSuccess ||
      cudaMalloc(&pbins, (size_t)E * 4) != cudaSuccess || cudaMalloc(&ws, ws_bytes) != cudaSuccess)
    return fail("cudaMalloc", 0);

  cudaStream_t stream;
  if (cudaStreamCreate(&stream) != cudaSuccess) return fail("cudaStreamCreate", 0);
  moe_status st = moe_workspace_init(ws, ws_bytes, stream);
  if (st != MOE_OK) return fail("moe_workspace_init", st);
  st = moe_layer_fwd(x, W_r, W1, W3, W2, N, H, E, K, F, MOE_BF16, 0, 0, 0.0f, NULL, y, (int32_t*)top, (float*)w,
                     (int32_t*)idx, (int32_t*)bins, (int32_t*)pbins, ws, ws_bytes, stream);
  if (st != MOE_OK) return fail("moe_layer_fwd", st);
  int32_t dev_status = -1;
  st = moe_get_device_status(ws, &dev_status, stream);
  if (st != MOE_OK || dev_status != 0) return fail("device status", dev_status);

  void* hy = malloc(sx);
  void* htop = malloc((size_t)N * K * 4);
  void* hw = malloc((size_t)N * K * 4);
  if (!hy || !htop || !hw || cudaMemcpy(hy, y, sx, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(htop, top, (size_t)N * K * 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(hw, w, (size_t)N * K * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail("copying the outputs back", 0);
  if (save_file(out_dir, "y.bin", hy, sx) || save_file(out_dir, "top.bin", htop, (size_t)N * K * 4) ||
      save_file(out_dir, "weights.bin", hw, (size_t)N * K * 4))
    return fail("writing the outputs", 0);
  cudaStreamDestroy(stream);
  return 0;
}
