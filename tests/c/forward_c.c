/*
 * The whole layer from plain C with the CUDA runtime and no Python: reads
 * the shape and the layer's inputs (fp32 or bf16 raw files written by
 * tests/test_gpu_c_forward.py), allocates device memory with cudaMalloc,
 * packs the weights, zero-fills the workspace, runs moe_forward on its own
 * stream, checks the device status and writes y.  Usage:
 *   forward_c DIR T d E k f ep dtype(0 = fp32, 1 = bf16)
 * reading DIR/{x,wr,wg,wu,wd}.bin and writing DIR/y.bin.  Prints "ok".
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "moe.h"

static void* read_file(const char* dir, const char* name, size_t bytes) {
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

static void* to_device(const void* host, size_t bytes) {
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess) return NULL;
  if (cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
  return d;
}

#define FAIL(msg)                   \
  do {                              \
    printf("FAIL: %s\n", msg);      \
    return 1;                       \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 9) FAIL("usage: forward_c DIR T d E k f ep dtype");
  const char* dir = argv[1];
  moe_shape s;
  s.T = atoll(argv[2]);
  s.d = atoi(argv[3]);
  s.E = atoi(argv[4]);
  s.k = atoi(argv[5]);
  s.f = atoi(argv[6]);
  s.ep = atoi(argv[7]);
  s.dtype = atoi(argv[8]) ? MOE_BF16 : MOE_F32;
  const size_t es = s.dtype == MOE_BF16 ? 2 : 4;
  const size_t nx = (size_t)s.T * s.d, nr = (size_t)s.d * s.E, ne = (size_t)s.E * s.d * s.f;
  void* hx = read_file(dir, "x.bin", nx * es);
  void* hr = read_file(dir, "wr.bin", nr * es);
  void* hg = read_file(dir, "wg.bin", ne * es);
  void* hu = read_file(dir, "wu.bin", ne * es);
  void* hd = read_file(dir, "wd.bin", ne * es);
  if (!hx || !hr || !hg || !hu || !hd) FAIL("reading inputs");
  void *x = to_device(hx, nx * es), *wr = to_device(hr, nr * es), *wg = to_device(hg, ne * es),
       *wu = to_device(hu, ne * es), *wd = to_device(hd, ne * es);
  if (!x || !wr || !wg || !wu || !wd) FAIL("device inputs");

  cudaStream_t st;
  if (cudaStreamCreate(&st) != cudaSuccess) FAIL("stream");
  size_t pbytes = 0, wbytes = 0;
  if (moe_packed_weights_size(&s, &pbytes) != MOE_OK) FAIL("packed size");
  if (moe_forward_workspace_size(&s, &wbytes) != MOE_OK) FAIL("workspace size");
  void *packed = NULL, *ws = NULL, *y = NULL;
  if (cudaMalloc(&packed, pbytes) != cudaSuccess || cudaMalloc(&ws, wbytes) != cudaSuccess ||
      cudaMalloc(&y, nx * es) != cudaSuccess)
    FAIL("device buffers");
  if (moe_workspace_init(ws, wbytes, st) != MOE_OK) FAIL("workspace init");
  moe_status r = moe_pack_weights(&s, wr, wg, wu, wd, packed, pbytes, st);
  if (r != MOE_OK) FAIL(moe_status_string(r));
  r = moe_forward(&s, x, packed, NULL, NULL, y, NULL, ws, wbytes, st);
  if (r != MOE_OK) FAIL(moe_status_string(r));
  moe_status dev = MOE_OK;
  if (moe_get_device_status(ws, st, &dev) != MOE_OK || dev != MOE_OK) FAIL("device status");
  void* hy = malloc(nx * es);
  if (!hy || cudaMemcpy(hy, y, nx * es, cudaMemcpyDeviceToHost) != cudaSuccess) FAIL("copy y");
  char path[4096];
  snprintf(path, sizeof(path), "%s/y.bin", dir);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(hy, 1, nx * es, f) != nx * es) FAIL("writing y");
  fclose(f);
  cudaFree(x);
  cudaFree(wr);
  cudaFree(wg);
  cudaFree(wu);
  cudaFree(wd);
  cudaFree(packed);
  cudaFree(ws);
  cudaFree(y);
  cudaStreamDestroy(st);
  free(hx);
  free(hr);
  free(hg);
  free(hu);
  free(hd);
  free(hy);
  printf("ok\n");
  return 0;
}
