/* kl_fwd_bwd called from plain C with the CUDA runtime only (no PyTorch),
 * built and run by tests/test_c_caller_gpu.py.
 *
 *   c_fwd_bwd DIR N d V K T
 *
 * Reads the bf16 top-K problem from raw little-endian files in DIR:
 *   H.bin [N, d] bf16, W.bin [V, d] bf16, idx.bin [N, K] int32,
 *   val.bin [N, K] float32, lse.bin [N] float32;
 * runs kl_fwd_bwd (partial-mass mode, grad_loss 1) on the legacy default
 * stream and writes loss.bin (1 float32), dH.bin [N, d] bf16, dW.bin [V, d]
 * float32 and status.txt (the device status).  Exits non-zero on any error. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "chunked_kl.h"

static int fail(const char* what, const char* detail) {
  fprintf(stderr, "c_fwd_bwd: %s: %s\n", what, detail);
  return 1;
}

/* Reads exactly n bytes of DIR/name into a new device buffer. */
static int upload(const char* dir, const char* name, size_t n, void** dev) {
  char path[1024];
  void* host = malloc(n > 0 ? n : 1);
  FILE* f;
  int rc = 0;
  snprintf(path, sizeof path, "%s/%s", dir, name);
  f = fopen(path, "rb");
  if (host == NULL || f == NULL || fread(host, 1, n, f) != n) rc = fail("read", path);
  if (f != NULL) fclose(f);
  if (rc == 0 && cudaMalloc(dev, n > 0 ? n : 1) != cudaSuccess) rc = fail("cudaMalloc", name);
  if (rc == 0 && cudaMemcpy(*dev, host, n, cudaMemcpyHostToDevice) != cudaSuccess)
    rc = fail("cudaMemcpy", name);
  free(host);
  return rc;
}

/* Writes n bytes of a device buffer to DIR/name. */
static int download(const char* dir, const char* name, const void* dev, size_t n) {
  char path[1024];
  void* host = malloc(n > 0 ? n : 1);
  FILE* f;
  int rc = 0;
  snprintf(path, sizeof path, "%s/%s", dir, name);
  if (host == NULL || cudaMemcpy(host, dev, n, cudaMemcpyDeviceToHost) != cudaSuccess)
    rc = fail("cudaMemcpy", name);
  f = rc == 0 ? fopen(path, "wb") : NULL;
  if (rc == 0 && (f == NULL || fwrite(host, 1, n, f) != n)) rc = fail("write", path);
  if (f != NULL) fclose(f);
  free(host);
  return rc;
}

int main(int argc, char** argv) {
  kl_problem p;
  const char* dir;
  void *H = NULL, *W = NULL, *idx = NULL, *val = NULL, *lse = NULL;
  void *ws = NULL, *dH = NULL, *dW = NULL, *loss = NULL;
  size_t ws_bytes;
  int rc, status;
  FILE* f;
  char path[1024];

  if (argc != 7) return fail("usage", "c_fwd_bwd DIR N d V K T");
  dir = argv[1];
  memset(&p, 0, sizeof p);
  p.N = atoll(argv[2]);
  p.d = atoll(argv[3]);
  p.V = atoll(argv[4]);
  p.K = atoi(argv[5]);
  p.T = (float)atof(argv[6]);
  p.dtype = KL_DTYPE_BF16;
  p.teacher = KL_TEACHER_TOPK;

  if (upload(dir, "H.bin", (size_t)(p.N * p.d * 2), &H) ||
      upload(dir, "W.bin", (size_t)(p.V * p.d * 2), &W) ||
      upload(dir, "idx.bin", (size_t)(p.N * p.K * 4), &idx) ||
      upload(dir, "val.bin", (size_t)(p.N * p.K * 4), &val) ||
      upload(dir, "lse.bin", (size_t)(p.N * 4), &lse))
    return 1;
  p.H = H;
  p.W = W;
  p.topk_idx = (const int32_t*)idx;
  p.topk_logit = (const float*)val;
  p.teacher_lse = (const float*)lse;

  ws_bytes = kl_workspace_bytes(&p, KL_ENTRY_FWD_BWD);
  if (ws_bytes == 0) return fail("kl_workspace_bytes", "invalid problem");
  if (cudaMalloc(&ws, ws_bytes) != cudaSuccess ||
      cudaMalloc(&dH, (size_t)(p.N * p.d * 2)) != cudaSuccess ||
      cudaMalloc(&dW, (size_t)(p.V * p.d * 4)) != cudaSuccess ||
      cudaMalloc(&loss, 4) != cudaSuccess)
    return fail("cudaMalloc", "outputs");

  rc = kl_fwd_bwd(&p, ws, ws_bytes, 1.0f, (float*)loss, NULL, dH, (float*)dW, 0, NULL);
  if (rc != KL_OK) return fail("kl_fwd_bwd", kl_status_string(rc));
  status = kl_status(ws, NULL); /* synchronises the stream */

  snprintf(path, sizeof path, "%s/status.txt", dir);
  f = fopen(path, "w");
  if (f == NULL) return fail("write", path);
  fprintf(f, "%d\n", status);
  fclose(f);
  if (download(dir, "loss.bin", loss, 4) || download(dir, "dH.bin", dH, (size_t)(p.N * p.d * 2)) ||
      download(dir, "dW.bin", dW, (size_t)(p.V * p.d * 4)))
    return 1;

  cudaFree(H);
  cudaFree(W);
  cudaFree(idx);
  cudaFree(val);
  cudaFree(lse);
  cudaFree(ws);
  cudaFree(dH);
  cudaFree(dW);
  cudaFree(loss);
  return status == KL_OK ? 0 : 2;
}
