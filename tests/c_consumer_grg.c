/* A plain C program driving the block through the C ABI on the GPU: device
 * memory from cudaMalloc, the legacy default stream, no Python and no torch.
 * Inputs come from a fixed linear congruential generator; inputs and outputs
 * are written to the file named by argv[1] for the test to compare with the
 * Python binding.  Usage: c_consumer_grg OUT_FILE */
#include <cuda_runtime_api.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "coda.h"

enum { M = 512, K = 512, D = 512, F = 1024, N = 2 * F };

static uint64_t lcg = 12345u;
static float next_uniform(void) { /* in [-1, 1) */
  lcg = lcg * 6364136223846793005ull + 1442695040888963407ull;
  return (float)((double)(lcg >> 11) / 9007199254740992.0) * 2.0f - 1.0f;
}
static uint16_t to_bf16(float x) { /* round to nearest even; inputs are finite */
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static uint16_t* host_bf16(size_t n, float scale, float offset) {
  uint16_t* h = (uint16_t*)malloc(n * 2);
  for (size_t i = 0; i < n; ++i) h[i] = to_bf16(offset + scale * next_uniform());
  return h;
}
static void* dev_copy(const void* h, size_t bytes) {
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess) exit(3);
  if (h && cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) exit(3);
  return d;
}
static void dump(FILE* f, const void* d, size_t bytes) {
  void* h = malloc(bytes);
  if (cudaMemcpy(h, d, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) exit(4);
  fwrite(h, 1, bytes, f);
  free(h);
}

int main(int argc, char** argv) {
  if (argc != 2) return 2;
  const size_t sX = (size_t)M * K * 2, sR = (size_t)M * D * 2, sW1 = (size_t)D * K * 2, sW2 = (size_t)N * D * 2;
  const size_t sG = (size_t)D * 2, sDY = (size_t)M * F * 2;
  uint16_t *X = host_bf16(sX / 2, 1.7f, 0.f), *R = host_bf16(sR / 2, 1.7f, 0.f);
  uint16_t *W1 = host_bf16(sW1 / 2, 1.7f / sqrtf((float)K), 0.f), *W2 = host_bf16(sW2 / 2, 1.7f / sqrtf((float)D), 0.f);
  uint16_t *g = host_bf16(sG / 2, 0.17f, 1.f), *dY = host_bf16(sDY / 2, 1.7f, 0.f);
  void *dX_in = dev_copy(X, sX), *dR_in = dev_copy(R, sR), *dW1_in = dev_copy(W1, sW1), *dW2_in = dev_copy(W2, sW2);
  void *dg_in = dev_copy(g, sG), *ddY = dev_copy(dY, sDY);
  void *H = dev_copy(NULL, sR), *r = dev_copy(NULL, (size_t)M * 4), *Y = dev_copy(NULL, sDY);
  void *AB = dev_copy(NULL, (size_t)M * N * 2);
  void *dX = dev_copy(NULL, sX), *dR = dev_copy(NULL, sR), *dW1 = dev_copy(NULL, sW1), *dW2 = dev_copy(NULL, sW2);
  void* dgrad = dev_copy(NULL, (size_t)D * 4);
  size_t wsb = coda_grg_fwd_workspace_bytes(M, K, D, N, 0);
  const size_t wsb2 = coda_grg_bwd_workspace_bytes(M, K, D, N);
  if (wsb2 > wsb) wsb = wsb2;
  void* ws = dev_copy(NULL, wsb);
  if (coda_status_clear(ws, NULL) != CODA_OK) return 5;
  coda_status st = coda_grg_fwd(dX_in, dW1_in, dR_in, dg_in, dW2_in, NULL, H, (float*)r, Y, AB, M, K, D, N, 1e-6f, ws,
                                wsb, NULL);
  if (st != CODA_OK) { fprintf(stderr, "fwd: %s\n", coda_status_string(st)); return 6; }
  st = coda_grg_bwd(ddY, NULL, dX_in, dW1_in, H, (const float*)r, AB, dg_in, dW2_in, dX, dR, dW1, dW2, (float*)dgrad,
                    M, K, D, N, ws, wsb, NULL);
  if (st != CODA_OK) { fprintf(stderr, "bwd: %s\n", coda_status_string(st)); return 7; }
  uint32_t detail = 0;
  st = coda_status_query(ws, NULL, &detail);
  if (st != CODA_OK) { fprintf(stderr, "device: %s %u\n", coda_status_string(st), detail); return 8; }
  FILE* f = fopen(argv[1], "wb");
  if (!f) return 9;
  fwrite(X, 1, sX, f); fwrite(R, 1, sR, f); fwrite(W1, 1, sW1, f); fwrite(W2, 1, sW2, f);
  fwrite(g, 1, sG, f); fwrite(dY, 1, sDY, f);
  dump(f, H, sR); dump(f, r, (size_t)M * 4); dump(f, Y, sDY); dump(f, AB, (size_t)M * N * 2);
  dump(f, dX, sX); dump(f, dR, sR); dump(f, dW1, sW1); dump(f, dW2, sW2); dump(f, dgrad, (size_t)D * 4);
  fclose(f);
  printf("ok\n");
  return 0;
}
