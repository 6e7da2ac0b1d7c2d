/* Plain C99 client of the C ABI in include/moe.h: no Python, no C++.
 *
 * It builds a small seeded bf16 layer (300 tokens, d = 256, 8 routed experts + 1 shared,
 * top-2, SwiGLU, capacity factor 1.25), runs the fused moe_forward, then the same layer
 * through the split calls moe_route -> moe_permute -> moe_expert_ffn -> moe_combine, and
 * checks that both give the same output bits and the same routing.  Exit status 0 on
 * success; a message and a non-zero status otherwise.
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe.h"

#define CHECK_CUDA(call)                                                     \
  do {                                                                       \
    cudaError_t e_ = (call);                                                 \
    if (e_ != cudaSuccess) {                                                 \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #call,           \
              cudaGetErrorString(e_));                                       \
      return 2;                                                              \
    }                                                                        \
  } while (0)

#define CHECK_MOE(call)                                                      \
  do {                                                                       \
    moe_status s_ = (call);                                                  \
    if (s_ != MOE_OK) {                                                      \
      fprintf(stderr, "%s:%d %s: status %d: %s\n", __FILE__, __LINE__, #call, \
              (int)s_, moe_last_error());                                    \
      return 3;                                                              \
    }                                                                        \
  } while (0)

/* 64-bit linear congruential generator (Knuth's MMIX constants). */
static uint64_t lcg_state = 12345u;
static float uniform_pm1(void) {
  lcg_state = lcg_state * 6364136223846793005ull + 1442695040888963407ull;
  return (float)((double)(lcg_state >> 11) / (double)(1ull << 53)) * 2.0f - 1.0f;
}

/* float -> bf16 with round to nearest even (finite inputs). */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static int upload_bf16(void** dev, size_t n, float scale) {
  uint16_t* h = (uint16_t*)malloc(n * sizeof(uint16_t));
  size_t i;
  if (h == NULL) return 1;
  for (i = 0; i < n; ++i) h[i] = to_bf16(scale * uniform_pm1());
  if (cudaMalloc(dev, n * sizeof(uint16_t)) != cudaSuccess ||
      cudaMemcpy(*dev, h, n * sizeof(uint16_t), cudaMemcpyHostToDevice) != cudaSuccess) {
    free(h);
    return 1;
  }
  free(h);
  return 0;
}

static void* dev_alloc(size_t bytes) {
  void* p = NULL;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return NULL;
  return p;
}

int main(void) {
  moe_config c;
  size_t ws_bytes, y_bytes, i;
  void *x = NULL, *W_g = NULL, *W_gu = NULL, *W_down = NULL, *ws = NULL;
  void *y_fused, *y_split, *xp, *ye;
  int32_t *ids_f, *ids_s, *counts, *demand, *offsets, *slot_row;
  float* gates;
  uint8_t* drop;
  moe_route_out ro;
  unsigned char *h1, *h2;
  int32_t *hi1, *hi2;
  int64_t Nk;

  memset(&c, 0, sizeof c);
  c.N = 300;
  c.d = 256;
  c.E = 8;
  c.k = 2;
  c.F = 256;
  c.n_shared = 1;
  c.score_fn = MOE_SCORE_SOFTMAX;
  c.renorm = 1;
  c.act = MOE_ACT_SWIGLU;
  c.dtype = MOE_DT_BF16;
  c.clamp = 0.0f;
  c.capacity = moe_capacity(c.N, c.k, c.E, 5, 4);
  Nk = c.N * c.k;

  if (upload_bf16(&x, (size_t)c.N * c.d, 1.0f) ||
      upload_bf16(&W_g, (size_t)c.E * c.d, 0.08f) ||
      upload_bf16(&W_gu, (size_t)(c.E + 1) * 2 * c.F * c.d, 0.08f) ||
      upload_bf16(&W_down, (size_t)(c.E + 1) * c.d * c.F, 0.08f)) {
    fprintf(stderr, "input upload failed\n");
    return 2;
  }
  ws_bytes = moe_workspace_size(&c);
  if (ws_bytes == 0) {
    fprintf(stderr, "moe_workspace_size: %s\n", moe_last_error());
    return 3;
  }
  y_bytes = (size_t)c.N * c.d * 2;
  ws = dev_alloc(ws_bytes);
  y_fused = dev_alloc(y_bytes);
  y_split = dev_alloc(y_bytes);
  xp = dev_alloc((size_t)Nk * c.d * 2);
  ye = dev_alloc((size_t)(Nk + c.N) * c.d * 2);
  ids_f = (int32_t*)dev_alloc((size_t)Nk * 4);
  ids_s = (int32_t*)dev_alloc((size_t)Nk * 4);
  gates = (float*)dev_alloc((size_t)Nk * 4);
  counts = (int32_t*)dev_alloc((size_t)c.E * 4);
  demand = (int32_t*)dev_alloc((size_t)c.E * 4);
  offsets = (int32_t*)dev_alloc((size_t)(c.E + 1) * 4);
  slot_row = (int32_t*)dev_alloc((size_t)Nk * 4);
  drop = (uint8_t*)dev_alloc((size_t)Nk);
  if (!ws || !y_fused || !y_split || !xp || !ye || !ids_f || !ids_s || !gates || !counts ||
      !demand || !offsets || !slot_row || !drop) {
    fprintf(stderr, "device allocation failed\n");
    return 2;
  }
  CHECK_MOE(moe_workspace_init(ws, NULL));

  /* the fused layer */
  memset(&ro, 0, sizeof ro);
  ro.ids = ids_f;
  CHECK_MOE(moe_forward(&c, x, W_g, NULL, NULL, NULL, W_gu, W_down, y_fused, &ro, ws, NULL));
  CHECK_MOE(moe_check_status(ws, NULL));

  /* the same layer through the split calls */
  CHECK_MOE(moe_route(&c, NULL, x, W_g, NULL, NULL, NULL, ids_s, gates, counts, demand, drop,
                      NULL, ws, NULL));
  CHECK_MOE(moe_permute(&c, ids_s, drop, x, offsets, NULL, slot_row, xp, ws, NULL));
  CHECK_MOE(moe_expert_ffn(&c, xp, offsets, x, W_gu, W_down, ye, ws, NULL));
  CHECK_MOE(moe_combine(&c, ye, slot_row, gates, y_split, NULL));
  CHECK_MOE(moe_check_status(ws, NULL));

  h1 = (unsigned char*)malloc(y_bytes);
  h2 = (unsigned char*)malloc(y_bytes);
  hi1 = (int32_t*)malloc((size_t)Nk * 4);
  hi2 = (int32_t*)malloc((size_t)Nk * 4);
  if (!h1 || !h2 || !hi1 || !hi2) return 2;
  CHECK_CUDA(cudaMemcpy(h1, y_fused, y_bytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(h2, y_split, y_bytes, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hi1, ids_f, (size_t)Nk * 4, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hi2, ids_s, (size_t)Nk * 4, cudaMemcpyDeviceToHost));
  if (memcmp(hi1, hi2, (size_t)Nk * 4) != 0) {
    fprintf(stderr, "routing differs between moe_forward and moe_route\n");
    return 1;
  }
  for (i = 0; i < (size_t)Nk; ++i)
    if (hi1[i] < 0 || hi1[i] >= c.E) {
      fprintf(stderr, "expert id out of range\n");
      return 1;
    }
  if (memcmp(h1, h2, y_bytes) != 0) {
    fprintf(stderr, "moe_forward and the split calls give different outputs\n");
    return 1;
  }
  printf("C ABI: moe_forward == route/permute/expert_ffn/combine (%lld tokens, C = %lld)\n",
         (long long)c.N, (long long)c.capacity);
  free(h1);
  free(h2);
  free(hi1);
  free(hi2);
  cudaFree(x);
  cudaFree(W_g);
  cudaFree(W_gu);
  cudaFree(W_down);
  cudaFree(ws);
  cudaFree(y_fused);
  cudaFree(y_split);
  cudaFree(xp);
  cudaFree(ye);
  cudaFree(ids_f);
  cudaFree(ids_s);
  cudaFree(gates);
  cudaFree(counts);
  cudaFree(demand);
  cudaFree(offsets);
  cudaFree(slot_row);
  cudaFree(drop);
  return 0;
}
