/* abi_c_decode.c — one decode step through libpaged from plain C, with the
 * CUDA runtime for device memory and no other framework.
 *
 * Built by tests/test_abi_c.py (gcc -std=c11, linked with libcudart and the
 * in-tree libpaged.so) and run with an output directory: it fills a bf16
 * cache of 3 sequences (contexts 1, 37 and 300, 8 query / 2 kv heads,
 * head_dim 128, 16-token blocks spread over a 32-block pool), writes each
 * sequence's new token with pa_reshape_and_cache, runs pa_decode, and dumps
 * the inputs and results as raw little-endian files for the test to check
 * against the oracle.
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "paged.h"

enum { S = 3, H = 8, HKV = 2, D = 128, BS = 16, NB = 32, MAXB = 19 };

#define CHECK_CUDA(x)                                                          \
  do {                                                                         \
    cudaError_t e_ = (x);                                                      \
    if (e_ != cudaSuccess) {                                                   \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));                 \
      return 1;                                                                \
    }                                                                          \
  } while (0)
#define CHECK_PA(x)                                                            \
  do {                                                                         \
    pa_status s_ = (x);                                                        \
    if (s_ != PA_OK) {                                                         \
      fprintf(stderr, "%s: status %d: %s\n", #x, (int)s_, pa_last_error());   \
      return 1;                                                                \
    }                                                                          \
  } while (0)

/* bf16 code of a float, round to nearest even (the inputs are finite) */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* a deterministic value in [-1, 1] for index i of stream k */
static float value_of(uint32_t k, uint32_t i) {
  uint32_t x = i * 2654435761u ^ (k * 0x9e3779b9u);
  x ^= x >> 15;
  x *= 0x85ebca6bu;
  x ^= x >> 13;
  return (float)((int)(x % 2001u) - 1000) / 1000.0f;
}

static int dump(const char* dir, const char* name, const void* p, size_t n) {
  char path[1024];
  snprintf(path, sizeof path, "%s/%s", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f) return 1;
  const size_t w = fwrite(p, 1, n, f);
  fclose(f);
  return w == n ? 0 : 1;
}

int main(int argc, char** argv) {
  if (argc != 2) return 2;
  const char* dir = argv[1];
  const int32_t ctx[S] = {1, 37, 300};
  const size_t cache_elems = (size_t)NB * BS * HKV * D;
  uint16_t* kc = malloc(cache_elems * 2);
  uint16_t* vc = malloc(cache_elems * 2);
  uint16_t* q = malloc((size_t)S * H * D * 2);
  uint16_t* nk = malloc((size_t)S * HKV * D * 2);
  uint16_t* nv = malloc((size_t)S * HKV * D * 2);
  uint16_t* out = malloc((size_t)S * H * D * 2);
  if (!kc || !vc || !q || !nk || !nv || !out) return 1;
  for (size_t i = 0; i < cache_elems; ++i) {
    kc[i] = to_bf16(value_of(1, (uint32_t)i));
    vc[i] = to_bf16(value_of(2, (uint32_t)i));
  }
  for (size_t i = 0; i < (size_t)S * H * D; ++i) q[i] = to_bf16(value_of(3, (uint32_t)i));
  for (size_t i = 0; i < (size_t)S * HKV * D; ++i) {
    nk[i] = to_bf16(value_of(4, (uint32_t)i));
    nv[i] = to_bf16(value_of(5, (uint32_t)i));
  }

  /* block tables from the allocator over a shuffled pool */
  int32_t order[NB];
  for (int i = 0; i < NB; ++i) order[i] = (i * 7 + 3) % NB;
  pa_alloc* a = NULL;
  CHECK_PA(pa_alloc_create(NB, order, &a));
  int32_t ids[S][MAXB];
  const int32_t* id_ptrs[S];
  int32_t nblk[S];
  for (int s = 0; s < S; ++s) {
    nblk[s] = (ctx[s] + BS - 1) / BS;
    CHECK_PA(pa_alloc_allocate(a, nblk[s], ids[s]));
    id_ptrs[s] = ids[s];
  }
  int32_t table[S * MAXB];
  CHECK_PA(pa_build_block_table(id_ptrs, nblk, S, MAXB, table));
  int32_t pos[S], slots[S];
  for (int s = 0; s < S; ++s) pos[s] = ctx[s] - 1;
  CHECK_PA(pa_build_slot_mapping(table, S, MAXB, NULL, pos, S, BS, slots));
  pa_alloc_destroy(a);

  if (dump(dir, "key_cache_in.bin", kc, cache_elems * 2) ||
      dump(dir, "value_cache_in.bin", vc, cache_elems * 2) ||
      dump(dir, "query.bin", q, (size_t)S * H * D * 2) ||
      dump(dir, "new_key.bin", nk, (size_t)S * HKV * D * 2) ||
      dump(dir, "new_value.bin", nv, (size_t)S * HKV * D * 2) ||
      dump(dir, "block_tables.bin", table, sizeof table) ||
      dump(dir, "context_lens.bin", ctx, sizeof ctx) || dump(dir, "slots.bin", slots, sizeof slots))
    return 1;

  void *d_kc, *d_vc, *d_q, *d_nk, *d_nv, *d_out, *d_table, *d_ctx, *d_slots, *d_ws;
  CHECK_CUDA(cudaMalloc(&d_kc, cache_elems * 2));
  CHECK_CUDA(cudaMalloc(&d_vc, cache_elems * 2));
  CHECK_CUDA(cudaMalloc(&d_q, (size_t)S * H * D * 2));
  CHECK_CUDA(cudaMalloc(&d_nk, (size_t)S * HKV * D * 2));
  CHECK_CUDA(cudaMalloc(&d_nv, (size_t)S * HKV * D * 2));
  CHECK_CUDA(cudaMalloc(&d_out, (size_t)S * H * D * 2));
  CHECK_CUDA(cudaMalloc(&d_table, sizeof table));
  CHECK_CUDA(cudaMalloc(&d_ctx, sizeof ctx));
  CHECK_CUDA(cudaMalloc(&d_slots, sizeof slots));
  const size_t ws_bytes = pa_decode_workspace_size(S, H, HKV, D, BS, 300, 0, PA_F16);
  if (ws_bytes < 256) return 1;
  CHECK_CUDA(cudaMalloc(&d_ws, ws_bytes));
  CHECK_CUDA(cudaMemcpy(d_kc, kc, cache_elems * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_vc, vc, cache_elems * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_q, q, (size_t)S * H * D * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_nk, nk, (size_t)S * HKV * D * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_nv, nv, (size_t)S * HKV * D * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_table, table, sizeof table, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_ctx, ctx, sizeof ctx, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(d_slots, slots, sizeof slots, cudaMemcpyHostToDevice));

  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreate(&stream));
  CHECK_PA(pa_workspace_init(d_ws, ws_bytes, stream));
  CHECK_PA(pa_reshape_and_cache(d_nk, d_nv, d_kc, d_vc, d_slots, S, HKV, D, BS, NB, PA_BF16,
                                PA_BF16, NULL, NULL, stream));
  CHECK_PA(pa_decode(d_out, d_q, d_kc, d_vc, d_table, MAXB, d_ctx, 300, S, H, HKV, D, BS, NB,
                     0.08838834764831845f, PA_BF16, PA_BF16, NULL, NULL, 0, d_ws, ws_bytes,
                     stream));
  CHECK_PA(pa_decode_check(d_ws, stream));
  CHECK_CUDA(cudaStreamSynchronize(stream));
  CHECK_CUDA(cudaMemcpy(out, d_out, (size_t)S * H * D * 2, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(kc, d_kc, cache_elems * 2, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(vc, d_vc, cache_elems * 2, cudaMemcpyDeviceToHost));
  if (dump(dir, "out.bin", out, (size_t)S * H * D * 2) ||
      dump(dir, "key_cache_out.bin", kc, cache_elems * 2) ||
      dump(dir, "value_cache_out.bin", vc, cache_elems * 2))
    return 1;
  CHECK_CUDA(cudaStreamDestroy(stream));
  void* bufs[] = {d_kc, d_vc, d_q, d_nk, d_nv, d_out, d_table, d_ctx, d_slots, d_ws};
  for (size_t i = 0; i < sizeof bufs / sizeof bufs[0]; ++i) CHECK_CUDA(cudaFree(bufs[i]));
  free(kc);
  free(vc);
  free(q);
  free(nk);
  free(nv);
  free(out);
  printf("decode ok\n");
  return 0;
}
