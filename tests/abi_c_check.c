/* abi_c_check.c — a plain C11 client of libpaged's host calls.
 *
 * Built by tests/test_abi_c.py with gcc (-std=c11 -pedantic -Werror) against
 * include/paged.h and the in-tree libpaged.so, then run on the host; it makes
 * no device call. It prints one "key value" line per result, which the test
 * compares with Python's hashlib, the Python binding and the oracle's
 * allocator model.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "paged.h"

static void print_hex(const char* key, const uint8_t* h) {
  printf("%s ", key);
  for (int i = 0; i < 32; ++i) printf("%02x", h[i]);
  printf("\n");
}

int main(void) {
  /* SHA-256 and the chained block hashes of a 34-token prompt (2 full blocks of 16) */
  uint8_t h[32];
  if (pa_sha256("abc", 3, h) != PA_OK) return 1;
  print_hex("sha256_abc", h);
  int32_t tokens[34];
  for (int i = 0; i < 34; ++i) tokens[i] = 1000 + 7 * i;
  uint8_t hashes[2 * 32];
  if (pa_prompt_block_hashes(tokens, 34, 16, hashes) != PA_OK) return 1;
  print_hex("block_hash_0", hashes);
  print_hex("block_hash_1", hashes + 32);

  /* allocator: a seeded order, allocate 3, share the first, free all three */
  const int32_t order[8] = {5, 2, 7, 0, 1, 6, 3, 4};
  pa_alloc* a = NULL;
  if (pa_alloc_create(8, order, &a) != PA_OK) return 1;
  int32_t ids[3];
  if (pa_alloc_allocate(a, 3, ids) != PA_OK) return 1;
  printf("allocated %d %d %d\n", ids[0], ids[1], ids[2]);
  if (pa_alloc_share(a, ids[0]) != PA_OK) return 1;
  if (pa_alloc_free(a, ids, 3) != PA_OK) return 1;
  printf("refcount_first %d\n", pa_alloc_refcount(a, ids[0]));
  printf("num_free %lld\n", (long long)pa_alloc_num_free(a));
  int32_t fl[8];
  const int64_t nf = pa_alloc_free_list(a, fl, 8);
  printf("free_list");
  for (int64_t i = 0; i < nf; ++i) printf(" %d", fl[i]);
  printf("\n");
  int32_t big[9];
  printf("oom %d\n", (int)pa_alloc_allocate(a, 9, big));
  pa_alloc_destroy(a);

  /* slot mapping of a 2-sequence table, block size 16 (one padding token) */
  const int32_t table[2 * 3] = {4, 9, -1, 3, 8, 11};
  const int32_t seq_ids[4] = {0, 0, 1, 1};
  const int32_t positions[4] = {0, 17, 40, -1};
  int32_t slots[4];
  if (pa_build_slot_mapping(table, 2, 3, seq_ids, positions, 4, 16, slots) != PA_OK) return 1;
  printf("slots %d %d %d %d\n", slots[0], slots[1], slots[2], slots[3]);

  /* workspace sizing and an argument error reported through pa_last_error */
  printf("prefill_ws %zu\n",
         pa_chunked_prefill_workspace_size(16, 16 * 512, 32, 32, 128, 512, 4096, PA_F16));
  const pa_status st = pa_decode(NULL, NULL, NULL, NULL, NULL, 0, NULL, 0, 1, 8, 3, 128, 16, 16,
                                 0.1f, PA_F16, PA_F16, NULL, NULL, 0, NULL, 0, NULL);
  printf("bad_decode %d %s\n", (int)st, strlen(pa_last_error()) > 0 ? "message" : "none");
  return 0;
}
