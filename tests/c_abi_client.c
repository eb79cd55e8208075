/* A plain C99 client of libpa.so: include/pa.h must compile as strict C
 * (no C++ constructs) and the host allocator (fork, copy-on-write, prefix
 * groups for the shared-prefix decode) must be usable through it alone.
 * Built and run by tests/test_c_client.py; needs no GPU. */
#include <stdio.h>

#include "pa.h"

int main(void) {
  pa_allocator* a = NULL;
  int64_t slots[20];
  int64_t pair[2];
  int32_t ncow = 0;
  int32_t table[4];
  int32_t n = 0;
  if (pa_version() != 1) return 10;
  if (pa_alloc_create(8, 16, NULL, &a) != PA_OK) return 11;
  if (pa_seq_add(a, 7) != PA_OK) return 12;
  /* 20 tokens: block 0 fills, token 16 opens block 1 */
  if (pa_seq_append(a, 7, 20, slots, pair, &ncow) != PA_OK || ncow != 0) return 13;
  if (pa_seq_fork(a, 7, 8) != PA_OK) return 14;
  /* the child writes into the shared, partly filled block 1: copy-on-write */
  if (pa_seq_append(a, 8, 1, slots, pair, &ncow) != PA_OK || ncow != 1) return 15;
  if (pa_seq_block_table(a, 8, table, 4, &n) != PA_OK || n != 2) return 16;
  printf("%lld %lld %d %d %d %d\n", (long long)pair[0], (long long)pair[1], table[0], table[1],
         pa_block_refcount(a, 0), pa_alloc_num_free(a));
  {
    /* parent and fork share their one full block: one group of two */
    const int64_t ids[2] = {7, 8};
    int32_t gs[3] = {-1, -1, -1}, gb[2] = {-1, -1}, ng = -1;
    if (pa_alloc_prefix_groups(a, ids, 2, 4, gs, gb, &ng) != PA_OK) return 19;
    printf("%d %d %d %d\n", ng, gs[0], gs[1], gb[0]);
  }
  if (pa_seq_free(a, 7) != PA_OK || pa_seq_free(a, 8) != PA_OK) return 17;
  if (pa_seq_free(a, 8) != PA_ERR_INVALID_ARG) return 18; /* double free */
  printf("%d %s\n", pa_alloc_num_free(a), pa_status_string(PA_ERR_OUT_OF_BLOCKS));
  pa_alloc_destroy(a);
  return 0;
}
