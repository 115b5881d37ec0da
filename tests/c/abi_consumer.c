/* A plain C99 program against include/pa.h and libpa.so: the header must compile as C
 * with every warning on, and the host-only entry points (block manager, partition
 * choice, argument checks) must work without a GPU.  Prints one line of results. */
#include <stdint.h>
#include <stdio.h>

#include "pa.h"

int main(void) {
  pa_alloc_t* a = NULL;
  int64_t slot = -1;
  int32_t src = 0, dst = 0;
  pa_stats_t st;
  int rc = pa_alloc_create(16, 4, NULL, &a);
  if (rc != PA_OK) return 1;
  rc |= pa_seq_add(a, 7, 5);                               /* 2 blocks, 3 free slots */
  rc |= pa_seq_fork(a, 7, 8);                              /* shares both blocks      */
  rc |= pa_seq_append_slot(a, 8, &slot, &src, &dst);       /* a shared block: a copy  */
  rc |= pa_alloc_stats(a, &st);
  printf("rc=%d slot=%lld copy=%d->%d used=%lld shared=%lld ps=%d bad=%d\n", rc,
         (long long)slot, (int)src, (int)dst, (long long)st.used_blocks,
         (long long)st.shared_blocks,
         pa_decode_partition_size(PA_BF16, 64, 32, 32, 128, 16, 2050, 148),
         pa_decode(NULL));
  pa_alloc_destroy(a);
  return rc == PA_OK ? 0 : 2;
}
