/* A plain C99 consumer of the library's C ABI (include/dsa.h).  It touches no
 * device: every call below is refused or answered on the host, so the
 * program runs on a machine without a GPU.  Exit status 0 and "ok" on
 * stdout mean every check passed; a nonzero status names the failed check. */
#include <stdio.h>
#include <string.h>

#include "dsa.h"

int main(void) {
  static char dummy[64];
  void *p = dummy + (16 - ((size_t)dummy & 15)) % 16; /* 16-byte aligned, never read */
  dsa_dims dims;
  dsa_layer_io layers[2];
  size_t small, large;

  memset(&dims, 0, sizeof dims);
  memset(layers, 0, sizeof layers);

  /* [IC] 1.1: the first layer must be F; refused before any launch */
  if (indexcache_forward("SF", 2, layers, &dims, (int32_t *)p, p, 0, NULL) != DSA_ERR_BAD_PATTERN) return 1;
  if (indexcache_forward("FX", 2, layers, &dims, (int32_t *)p, p, 0, NULL) != DSA_ERR_BAD_PATTERN) return 2;
  if (strlen(dsa_last_error()) == 0) return 3;

  /* null inputs are refused with an argument error */
  if (dsa_indexer_topk(NULL, NULL, NULL, 1, 1, 1, 0, 64, 128, 8, NULL, p, 64, NULL) != DSA_ERR_INVALID_ARG) return 4;
  if (dsa_sparse_attn(NULL, NULL, 576, NULL, 576, NULL, 1, 1, 1, 0, 128, 576, 512, 8, 1.0f, NULL, NULL, p, 64,
                      NULL) != DSA_ERR_INVALID_ARG)
    return 5;
  if (dsa_check_indices(NULL, 1, 1, 0, 8, NULL, NULL) != DSA_ERR_INVALID_ARG) return 6;

  /* start_pos + Lq - 1 must not pass Lk */
  if (dsa_indexer_topk((const dsa_bf16 *)p, (const dsa_bf16 *)p, (const float *)p, 1, 6, 4, 0, 64, 128, 8,
                       (int32_t *)p, p, 64, NULL) != DSA_ERR_INVALID_ARG)
    return 7;

  /* CSA: several rows must start on a block boundary */
  if (dsa_csa_indexer_topk((const dsa_bf16 *)p, (const dsa_bf16 *)p, (const float *)p, 1, 8, 10, 6, 4, 64, 128, 8,
                           (int32_t *)p, p, 64, NULL) != DSA_ERR_UNSUPPORTED)
    return 8;

  /* workspace queries are host arithmetic and grow with the sequence */
  small = dsa_indexer_topk_workspace(1, 4096, 4096, 0, 64, 128, 2048);
  large = dsa_indexer_topk_workspace(1, 200000, 200000, 0, 64, 128, 2048);
  if (small == 0 || large < small) return 9;
  if (dsa_sparse_attn_workspace(0, 1, 128, 512, 8) != 0) return 10;
  if (dsa_indexer_launch_count() < 0) return 11;

  printf("ok\n");
  return 0;
}
