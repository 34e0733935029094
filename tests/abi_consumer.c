/* A plain C11 consumer of the library's public header, built with -std=c11 -pedantic
 * -Werror and linked against libaqnf4.so by tests/test_abi_host.py.  It calls only entry
 * points that work on the host or that must reject their arguments before any launch, and
 * prints what the test compares with the oracle (hex floats, so nothing is rounded). */
#include <stdio.h>

#include "aqnf4.h"

int main(void) {
  float levels[16], mids[15];
  const int64_t ns[] = {1, 63, 64, 65, 16384, 16385, (int64_t)4096 * 11008};
  aqnf4_layer layer = {0};
  uint64_t before;
  int i;

  if (aqnf4_codebook(0.0, levels, mids) != AQNF4_OK) return 1;
  for (i = 0; i < 16; ++i) printf("level %d %a\n", i, (double)levels[i]);
  for (i = 0; i < 15; ++i) printf("mid %d %a\n", i, (double)mids[i]);
  for (i = 0; i < (int)(sizeof ns / sizeof ns[0]); ++i)
    printf("cost %lld %lld\n", (long long)ns[i], (long long)aqnf4_cost_bytes(ns[i]));

  before = aqnf4_launch_count();
  layer.numel = 64; /* w is NULL */
  layer.dtype = AQNF4_BF16;
  printf("layer_error_null_w %d\n",
         (int)aqnf4_layer_error(&layer, 1, NULL, 0, NULL, NULL, NULL, NULL, NULL));
  printf("dequantize_null %d\n",
         (int)aqnf4_dequantize(NULL, NULL, NULL, NULL, 64, AQNF4_BF16, NULL, NULL));
  printf("nf4_linear_bad_k %d\n",
         (int)aqnf4_nf4_linear((const void*)16, AQNF4_BF16, 4, 96, (const uint8_t*)16,
                               (const uint8_t*)16, (const float*)16, 8, (void*)16, 1, NULL,
                               NULL));
  printf("nf4_linear_splits_bad_k %d\n", (int)aqnf4_nf4_linear_splits(4, 8, 96));
  printf("launches %llu\n", (unsigned long long)(aqnf4_launch_count() - before));
  printf("status %s\n", aqnf4_status_string(AQNF4_ERR_ALIGNMENT));
  return 0;
}
