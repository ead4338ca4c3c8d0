/*
 * Plain C client of the library: includes only include/tps.h, links libtps.so,
 * and exercises the host-only entry points (no GPU needed). Prints one line per
 * check; exits non-zero on the first failure.
 */
#include <stdio.h>
#include <string.h>

#include "tps.h"

static int fail(const char* what) {
  printf("FAIL %s\n", what);
  return 1;
}

int main(void) {
  int32_t qf[8], qc[8], kf[8], kc[8];
  /* the page's 32 query heads over tp = 4: heads 0-7, 8-15, 16-23, 24-31; 8 KV heads -> 2 per shard */
  if (tp_head_map(32, 8, 4, qf, qc, kf, kc) != TPS_OK) return fail("tp_head_map status");
  for (int r = 0; r < 4; ++r)
    if (qf[r] != 8 * r || qc[r] != 8 || kf[r] != 2 * r || kc[r] != 2) return fail("tp_head_map values");
  /* tp = 8 over 4 KV heads: each KV head on two shards */
  if (tp_head_map(32, 4, 8, qf, qc, kf, kc) != TPS_OK) return fail("tp_head_map replicated");
  for (int r = 0; r < 8; ++r)
    if (kf[r] != r / 2 || kc[r] != 1) return fail("tp_head_map replicated values");
  if (tp_head_map(32, 8, 3, NULL, NULL, NULL, NULL) != TPS_ERR_DIVISIBILITY) return fail("tp_head_map divisibility");
  printf("ok tp_head_map\n");

  /* COLUMN pack of W[1024, 4096] over 8 shards: 512 rows, 1024 K per shard, 128x64 tiles */
  if (tp_packed_bytes(TPS_KIND_COLUMN, 1024, 4096, 8, NULL) != (size_t)8 * 512 * 1024 * 2)
    return fail("tp_packed_bytes column");
  /* ROW pack of V[4096, 1024] over 8 shards: 1024 rows of 512 K each */
  if (tp_packed_bytes(TPS_KIND_ROW, 4096, 1024, 8, NULL) != (size_t)8 * 1024 * 512 * 2)
    return fail("tp_packed_bytes row");
  if (tp_packed_bytes(TPS_KIND_ROW, 4096, 1024, 3, NULL) != 0) return fail("tp_packed_bytes invalid");
  printf("ok tp_packed_bytes\n");

  if (tps_workspace_bytes(TPS_FN_ROW, 512, 1024, 4096, 8) == 0) return fail("tps_workspace_bytes row");
  if (tps_workspace_bytes(TPS_FN_ARGMAX, 64, 128256, 4096, 8) == 0) return fail("tps_workspace_bytes argmax");
  printf("ok tps_workspace_bytes\n");

  if (strncmp(tps_status_string(TPS_ERR_DIVISIBILITY), "TPS_ERR_DIVISIBILITY", 20) != 0)
    return fail("tps_status_string");
  printf("ok tps_status_string\n");

  /* argument validation happens before any CUDA call: fake, aligned, never dereferenced addresses */
  const void* fake = (const void*)(uintptr_t)(1u << 20);
  tps_heads h = {32, 8, 64};
  if (sharded_gqa_attention(fake, 1, 16, &h, 8, 1, (void*)fake, NULL) != TPS_ERR_UNIMPLEMENTED)
    return fail("sharded_gqa_attention head_dim");
  if (row_parallel_forward(fake, 4, 64, fake, 64, 3, NULL, TPS_REDUCE_FUSED, NULL, (void*)fake, TPS_DTYPE_BF16,
                           NULL, 0, NULL) != TPS_ERR_DIVISIBILITY)
    return fail("row_parallel_forward divisibility");
  if (column_parallel_forward(fake, 0, 64, fake, TPS_KIND_COLUMN, 256, 2, NULL, NULL, TPS_ACT_NONE, (void*)fake,
                              TPS_DTYPE_BF16, NULL, 0, NULL) != TPS_OK)
    return fail("column_parallel_forward m = 0");
  printf("ok validation\n");
  printf("all ok\n");
  return 0;
}
