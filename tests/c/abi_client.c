/* A plain C client of libengram: compiles against include/engram.h alone
 * (no CUDA headers), links libengram.so and calls the host-side entry points
 * (version, workspace sizes, shard sizes, argument checks).  No kernel runs,
 * so it needs no GPU.  Prints one "name value" line per check; exit 0 when
 * every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "engram.h"

static int failures = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", what, ok ? "ok" : "FAIL");
  if (!ok) ++failures;
}

int main(void) {
  engram_config c;
  memset(&c, 0, sizeof c);
  c.n_orders = 2;
  c.orders[0] = 2;
  c.orders[1] = 3;
  c.heads_per_order = 8;
  c.row_dim = 64;
  c.hidden = 1024;
  c.hc_mult = 4;
  c.conv_kernel = 4;
  c.dilation = 3;
  c.pad_id = 0;
  c.vocab = 98304;
  c.rms_eps = 1e-6f;
  c.gate_eps = 1e-6f;
  c.dtype = ENGRAM_BF16;

  check(engram_version() >= 100, "version");

  size_t ws = 0;
  check(engram_forward_workspace_size(&c, 4, 2048, &ws) == ENGRAM_OK && ws >= (size_t)4 * 2048 * 1024 * 2,
        "forward_workspace_size");

  int64_t total = 0;
  for (int r = 0; r < 8; ++r) total += engram_shard_rows(1000003, 8, r);
  check(total == 1000003, "shard_rows_sum");
  check(engram_shard_rows(10, 4, 4) == -1, "shard_rows_out_of_range");
  check(engram_shard_route_workspace_size(&c, 4, 2048, 8) > 0, "shard_route_workspace_size");

  /* a config error is reported on the host, with text */
  engram_config bad = c;
  bad.n_orders = 0;
  check(engram_forward_workspace_size(&bad, 4, 2048, &ws) == ENGRAM_ERR_INVALID_ARG, "bad_config_rejected");
  char msg[256];
  engram_last_error(msg, sizeof msg);
  check(strstr(msg, "n_orders") != NULL, "error_text");

  /* arguments checked before any launch: the pointers are never dereferenced */
  check(engram_shard_place(&c, (const void*)256, NULL, 4, (void*)256, 8, NULL, NULL) == ENGRAM_ERR_INVALID_ARG,
        "place_null_rejected");
  return failures == 0 ? 0 : 1;
}
