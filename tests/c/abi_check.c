/* Plain C11 client of the library's C ABI (include/gca.h): compiles the header as C and calls
 * the host-side entry points, which need no GPU. Prints one line per check; exits non-zero on the
 * first failure. Built and run by tests/test_abi_c.py. */
#include <stdio.h>
#include <string.h>

#include "gca.h"

static int fails = 0;

static void expect(int cond, const char* what) {
  printf("%s %s\n", cond ? "ok  " : "FAIL", what);
  if (!cond) ++fails;
}

int main(void) {
  /* one GCA layer at 518x378: 27 x 37 patches + 5 special tokens, 16 heads of 64 */
  gca_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.num_heads = 16;
  cfg.head_dim = 64;
  cfg.page_size = 16;
  cfg.grid_h = 27;
  cfg.grid_w = 37;
  cfg.num_special = 5;
  cfg.anchor_frames = 1;
  cfg.window_frames = 16;
  cfg.keep_tokens = 12;
  cfg.max_frames = 320;
  cfg.num_pages = 1400;
  cfg.rope_base = 10000.0f;

  expect(gca_validate_config(&cfg) == GCA_OK, "valid config accepted");
  const size_t ws = gca_workspace_bytes(&cfg);
  /* the K and V pools alone: 2 x pages x heads x 16 slots x 64 dims x 2 bytes */
  const size_t pools = (size_t)2 * 1400 * 16 * 16 * 64 * 2;
  expect(ws >= pools, "workspace holds both pools");
  expect(ws % 1024 == 0, "workspace size is a multiple of 1024 bytes");

  gca_config bad = cfg;
  bad.head_dim = 128;
  expect(gca_validate_config(&bad) != GCA_OK, "head_dim other than 64 rejected");
  bad = cfg;
  bad.window_frames = 0;
  expect(gca_validate_config(&bad) == GCA_ERR_INVALID_ARG, "empty window rejected");
  bad = cfg;
  bad.rope_base = -1.0f;
  expect(gca_validate_config(&bad) == GCA_ERR_INVALID_ARG, "negative RoPE base rejected");
  expect(gca_validate_config(NULL) == GCA_ERR_INVALID_ARG, "NULL config rejected");
  expect(gca_workspace_bytes(&bad) == 0, "no workspace size for an invalid config");

  expect(strcmp(gca_status_string(GCA_OK), "GCA_OK") == 0, "status string of GCA_OK");
  expect(strcmp(gca_status_string(GCA_ERR_OUT_OF_PAGES), "GCA_ERR_OUT_OF_PAGES") == 0,
         "status string of GCA_ERR_OUT_OF_PAGES");
  expect(gca_cache_destroy(NULL) == GCA_OK, "destroying NULL is accepted");
  return fails == 0 ? 0 : 1;
}
