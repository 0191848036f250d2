/* Host-only use of libvt's C ABI from plain C99 (no C++, no Python): configuration
 * checks, the thread's error message, the workspace plan and the index maps of a grid.
 * Needs no GPU.  Prints "c abi ok" and returns 0 when every check holds; otherwise it
 * prints the failed check and returns 1.  Built and run by tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "vt.h"

#define CHECK(cond)                                                         \
  do {                                                                      \
    if (!(cond)) {                                                          \
      fprintf(stderr, "c abi check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                             \
    }                                                                       \
  } while (0)

/* The 32-layer tower of the model card: hidden 1280, 16 heads of 80, MLP 5120, patch 14,
 * temporal patch 2, 2x2 merge, projector 6144, RoPE sections 16/32/32. */
static vt_config tower_config(void) {
  vt_config c;
  memset(&c, 0, sizeof c);
  c.layers = 32;
  c.hidden = 1280;
  c.heads = 16;
  c.head_dim = 80;
  c.mlp = 5120;
  c.patch = 14;
  c.temporal_patch = 2;
  c.merge = 2;
  c.rope_sections[0] = 16;
  c.rope_sections[1] = 32;
  c.rope_sections[2] = 32;
  c.rope_theta = 10000.0f;
  c.ln_eps = 1e-6f;
  c.gelu_tanh = 1;
  c.proj_gelu_tanh = 1;
  c.proj_hidden = 6144;
  c.proj_out = 6144;
  c.use_rope = 1;
  return c;
}

int main(void) {
  vt_config cfg = tower_config();
  vt_handle* h = NULL;
  CHECK(vt_create(&cfg, &h) == VT_OK);
  CHECK(h != NULL);

  /* configuration errors: status codes and a message for this thread */
  vt_config bad = cfg;
  vt_handle* h2 = NULL;
  bad.heads = 15; /* heads * head_dim != hidden */
  CHECK(vt_create(&bad, &h2) == VT_ERR_INVALID_ARG);
  CHECK(h2 == NULL);
  CHECK(vt_last_error() != NULL && strlen(vt_last_error()) > 0);
  bad = cfg;
  bad.rope_sections[2] = 30; /* sections must sum to head_dim */
  CHECK(vt_create(&bad, &h2) == VT_ERR_INVALID_ARG);
  bad = cfg;
  bad.merge = 3;
  CHECK(vt_create(&bad, &h2) == VT_ERR_UNSUPPORTED);
  CHECK(vt_create(NULL, &h2) == VT_ERR_INVALID_ARG);

  /* workspace: affine in tokens (equal increments for equal token steps, up to the
   * per-buffer 256-byte rounding), linear in the batch, grids checked */
  const int32_t g1[3] = {1, 32, 32}, g2[3] = {1, 64, 64}, g3[3] = {1, 96, 96};
  size_t w1 = 0, w2 = 0, w3 = 0, w8 = 0;
  CHECK(vt_workspace_bytes(h, 1, g1, &w1) == VT_OK);
  CHECK(vt_workspace_bytes(h, 1, g2, &w2) == VT_OK);
  CHECK(vt_workspace_bytes(h, 1, g3, &w3) == VT_OK);
  CHECK(w1 > 0 && w2 > w1 && w3 > w2);
  {
    /* tokens: 1024, 4096, 9216 -> slope over the two steps */
    const double s12 = (double)(w2 - w1) / (4096 - 1024);
    const double s23 = (double)(w3 - w2) / (9216 - 4096);
    CHECK(s12 > 0.0 && (s23 - s12) * (s23 - s12) < (0.001 * s12) * (0.001 * s12));
  }
  CHECK(vt_workspace_bytes(h, 8, g1, &w8) == VT_OK);
  CHECK(w8 <= 8 * w1 + 16 * 256);
  {
    const int32_t odd[3] = {1, 7, 8}; /* h not even: no 2x2 merge */
    size_t w = 0;
    CHECK(vt_workspace_bytes(h, 1, odd, &w) == VT_ERR_SHAPE);
    CHECK(vt_workspace_bytes(h, 0, g1, &w) == VT_ERR_INVALID_ARG);
    CHECK(vt_workspace_bytes(h, 1, g1, NULL) == VT_ERR_INVALID_ARG);
  }

  /* index maps of a 4 x 6 grid: block order groups each 2x2 block's four tokens in
   * member order (0,0), (0,1), (1,0), (1,1), blocks in raster order; the merge map
   * gathers the same four raster tokens; positions are (0, row, col) */
  {
    const int32_t grid[3] = {1, 4, 6};
    int32_t order[24], pos[72], merge[24];
    CHECK(vt_index_maps(grid, order, pos, merge) == VT_OK);
    int seen[24] = {0};
    for (int i = 0; i < 24; ++i) {
      CHECK(order[i] >= 0 && order[i] < 24);
      seen[order[i]] += 1;
    }
    for (int i = 0; i < 24; ++i) CHECK(seen[i] == 1);
    for (int g = 0; g < 6; ++g) {
      const int bi = g / 3, bj = g % 3;
      for (int m = 0; m < 4; ++m) {
        const int raster = (2 * bi + m / 2) * 6 + (2 * bj + m % 2);
        CHECK(order[4 * g + m] == raster);
        CHECK(merge[4 * g + m] == raster);
      }
    }
    for (int n = 0; n < 24; ++n) {
      CHECK(pos[3 * n] == 0);
      CHECK(pos[3 * n + 1] == n / 6);
      CHECK(pos[3 * n + 2] == n % 6);
    }
    CHECK(vt_index_maps(grid, NULL, NULL, NULL) == VT_OK);
  }

  CHECK(vt_destroy(h) == VT_OK);
  printf("c abi ok\n");
  return 0;
}
