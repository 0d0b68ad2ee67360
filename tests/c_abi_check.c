/* Plain C99 client of libhimuon: the header compiles as C, the library links
 * and the host-side entry points answer without a GPU.  Built and run by
 * tests/test_c_abi.py; prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "himuon.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  static char storage[16];
  const float coeffs[15] = {3.4445f, -4.7750f, 2.0315f, 3.4445f, -4.7750f, 2.0315f, 3.4445f, -4.7750f,
                            2.0315f, 3.4445f, -4.7750f, 2.0315f, 3.4445f, -4.7750f, 2.0315f};
  himuon_ns_params p;
  himuon_mat mats[2];
  int64_t records[5 * 16];
  int32_t tiles[2] = {128, 512};
  int64_t n;

  CHECK(himuon_version() == HIMUON_VERSION);
  CHECK(strstr(himuon_status_string(HIMUON_ERR_WORKSPACE), "workspace") != NULL);

  memset(&p, 0, sizeof p);
  p.tile = 128;
  p.steps = 5;
  p.coeffs = coeffs;
  p.eps = 1e-7f;
  p.compute = HIMUON_BF16;
  p.safety = 1.0f;

  /* a 300 x 500 matrix at T = 128: 3 x 4 tiles, ragged at the bottom and right */
  mats[0].data = storage;
  mats[0].rows = 300;
  mats[0].cols = 500;
  mats[0].ld = 504;
  mats[0].dtype = HIMUON_BF16;
  n = himuon_plan_tiles(mats, 1, NULL, 128, records, 16);
  CHECK(n == 12);
  CHECK(records[0] == 0 && records[1] == 0 && records[2] == 0 && records[3] == 128 && records[4] == 128);
  CHECK(records[5 * 11 + 1] == 256 && records[5 * 11 + 2] == 384);   /* last tile: row 256, column 384 */
  CHECK(records[5 * 11 + 3] == 44 && records[5 * 11 + 4] == 116);    /* 300 - 256, 500 - 384 */

  /* on chip at T = 128 (and 256) needs no workspace; a per-matrix T of 512 does */
  mats[1] = mats[0];
  mats[1].data = storage + 0;
  CHECK(himuon_workspace_size(mats, 1, NULL, &p, HIMUON_OP_NS_TILED) == 0);
  p.tiles = tiles;
  CHECK(himuon_workspace_size(mats, 2, NULL, &p, HIMUON_OP_NS_TILED) > 0);
  CHECK(himuon_ns_static(mats, mats, 2, NULL, &p, NULL) == HIMUON_ERR_UNSUPPORTED);
  p.tiles = NULL;

  /* argument errors come back before anything touches a device; an empty
     call (no matrices) is one of them */
  CHECK(himuon_ns_tiled(NULL, mats, 1, NULL, &p, NULL, 0, NULL) == HIMUON_ERR_INVALID);
  CHECK(himuon_ns_tiled(mats, mats, 0, NULL, &p, NULL, 0, NULL) == HIMUON_ERR_INVALID);
  CHECK(himuon_workspace_size(mats, 0, NULL, &p, HIMUON_OP_NS_TILED) == HIMUON_ERR_INVALID);
  CHECK(himuon_plan_tiles(mats, 0, NULL, 128, records, 16) == HIMUON_ERR_INVALID);
  p.steps = 17;
  CHECK(himuon_ns_tiled(mats, mats, 1, NULL, &p, NULL, 0, NULL) == HIMUON_ERR_UNSUPPORTED);
  p.steps = 5;
  CHECK(himuon_momentum_step(NULL, mats, mats, 1, 0.95f, 0.02f, NULL, &p, NULL, NULL, 0, NULL) ==
        HIMUON_ERR_INVALID);

  printf("ok\n");
  return 0;
}
