/* A plain C (C99) consumer of include/flexattn.h: the header compiles as C and
 * the host-side checks answer without touching a GPU.  Built and run by
 * tests/test_c_consumer.py; prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "flexattn.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    printf("FAILED: %s (last error: %s)\n", what, flexattn_last_error());
    ++failures;
  }
}

int main(void) {
  int32_t mb = 0, nb = 0;
  expect(flexattn_version() > 0, "version is positive");

  /* tile grid of a 2048 x 2048 problem in 128 x 128 tiles, and of a ragged one */
  expect(flexattn_block_mask_dims(2048, 2048, 128, 128, &mb, &nb) == FA_OK && mb == 16 && nb == 16,
         "16 x 16 tiles for 2048 x 2048");
  expect(flexattn_block_mask_dims(200, 333, 64, 32, &mb, &nb) == FA_OK && mb == 4 && nb == 11,
         "ragged grid rounds up");
  expect(flexattn_block_mask_dims(0, 16, 16, 16, &mb, &nb) == FA_ERR_SHAPE, "L = 0 is a shape error");
  expect(flexattn_block_mask_dims(16, 16, 256, 16, &mb, &nb) == FA_ERR_SHAPE, "BM above 128 is a shape error");
  expect(flexattn_block_mask_dims(16, 16, 16, 16, NULL, &nb) == FA_ERR_NULL, "NULL output is rejected");
  expect(strlen(flexattn_last_error()) > 0, "a failing call leaves a message");

  /* a forward call with NULL tensors is rejected on the host */
  expect(flexattn_forward(NULL, NULL, NULL, NULL, NULL, 0.0f, 0, NULL, NULL, NULL, 0, NULL, NULL, 0, NULL) ==
             FA_ERR_NULL,
         "forward with NULL tensors");
  {
    /* the options struct is plain C and its defaults are all zero */
    fa_forward_options opts;
    memset(&opts, 0, sizeof(opts));
    opts.flags = FA_FLAG_ROWS_GUARANTEED_SAFE;
    expect(sizeof(opts) == 40, "fa_forward_options is 40 bytes");
    expect(flexattn_forward(NULL, NULL, NULL, NULL, NULL, 0.0f, 0, NULL, NULL, NULL, 0, &opts, NULL, 0, NULL) ==
               FA_ERR_NULL,
           "forward with options and NULL tensors");
  }
  expect(flexattn_build_block_mask(NULL, NULL, NULL) == FA_ERR_NULL, "block mask with NULL arguments");

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
