/* A plain C99 client of libmla's C ABI: include/mla.h compiles as C, and the
 * host-side entry points (sizes, status strings, argument checks that return
 * before any CUDA call) work when linked from C.  No GPU is needed. */
#include <stdio.h>
#include <string.h>

#include "mla.h"

static int fails = 0;
#define CHECK(c)                                                         \
  do {                                                                   \
    if (!(c)) {                                                          \
      fprintf(stderr, "FAIL %s:%d: %s\n", __FILE__, __LINE__, #c);       \
      ++fails;                                                           \
    }                                                                    \
  } while (0)

static mla_dims dsv2_dims(void) {
  mla_dims d;
  memset(&d, 0, sizeof d);
  d.n_h = 128;
  d.d_h = 128;
  d.d_v = 128;
  d.d_c = 512;
  d.d_r = 64;
  d.d_model = 5120;
  d.d_cq = 1536;
  d.rope_base = 10000.0f;
  d.softmax_scale = 0.0f;
  d.page_size = 64;
  d.dtype = MLA_BF16;
  return d;
}

int main(void) {
  mla_dims d = dsv2_dims();
  float out = 0.0f;
  mla_weights* w = NULL;

  /* Sizes. */
  CHECK(mla_absorbed_weights_bytes(&d) > 0);
  CHECK(mla_append_workspace_bytes(&d, 64) > 0);
  CHECK(mla_decode_workspace_bytes(&d, 64, 1, 8193) > 0);
  CHECK(mla_prefill_workspace_bytes(&d, 4, 4096) > mla_decode_workspace_bytes(&d, 64, 1, 8193));
  CHECK(mla_decode_cp_workspace_bytes(&d, 64, 1) >= mla_decode_workspace_bytes(&d, 64, 1, 8193));
  d.d_r = 63;
  CHECK(mla_absorbed_weights_bytes(&d) == 0);
  d = dsv2_dims();
  d.dtype = MLA_F32;
  CHECK(mla_decode_cp_workspace_bytes(&d, 64, 1) == 0);
  d = dsv2_dims();

  /* Status strings. */
  CHECK(strcmp(mla_status_string(MLA_OK), "MLA_OK") == 0);
  CHECK(strcmp(mla_status_string(MLA_ERR_TIMEOUT), "MLA_ERR_TIMEOUT") == 0);
  CHECK(strcmp(mla_status_string(MLA_ERR_DEVICE_BOUNDS), "MLA_ERR_DEVICE_BOUNDS") == 0);

  /* Argument checks that return before any launch. */
  CHECK(mla_absorb_weights(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, &w, NULL) ==
        MLA_ERR_INVALID_ARG);
  CHECK(w == NULL);
  CHECK(mla_append_latent(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, NULL, 1, NULL, 0, NULL) == MLA_ERR_INVALID_ARG);
  CHECK(mla_decode(NULL, NULL, NULL, NULL, 1, 1, NULL, &out, 1, 1, 1, NULL, 0, NULL) == MLA_ERR_INVALID_ARG);
  CHECK(mla_prefill(NULL, NULL, NULL, 1, 1, NULL, &out, 1, 1, NULL, 0, NULL) == MLA_ERR_INVALID_ARG);
  CHECK(mla_decode_cp_partial(NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, NULL, NULL, &out, 1, 1, 1, NULL, 0,
                              NULL) == MLA_ERR_INVALID_ARG);
  CHECK(mla_decode_cp_combine(NULL, 2, NULL, NULL, &out, 1, 1, NULL, 0, NULL) == MLA_ERR_INVALID_ARG);
  CHECK(mla_weights_dims(NULL, &d) == MLA_ERR_INVALID_ARG);
  CHECK(mla_get_error(NULL, NULL) == MLA_ERR_INVALID_ARG);
  mla_release_weights(NULL);

  if (fails) return 1;
  printf("ok\n");
  return 0;
}
