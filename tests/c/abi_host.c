/* Links against libhstu.so through include/hstu.h only (no Python) and calls
 * the entry points that run on the host: version, workspace sizing, the
 * Stochastic Length keep count, and argument checks that return before any
 * launch.  Prints one line per check; exits non-zero on the first failure. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "hstu.h"

#define CHECK(cond, what)                                   \
  do {                                                      \
    if (!(cond)) {                                          \
      printf("FAIL %s\n", what);                            \
      return 1;                                             \
    }                                                       \
    printf("ok %s\n", what);                                \
  } while (0)

int main(void) {
  CHECK(hstu_version() >= 1, "version");
  hstu_layer_desc d;
  memset(&d, 0, sizeof d);
  d.d_model = 1024;
  d.n_heads = 8;
  d.d_qk = 128;
  d.d_v = 128;
  d.n_pos_buckets = 128;
  d.n_time_buckets = 128;
  d.pos_sub_bits = 4;
  d.time_sub_bits = 2;
  d.ln_eps = 1e-6f;
  d.dtype = HSTU_BF16;
  const size_t ws = hstu_workspace_size(&d, 8, 128, 42157, 776, 0, 0, 0);
  CHECK(ws > 0 && ws % 256 == 0, "stack workspace size");
  CHECK(hstu_sl_keep_count(4096) == 776 && hstu_sl_keep_count(0) == 0 &&
            hstu_sl_keep_count(-1) == -1,
        "keep count");
  CHECK(hstu_retrieval_workspace_size(128, 1000000, 1024, 100, 1) > (size_t)128 * 1000000 * 4,
        "retrieval workspace size");
  CHECK(hstu_transformer_workspace_size(512, 8, 2048, 16, 82351) > 0 &&
            hstu_transformer_workspace_size(500, 8, 2048, 16, 82351) == 0,
        "transformer workspace size");
  const int64_t before = hstu_launch_count();
  /* null offsets: rejected on the host */
  hstu_layer_weights w;
  memset(&w, 0, sizeof w);
  CHECK(hstu_layer_fwd(&d, 2, 10, 8, NULL, (void*)0x1000, &w, (void*)0x1000, (void*)0x2000,
                       (void*)0x10000, 1 << 20, NULL) == HSTU_ERR_INVALID_ARG,
        "layer rejects null offsets");
  CHECK(hstu_bf16_to_f16((void*)0x1000, (void*)0x2000, 7, NULL) == HSTU_ERR_INVALID_ARG,
        "conversion rejects a length not a multiple of 8");
  CHECK(hstu_launch_count() == before, "nothing launched");
  CHECK(strlen(hstu_status_string(HSTU_ERR_BAD_IDS)) > 0, "status strings");
  return 0;
}
