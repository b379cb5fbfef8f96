/*
 * Plain-C client of include/fr.h: the library's boundary used without Python or C++.
 * Exercises the calls that need no GPU (host number formats, capsule sizing, argument
 * checks); prints "ok" and exits 0 when every check holds.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fr.h"

static int failures = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  /* RoPE tables: position 0 is the identity rotation */
  float c[4 * 8], s[4 * 8];
  CHECK(fr_rope_tables(4, 16, 10000.0, c, s) == FR_OK);
  for (int j = 0; j < 8; ++j) CHECK(c[j] == 1.0f && s[j] == 0.0f);
  CHECK(fabsf(c[8] - cosf(1.0f)) < 1e-6f && fabsf(s[8] - sinf(1.0f)) < 1e-6f);   /* pos 1, j 0: angle 1 */

  /* bf16 rounding: round to nearest even, exact values pass through */
  const float in[4] = {1.0f, 1.00390625f, 1.01171875f, -2.5f};   /* 1 + 2^-8 ties to even (1.0); 1 + 3*2^-8 ties up */
  uint16_t out[4];
  fr_round_bf16(in, out, 4);
  CHECK(out[0] == 0x3F80 && out[1] == 0x3F80 && out[2] == 0x3F82 && out[3] == 0xC020);

  /* 4-bit group quantiser: max |w| maps to 7 */
  float w[128];
  for (int i = 0; i < 128; ++i) w[i] = (float)(i - 64) / 64.0f;
  int8_t q[128];
  uint16_t sb[1];
  CHECK(fr_quantize_w4(w, 1, 128, q, sb) == FR_OK);
  CHECK(q[0] == -7 && q[64] == 0);
  CHECK(fr_quantize_w4(NULL, 1, 128, q, sb) == FR_ERR_ARG);

  /* capsule sizing: K and V [L][B][Hkv][P][dh] bf16, then x, each part 256-byte aligned */
  fr_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.L = 2; cfg.D = 256; cfg.Hq = 4; cfg.Hkv = 1; cfg.dh = 64; cfg.F = 1024; cfg.H = 16; cfg.A = 8;
  cfg.B_max = 2; cfg.P_max = 64; cfg.K = 2; cfg.dtype = FR_DTYPE_BF16; cfg.path = FR_PATH_AUTO;
  cfg.rope_theta = 10000.0f; cfg.eps = 1e-6f; cfg.time_dim = 256; cfg.time_base = 10000.0f;
  const size_t kv = (size_t)2 * 2 * 1 * 64 * 64 * 2;
  CHECK(fr_capsule_bytes(&cfg, 2, 64, 0) == 2 * kv);
  CHECK(fr_capsule_bytes(&cfg, 2, 64, 1) == 2 * kv + 1024);
  CHECK(fr_capsule_bytes(&cfg, 3, 64, 0) == 0);
  CHECK(fr_capsule_bytes(NULL, 1, 1, 0) == 0);

  /* argument checks before any device work */
  fr_handle* h = NULL;
  CHECK(fr_create(NULL, 0, &h) == FR_ERR_ARG && h == NULL);
  CHECK(fr_denoise(NULL, NULL, NULL, 1, NULL) == FR_ERR_ARG);
  CHECK(fr_prefill(NULL, NULL, 1, 1, NULL, NULL) == FR_ERR_ARG);
  CHECK(fr_graph_count(NULL) == FR_ERR_ARG);
  CHECK(strlen(fr_last_error()) > 0);
  fr_destroy(NULL);

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
