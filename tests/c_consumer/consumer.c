/* A plain C99 consumer of the library: it compiles against include/wush.h with no
 * C++ and no CUDA headers, links libwush.so and makes host-only calls (no GPU).
 * Exit status 0 means every check passed; the first failing check's line is printed. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "wush.h"

#define CHECK(c)                                      \
  do {                                                \
    if (!(c)) {                                       \
      fprintf(stderr, "check failed line %d: %s\n", __LINE__, #c); \
      return 1;                                       \
    }                                                 \
  } while (0)

/* splitmix64, for seeded inputs */
static unsigned long long sm_state = 0x5EEDull;
static double uniform01(void) {
  unsigned long long z = (sm_state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (double)(z >> 11) * (1.0 / 9007199254740992.0);
}

int main(int argc, char** argv) {
  const char* path = argc > 1 ? argv[1] : "consumer.wush";
  /* formats and sizes */
  CHECK(wush_block_size(WUSH_FMT_MXFP4) == 32 && wush_block_size(WUSH_FMT_NVFP4) == 16);
  CHECK(wush_codes_bytes(300, 256, WUSH_FMT_MXFP4) == 300 * 128);
  CHECK(wush_scales_bytes(300, 256, WUSH_FMT_MXFP4) == 3 * 2 * 512);  /* 128 x 4 atoms */
  CHECK(wush_scales_bytes(300, 256, WUSH_FMT_INT4) == 300 * 8 * 2);
  CHECK(strcmp(wush_status_string(WUSH_ERR_TIMEOUT), "a bounded device wait gave up") == 0);

  /* calibrate a 64-wide layer with 16-blocks, from seeded data */
  enum { N_CAL = 256, D_OUT = 96, D_IN = 64, B = 16, NB = D_IN / B };
  float* x = malloc(sizeof(float) * N_CAL * D_IN);
  float* w = malloc(sizeof(float) * D_OUT * D_IN);
  float* tx = malloc(sizeof(float) * NB * B * B);
  float* tw = malloc(sizeof(float) * NB * B * B);
  CHECK(x && w && tx && tw);
  for (int i = 0; i < N_CAL * D_IN; ++i) x[i] = (float)(2.0 * uniform01() - 1.0) * (i % D_IN == 5 ? 30.f : 1.f);
  for (int i = 0; i < D_OUT * D_IN; ++i) w[i] = (float)(0.04 * uniform01() - 0.02);
  CHECK(wush_calibrate(x, N_CAL, w, D_OUT, D_IN, B, WUSH_T_WUSH, tx, tw) == WUSH_OK);
  /* T_W^T T_X = I per block */
  double worst = 0.0;
  for (int j = 0; j < NB; ++j)
    for (int r = 0; r < B; ++r)
      for (int c = 0; c < B; ++c) {
        double s = 0.0;
        for (int k = 0; k < B; ++k) s += (double)tw[(j * B + k) * B + r] * tx[(j * B + k) * B + c];
        worst = fmax(worst, fabs(s - (r == c ? 1.0 : 0.0)));
      }
  CHECK(worst < 1e-4);
  /* a non-finite calibration value is refused */
  x[17] = NAN;
  CHECK(wush_calibrate(x, N_CAL, w, D_OUT, D_IN, B, WUSH_T_WUSH, tx, tw) == WUSH_ERR_INVALID_ARG);

  /* checkpoint round trip */
  CHECK(wush_save_transforms(path, B, WUSH_T_WUSH, WUSH_NORM_MEAN, NB, tx, tw, NULL, 0) == WUSH_OK);
  int blk = 0, kind = 0, norm = 0, has_index = 1;
  int64_t n_t = 0, n_blocks = 0;
  CHECK(wush_transforms_file_info(path, &blk, &kind, &norm, &n_t, &n_blocks, &has_index) == WUSH_OK);
  CHECK(blk == B && kind == WUSH_T_WUSH && norm == WUSH_NORM_MEAN && n_t == NB && n_blocks == NB && !has_index);
  float* lx = malloc(sizeof(float) * NB * B * B);
  float* lw = malloc(sizeof(float) * NB * B * B);
  CHECK(lx && lw);
  CHECK(wush_load_transforms(path, lx, lw, NB * B * B - 1, NULL, 0) == WUSH_ERR_BUFFER_TOO_SMALL);
  CHECK(wush_load_transforms(path, lx, lw, NB * B * B, NULL, 0) == WUSH_OK);
  CHECK(memcmp(lx, tx, sizeof(float) * NB * B * B) == 0 && memcmp(lw, tw, sizeof(float) * NB * B * B) == 0);

  /* a device entry point refuses a bad shape before touching the device */
  CHECK(wush_qgemm((const uint8_t*)16, (const void*)16, (const uint8_t*)16, (const void*)16, 100, 256, 256,
                   WUSH_FMT_MXFP4, 1.0f, (float*)16, NULL) == WUSH_ERR_INVALID_ARG);
  free(x); free(w); free(tx); free(tw); free(lx); free(lw);
  printf("c consumer ok\n");
  return 0;
}
