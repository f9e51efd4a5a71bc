/*
 * A plain C99 user of the library: includes include/vdit.h, links libvdit.so
 * and checks calls whose arguments the library rejects before it touches CUDA
 * (so it runs without a GPU).  Prints one line per failed check and exits with
 * the number of failures.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "vdit.h"

static int fails = 0;

static void expect(const char* what, int got, int want) {
  if (got != want) {
    printf("FAIL %s: got %d (%s), want %d\n", what, got, vdit_status_string(got), want);
    ++fails;
  }
}

int main(void) {
  /* 16-byte aligned addresses that are never dereferenced: every call below returns first */
  void* const fake = (void*)(uintptr_t)0x7f0000000000ull;
  void* const mis = (void*)(uintptr_t)(0x7f0000000000ull + 8);

  if (vdit_version() != 10100) { printf("FAIL version %d\n", vdit_version()); ++fails; }
  for (int s = 0; s <= VDIT_ERR_TIMEOUT; ++s)
    if (vdit_status_string(s) == NULL || strlen(vdit_status_string(s)) == 0) {
      printf("FAIL status string %d\n", s);
      ++fails;
    }

  expect("patchify null", vdit_patchify_3d(NULL, fake, VDIT_F32, 1, 4, 8, 16, 16, 1, 2, 2, NULL), VDIT_ERR_NULL);
  expect("patchify dtype", vdit_patchify_3d(fake, fake, 7, 1, 4, 8, 16, 16, 1, 2, 2, NULL), VDIT_ERR_UNSUPPORTED);
  expect("patchify shape", vdit_patchify_3d(fake, fake, VDIT_BF16, 0, 4, 8, 16, 16, 1, 2, 2, NULL),
         VDIT_ERR_SHAPE);

  expect("rope null", vdit_rope_3d(NULL, fake, fake, fake, 1, 5, 30, 52, 40, 128, 44, 42, 42, 10000.f, NULL),
         VDIT_ERR_NULL);
  expect("rope split", vdit_rope_3d(fake, fake, fake, fake, 1, 5, 30, 52, 40, 128, 44, 42, 40, 10000.f, NULL),
         VDIT_ERR_SHAPE);
  expect("rope align", vdit_rope_3d(mis, fake, fake, fake, 1, 5, 30, 52, 40, 128, 44, 42, 42, 10000.f, NULL),
         VDIT_ERR_ALIGN);

  expect("full null", vdit_attn_full(NULL, fake, fake, fake, NULL, 1, 256, 2, 128, 0.f, NULL), VDIT_ERR_NULL);
  expect("full align", vdit_attn_full(fake, fake, mis, fake, NULL, 1, 256, 2, 128, 0.f, NULL), VDIT_ERR_ALIGN);
  expect("full head_dim", vdit_attn_full(fake, fake, fake, fake, NULL, 1, 256, 2, 48, 0.f, NULL),
         VDIT_ERR_UNSUPPORTED);
  expect("full shape", vdit_attn_full(fake, fake, fake, fake, NULL, 1, -5, 2, 128, 0.f, NULL), VDIT_ERR_SHAPE);
  expect("time null", vdit_attn_divided_time(fake, NULL, fake, fake, NULL, 1, 21, 1560, 40, 128, 0.f, NULL),
         VDIT_ERR_NULL);
  expect("time shape", vdit_attn_divided_time(fake, fake, fake, fake, NULL, 1, 0, 1560, 40, 128, 0.f, NULL),
         VDIT_ERR_SHAPE);
  expect("space head_dim",
         vdit_attn_divided_space(fake, fake, fake, fake, NULL, 1, 21, 1560, 40, 96, 0.f, NULL),
         VDIT_ERR_UNSUPPORTED);
  expect("cross key length", vdit_attn_cross(fake, fake, fake, fake, NULL, 1, 256, 0, 2, 128, 0.f, NULL),
         VDIT_ERR_SHAPE);
  expect("cross lse align",
         vdit_attn_cross(fake, fake, fake, fake, (float*)((char*)fake + 2), 1, 256, 77, 2, 128, 0.f, NULL),
         VDIT_ERR_ALIGN);
  expect("watchdog self-test site", vdit_watchdog_selftest(0, NULL), VDIT_ERR_SHAPE);
  expect("rope K only", vdit_rope_3d(NULL, fake, NULL, mis, 1, 5, 30, 52, 40, 128, 44, 42, 42, 10000.f, NULL),
         VDIT_ERR_ALIGN);
  expect("rope half Q", vdit_rope_3d(NULL, fake, fake, fake, 1, 5, 30, 52, 40, 128, 44, 42, 42, 10000.f, NULL),
         VDIT_ERR_NULL);
  if (vdit_rope_3d_table_entries(21, 30, 52, 128, 44, 42, 42) != 2184) {
    printf("FAIL table entries\n");
    ++fails;
  }
  expect("table split", vdit_rope_3d_table((float*)fake, 21, 30, 52, 128, 44, 42, 40, 10000.f, NULL),
         VDIT_ERR_SHAPE);
  expect("rope-q table null",
         vdit_attn_full_rope_q(fake, fake, fake, fake, NULL, 1, 5, 30, 52, 40, 128, 0.f, 44, 42, 42, NULL, NULL, 0,
                               1e-6f, NULL),
         VDIT_ERR_NULL);
  expect("rope-q token group",
         vdit_attn_full_rope_q(fake, fake, fake, fake, NULL, 1, 5, 30, 52, 40, 128, 0.f, 44, 42, 42, (float*)fake,
                               NULL, 5120, 1e-6f, NULL),
         VDIT_ERR_UNSUPPORTED);
  return fails;
}
