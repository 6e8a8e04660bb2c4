/* The C ABI used from plain C (no C++, no torch): host-only entry points.
 * Built and run by tests/test_abi_host.py::test_c_program_uses_the_abi. Prints "ok" and
 * exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "fourier_attention.h"

#define CHECK(c)                                                  \
  do {                                                            \
    if (!(c)) {                                                   \
      printf("check failed at line %d: %s\n", __LINE__, #c);       \
      return 1;                                                   \
    }                                                             \
  } while (0)

int main(void) {
  /* LLaMA-3-8B-shaped layer: B = 2, 32 query heads, 8 KV heads, L = 4096, S = 32, R = 64 */
  fa_shape shape = {2, 32, 8, 128, 4096, 32, 64, 255};
  static uint8_t mask[8 * 128];
  for (int g = 0; g < 8; ++g)
    for (int d = 0; d < 128; ++d) mask[g * 128 + d] = (uint8_t)(d >= 32); /* 96 compressed */
  fa_plan plan;
  CHECK(fa_plan_init(&shape, mask, &plan) == FA_OK);
  CHECK(plan.S == 32 && plan.R == 64 && plan.M == 4000 && plan.P == 4000 && plan.G == 4);
  CHECK(plan.dc[0] == 96 && plan.de[0] == 32 && plan.perm[0][0] == 32 && plan.perm[0][96] == 0);
  CHECK(plan.c_elems == 2LL * 8 * 255 * 96);
  CHECK(plan.f_elems == 2LL * 8 * 96 * 128);

  /* room for 1000 appended tokens: E grows to P rows, C and F do not */
  const long long e0 = plan.e_elems, c0 = plan.c_elems;
  CHECK(fa_plan_reserve(&plan, 5096) == FA_OK);
  CHECK(plan.P == 5000 && plan.phi_ld == 5000 && plan.c_elems == c0);
  CHECK(plan.e_elems * 4000 == e0 * 5000);
  CHECK(fa_plan_reserve(&plan, 6000) == FA_ERR_UNSUPPORTED); /* reserved once only */
  CHECK(strlen(fa_last_error()) > 0);

  /* a plan without room refuses an append before touching any pointer */
  fa_plan fresh;
  CHECK(fa_plan_init(&shape, mask, &fresh) == FA_OK);
  fa_cache cache = {0, 0, 0, 0, 0, 0};
  CHECK(fa_append(&fresh, (void*)0x1000, (void*)0x1000, &cache, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fresh.M == 4000 && fresh.shape.L == 4096);

  /* dim selection from host scores: the 96 lowest of each KV head are compressed */
  static float scores[8 * 128];
  for (int g = 0; g < 8; ++g)
    for (int d = 0; d < 128; ++d) scores[g * 128 + d] = (float)((d * 37 + g) % 128);
  static uint8_t sel[8 * 128];
  CHECK(fa_select_dims(scores, 8, 96, sel) == FA_OK);
  for (int g = 0; g < 8; ++g) {
    int n = 0;
    for (int d = 0; d < 128; ++d) {
      n += sel[g * 128 + d];
      CHECK(sel[g * 128 + d] == (scores[g * 128 + d] < 96.0f));
    }
    CHECK(n == 96);
  }
  CHECK(fa_select_dims(scores, 8, 129, sel) == FA_ERR_INVALID);
  printf("ok\n");
  return 0;
}
