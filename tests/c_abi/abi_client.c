/* A plain C client of liblamp.so: compiled and run by tests/test_abi.py on a
 * machine without a GPU. It uses only include/lamp.h and checks the calls that
 * need no device: the version, the struct sizes, and argument errors returned
 * before any CUDA call. */
#include <stdio.h>
#include <string.h>

#include "lamp.h"

static int fails = 0;
#define CHECK(cond)                                                     \
  do {                                                                  \
    if (!(cond)) {                                                      \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++fails;                                                          \
    }                                                                   \
  } while (0)

int main(void) {
  CHECK(strncmp(lamp_version(), "lamp-b200", 9) == 0);
  CHECK(lamp_args_size() == sizeof(lamp_args));
  CHECK(lamp_gelu_args_size() == sizeof(lamp_gelu_args));
  CHECK(lamp_ln_args_size() == sizeof(lamp_ln_args));

  lamp_dims d = {1, 1, 8, 8, 64};
  char buf[64];
  void *p = (void *)(((size_t)buf + 15) & ~(size_t)15);
  CHECK(lamp_attention(&d, p, p, p, p, NULL, 0, 0.1f, LAMP_STRICT, 1, NULL) == LAMP_ERR_ARG);  /* mu = 0 */
  CHECK(strstr(lamp_last_error(), "mu") != NULL);
  d.d = 80;
  CHECK(lamp_attention(&d, p, p, p, p, NULL, 4, 0.1f, LAMP_STRICT, 1, NULL) == LAMP_ERR_UNSUPPORTED);

  lamp_args a;
  memset(&a, 0, sizeof(a));
  a.dims.B = 1; a.dims.H = 1; a.dims.n_q = 8; a.dims.n_k = 8; a.dims.d = 64;
  a.Q = a.K = a.V = p; a.out = p; a.mu = 4; a.variant = LAMP_GIVEN_MASK; a.causal = 1;
  CHECK(lamp_attention_ex(&a) == LAMP_ERR_ARG);  /* given mask without mask_in */

  lamp_gelu_args g;
  memset(&g, 0, sizeof(g));
  g.M = 4; g.N = 4; g.K = 12; g.x = g.W = p; g.out = p; g.mu = 4; g.tau = 1.0f;
  CHECK(lamp_linear_gelu(&g) == LAMP_ERR_UNSUPPORTED);  /* K not a multiple of 8 */

  lamp_ln_args l;
  memset(&l, 0, sizeof(l));
  l.M = 4; l.N = 9000; l.K = 16; l.x = l.W = p; l.out = p; l.mu = 4; l.tau = 1.0f;
  CHECK(lamp_linear_layernorm(&l) == LAMP_ERR_UNSUPPORTED);  /* N > 8192 */
  CHECK(lamp_ln_workspace_size(16, 32) == 16 * 32 * 4);

  if (fails) return 1;
  printf("abi client ok\n");
  return 0;
}
