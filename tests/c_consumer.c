/* A plain C program that uses the library only through include/sdm.h: it
 * checks that the header compiles as C (C11), that the ABI version matches,
 * and that host-side validation and the workspace queries answer without a
 * GPU. Built and run by tests/test_c_consumer.py. */
#include <stdio.h>
#include <string.h>

#include "sdm.h"

static int fails = 0;
#define CHECK(cond)                                           \
  do {                                                        \
    if (!(cond)) {                                            \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++fails;                                                \
    }                                                         \
  } while (0)

int main(void) {
  CHECK(sdm_abi_version() == SDM_ABI_VERSION);
  CHECK(strcmp(sdm_status_string(SDM_OK), "ok") == 0);

  sdm_shape_t s;
  memset(&s, 0, sizeof s);
  s.B = 2; s.T = 300; s.H = 2; s.sqrt_n = 32; s.W = 64; s.R = 64; s.d_v = 128;
  s.in_dtype = SDM_BF16; s.state_dtype = SDM_F32; s.rms_eps = 1e-6f; s.variant = SDM_VARIANT_AUTO;

  /* Workspace sizes are pure host arithmetic. */
  CHECK(sdm_scan_workspace_bytes(&s) > 0);
  CHECK(sdm_layer_forward_workspace_bytes(&s) > sdm_scan_workspace_bytes(&s));
  CHECK(sdm_layer_step_workspace_bytes(&s) == sdm_layer_forward_workspace_bytes(&s));
  CHECK(sdm_scan_backward_workspace_bytes(&s) > 0);
  CHECK(sdm_layer_backward_workspace_bytes(&s) > sdm_scan_backward_workspace_bytes(&s));

  /* Invalid shapes and arguments are refused before any CUDA call. */
  sdm_shape_t bad = s;
  bad.sqrt_n = 0;
  CHECK(sdm_scan_workspace_bytes(&bad) == 0);
  CHECK(sdm_layer_forward(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
        SDM_ERR_INVALID_ARGUMENT);
  CHECK(strstr(sdm_last_error(), "sqrt_n") != NULL);
  CHECK(sdm_pkm_topk(NULL, SDM_F32, 1, 1, 1, 4, 3, NULL, NULL, NULL) == SDM_ERR_INVALID_ARGUMENT);
  CHECK(strstr(sdm_last_error(), "scores") != NULL);
  CHECK(sdm_slot_counts(NULL, 1, 4, 1, 0, 64, NULL, NULL) == SDM_ERR_INVALID_ARGUMENT);
  /* Empty problems are no-ops. */
  CHECK(sdm_pkm_topk(NULL, SDM_F32, 0, 7, 3, 4, 3, NULL, NULL, NULL) == SDM_OK);

  /* The decode launch count is host logic too. */
  sdm_shape_t dec = s;
  dec.T = 1;
  CHECK(sdm_layer_step_launches(&dec) == 1);
  dec.R = 32;
  CHECK(sdm_layer_step_launches(&dec) == 4);

  if (fails == 0) printf("c consumer ok\n");
  return fails == 0 ? 0 : 1;
}
