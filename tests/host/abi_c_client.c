/* A plain C client of libdiffattn.so: includes the boundary header, links the
 * library and calls the entry points that need no GPU (version, lambda_init,
 * workspace sizes and argument validation).  Exit status 0 when every check
 * holds; the failing check's line otherwise. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "diffattn.h"

#define CHECK(cond)                                            \
  do {                                                         \
    if (!(cond)) {                                             \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return __LINE__;                                         \
    }                                                          \
  } while (0)

int main(void) {
  const char* v = diffattn_version();
  CHECK(v != NULL && strstr(v, "sm_100a") != NULL);
  CHECK(fabs(diffattn_lambda_init(1) - 0.2) < 1e-15);
  CHECK(fabs(diffattn_lambda_init(12) - (0.8 - 0.6 * exp(-0.3 * 11))) < 1e-15);

  /* Argument errors come back before any device call, with a message. */
  char buf[64];
  void* p = buf;   /* never dereferenced: validation fails first */
  int rc = diffattn_fwd_v2(p, p, p, (const float*)p, p, DIFFATTN_BF16, 1, 3, 1, 8, 8, 128, 1, NULL);
  CHECK(rc == DIFFATTN_ERR_INVALID_ARG);
  CHECK(strlen(diffattn_last_error()) > 0);
  rc = diffattn_fwd_v1(p, p, p, p, p, (const float*)p, p, DIFFATTN_BF16, 1, 3, 2, 8, 8, 64, 128, 1, 0, 0.f, NULL);
  CHECK(rc == DIFFATTN_ERR_INVALID_ARG);
  rc = diffattn_bwd_v2(p, p, p, (const float*)p, p, (const float*)p, p, p, p, p, (float*)p, DIFFATTN_F32, 1, 4, 2, 8,
                       8, 128, 1, p, 1024, NULL);
  CHECK(rc == DIFFATTN_ERR_UNSUPPORTED);

  /* Workspace sizes are pure functions of the sizes. */
  CHECK(diffattn_decode_v2_workspace_size(2, 63, 8192, 128) == 0);   /* odd Hq: invalid, no device needed */
  CHECK(diffattn_decode_v2_workspace_size(2, 64, -1, 128) == 0);
  CHECK(diffattn_bwd_v2_workspace_size(2, 64, 8192) > 0);
  CHECK(diffattn_bwd_v2_workspace_size(2, 63, 8192) == 0);
  CHECK(diffattn_bwd_v1_workspace_size(8, 16, 16, 4096, 4096, 1) > diffattn_bwd_v1_workspace_size(8, 16, 16, 4096,
                                                                                                  4096, 0));
  CHECK(diffattn_fwd_lowrank_workspace_size(2, 32, 8192, 8192, 16, 1) > 0);
  CHECK(diffattn_fwd_lowrank_workspace_size(2, 32, 8192, 8192, 17, 1) == 0);
  printf("ok\n");
  return 0;
}
