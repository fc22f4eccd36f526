/* A plain C (C99) consumer of include/wam.h: the header compiles as C, the
 * library links from C, and the entry points that need no device behave as
 * documented (argument errors before any device work). */
#include <stdio.h>
#include <string.h>

#include "wam.h"

static int failures = 0;

#define EXPECT(cond)                                           \
  do {                                                         \
    if (!(cond)) {                                             \
      fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                              \
    }                                                          \
  } while (0)

int main(void) {
  wam_config c;
  memset(&c, 0, sizeof c);
  EXPECT(wam_preset(2, &c) == WAM_OK);
  EXPECT(c.n_blocks == 28 && c.d_video == 1536 && c.d_action == 768 && c.n_heads == 24 && c.head_dim == 64);
  EXPECT(c.l_cond == 64 && c.l_video == 1024 && c.l_action == 32 && c.action_dim == 30 && c.batch == 1);
  EXPECT(c.dtype == WAM_BF16);
  EXPECT(wam_preset(9, &c) == WAM_ERR_INVALID_ARG);
  EXPECT(wam_preset(1, NULL) == WAM_ERR_INVALID_ARG);

  /* a shape the kernels do not cover is rejected before any device work */
  wam_ctx* ctx = NULL;
  EXPECT(wam_preset(2, &c) == WAM_OK);
  c.head_dim = 48;
  EXPECT(wam_init(&c, 0, &ctx) == WAM_ERR_INVALID_ARG && ctx == NULL);
  EXPECT(wam_init(NULL, 0, &ctx) == WAM_ERR_INVALID_ARG);

  /* a NULL context is an argument error, never a crash */
  float t[2] = {1.0f, 0.0f};
  EXPECT(wam_infer_chunk(NULL, NULL, NULL, NULL, NULL, 1, t, WAM_SCHED_CEWP, 1, NULL, NULL) == WAM_ERR_INVALID_ARG);
  EXPECT(wam_action_step(NULL, NULL, 1.0f, 0.0f, NULL) == WAM_ERR_INVALID_ARG);
  EXPECT(strcmp(wam_last_error(NULL), "") == 0);
  wam_destroy(NULL);

  EXPECT(strcmp(wam_status_str(WAM_OK), "ok") == 0);
  EXPECT(wam_status_str(WAM_ERR_TIMEOUT) != NULL);
  if (failures == 0) printf("c abi ok\n");
  return failures == 0 ? 0 : 1;
}
