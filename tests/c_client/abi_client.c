/* A plain C99 client of libbsattn.so, compiled and run by tests/test_c_client.py without
 * a GPU.  It uses only calls that need no device: workspace sizes, status strings and
 * argument checks that fail on the host before anything is launched.  It prints one line
 * per operation, "<op> <workspace bytes>", for the 720p Wan-14B-like shape and a small
 * ragged one, then the results of the rejection checks. */
#include <stdio.h>
#include <string.h>

#include "bsattn.h"

static int expect(const char* what, bsa_status got, bsa_status want) {
  if (got != want) {
    printf("FAIL %s: %d (%s), expected %d\n", what, (int)got, bsa_status_string(got), (int)want);
    return 1;
  }
  return 0;
}

int main(void) {
  bsa_shape shapes[2];
  bsa_shape bad;
  int ops[5] = {BSA_OP_BLOCK_MASS, BSA_OP_TOPP_SELECT, BSA_OP_FWD, BSA_OP_PATTERN,
                BSA_OP_POOLED_MASS};
  int i, o, fails = 0;
  float mass_dummy[4];
  memset(shapes, 0, sizeof shapes);
  /* batch, heads, head_dim, T, H, W, Tp, Hp, Wp, q_block, kv_block */
  shapes[0].batch = 1; shapes[0].heads = 40; shapes[0].head_dim = 128;
  shapes[0].T = 21; shapes[0].H = 45; shapes[0].W = 80;
  shapes[0].Tp = 24; shapes[0].Hp = 48; shapes[0].Wp = 80;
  shapes[0].q_block = 64; shapes[0].kv_block = 64;
  shapes[1] = shapes[0];
  shapes[1].batch = 2; shapes[1].heads = 3; shapes[1].head_dim = 64;
  shapes[1].T = 6; shapes[1].H = 10; shapes[1].W = 11;
  shapes[1].Tp = 8; shapes[1].Hp = 12; shapes[1].Wp = 12; shapes[1].q_block = 128;
  for (i = 0; i < 2; ++i)
    for (o = 0; o < 5; ++o)
      printf("shape%d op%d %lu\n", i, ops[o], (unsigned long)bsa_workspace_bytes(&shapes[i], ops[o]));

  bad = shapes[0];
  bad.head_dim = 96;
  if (bsa_workspace_bytes(&bad, BSA_OP_FWD) != 0) { printf("FAIL head_dim 96 sized\n"); ++fails; }
  bad = shapes[0];
  bad.Tp = 22;  /* not a multiple of 4 */
  if (bsa_workspace_bytes(&bad, BSA_OP_BLOCK_MASS) != 0) { printf("FAIL Tp 22 sized\n"); ++fails; }
  if (bsa_workspace_bytes(NULL, BSA_OP_FWD) != 0) { printf("FAIL null shape sized\n"); ++fails; }

  fails += expect("block_mass null q", bsa_block_mass(&shapes[0], NULL, NULL, 0.088f, mass_dummy,
                                                      NULL, 0, NULL), BSA_ERR_INVALID_ARG);
  fails += expect("block_mass Tp 22", bsa_block_mass(&bad, NULL, NULL, 0.088f, NULL, NULL, 0,
                                                     NULL), BSA_ERR_INVALID_ARG);
  bad = shapes[0];
  bad.head_dim = 96;
  fails += expect("block_mass head_dim 96", bsa_block_mass(&bad, NULL, NULL, 0.088f, NULL, NULL,
                                                           0, NULL), BSA_ERR_UNSUPPORTED);
  fails += expect("clear_status null", bsa_clear_status(NULL, NULL), BSA_ERR_INVALID_ARG);
  if (strlen(bsa_status_string(BSA_ERR_TIMEOUT)) == 0) { printf("FAIL empty status string\n"); ++fails; }
  printf("status %s\n", bsa_status_string(BSA_ERR_CAPACITY));
  printf("fails %d\n", fails);
  return fails == 0 ? 0 : 1;
}
