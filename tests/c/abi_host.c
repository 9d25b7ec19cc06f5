/* Host-only use of the C ABI from plain C (no GPU needed): the header compiles as C, the library
 * links, and the size queries, the CG table and the error reporting answer as documented.
 * Prints one line per check; exits non-zero on the first failure. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "e3b.h"

static int fails = 0;
#define CHECK(cond, what)                      \
  do {                                         \
    if (!(cond)) {                             \
      printf("FAIL %s\n", what);               \
      fails++;                                 \
    } else {                                   \
      printf("ok %s\n", what);                 \
    }                                          \
  } while (0)

int main(void) {
  size_t bytes = 0;
  CHECK(e3_csr_workspace_size(3000, 156278, &bytes) == E3_OK && bytes > 0, "csr workspace size");
  CHECK(e3_backward_workspace_size(3000, &bytes) == E3_OK && bytes >= 16 + 4 * 3000, "backward workspace size");
  CHECK(e3_conv_topology_size(3000, 156278, &bytes) == E3_OK && bytes % 256 == 0, "topology size");
  CHECK(e3_morton_workspace_size(3000, &bytes) == E3_OK && bytes > 0, "morton workspace size");
  CHECK(e3_csr_workspace_size(-1, 5, &bytes) == E3_ERR_SHAPE && strlen(e3_last_error()) > 0, "error message");

  /* the 1 x 1 -> 1 real CG block: proportional to the cross product, Frobenius norm 1 */
  double cg[27];
  CHECK(e3_cg_dense(1, 1, 1, cg) == E3_OK, "cg table call");
  double norm = 0.0, diag = 0.0;
  for (int i = 0; i < 27; ++i) norm += cg[i] * cg[i];
  for (int i = 0; i < 3; ++i) diag += fabs(cg[i * 9 + i * 3 + 0]) + fabs(cg[i * 9 + i * 3 + 1]) + fabs(cg[i * 9 + i * 3 + 2]);
  CHECK(fabs(norm - 1.0) < 1e-12 && diag < 1e-15, "cg 1x1->1 normalised, zero when two indices agree");
  CHECK(e3_cg_dense(1, 1, 3, cg) == E3_ERR_INSTRUCTION || e3_cg_dense(1, 1, 3, cg) != E3_OK, "cg triangle rule");
  CHECK(strlen(e3_supported()) > 0, "supported list");
  return fails != 0;
}
