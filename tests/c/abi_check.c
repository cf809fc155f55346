/* Plain-C client of libsvg_b200.so: includes svg.h, links the library and
 * exercises the calls that need no GPU (version, workspace sizes, the
 * epsilon schedule, and argument validation that rejects before any
 * launch).  Exits 0 when every check holds. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "svg.h"

static int failures = 0;

#define CHECK(cond, what)                                    \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "FAIL: %s (%s)\n", what, svg_last_error()); \
      ++failures;                                            \
    }                                                        \
  } while (0)

int main(void) {
  /* never dereferenced: every call below is rejected on the host */
  void* fake = (void*)(uintptr_t)(1u << 20);
  void* fake2 = (void*)(uintptr_t)(2u << 20);

  CHECK(strstr(svg_version(), "sm_100a") != NULL, "version names sm_100a");
  CHECK(svg_profile_workspace_size(1, 2, 256, 64, 16) > 0, "profile workspace size");
  CHECK(svg_block_energy_workspace_size(1, 2, 256) >= 2 * 256 * sizeof(float),
        "energy workspace holds one lse per row");
  CHECK(svg_row_similarity_workspace_size(SVG_BF16, 1, 2, 4, 16, 1) > 0,
        "row similarity workspace size");

  double eps[5];
  CHECK(svg_epsilon_schedule(5, 0.99, 0.84, eps) == SVG_OK, "epsilon schedule");
  CHECK(fabs(eps[0] - 0.99) < 1e-15 && fabs(eps[4] - 0.84) < 1e-15, "schedule end points");
  CHECK(fabs(eps[2] - sqrt(0.99 * 0.84)) < 1e-15, "schedule midpoint is the geometric mean");
  CHECK(svg_epsilon_schedule(3, 1.5, 0.84, eps) == SVG_ERR_INVALID_ARG, "threshold > 1 rejected");

  /* d = 96 is not supported: rejected before launch, with a message */
  svg_status st = svg_sparse_attn(fake, fake, fake, fake2, SVG_BF16, 1, 2, 256, 96, fake, 3, 2,
                                  fake, fake, 0.f, NULL, NULL, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG && strstr(svg_last_error(), "d=96") != NULL, "d=96 rejected");
  /* a successful host-only call clears the error text */
  CHECK(svg_epsilon_schedule(1, 0.9, 0.9, eps) == SVG_OK && svg_last_error()[0] == '\0',
        "last error cleared");
  st = svg_permute_token_major(fake, fake, SVG_BF16, 1, 2, 12, 64, 3, 4, NULL, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG, "in-place permutation rejected");
  st = svg_qk_norm_rope(fake, fake2, fake, fake2, NULL, NULL, SVG_BF16, 1, 2, 256, 64, 0, 0,
                        SVG_QK_NORM | SVG_QK_ROPE, NULL, NULL, 1e-6f, NULL, NULL, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG && strstr(svg_last_error(), "cos and sin") != NULL,
        "RoPE without tables rejected");
  st = svg_row_broadcast(fake, SVG_BF16, 1, 2, 256, 64, 4, 4, 15, 5, fake2, 3, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG, "frame shape that does not tile N rejected");
  /* the temporal-heads copy needs the modes */
  st = svg_permute_temporal_heads(fake, fake2, SVG_BF16, 1, 2, 12, 64, 3, 4, NULL, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG && strstr(svg_last_error(), "mode is required") != NULL,
        "temporal-heads copy without modes rejected");
  /* pairing order: one bitmap word per 32 key blocks, per row and list */
  CHECK(svg_pair_query_tiles_workspace_size(2, 5, 33) == 2 * 5 * 2 * sizeof(uint32_t),
        "pairing workspace size");
  CHECK(svg_pair_query_tiles_workspace_size(0, 5, 33) == 0, "pairing workspace of no lists");
  st = svg_pair_query_tiles(fake, fake2, 2, 5, 33, fake, NULL, fake2, 4, NULL);
  CHECK(st == SVG_ERR_INVALID_ARG && strstr(svg_last_error(), "workspace") != NULL,
        "short pairing workspace rejected");

  if (failures == 0) printf("c abi ok: %s\n", svg_version());
  return failures == 0 ? 0 : 1;
}
