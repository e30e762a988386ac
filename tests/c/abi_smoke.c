/* Plain C (C99) use of the C ABI in include/muon.h, with no GPU: the entry points that need no
 * device must answer, argument errors must come back as status codes, and the workspace size of
 * a parameter set must be printed for the test to compare with the Python binding. */
#include <stdio.h>
#include <string.h>

#include "muon.h"

static int fails = 0;
#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++fails;                                                   \
    }                                                            \
  } while (0)

int main(void) {
  muon_shape_t shapes[3] = {{1536, 1536}, {1536, 6144}, {6144, 1536}};
  size_t bytes = 0;
  CHECK(muon_workspace_size(shapes, 3, MUON_BF16, MUON_MODE_FAST, &bytes) == MUON_OK);
  CHECK(bytes > 0 && bytes % 1024 == 0);
  printf("workspace %zu\n", bytes);

  /* argument errors are status codes, never crashes */
  CHECK(muon_workspace_size(NULL, 3, MUON_BF16, MUON_MODE_FAST, &bytes) == MUON_ERR_INVALID_ARG);
  CHECK(muon_workspace_size(shapes, 0, MUON_BF16, MUON_MODE_FAST, &bytes) == MUON_ERR_INVALID_ARG);
  muon_shape_t bad = {0, 5};
  CHECK(muon_workspace_size(&bad, 1, MUON_BF16, MUON_MODE_FAST, &bytes) == MUON_ERR_INVALID_ARG);
  CHECK(muon_step(NULL, NULL, NULL, NULL, NULL, 0) == MUON_ERR_INVALID_ARG);
  CHECK(muon_destroy(NULL) == MUON_ERR_INVALID_ARG);

  /* every status has a name */
  for (int s = MUON_OK; s <= MUON_ERR_NO_DEVICE; ++s) {
    const char* name = muon_status_string((muon_status_t)s);
    CHECK(name != NULL && strlen(name) > 0);
  }
  /* creating a handle without a device reports it instead of failing silently */
  muon_handle_t h = NULL;
  muon_status_t st = muon_create(&h, shapes, 3, MUON_BF16, MUON_MODE_FAST, NULL, bytes);
  CHECK(st != MUON_OK && h == NULL);
  printf("create without workspace: %s\n", muon_status_string(st));
  return fails == 0 ? 0 : 1;
}
