/* Plain C client of libcsa.so: compiles against include/csa.h as C99, links
 * the library, and exercises the host-side paths that need no GPU (version,
 * status strings, workspace arithmetic, argument validation before any launch). */
#include <stdio.h>
#include <string.h>
#include "csa.h"

static int fails = 0;
#define CHECK(cond) do { if (!(cond)) { printf("FAIL %s:%d: %s\n", __FILE__, __LINE__, #cond); ++fails; } } while (0)

int main(void) {
  CHECK(csa_abi_version() == 1);
  CHECK(strcmp(csa_status_string(CSA_OK), "CSA_OK") == 0);
  CHECK(strcmp(csa_status_string(CSA_ERR_INVALID_ARG), "CSA_ERR_INVALID_ARG") == 0);

  /* workspace of the prefill indexer call: the score matrix plus the item counter */
  CHECK(csa_index_topk_workspace(1, 16384, 4096, 512) == (size_t)16384 * 4096 * 4 + 256);
  CHECK(csa_workspace_size(1, 16384, 4096, 512, 64, 512, 1) == csa_index_topk_workspace(1, 16384, 4096, 512));

  /* argument errors are reported before any device work */
  void* p = (void*)(uintptr_t)16;
  CHECK(csa_grouped_out_proj(p, p, p, 4, 64, 512, 7, 1024, 4096, p, p, CSA_BF16, 0) == CSA_ERR_INVALID_ARG);
  CHECK(strstr(csa_last_error(), "divide") != NULL);
  CHECK(strcmp(csa_get_last_error_string(), csa_last_error()) == 0);
  CHECK(csa_grouped_out_proj(p, p, p, 4, 64, 512, 8, 1000, 4096, p, p, CSA_BF16, 0) == CSA_ERR_UNSUPPORTED);
  CHECK(csa_grouped_out_proj(NULL, NULL, NULL, 0, 64, 512, 8, 1024, 4096, NULL, NULL, CSA_F32, 0) == CSA_OK);
  CHECK(csa_rmsnorm_rope(p, CSA_BF16, 10, 100, 1, 0, 1, 64, 10000.f, 1e-6f, p, CSA_BF16, 0) == CSA_ERR_INVALID_ARG);
  CHECK(csa_rmsnorm_rope(NULL, CSA_BF16, 0, 512, 1, 0, 1, 64, 10000.f, 1e-6f, NULL, CSA_BF16, 0) == CSA_OK);

  printf(fails ? "check_abi: %d failure(s)\n" : "check_abi: ok\n", fails);
  return fails != 0;
}
