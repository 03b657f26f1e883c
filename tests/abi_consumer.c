/* A plain C11 program built against include/mlra.h and linked with libmlra.so.
 * It shows that the header is C (not only C++), that every entry point links
 * under its declared type, and that argument validation answers without a
 * GPU: each call below is rejected before anything is enqueued.  Exit status
 * 0 means every check held; otherwise the failing check is printed. */
#include <stdio.h>
#include <string.h>

#include "mlra.h"

static int failures = 0;

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
      ++failures;                                                \
    }                                                            \
  } while (0)

/* Every entry point the header declares: each must be declared for a C
 * caller (an undeclared name fails to compile under -Werror) and must link. */
static void* const entry_points[] = {
    (void*)mlra_workspace_bytes,  (void*)mla_decode,           (void*)mlra_decode,
    (void*)mlra_decode_profiled,  (void*)mlra_decode_host_workspace_bytes,
    (void*)mlra_decode_host,      (void*)latent_append_workspace_bytes,
    (void*)latent_append,         (void*)latent_store,         (void*)latent_append_noalloc,
    (void*)mlra_selftest_wait_timeout, (void*)mlra_check_status, (void*)mlra_last_error,
    (void*)mlra_shutdown,         (void*)mlra_version,          (void*)mlra_describe_plan,
    (void*)mlra_attend_partial,   (void*)mlra_merge_workspace_bytes, (void*)mlra_merge_upproj,
    (void*)mlra_quantize_pages_fp8, (void*)mlra_decode_fp8,
};

static mlra_dims dims_dsv2(void) {
  mlra_dims d;
  memset(&d, 0, sizeof d);
  d.B = 4;
  d.H = 128;
  d.d_h = 128;
  d.d_v = 128;
  d.d_c = 512;
  d.d_r = 64;
  d.n_branch = 1;
  d.page_size = 64;
  d.max_pages_per_seq = 8;
  d.num_pages = 32;
  d.branch_scale = 1.0f;
  d.dtype = MLRA_BF16;
  d.num_splits = 74;
  d.kernel = MLRA_KERNEL_AUTO;
  return d;
}

int main(void) {
  for (size_t i = 0; i < sizeof entry_points / sizeof entry_points[0]; ++i) CHECK(entry_points[i] != NULL);
  CHECK(mlra_version() == 1);

  /* NULL dims: no workspace size, and a message */
  CHECK(mlra_workspace_bytes(NULL) == 0);
  CHECK(strlen(mlra_last_error()) > 0);

  /* valid dims with explicit split count: a size without touching a device */
  mlra_dims d = dims_dsv2();
  CHECK(mlra_workspace_bytes(&d) > 0);

  /* odd RoPE width: rejected as an invalid argument */
  d.d_r = 63;
  void* fake = (void*)(size_t)(1u << 20); /* aligned, never dereferenced on this path */
  const int32_t* ifake = (const int32_t*)fake;
  mlra_status st = mla_decode(&d, fake, fake, ifake, fake, fake, fake, fake, ifake, ifake, fake, fake,
                              (size_t)1 << 30, (cudaStream_t)0);
  CHECK(st == MLRA_ERR_INVALID_ARG);
  CHECK(strstr(mlra_last_error(), "d_r") != NULL);

  /* MLA entry point with two branches: rejected */
  d = dims_dsv2();
  d.n_branch = 2;
  st = mla_decode(&d, fake, fake, ifake, fake, fake, fake, fake, ifake, ifake, fake, fake, (size_t)1 << 30,
                  (cudaStream_t)0);
  CHECK(st == MLRA_ERR_INVALID_ARG);

  /* page size other than 64: valid in principle, not implemented */
  d = dims_dsv2();
  d.page_size = 32;
  CHECK(mlra_workspace_bytes(&d) == 0);

  /* too small a workspace: reported as such */
  d = dims_dsv2();
  const size_t need = mlra_workspace_bytes(&d);
  st = mlra_decode(&d, fake, fake, ifake, fake, fake, fake, fake, ifake, ifake, fake, fake, need - 256,
                   (cudaStream_t)0);
  CHECK(st == MLRA_ERR_WORKSPACE);

  /* append with a zero model width: no workspace size */
  CHECK(latent_append_workspace_bytes(&d, 0) == 0);

  if (failures) return 1;
  printf("ok %zu entry points\n", sizeof entry_points / sizeof entry_points[0]);
  return 0;
}
