/*
 * A plain C11 consumer of the library's C ABI (include/qlora_nf4.h): it compiles
 * against the header alone and links libqlora_nf4.so, with no Python and no
 * PyTorch in between.  It runs without a GPU, so it calls only what needs no
 * device: version and status strings, the NF4 level table, the storage sizes,
 * the workspace size, the wait-limit setter, and the argument checks that every
 * entry point makes before it launches anything.
 * Exit status: the number of failed checks.
 */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "qlora_nf4.h"

static int failures = 0;

#define CHECK(cond)                                                        \
  do {                                                                     \
    if (!(cond)) {                                                         \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                          \
    }                                                                      \
  } while (0)

/* Stand-ins for device pointers: never dereferenced, only checked for NULL and
 * alignment by the entry points before they launch. */
#define PTR(a) ((void *)(uintptr_t)(a))

int main(void) {
  CHECK(qlora_version() > 0);
  for (int s = QLORA_OK; s <= QLORA_ERR_NO_DEVICE; ++s) {
    const char *t = qlora_status_string((qlora_status)s);
    CHECK(t != NULL && strlen(t) > 0);
  }

  /* the level table: 16 ascending levels, 7 negative, an exact zero, 8 positive, in [-1, 1] */
  float L[16];
  qlora_nf4_levels(L);
  CHECK(L[0] == -1.0f && L[7] == 0.0f && L[15] == 1.0f);
  for (int i = 1; i < 16; ++i) CHECK(L[i] > L[i - 1]);

  /* storage: n/2 + n/64 + 4 n/16384 bytes, rounded up per array */
  size_t cb = 0, qb = 0, sb = 0;
  CHECK(qlora_nf4_bytes(4096, 4096, &cb, &qb, &sb) == 8388608u + 262144u + 4096u);
  CHECK(cb == 8388608u && qb == 262144u && sb == 4096u);
  CHECK(qlora_nf4_bytes(1, 65, &cb, &qb, &sb) == 33u + 2u + 4u);
  CHECK(qlora_nf4_bytes(3, 5, NULL, NULL, NULL) == 8u + 1u + 4u);
  /* single-level constants: one fp32 per 64-value block */
  CHECK(qlora_nf4_single_bytes(4096, 4096, &cb, &sb) == 8388608u + 4u * 262144u);
  CHECK(qlora_nf4_single_bytes(1, 65, NULL, NULL) == 33u + 8u);

  /* workspace: positive for a valid call, 0 for an invalid one */
  CHECK(qlora_linear_workspace_bytes(4096, 4096, 4096, 16) > 0);
  CHECK(qlora_linear_workspace_bytes(0, 4096, 4096, 16) == 0);

  /* the wait limit round-trips */
  const uint32_t old = qlora_set_wait_limit_us(1234);
  CHECK(qlora_set_wait_limit_us(old) == 1234);

  /* argument errors are returned before anything is launched */
  qlora_nf4_t none = {NULL, NULL, NULL, 4, 4};
  CHECK(qlora_nf4_quantize(NULL, 4, 4, &none, NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_nf4_dequant(&none, PTR(16), NULL) == QLORA_ERR_INVALID_ARG);
  qlora_nf4_t skew = {PTR(16), PTR(18), PTR(32), 128, 128};   /* q8 not 16-byte aligned */
  CHECK(qlora_nf4_dequant(&skew, PTR(64), NULL) == QLORA_ERR_MISALIGNED);

  qlora_nf4_t w = {PTR(16), PTR(32), PTR(48), 128, 128};
  const int bad_r[] = {0, 4, 12, 136};
  for (int i = 0; i < 4; ++i)
    CHECK(qlora_linear_fwd(PTR(16), 4, &w, PTR(16), PTR(16), bad_r[i], 1.0f, PTR(16), NULL, PTR(16),
                           1u << 20, NULL) == QLORA_ERR_INVALID_ARG);
  qlora_nf4_t odd = {PTR(16), PTR(32), PTR(48), 100, 128};    /* N not a multiple of the tile */
  CHECK(qlora_linear_fwd(PTR(16), 4, &odd, PTR(16), PTR(16), 8, 1.0f, PTR(16), NULL, PTR(16), 1u << 20,
                         NULL) == QLORA_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlora_linear_fwd(PTR(18), 4, &w, PTR(16), PTR(16), 8, 1.0f, PTR(16), NULL, PTR(16), 1u << 20,
                         NULL) == QLORA_ERR_MISALIGNED);
  CHECK(qlora_linear_fwd(PTR(16), 4, &w, PTR(16), PTR(16), 8, NAN, PTR(16), NULL, PTR(16), 1u << 20,
                         NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_linear_bwd(NULL, PTR(16), NULL, 4, &w, PTR(16), PTR(16), 8, 1.0f, NULL, PTR(16), PTR(16),
                         PTR(16), 1u << 20, NULL) == QLORA_ERR_INVALID_ARG);
  /* merge: exactly one base, r a multiple of 8 in [8, 128], N % 8 == 0, K % 64 == 0 */
  CHECK(qlora_nf4_merge(NULL, NULL, 128, 128, PTR(16), PTR(16), 16, 1.0f, PTR(16), NULL) ==
        QLORA_ERR_INVALID_ARG);
  CHECK(qlora_nf4_merge(&w, PTR(16), 128, 128, PTR(16), PTR(16), 16, 1.0f, PTR(16), NULL) ==
        QLORA_ERR_INVALID_ARG);
  CHECK(qlora_nf4_merge(NULL, PTR(16), 128, 128, PTR(16), PTR(16), 12, 1.0f, PTR(16), NULL) ==
        QLORA_ERR_INVALID_ARG);
  CHECK(qlora_nf4_merge(NULL, PTR(16), 100, 128, PTR(16), PTR(16), 16, 1.0f, PTR(16), NULL) ==
        QLORA_ERR_UNSUPPORTED_SHAPE);
  CHECK(qlora_nf4_merge(NULL, PTR(16), 128, 128, PTR(16), PTR(16), 16, 1.0f, PTR(24), NULL) ==
        QLORA_ERR_MISALIGNED);
  CHECK(qlora_selftest_wait_timeout(0, NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_get_device_status(NULL, NULL) == QLORA_ERR_INVALID_ARG);
  CHECK(qlora_profile_read(0, NULL, NULL) == 0);   /* nothing recorded: profiling never enabled */

  if (failures == 0) printf("abi_consumer: all checks passed\n");
  return failures;
}
