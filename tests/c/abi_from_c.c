/*
 * The C ABI used from plain C: include/ulysses.h compiles as C11 with every
 * warning an error, libulysses.so links, and the host-side calls behave as
 * the header documents.  Built and run by tests/test_c_abi.py.
 *
 *   abi_from_c              workspace queries and status strings (no device
 *                           memory is touched: safe on any host)
 *   abi_from_c --refusals   also bad arguments, with null or fake device
 *                           addresses that a correct library never touches;
 *                           run only on a host without a GPU
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ulysses.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static void queries(void) {
  const uly_shape s = {1, 1024, 32, 8, 128, 4};
  uly_shape bad = s;
  /* status word (256 B) plus the per-token sample start and end tables */
  CHECK(ulysses_attn_fwd_workspace(&s) >= 256 + 2 * 4 * 1024);
  CHECK(ulysses_attn_bwd_workspace(&s, ULY_F32) >= ulysses_attn_fwd_workspace(&s));
  bad.n = 1001; /* not a multiple of P: no workspace size */
  CHECK(ulysses_attn_fwd_workspace(&bad) == 0);
  CHECK(ulysses_attn_bwd_workspace(&bad, ULY_BF16) == 0);
  CHECK(ulysses_attn_fwd_workspace(NULL) == 0);
  CHECK(strcmp(ulysses_status_string(ULY_OK), "ok") == 0);
  for (int c = ULY_OK; c <= ULY_ERR_TIMEOUT; ++c) {
    const char* text = ulysses_status_string((uly_status)c);
    CHECK(text != NULL && strcmp(text, "unknown status") != 0);
  }
  CHECK(strcmp(ulysses_status_string((uly_status)99), "unknown status") == 0);
}

static void refusals(void) {
  char* const F = (char*)(uintptr_t)0x100000; /* fake, 256-byte aligned, never dereferenced */
  const int64_t G = (int64_t)1 << 30;
  const uly_shape s = {1, 1024, 32, 8, 128, 4};
  uly_shape odd = s;
  int32_t code = -1;
  float* lse = (float*)(F + 5 * G);
  odd.n = 1002; /* n % P != 0 */

  CHECK(ulysses_seq_to_head(NULL, F, 1, 64, 8, 64, 4, ULY_BF16, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_seq_to_head(F, F + G, 1, 62, 8, 64, 4, ULY_BF16, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_head_to_seq(F, F + 1, 1, 64, 8, 64, 4, ULY_BF16, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_kv_seq_to_head(F, F + G, 1, 64, 3, 64, 4, ULY_BF16, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_transpose_runs(F, F + 32, 2, 2, 16, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_attn_fwd(F, F + G, F + 2 * G, (const int64_t*)(F + 3 * G), &odd, -1, 0.f, F + 4 * G, ULY_F32,
                         lse, F + 6 * G, (size_t)1 << 24, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_attn_fwd(F, F + G, F + 2 * G, (const int64_t*)(F + 3 * G), &s, 4, 0.f, F + 4 * G, ULY_F32,
                         lse, F + 6 * G, (size_t)1 << 24, NULL) == ULY_ERR_INVALID_ARG); /* rank >= P */
  CHECK(ulysses_attn_fwd(F, F + G, F + 2 * G, (const int64_t*)(F + 3 * G), &s, -1, 0.f, F + 4 * G, ULY_F32,
                         lse, F + 6 * G, 16, NULL) == ULY_ERR_WORKSPACE);
  CHECK(ulysses_attn_fwd_kv_range(F, F + G, F + 2 * G, (const int64_t*)(F + 3 * G), &s, -1, 0.f, 5, 5, F + 4 * G,
                                  ULY_F32, lse, F + 6 * G, (size_t)1 << 24, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_attn_lse_merge((const float*)F, (const float*)(F + G), 0, &s, F + 2 * G, ULY_F32,
                               (float*)(F + 3 * G), NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_attn_bwd_timed(F, F + G, F + 2 * G, F + 3 * G, ULY_F32, lse, F + 4 * G,
                               (const int64_t*)(F + 6 * G), &s, -1, 0.f, F + 7 * G, F + 8 * G, F + 9 * G, ULY_F32,
                               F + 10 * G, (size_t)1 << 24, NULL, NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_sp_loss_aggregate((const float*)F, (const int64_t*)(F + G), 1, 64, 0, -100, (float*)(F + 2 * G),
                                  (int64_t*)(F + 3 * G), (float*)(F + 4 * G), NULL) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_workspace_status(NULL, NULL, &code) == ULY_ERR_INVALID_ARG);
  CHECK(ulysses_workspace_status(F + 16, NULL, &code) == ULY_ERR_INVALID_ARG); /* not 256-byte aligned */
}

int main(int argc, char** argv) {
  queries();
  if (argc > 1 && strcmp(argv[1], "--refusals") == 0) refusals();
  if (failures) fprintf(stderr, "%d check(s) failed\n", failures);
  else printf("ok\n");
  return failures ? 1 : 0;
}
