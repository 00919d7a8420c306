/* Plain-C use of the libaal boundary without any GPU work: the host-side
 * table query, the product counts, argument checking and status strings.
 * Built and run by tests/test_abi_cpu.py with gcc; prints one line per check
 * and exits non-zero on the first mismatch. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "aal.h"

static int fail(const char* what) {
  printf("FAIL %s\n", what);
  return 1;
}

int main(void) {
  /* Q_3: S(i, i) = {i}, S(i, k) = {i, k} */
  uint8_t S[27];
  if (aal_block_table(AAL_LAW_Q, 3, S) != AAL_OK) return fail("table status");
  for (int i = 0; i < 3; ++i)
    for (int k = 0; k < 3; ++k)
      for (int a = 0; a < 3; ++a) {
        const int want = (a == i || a == k) ? 1 : 0;
        if (S[(i * 3 + k) * 3 + a] != want) return fail("table entry");
      }
  printf("table ok\n");
  if (aal_block_product_count(AAL_LAW_Q, 2, 0) != 6) return fail("count q=2 square");
  if (aal_block_product_count(AAL_LAW_Q, 5, 1) != 9) return fail("count q=5 row");
  if (aal_block_product_count(AAL_LAW_Q2XQ2, 4, 1) != 9) return fail("count Q2xQ2 row");
  if (aal_block_product_count(AAL_LAW_Q2XQ2, 4, 0) != 36) return fail("count Q2xQ2 square");
  printf("counts ok\n");
  /* a decode call without positions is rejected before anything runs */
  aal_mat x = {(void*)0x10000, AAL_BF16, 4, 8, 8};
  aal_mat W = {(void*)0x20000, AAL_BF16, 8, 8, 8};
  aal_mat y = {(void*)0x30000, AAL_BF16, 4, 8, 8};
  if (aal_decode_matvec(AAL_LAW_Q, 2, NULL, x, W, y, NULL) != AAL_ERR_INVALID_ARG)
    return fail("decode argument check");
  printf("argument check ok\n");
  if (strlen(aal_status_string(AAL_OK)) == 0) return fail("status string");
  printf("version %d\n", (int)aal_version());
  return 0;
}
