/* A plain C99 client of the library's C ABI (include/qlora.h), built by
 * tests/test_c_abi.py with -std=c99 -pedantic -Werror (and as C++ to check the
 * extern "C" block) and linked against libqlora.so.  It calls only the host
 * side of the ABI, so it runs without a GPU, and prints what it got, one
 * "key value..." line each, for the test to compare with the oracle and the
 * Python binding. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "qlora.h"

static uint32_t bits(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return u;
}

int main(void) {
  float lv[16], th[15];
  int i, fmt;
  if (qlora_nf4_codebook(lv) != QLORA_OK) return 1;
  printf("nf4");
  for (i = 0; i < 16; ++i) printf(" %08x", (unsigned)bits(lv[i]));
  printf("\n");
  for (fmt = QLORA_FORMAT_NF4; fmt <= QLORA_FORMAT_INT4; ++fmt) {
    if (qlora_format_codebook(fmt, lv, th) != QLORA_OK) return 2;
    printf("levels%d", fmt);
    for (i = 0; i < 16; ++i) printf(" %08x", (unsigned)bits(lv[i]));
    printf("\nthresh%d", fmt);
    for (i = 0; i < 15; ++i) printf(" %08x", (unsigned)bits(th[i]));
    printf("\n");
  }
  /* argument errors come back before anything touches a device */
  printf("bad_format %d\n", (int)qlora_format_codebook(7, lv, th));
  printf("null_levels %d\n", (int)qlora_format_codebook(QLORA_FORMAT_NF4, NULL, th));
  printf("null_codebook %d\n", (int)qlora_nf4_codebook(NULL));
  printf("sizes %zu %zu %zu %zu\n", qlora_codes_bytes(4096, 11008), qlora_absmax_bytes(4096, 11008),
         qlora_group_scale_bytes(4096, 11008), qlora_group_scale_bytes_dq(4096, 11008, QLORA_DQ_SIGNED));
  printf("ws %zu %zu %zu\n", qlora_workspace_bytes(QLORA_OP_FWD, 4096, 11008, 4096, 64),
         qlora_workspace_bytes(QLORA_OP_BWD, 4096, 11008, 4096, 64),
         qlora_workspace_min_bytes(QLORA_OP_FWD, 4096, 11008, 4096, 64));
  printf("status %s|%s\n", qlora_status_string(QLORA_OK), qlora_status_string(QLORA_ERR_INVALID_ARG));
  return 0;
}
