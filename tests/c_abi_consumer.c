/*
 * c_abi_consumer.c -- a plain C11 program that uses libattn.so through
 * include/attn.h only (test infrastructure; built and run by
 * tests/test_c_abi.py).  It makes no call that needs a GPU: host-only helpers,
 * and calls whose arguments are invalid, which the library must reject before
 * touching any CUDA API.  Prints one "name value" line per check and exits 0
 * when every check holds.
 */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "attn.h"

static int failures = 0;

static void check(const char* name, long long got, long long want) {
  printf("%s %lld\n", name, got);
  if (got != want) {
    fprintf(stderr, "FAIL %s: got %lld, want %lld\n", name, got, want);
    ++failures;
  }
}

int main(void) {
  /* accounting helpers: N(N+1)/2 kept pairs causal, one block per causal tile pair */
  check("unmasked_pairs_causal_4096", attn_unmasked_pairs(4096, 1, 0, 0), 4096LL * 4097 / 2);
  check("unmasked_pairs_full_100", attn_unmasked_pairs(100, 0, 0, 0), 100LL * 100);
  check("visited_blocks_causal_4096", attn_visited_blocks(4096, 1, 0, 0), 32 * 33 / 2);
  check("unmasked_pairs_bad", attn_unmasked_pairs(-1, 1, 0, 0), -1);
  check("unit_kind_c3", attn_fwd_unit_kind(4, 16, 16, 4096, 0, 0, 148), 0);
  check("unit_kind_c2", attn_fwd_unit_kind(2, 8, 8, 1024, 0, 0, 148), 1);
  check("unit_kind_c5", attn_fwd_unit_kind(8, 32, 1, 8192, 1024, 0, 148), 2);
  check("unit_kind_bad", attn_fwd_unit_kind(1, 4, 3, 64, 0, 0, 148), ATTN_ERR_INVALID_ARG);

  /* the pages' ALiBi slopes for H = 8 are 2^-1 .. 2^-8, exact in float */
  float slopes[8];
  check("alibi_slopes_rc", attn_alibi_slopes(8, slopes), ATTN_OK);
  int exact = 1;
  for (int h = 0; h < 8; ++h) exact &= slopes[h] == ldexpf(1.0f, -(h + 1));
  check("alibi_slopes_exact", exact, 1);
  check("alibi_slopes_bad", attn_alibi_slopes(0, slopes), ATTN_ERR_INVALID_ARG);

  /* workspace queries */
  check("bwd_workspace_f32", attn_bwd_workspace_bytes(1, 1, 64, 64, ATTN_BF16 | ATTN_OUT_F32), 256);
  check("bwd_workspace_16", attn_bwd_workspace_bytes(1, 1, 64, 64, ATTN_BF16), 256 + 64 * 64 * 4);
  /* 8 groups: at most ceil(148 / 8) + 1 = 20 parts of 4 rows, each an LSE
     (2560 bytes in all, already 256-aligned) and a 128-wide fp32 row */
  check("decode_workspace", attn_decode_workspace_bytes(4, 8, 2, 1, 200, 128),
        2560 + 20 * 8 * 4 * 128 * 4);

  /* invalid calls are rejected before any CUDA call */
  check("fwd_null", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 64, 64, 1, 0, 0, 0.125f,
                             ATTN_BF16, NULL), ATTN_ERR_INVALID_ARG);
  check("fwd_empty", attn_fwd(NULL, NULL, NULL, NULL, NULL, 0, 1, 1, 64, 64, 1, 0, 0, 0.125f,
                              ATTN_BF16, NULL), ATTN_OK);
  check("fwd_bad_d", attn_fwd((void*)0x1000, (void*)0x2000, (void*)0x3000, (void*)0x4000, NULL,
                              1, 1, 1, 64, 48, 1, 0, 0, 0.125f, ATTN_BF16, NULL),
        ATTN_ERR_UNSUPPORTED);
  check("bwd_null_o", attn_bwd((void*)0x100000, (void*)0x200000, (void*)0x300000, NULL,
                               (void*)0x500000, (float*)0x600000, NULL, (void*)0x700000,
                               (void*)0x800000, (void*)0x900000, (void*)0xA00000, 1 << 20,
                               1, 1, 1, 64, 64, 1, 0, 0, 0.125f, ATTN_BF16, NULL),
        ATTN_ERR_INVALID_ARG);
  check("decode_nq_gt_nkv", attn_decode((void*)0x1000, (void*)0x2000, (void*)0x3000,
                                        (void*)0x4000, NULL, NULL, 0, 1, 8, 2, 5, 4, 128, 1, 0,
                                        0, 0.1f, ATTN_BF16, NULL),
        ATTN_ERR_INVALID_ARG);

  /* status names */
  check("error_string_ok", strlen(attn_error_string(ATTN_OK)) > 0, 1);
  check("error_string_unknown", attn_error_string(12345) != NULL, 1);

  printf("failures %d\n", failures);
  return failures == 0 ? 0 : 1;
}
