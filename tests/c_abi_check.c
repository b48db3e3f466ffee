/*
 * c_abi_check.c -- the boundary seen from plain C (C11, no C++ and no torch): compiled
 * against include/dsa.h and linked to libdsa.so by tests/test_c_abi.py.  It checks that
 * the header is valid C, that every declared entry point links, and that the calls that
 * need no GPU behave as the header documents (argument errors are returned before
 * anything touches a device).  Prints "OK" and exits 0 on success.
 */
#include <stdio.h>
#include <string.h>

#include "dsa.h"

static int fails = 0;

static void check(int cond, const char* what) {
    if (!cond) {
        printf("failed: %s\n", what);
        ++fails;
    }
}

int main(void) {
    /* every entry point, so that the link step proves each one is exported */
    void* volatile entry[] = {
        (void*)dsa_status_string, (void*)dsa_last_error, (void*)dsa_version,
        (void*)dsa_indexer_scores, (void*)dsa_topk_select, (void*)dsa_index_select,
        (void*)dsa_index_select_workspace_size, (void*)dsa_sparse_mla_fwd,
        (void*)dsa_sparse_mla_workspace_size, (void*)dsa_sparse_mla_decode_noalloc,
        (void*)dsa_index_varlen, (void*)dsa_index_varlen_workspace_size,
        (void*)dsa_sparse_mla_fp8_fwd, (void*)dsa_latent_quantize_fp8, (void*)dsa_layer_stack,
        (void*)dsa_layer_stack_workspace_size, (void*)dsa_pattern_from_freq,
        (void*)dsa_selftest_wait_timeout, (void*)dsa_check_device_errors,
        (void*)dsa_launch_count, (void*)dsa_reset_launch_counts};
    for (size_t i = 0; i < sizeof(entry) / sizeof(entry[0]); ++i) check(entry[i] != NULL, "entry");

    check((dsa_version() >> 16) == 1, "ABI major version 1");
    check(strcmp(dsa_status_string(DSA_ERR_WORKSPACE), "DSA_ERR_WORKSPACE") == 0, "status string");

    char pat[8];
    check(dsa_pattern_from_freq(3, 7, pat, 8) == DSA_OK && strcmp(pat, "FSSFSSF") == 0,
          "index_topk_freq 3 over 7 layers");
    check(dsa_pattern_from_freq(0, 7, pat, 8) == DSA_ERR_INVALID_ARG, "freq 0 rejected");
    check(dsa_pattern_from_freq(2, 8, pat, 8) == DSA_ERR_INVALID_ARG, "no room for the NUL");

    /* ld_idx < k: refused before any launch, with a message */
    check(dsa_topk_select((const float*)16, 64, 4, 0, NULL, 64, 8, (int*)16, 4, NULL) ==
              DSA_ERR_INVALID_ARG && strlen(dsa_last_error()) > 0,
          "top-k argument error");
    /* kv_scale must be finite and positive */
    check(dsa_latent_quantize_fp8((const void*)16, 8, 0.0f, (void*)16, NULL) ==
              DSA_ERR_INVALID_ARG, "quantize with kv_scale 0");
    check(dsa_latent_quantize_fp8((const void*)16, 0, 0.01f, (void*)16, NULL) == DSA_OK,
          "empty quantize is a no-op");

    check(dsa_sparse_mla_workspace_size(DSA_PREFILL, 10, 16, 512, 2048) == 0,
          "prefill needs no workspace");
    check(dsa_layer_stack_workspace_size(1000, 16) == (size_t)16 * 1000 * 4, "stack workspace");
    check(dsa_index_varlen_workspace_size(100, 7) == (size_t)7 * 100 * 4, "varlen workspace");

    dsa_reset_launch_counts();
    check(dsa_launch_count(DSA_KERNEL_INDEXER) == 0 && dsa_launch_count(99) == -1,
          "launch counters");

    printf("%s\n", fails ? "FAIL" : "OK");
    return fails ? 1 : 0;
}
