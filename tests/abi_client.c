/* A plain C client of libcalibatt.so: compiled by tests/test_abi.py with gcc -std=c99
 * against include/calibatt.h and linked to the library, with no Python or torch.  It
 * calls the entry points whose answers are decided on the host (status strings, the
 * anchor count, argument validation) and the full sizing path of the API, and exits 0
 * when every answer is the documented one; otherwise it prints the failing check. */
#include <stdio.h>
#include <string.h>

#include "calibatt.h"

static int failures = 0;

static void expect(int cond, const char* what) {
    if (!cond) {
        printf("FAIL: %s\n", what);
        ++failures;
    }
}

int main(void) {
    void* fake = (void*)(uintptr_t)256;          /* aligned, never dereferenced on error */
    const int32_t* rp = (const int32_t*)fake;
    const int16_t* ci = (const int16_t*)fake;
    calib_block_list bl = {1, 1, 1, 128, rp, ci, NULL, 0};
    calib_block_list bl_bad = {1, 2, 2, 128, rp, ci, NULL, 0};
    uint8_t rep[1] = {1};

    expect(strcmp(calib_status_string(CALIB_OK), "CALIB_OK") == 0, "status string OK");
    expect(strcmp(calib_status_string(CALIB_ERR_TIMEOUT), "CALIB_ERR_TIMEOUT") == 0, "status string TIMEOUT");

    /* anchors: 21 frames x ceil(45/4) latent rows x 80 columns; stride 0 is invalid */
    expect(calib_anchor_count(21, 45, 80, 0, 4) == 21 * 12 * 80, "anchor count wan14b");
    expect(calib_anchor_count(4, 8, 16, 0, 2) == 256, "anchor count tiny");
    expect(calib_anchor_count(1, 1, 1, 0, 0) == -1, "anchor count stride 0");

    /* selection: null energy, tau outside (0, 1], nk beyond 1024 */
    expect(calib_select_mask(NULL, 1, 1, 1, 0.9, NULL, NULL, NULL, NULL) == CALIB_ERR_INVALID, "select null");
    expect(calib_select_mask((const float*)fake, 1, 1, 1, 0.0, NULL, (uint8_t*)fake, NULL, NULL) ==
               CALIB_ERR_INVALID, "select tau 0");
    expect(calib_select_mask((const float*)fake, 1, 1, 1025, 0.9, NULL, (uint8_t*)fake, NULL, NULL) ==
               CALIB_ERR_UNSUPPORTED, "select nk 1025");

    /* vote: rho above 1 */
    expect(calib_aggregate_masks((const int32_t*)fake, 1, 1, 1, 3, 3, 2, (uint8_t*)fake, NULL) ==
               CALIB_ERR_INVALID, "vote rho > 1");

    /* energies: block size 96, misaligned q, N beyond the supported 131072 tokens */
    expect(calib_block_energy(fake, fake, NULL, 1, 128, 128, 96, 0.1f, NULL, 0, (float*)fake, 0, NULL) ==
               CALIB_ERR_INVALID, "energy block 96");
    expect(calib_block_energy((void*)(uintptr_t)258, fake, NULL, 1, 128, 128, 128, 0.1f, NULL, 0, (float*)fake, 0,
                              NULL) == CALIB_ERR_INVALID, "energy misaligned q");
    expect(calib_block_energy(fake, fake, NULL, 1, 131073, 128, 128, 0.1f, NULL, 0, (float*)fake, 0, NULL) ==
               CALIB_ERR_UNSUPPORTED, "energy N beyond limit");

    /* attention: no list, head dim 96, list shape mismatch, negative scale, unknown flags */
    expect(sparse_attn_fwd(fake, fake, fake, fake, NULL, 1, 128, 128, 0.1f, NULL, 0, NULL) == CALIB_ERR_INVALID,
           "attn no list");
    expect(sparse_attn_fwd(fake, fake, fake, fake, NULL, 1, 128, 96, 0.1f, &bl, 0, NULL) == CALIB_ERR_UNSUPPORTED,
           "attn D 96");
    expect(sparse_attn_fwd(fake, fake, fake, fake, NULL, 1, 128, 128, 0.1f, &bl_bad, 0, NULL) == CALIB_ERR_INVALID,
           "attn list shape");
    expect(sparse_attn_fwd(fake, fake, fake, fake, NULL, 1, 128, 128, -1.0f, &bl, 0, NULL) == CALIB_ERR_INVALID,
           "attn negative scale");
    expect(sparse_attn_fwd(fake, fake, fake, fake, NULL, 1, 128, 128, 0.1f, &bl, 6u, NULL) == CALIB_ERR_INVALID,
           "attn unknown flags");
    expect(sparse_attn_fwd_repeat(fake, fake, fake, fake, NULL, 1, 128, 1, 1, 128, 0, 1, NULL, 0.1f, &bl, 0,
                                  NULL) == CALIB_ERR_INVALID, "repeat without head flags");

    /* host-buffer attention: null host pointer, chunk size 0 */
    expect(sparse_attn_fwd_host(NULL, fake, fake, fake, fake, fake, fake, fake, NULL, 1, 128, 128, 0.1f, &bl, 0, 1,
                                NULL, NULL, NULL) == CALIB_ERR_INVALID, "host attn null q_host");
    expect(sparse_attn_fwd_host(fake, fake, fake, fake, fake, fake, fake, fake, NULL, 1, 128, 128, 0.1f, &bl, 0, 0,
                                NULL, NULL, NULL) == CALIB_ERR_INVALID, "host attn chunk 0");
    expect(sparse_attn_fwd_repeat_host(fake, fake, fake, fake, fake, fake, fake, fake, NULL, 1, 128, 1, 1, 128, 0, 1,
                                       rep, 0.1f, &bl_bad, 0, 1, NULL, NULL, NULL) == CALIB_ERR_INVALID,
           "host repeat list shape");

    /* batched selection: no output, too many entries, a tau outside (0, 1] */
    {
        double taus[2] = {0.9, 1.5};
        expect(calib_select_mask_batched((const float*)fake, 1, 1, 1, 1, taus, NULL, NULL, NULL, NULL) ==
                   CALIB_ERR_INVALID, "batched select without outputs");
        expect(calib_select_mask_batched((const float*)fake, 257, 1, 1, 1, taus, NULL, (uint8_t*)fake, NULL, NULL) ==
                   CALIB_ERR_INVALID, "batched select 257 entries");
        expect(calib_select_mask_batched((const float*)fake, 2, 1, 1, 1, taus, NULL, (uint8_t*)fake, NULL, NULL) ==
                   CALIB_ERR_INVALID, "batched select tau 1.5");
    }
    /* energy mean: zero inputs */
    expect(calib_energy_mean((const float*)fake, 4, 0, (float*)fake, NULL) == CALIB_ERR_INVALID, "mean 0 inputs");

    /* host-side skip-list check: a valid 2 x 2 list, then an index past nk and a bad work item */
    {
        int32_t rp2[3] = {0, 2, 3};
        int16_t ci2[3] = {0, 1, 1};
        int32_t wk[2] = {1, 0};
        int32_t wk_bad[2] = {1, 2};
        int16_t ci_bad[3] = {0, 2, 1};
        expect(calib_validate_block_list_host(1, 2, 2, rp2, ci2, 3, wk, 2) == CALIB_OK, "valid list");
        expect(calib_validate_block_list_host(1, 2, 2, rp2, ci_bad, 3, wk, 2) == CALIB_ERR_INVALID, "index >= nk");
        expect(calib_validate_block_list_host(1, 2, 2, rp2, ci2, 3, wk_bad, 2) == CALIB_ERR_INVALID, "work i >= nq");
        expect(calib_validate_block_list_host(1, 2, 2, rp2, ci2, 2, wk, 2) == CALIB_ERR_INVALID, "beyond capacity");
    }

    if (failures == 0) printf("ok\n");
    return failures == 0 ? 0 : 1;
}
