/* Plain C use of the library's C ABI (no Python, no torch): host-only entry points and
 * argument validation.  Built and run by tests/test_c_abi.py; prints one line per result. */
#include <stdio.h>
#include <stdint.h>

#include "rf2.h"

int main(void) {
    rf2_geom g = {1, 40, 21, 45, 80, 128, 2, 8, 8}; /* 720p video grid, 2x8x8 windows */
    printf("kept %d\n", rf2_kept_count(&g, 0.8, 1, 0));
    printf("kept_additive %d\n", rf2_kept_count(&g, 0.8, 1, RF2_SINK_ADDITIVE));
    printf("kept_no_permute %d\n", rf2_kept_count(&g, 0.8, 1, RF2_NO_PERMUTE));
    printf("ws_nonzero %d\n", rf2_workspace_size(&g, 0.8, 1, 0, 1) > 0);
    rf2_v1_params p = {0.25, 2, 0.9, 0, 0, 0.9};
    printf("v1_kmax %d\n", rf2_v1_kmax(&g, &p, 0));
    p.dynamic = 1;
    printf("v1_kmax_dynamic %d\n", rf2_v1_kmax(&g, &p, 0));
    rf2_schedule sc = {10, 0.15, 3};
    printf("schedule");
    for (int s = 0; s < 10; ++s) printf(" %d", rf2_schedule_action(&sc, s));
    printf("\n");
    /* invalid calls are refused on the host, before any device work */
    printf("attention_null %d\n", rf2_attention(NULL, NULL, NULL, &g, 0.8, 1, 0.f, NULL, NULL, NULL, 0, 0, NULL));
    printf("kept_bad_sparsity %d\n", rf2_kept_count(&g, 1.5, 1, 0));
    rf2_geom bad = g;
    bad.D = 96;
    printf("kept_bad_D %d\n", rf2_kept_count(&bad, 0.8, 1, 0));
    printf("status_text %s\n", rf2_status_string(RF2_ERR_UNSUPPORTED));
    return 0;
}
