/* Compiled as C99 against include/moe.h and linked to the library: the
 * boundary is plain C (no C++ types), and its host-only calls work without a
 * GPU.  Prints one line per check; exits nonzero on the first failure. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int fail(const char* what) {
    printf("FAIL %s\n", what);
    return 1;
}

int main(void) {
    moe_problem p;
    memset(&p, 0, sizeof(p));
    p.T = 4096;
    p.H = 6144;
    p.E = 256;
    p.I = 2048;
    p.top_k = 8;
    p.num_shared = 1;
    p.routed_scale = 2.827f;
    p.clip_limit = 10.0f;
    p.dtype = MOE_BF16;

    size_t fwd = moe_workspace_size(&p, MOE_CALL_FORWARD);
    size_t fp8 = moe_workspace_size(&p, MOE_CALL_FORWARD_FP8);
    size_t route = moe_workspace_size(&p, MOE_CALL_ROUTE);
    if (fwd == 0 || fp8 == 0 || route == 0) return fail("workspace sizes");
    if (route >= fwd) return fail("route workspace smaller than forward");
    printf("workspace forward=%zu fp8=%zu route=%zu\n", fwd, fp8, route);

    p.top_k = 0; /* outside the supported set */
    if (moe_workspace_size(&p, MOE_CALL_FORWARD) != 0) return fail("bad problem rejected");
    p.top_k = 8;

    const char* s = moe_status_string(MOE_ERR_WORKSPACE);
    if (s == NULL || strlen(s) == 0) return fail("status string");
    printf("status %d: %s\n", (int)MOE_ERR_WORKSPACE, s);

    /* argument validation happens before any CUDA call */
    if (moe_forward(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) !=
        MOE_ERR_INVALID_ARG)
        return fail("null pointers rejected");
    printf("ok\n");
    return 0;
}
