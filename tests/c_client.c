/* A plain C99 client of libmss.so: it includes include/mss.h, links the
 * library and makes calls that need no GPU (the version, the error strings,
 * workspace-size queries and argument errors, which the library reports
 * before touching any device).  It prints "ok" on success and exits 0. */
#include <stdio.h>
#include <string.h>

#include "mss.h"

static int fail(const char *what) {
    fprintf(stderr, "c client: %s\n", what);
    return 1;
}

int main(void) {
    if (mss_version() != MSS_VERSION) return fail("version mismatch");
    if (!mss_strerror(MSS_ERR_NULL) || strlen(mss_strerror(MSS_ERR_NULL)) == 0) return fail("no error string");
    /* a required pointer missing: reported before any launch */
    if (mss_scan_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, NULL, NULL, 2, 16, 16, 64,
                     MSS_DTYPE_BF16, NULL) != MSS_ERR_NULL)
        return fail("mss_scan_fwd did not report the missing pointers");
    if (mss_state_update(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, NULL, 2, 16, 3,
                         MSS_DTYPE_BF16, NULL) != MSS_ERR_UNSUPPORTED_N)
        return fail("mss_state_update did not reject N = 3");
    if (mss_scan_fwd_workspace_size(1, 16, 16, 4096, 7, 0) != MSS_ERR_DTYPE) return fail("dtype not rejected");
    if (mss_scan_fwd_host_workspace_size(0, 8, 16, 32, MSS_DTYPE_BF16, 0, 0, 0, 0, 0) != 0)
        return fail("empty host call needs a workspace");
    printf("ok\n");
    return 0;
}
