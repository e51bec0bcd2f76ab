/* A plain C99 client of libonebit's host-only calls (no GPU needed): the
 * header must compile as C and the calls must link from C.  Prints the
 * results for tests/test_c_abi.py to compare with the Python binding. */
#include <stdio.h>

#include "onebit.h"

int main(void) {
    int64_t numel[3] = {100003, 31, 0}, offs[3], npad = 0, b = 0, e = 0, wb = 0, we = 0;
    size_t ws = 0;
    int cb = 0, ce = 0;
    if (ob_abi_version() != OB_ABI_VERSION) return 1;
    if (ob_layout(3, numel, offs, &npad) != OB_OK) return 2;
    if (ob_chunk_range(numel[0], 8, 3, &b, &e) != OB_OK) return 3;
    if (ob_workspace_bytes(3, numel, 8, &ws) != OB_OK || ws == 0) return 4;
    if (ob_server_shard_range(3, numel, 8, 4, 1, &cb, &ce, &wb, &we) != OB_OK) return 5;
    if (ob_layout(0, numel, offs, &npad) != OB_ERR_INVALID_ARG) return 6;
    if (ob_compressed_step(NULL, NULL) != OB_ERR_INVALID_ARG) return 7;
    printf("%lld %lld %lld %lld %zu %d %d %lld %lld %s\n", (long long)offs[1], (long long)npad,
           (long long)b, (long long)e, ws, cb, ce, (long long)wb, (long long)we,
           ob_status_string(OB_ERR_PHASE));
    return 0;
}
