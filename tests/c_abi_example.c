/* A plain C99 caller of the library's C ABI: compiles against include/sv.h
 * alone, links libsv.so, and uses only calls that do no CUDA work (sizes,
 * strings, and argument errors, which are returned before anything is
 * launched), so it runs on a machine without a GPU. */
#include <stdio.h>
#include <string.h>

#include "sv.h"

int main(void) {
    if (sv_version() < 1) return 1;
    if (sv_verify_workspace_bytes(256, 8, 129280, SV_BF16) == 0) return 2;
    if (sv_verify_workspace_bytes(0, 8, 100, SV_F32) != 0) return 3;
    if (sv_verify(NULL, NULL, SV_BF16, 4, 4, 100, NULL, NULL, NULL, 0u, 0, NULL, NULL, NULL, 0,
                  NULL, NULL) != SV_ERR_ARG)
        return 4;
    sv_vp_slice s;
    memset(&s, 0, sizeof s);
    if (sv_vp_stats_bytes(&s) != 0) return 5;
    s.dtype = SV_BF16; s.B = 4; s.K = 4; s.V = 1000; s.v0 = 0; s.Vs = 500; s.nshards = 2; s.shard = 0;
    if (sv_vp_stats_bytes(&s) != (size_t)4 * 9 * 16) return 6;
    if (sv_verify_host_workspace_bytes(4, 4, 1000, SV_F32) == 0) return 7;
    if (strcmp(sv_status_string(SV_ERR_WORKSPACE), "SV_ERR_WORKSPACE") != 0) return 8;
    printf("c abi ok\n");
    return 0;
}
