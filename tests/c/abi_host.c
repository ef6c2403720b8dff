/*
 * Host-only use of libalspec.so from plain C (no Python): compiled against
 * include/alspec.h by tests/test_c_abi.py, which compares what it prints
 * with the ctypes binding's view of the same calls.  No CUDA call that needs
 * a GPU is made: workspace sizing, planning, argument checks and status
 * strings only.
 */
#include <stdio.h>
#include <string.h>

#include "alspec.h"

int main(void) {
    alspec_desc d;
    memset(&d, 0, sizeof d);
    d.batch = 1;
    d.n_q_heads = 32;
    d.n_kv_heads = 8;
    d.head_dim = 128;
    d.max_seq_len = 131072;
    d.dtype = ALSPEC_BF16;
    printf("sizeof_desc %zu\n", sizeof(alspec_desc));
    printf("version %d\n", alspec_version());
    for (int sch = ALSPEC_SCHEDULE_AUTO; sch <= ALSPEC_SCHEDULE_SINK_FIRST; ++sch) {
        d.schedule = sch;
        int info[12];
        const alspec_status st = alspec_query_plan(&d, 4, 1024, info, 12);
        printf("schedule %d status %d workspace %zu plan", sch, (int)st,
               alspec_workspace_size(&d, 4, 1024));
        for (int i = 0; i < 12; ++i) printf(" %d", info[i]);
        printf("\n");
    }
    int scratch[11];
    d.schedule = 7;
    printf("bad_schedule %d\n", (int)alspec_query_plan(&d, 4, 1024, scratch, 11));
    d.schedule = ALSPEC_SCHEDULE_AUTO;
    d.n_q_heads = 12; /* not a multiple of 8 KV heads */
    printf("bad_heads %d\n", (int)alspec_query_plan(&d, 4, 1024, scratch, 11));
    printf("status_string %s\n", alspec_status_string(ALSPEC_ERR_WORKSPACE));
    return 0;
}
