/* A plain C caller of libzero.so: builds the plan of the GPT-2-small-shaped
 * workload (124,439,808 parameters, Nd = 8, stage 2, 25M-element buckets)
 * and of a three-unit stage-3 plan, and prints what the C ABI reports, one
 * "key value" pair per line, for the test that compares it with the oracle.
 * Host calls only: it needs no GPU. */
#include <stdio.h>
#include <string.h>

#include "zero.h"

static int check(zero_status_t s, const char *what) {
    if (s != ZERO_OK) {
        fprintf(stderr, "%s: %s (%s)\n", what, zero_status_str(s), zero_last_error());
        return 1;
    }
    return 0;
}

int main(void) {
    zero_plan_desc_t d;
    memset(&d, 0, sizeof d);
    d.psi = 124439808ull;
    d.nd = 8;
    d.stage = 2;
    d.bucket_elems = 25000000ull;
    zero_plan_t *p = NULL;
    if (check(zero_plan(&d, &p), "zero_plan")) return 1;
    uint64_t v = 0;
    const zero_query_t qs[] = {ZERO_Q_PSI_PAD, ZERO_Q_S, ZERO_Q_N_BUCKETS, ZERO_Q_WORKSPACE_BYTES};
    const char *names[] = {"psi_pad", "S", "n_buckets", "workspace_bytes"};
    for (int i = 0; i < 4; ++i) {
        if (check(zero_plan_query(p, qs[i], 0, &v), names[i])) return 1;
        printf("gpt2.%s %llu\n", names[i], (unsigned long long)v);
    }
    for (uint64_t st = 0; st < 4; ++st) {
        if (check(zero_plan_query(p, ZERO_Q_MEM_BYTES_PER_RANK, st, &v), "mem")) return 1;
        printf("gpt2.mem_stage%llu %llu\n", (unsigned long long)st, (unsigned long long)v);
    }
    if (check(zero_bytes_moved(p, ZERO_BYTES_COMM_ELEMS_PER_RANK, 0, &v), "comm")) return 1;
    printf("gpt2.comm_elems %llu\n", (unsigned long long)v);
    if (check(zero_bytes_moved(p, ZERO_BYTES_HBM_STEP, 0, &v), "hbm")) return 1;
    printf("gpt2.hbm_step %llu\n", (unsigned long long)v);
    if (check(zero_plan_query(p, ZERO_Q_OWNER, 77777777ull, &v), "owner")) return 1;
    printf("gpt2.owner_of_77777777 %llu\n", (unsigned long long)v);
    zero_plan_destroy(p);

    const uint64_t units[3] = {100000, 7, 250001};
    memset(&d, 0, sizeof d);
    d.psi = 350008;
    d.nd = 5;
    d.stage = 3;
    d.bucket_elems = 65536;
    d.align_elems = 8;
    d.n_units = 3;
    d.unit_elems = units;
    if (check(zero_plan(&d, &p), "zero_plan stage 3")) return 1;
    for (uint64_t u = 0; u < 3; ++u) {
        uint64_t pad, shard, off;
        if (check(zero_plan_query(p, ZERO_Q_UNIT_PAD, u, &pad), "pad") ||
            check(zero_plan_query(p, ZERO_Q_UNIT_SHARD, u, &shard), "shard") ||
            check(zero_plan_query(p, ZERO_Q_UNIT_OFFSET, u, &off), "offset"))
            return 1;
        printf("st3.unit%llu %llu %llu %llu\n", (unsigned long long)u, (unsigned long long)pad,
               (unsigned long long)shard, (unsigned long long)off);
    }
    /* an error comes back as a status with a message, never an abort */
    zero_status_t s = zero_release_layer(p, 0);
    printf("st3.release_unheld %d %s\n", (int)s, s == ZERO_ESTATE ? "ESTATE" : "other");
    zero_plan_destroy(p);
    printf("abi %u\n", zero_abi_version());
    return 0;
}
