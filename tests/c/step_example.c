/* A plain C caller of libzero.so on the GPU: one ZeRO step of a four-rank
 * toy (65,536 parameters, stage 2, 16,384-element buckets) with device
 * memory from the CUDA runtime, then a second step.  Inputs are bit
 * patterns from an integer hash (no rounding, no arithmetic of the method):
 * bf16 gradients of magnitude 2^-10 .. 2^-6 with random sign and mantissa,
 * fp32 master weights of magnitude 2^-8 .. 2^-5.  Writes the inputs of both
 * steps and every output, raw, to the file named on the command line, for
 * the test that compares them with the oracle.
 *     step_example OUT.bin */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "zero.h"

#define PSI 65536u
#define ND 4u

static uint32_t mix(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

static uint16_t grad_bits(uint32_t i) {
    const uint32_t h = mix(i * 2654435761u + 12345u);
    const uint32_t sign = (h >> 31) & 1u, exp = 127u - 10u + (h >> 24) % 5u, man = h & 0x7fu;
    return (uint16_t)((sign << 15) | (exp << 7) | man);
}

static uint32_t master_bits(uint32_t i) {
    const uint32_t h = mix(i ^ 0x9e3779b9u);
    const uint32_t sign = (h >> 31) & 1u, exp = 127u - 8u + (h >> 23) % 4u, man = mix(h) & 0x7fffffu;
    return (sign << 31) | (exp << 23) | man;
}

#define CK(x)                                                                      \
    do {                                                                           \
        cudaError_t e_ = (x);                                                      \
        if (e_ != cudaSuccess) {                                                   \
            fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));               \
            return 1;                                                              \
        }                                                                          \
    } while (0)

#define ZK(x)                                                                      \
    do {                                                                           \
        zero_status_t s_ = (x);                                                    \
        if (s_ != ZERO_OK) {                                                       \
            fprintf(stderr, "%s: %s (%s)\n", #x, zero_status_str(s_), zero_last_error()); \
            return 1;                                                              \
        }                                                                          \
    } while (0)

int main(int argc, char **argv) {
    if (argc != 2) {
        fprintf(stderr, "usage: %s OUT.bin\n", argv[0]);
        return 2;
    }
    zero_plan_desc_t d;
    memset(&d, 0, sizeof d);
    d.psi = PSI;
    d.nd = ND;
    d.stage = 2;
    d.bucket_elems = 16384;
    zero_plan_t *plan = NULL;
    ZK(zero_plan(&d, &plan));
    uint64_t psi_pad = 0, S = 0, ws_bytes = 0;
    ZK(zero_plan_query(plan, ZERO_Q_PSI_PAD, 0, &psi_pad));
    ZK(zero_plan_query(plan, ZERO_Q_S, 0, &S));
    ZK(zero_plan_query(plan, ZERO_Q_WORKSPACE_BYTES, 0, &ws_bytes));
    const size_t n = (size_t)ND * S; /* owner storage = logical order here (one unit) */

    uint16_t *hg = malloc(2 * (size_t)ND * psi_pad * 2);
    uint32_t *hw = malloc(n * 4);
    float *hout = malloc(n * 4 * 4);
    uint16_t *hp = malloc((size_t)ND * psi_pad * 2);
    if (!hg || !hw || !hout || !hp) return 1;
    for (uint32_t k = 0; k < 2u * ND * psi_pad; ++k) hg[k] = grad_bits(k);
    for (uint32_t k = 0; k < n; ++k) hw[k] = master_bits(k);

    void *g, *params, *ws;
    float *w, *m, *v, *red;
    double *norm;
    int32_t *ovf;
    CK(cudaMalloc(&g, (size_t)ND * psi_pad * 2));
    CK(cudaMalloc((void **)&w, n * 4));
    CK(cudaMalloc((void **)&m, n * 4));
    CK(cudaMalloc((void **)&v, n * 4));
    CK(cudaMalloc((void **)&red, n * 4));
    CK(cudaMalloc(&params, (size_t)ND * psi_pad * 2));
    CK(cudaMalloc((void **)&norm, 8));
    CK(cudaMalloc((void **)&ovf, 4));
    CK(cudaMalloc(&ws, ws_bytes));
    CK(cudaMemcpy(w, hw, n * 4, cudaMemcpyHostToDevice));
    CK(cudaMemset(m, 0, n * 4));
    CK(cudaMemset(v, 0, n * 4));

    zero_bufs_t b;
    memset(&b, 0, sizeof b);
    b.grads = g;
    b.grad_stride = psi_pad;
    b.master = w;
    b.exp_avg = m;
    b.exp_avg_sq = v;
    b.params = params;
    b.param_stride = psi_pad;
    b.reduced_grad = red;
    b.grad_norm_sq = norm;
    b.overflow = ovf;
    b.workspace = ws;
    b.workspace_bytes = ws_bytes;
    b.owner_view = -1;
    zero_adam_t adam = {1e-3, 0.9, 0.999, 1e-8, 1.0 / ND, 0.01};
    double norms[2];
    int32_t ovfs[2];
    for (uint64_t t = 1; t <= 2; ++t) {
        CK(cudaMemcpy(g, hg + (t - 1) * ND * psi_pad, (size_t)ND * psi_pad * 2, cudaMemcpyHostToDevice));
        ZK(zero_step(plan, &b, &adam, t, NULL));
        ZK(zero_stream_status(NULL));
        CK(cudaMemcpy(&norms[t - 1], norm, 8, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(&ovfs[t - 1], ovf, 4, cudaMemcpyDeviceToHost));
    }
    CK(cudaMemcpy(hout, w, n * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hout + n, m, n * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hout + 2 * n, v, n * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hout + 3 * n, red, n * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(hp, params, (size_t)ND * psi_pad * 2, cudaMemcpyDeviceToHost));

    FILE *f = fopen(argv[1], "wb");
    if (!f) return 1;
    const uint64_t hdr[3] = {ND, psi_pad, S};
    fwrite(hdr, 8, 3, f);
    fwrite(hg, 2, 2 * (size_t)ND * psi_pad, f);  /* gradients of steps 1 and 2 */
    fwrite(hw, 4, n, f);                          /* master before step 1 */
    fwrite(hout, 4, 4 * n, f);                    /* w, m, v, reduced after step 2 */
    fwrite(hp, 2, (size_t)ND * psi_pad, f);       /* replicas after step 2 */
    fwrite(norms, 8, 2, f);
    fwrite(ovfs, 4, 2, f);
    fclose(f);
    zero_plan_destroy(plan);
    printf("ok\n");
    return 0;
}
