/*
 * mep_plan_static_ws across a device reset, from C (no Python, no torch): the plan with
 * the library's own scratch array must equal, bit for bit, the plan of mep_plan with a
 * caller workspace, before cudaDeviceReset and again after it (the reset destroys the
 * context in which the array's device address was looked up; the library must look it
 * up again in the new one). Prints "static_ws_reset ok" and exits 0 on success.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "mep.h"

#define CHECK(x)                                                                 \
    do {                                                                         \
        if (!(x)) {                                                              \
            fprintf(stderr, "check failed: %s (line %d)\n", #x, __LINE__);       \
            return 1;                                                            \
        }                                                                        \
    } while (0)

enum { R = 4, E = 16, S = 500, K = 4, N = R * S * K };
#define NOUT 8

/* sizes (int32 words) of pos, hist, rank_off, load, rep_count, rep_key, rep_cu, stats */
static const size_t kWords[NOUT] = {N, E, R + 1, R, R, (size_t)R * E, (size_t)R * (E + 1), 8};

/* One round: upload ids, plan both ways, compare every output. */
static int round_trip(const int32_t *ids, int round)
{
    int32_t *d_ids, *a[NOUT], *b[NOUT];
    void *ws;
    size_t ws_bytes = mep_plan_workspace_size(R, E, S, K);
    CHECK(ws_bytes > 0 && ws_bytes <= MEP_PLAN_STATIC_WS_BYTES);
    CHECK(cudaMalloc((void **)&d_ids, sizeof(int32_t) * N) == cudaSuccess);
    CHECK(cudaMalloc(&ws, ws_bytes) == cudaSuccess);
    for (int i = 0; i < NOUT; i++) {
        CHECK(cudaMalloc((void **)&a[i], sizeof(int32_t) * kWords[i]) == cudaSuccess);
        CHECK(cudaMalloc((void **)&b[i], sizeof(int32_t) * kWords[i]) == cudaSuccess);
        CHECK(cudaMemset(a[i], 0x5a, sizeof(int32_t) * kWords[i]) == cudaSuccess);
        CHECK(cudaMemset(b[i], 0x33, sizeof(int32_t) * kWords[i]) == cudaSuccess);
    }
    CHECK(cudaMemcpy(d_ids, ids, sizeof(int32_t) * N, cudaMemcpyHostToDevice) == cudaSuccess);
    cudaStream_t st;
    CHECK(cudaStreamCreate(&st) == cudaSuccess);
    mep_status_t rs = mep_plan_static_ws(d_ids, NULL, R, E, S, K, MEP_PLAN_BALANCED, 0, a[0], a[1], a[2], a[3],
                                         a[4], a[5], a[6], (mep_plan_stats_t *)a[7], st);
    if (rs != MEP_OK) fprintf(stderr, "round %d: status %d, cuda %d\n", round, (int)rs, mep_last_cuda_error());
    CHECK(rs == MEP_OK);
    CHECK(mep_plan(d_ids, NULL, R, E, S, K, MEP_PLAN_BALANCED, 0, b[0], b[1], b[2], b[3], b[4], b[5], b[6],
                   (mep_plan_stats_t *)b[7], ws, ws_bytes, st) == MEP_OK);
    CHECK(cudaStreamSynchronize(st) == cudaSuccess);
    int32_t derr = -1;
    CHECK(mep_get_error(st, &derr, 1) == MEP_OK && derr == 0);
    for (int i = 0; i < NOUT; i++) {
        int32_t *ha = malloc(sizeof(int32_t) * kWords[i]), *hb = malloc(sizeof(int32_t) * kWords[i]);
        CHECK(cudaMemcpy(ha, a[i], sizeof(int32_t) * kWords[i], cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(hb, b[i], sizeof(int32_t) * kWords[i], cudaMemcpyDeviceToHost) == cudaSuccess);
        if (memcmp(ha, hb, sizeof(int32_t) * kWords[i]) != 0) {
            fprintf(stderr, "round %d: output %d differs\n", round, i);
            return 1;
        }
        free(ha);
        free(hb);
    }
    CHECK(cudaStreamDestroy(st) == cudaSuccess);
    return 0;
}

int main(void)
{
    int32_t *ids = malloc(sizeof(int32_t) * N);
    unsigned s = 2024;
    for (int n = 0; n < N; n++) {
        s = s * 1664525u + 1013904223u;
        int32_t e = (int32_t)((s >> 8) % 64);
        ids[n] = e < 24 ? 0 : e % E;   /* expert 0 hot: its rows straddle ranks */
    }
    CHECK(round_trip(ids, 0) == 0);
    CHECK(cudaDeviceReset() == cudaSuccess);
    CHECK(round_trip(ids, 1) == 0);
    CHECK(round_trip(ids, 2) == 0);
    printf("static_ws_reset ok\n");
    return 0;
}
