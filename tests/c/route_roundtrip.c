/*
 * A C caller of libmep, with no Python involved: plan, dispatch and combine of a small
 * balanced workload through the C ABI of include/mep.h, then the same round trip from
 * host memory in one mep_route_host call, checked against closed forms (every rank
 * receives exactly S*K rows; with gates summing to one, the identity expert gives every
 * token back). Then the int8 dispatch with all-ones smoothing scales, per token and
 * sorted by expert (with its workspace query), against the plain per-token int8
 * dispatch: the same codes and scales. Prints "route_roundtrip ok" and exits 0 on success.
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

static uint16_t bf16_of_int(int v) /* small integers are exact in bf16 */
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

int main(void)
{
    const int R = 4, E = 16, S = 64, K = 4, H = 256;
    const int T = R * S, N = T * K;
    int32_t *ids = malloc(sizeof(int32_t) * N);
    float *gates = malloc(sizeof(float) * N);
    uint16_t *x = malloc(sizeof(uint16_t) * T * H), *out = malloc(sizeof(uint16_t) * T * H);
    int32_t *pos = malloc(sizeof(int32_t) * N), *rank_off = malloc(sizeof(int32_t) * (R + 1));
    mep_plan_stats_t stats;
    unsigned s = 12345;
    for (int t = 0; t < T; t++)
        for (int k = 0; k < K; k++) {
            s = s * 1103515245u + 12345u;
            ids[t * K + k] = (int32_t)((t + k * 3 + (s >> 16) % 2) % E);
            gates[t * K + k] = 0.25f;   /* K = 4: gates sum to exactly one */
        }
    for (int i = 0; i < T * H; i++) x[i] = bf16_of_int((i * 7) % 255 - 127);

    int32_t *d_ids, *d_pos, *d_hist, *d_roff, *d_load, *d_rc, *d_rk, *d_rcu;
    float *d_g;
    uint16_t *d_x, *d_recv, *d_out;
    mep_plan_stats_t *d_stats;
    void *d_ws;
    size_t ws = mep_plan_workspace_size(R, E, S, K);
    CHECK(ws > 0);
    CHECK(cudaMalloc((void **)&d_ids, sizeof(int32_t) * N) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_pos, sizeof(int32_t) * N) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_hist, sizeof(int32_t) * E) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_roff, sizeof(int32_t) * (R + 1)) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_load, sizeof(int32_t) * R) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_rc, sizeof(int32_t) * R) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_rk, sizeof(int32_t) * R * E) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_rcu, sizeof(int32_t) * R * (E + 1)) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_stats, sizeof(mep_plan_stats_t)) == cudaSuccess);
    CHECK(cudaMalloc(&d_ws, ws) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_g, sizeof(float) * N) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_x, sizeof(uint16_t) * T * H) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_recv, sizeof(uint16_t) * N * H) == cudaSuccess);
    CHECK(cudaMalloc((void **)&d_out, sizeof(uint16_t) * T * H) == cudaSuccess);
    CHECK(cudaMemcpy(d_ids, ids, sizeof(int32_t) * N, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(d_g, gates, sizeof(float) * N, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(d_x, x, sizeof(uint16_t) * T * H, cudaMemcpyHostToDevice) == cudaSuccess);

    cudaStream_t st;
    CHECK(cudaStreamCreate(&st) == cudaSuccess);
    CHECK(mep_plan(d_ids, NULL, R, E, S, K, MEP_PLAN_BALANCED, 0, d_pos, d_hist, d_roff, d_load, d_rc,
                   d_rk, d_rcu, d_stats, d_ws, ws, st) == MEP_OK);
    CHECK(mep_dispatch(d_x, d_pos, T, K, H, 0, d_recv, NULL, N, st) == MEP_OK);
    CHECK(mep_combine(d_recv, N, d_pos, d_g, T, K, H, d_out, st) == MEP_OK);
    CHECK(cudaStreamSynchronize(st) == cudaSuccess);
    int32_t derr = -1;
    CHECK(mep_get_error(st, &derr, 1) == MEP_OK && derr == 0);

    CHECK(cudaMemcpy(pos, d_pos, sizeof(int32_t) * N, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(rank_off, d_roff, sizeof(int32_t) * (R + 1), cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(&stats, d_stats, sizeof stats, cudaMemcpyDeviceToHost) == cudaSuccess);
    CHECK(cudaMemcpy(out, d_out, sizeof(uint16_t) * T * H, cudaMemcpyDeviceToHost) == cudaSuccess);
    int *count = calloc(R, sizeof(int));
    int *seen = calloc(N, sizeof(int));
    for (int n = 0; n < N; n++) {
        CHECK(pos[n] >= 0 && pos[n] < N && !seen[pos[n]]);
        seen[pos[n]] = 1;
        count[pos[n] / (S * K)]++;
    }
    for (int r = 0; r < R; r++) CHECK(count[r] == S * K && rank_off[r] == r * S * K);
    CHECK(stats.max_chunk == S * K && stats.n_kept == N && stats.redundant <= R - 1);
    double mv_before = -9.0, mv_after = -9.0;
    CHECK(mep_maxvio(&stats, S, K, E, &mv_before, &mv_after, NULL) == MEP_OK);
    CHECK(mv_after == 0.0 && mv_before == (double)stats.max_load / (double)(S * K) - 1.0);
    CHECK(memcmp(out, x, sizeof(uint16_t) * T * H) == 0);
    /* the same round trip from host memory in one call (pageable buffers: the copies
       are synchronous, the kernels still run on the stream) */
    uint16_t *out2 = malloc(sizeof(uint16_t) * T * H);
    memset(out2, 0xff, sizeof(uint16_t) * T * H);
    CHECK(cudaMemset(d_out, 0, sizeof(uint16_t) * T * H) == cudaSuccess);
    mep_route_buffers_t rb;
    memset(&rb, 0, sizeof rb);
    rb.R = R; rb.E = E; rb.S = S; rb.K = K; rb.H = H; rb.quant = 0;
    rb.ids = d_ids; rb.gates = d_g; rb.x = d_x; rb.recv = d_recv; rb.recv_scale = NULL; rb.out = d_out;
    rb.pos = d_pos; rb.hist = d_hist; rb.rank_off = d_roff; rb.load = d_load; rb.rep_count = d_rc;
    rb.rep_key = d_rk; rb.rep_cu = d_rcu; rb.stats = d_stats; rb.workspace = d_ws; rb.workspace_bytes = ws;
    CHECK(mep_route_host(&rb, ids, gates, x, out2, st) == MEP_OK);
    CHECK(cudaStreamSynchronize(st) == cudaSuccess);
    CHECK(memcmp(out2, x, sizeof(uint16_t) * T * H) == 0);
    rb.quant = 5;
    CHECK(mep_route_host(&rb, ids, gates, x, out2, st) == MEP_ERR_DTYPE);
    /* smoothing scales of one: the smoothed codes and scales are the plain int8 dispatch's */
    {
        float *ones = malloc(sizeof(float) * E * H), *d_sm, *d_sc0, *d_sc1, *d_sc2;
        int8_t *d_q0, *d_q1, *d_q2;
        void *d_sws;
        for (int i = 0; i < E * H; i++) ones[i] = 1.0f;
        const size_t sws = mep_dispatch_int8_smooth_workspace_size(T, K);
        CHECK(sws >= sizeof(int32_t) * (size_t)N && sws % 256 == 0);
        CHECK(cudaMalloc((void **)&d_sm, sizeof(float) * E * H) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_q0, (size_t)N * H) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_q1, (size_t)N * H) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_q2, (size_t)N * H) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_sc0, sizeof(float) * N) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_sc1, sizeof(float) * N) == cudaSuccess);
        CHECK(cudaMalloc((void **)&d_sc2, sizeof(float) * N) == cudaSuccess);
        CHECK(cudaMalloc(&d_sws, sws) == cudaSuccess);
        CHECK(cudaMemcpy(d_sm, ones, sizeof(float) * E * H, cudaMemcpyHostToDevice) == cudaSuccess);
        CHECK(mep_dispatch(d_x, d_pos, T, K, H, 1, d_q0, d_sc0, N, st) == MEP_OK);
        CHECK(mep_dispatch_int8_smooth(d_x, d_ids, d_pos, T, K, H, d_sm, E, d_q1, d_sc1, N, st) == MEP_OK);
        CHECK(mep_dispatch_int8_smooth_grouped(d_x, d_ids, d_pos, T, K, H, d_sm, E, d_q2, d_sc2, N, NULL, sws, st) ==
              MEP_ERR_WORKSPACE);
        CHECK(mep_dispatch_int8_smooth_grouped(d_x, d_ids, d_pos, T, K, H, d_sm, E, d_q2, d_sc2, N, d_sws, sws, st) ==
              MEP_OK);
        CHECK(cudaStreamSynchronize(st) == cudaSuccess);
        CHECK(mep_get_error(st, &derr, 1) == MEP_OK && derr == 0);
        int8_t *q0 = malloc((size_t)N * H), *q1 = malloc((size_t)N * H), *q2 = malloc((size_t)N * H);
        float *sc0 = malloc(sizeof(float) * N), *sc1 = malloc(sizeof(float) * N), *sc2 = malloc(sizeof(float) * N);
        CHECK(cudaMemcpy(q0, d_q0, (size_t)N * H, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(q1, d_q1, (size_t)N * H, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(q2, d_q2, (size_t)N * H, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(sc0, d_sc0, sizeof(float) * N, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(sc1, d_sc1, sizeof(float) * N, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(cudaMemcpy(sc2, d_sc2, sizeof(float) * N, cudaMemcpyDeviceToHost) == cudaSuccess);
        CHECK(memcmp(q0, q1, (size_t)N * H) == 0 && memcmp(q0, q2, (size_t)N * H) == 0);
        CHECK(memcmp(sc0, sc1, sizeof(float) * N) == 0 && memcmp(sc0, sc2, sizeof(float) * N) == 0);
    }
    /* argument errors come back without touching the device */
    CHECK(mep_dispatch(d_x, d_pos, T, K, H, 7, d_recv, NULL, N, st) == MEP_ERR_DTYPE);
    CHECK(mep_plan(NULL, NULL, R, E, S, K, 0, 0, d_pos, d_hist, d_roff, NULL, d_rc, d_rk, d_rcu, d_stats, d_ws,
                   ws, st) == MEP_ERR_NULLPTR);
    printf("route_roundtrip ok: R=%d E=%d S=%d K=%d H=%d, redundant=%d, max_load=%d\n", R, E, S, K, H,
           stats.redundant, stats.max_load);
    return 0;
}
