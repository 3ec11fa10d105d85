// One dispatch row per (token, destination rank), and the expansion back to the
// expert-grouped rows on the receiving side (sm_100a).
//
// A token whose kept slots land on one destination rank several times crosses to it
// once (the MoonEP API reference, section 5.2 on communication performance, names a
// bounds-checked dedup encoding). A rank's deduplicated rows hold its tokens in
// ascending global token order. That order is the stable counting sort by destination
// rank of the slots that open a (token, rank) pair: slot n opens its pair when no
// earlier slot of its token lands on the same rank. So the plan's counting-sort passes
// (k_tile_count, k_scan_cols, k_rank) run unchanged on
//   key  = destination rank of the slot,  keep = the slot opens its pair,
// and give each opening slot its deduplicated row (the send list). k_dedup_finish then
// hands that row to the pair's other slots and inverts the plan rows.
#pragma once

#include "common.cuh"
#include "plan_kernels.cuh"

namespace mep {

// Largest r with off[r] <= p, for 0 <= p < off[R] (off non-decreasing, off[0] = 0): the
// rank whose rows [off[r], off[r+1]) hold row p, empty ranks included.
__device__ __forceinline__ int32_t rank_of_row(const int32_t *off, int32_t R, int64_t p)
{
    int32_t lo = 0, hi = R;   // invariant: off[lo] <= p < off[hi]
    while (hi - lo > 1) {
        const int32_t mid = (lo + hi) >> 1;
        if (off[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Destination rank of slot n (-1: dropped). Rows outside [-1, min(off[R], N)) flag
// MEP_DERR_ROW_RANGE and count as dropped (plan rows are below N = R*S*K).
__device__ __forceinline__ int32_t slot_rank(const int32_t *__restrict__ pos, int64_t n, int64_t N,
                                             const int32_t *off, int32_t R)
{
    const int32_t p = pos[n];
    if (p == -1) return -1;
    if (p < -1 || p >= off[R] || p >= N) {
        flag_error(MEP_DERR_ROW_RANGE);
        return -1;
    }
    return rank_of_row(off, R, p);
}

// dkey[n] = destination rank of slot n (0 when dropped), dkeep[n] = 1 when slot n is the
// first slot of its token on that rank. One thread per token; rank_off in shared memory.
__global__ void __launch_bounds__(256)
k_dedup_keys(const int32_t *__restrict__ pos, const int32_t *__restrict__ rank_off, int32_t R, int64_t T,
             int K, int32_t *__restrict__ dkey, uint8_t *__restrict__ dkeep)
{
    extern __shared__ int32_t off_sh[];
    for (int i = threadIdx.x; i <= R; i += blockDim.x) off_sh[i] = rank_off[i];
    __syncthreads();
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < T; g += (int64_t)gridDim.x * blockDim.x) {
        int32_t rk[MEP_MAX_K];
        for (int k = 0; k < K; k++) {
            const int64_t n = g * K + k;
            const int32_t r = slot_rank(pos, n, T * K, off_sh, R);
            rk[k] = r;
            bool opens = r >= 0;
            for (int j = 0; j < k && opens; j++) opens = rk[j] != r;
            dkey[n] = r >= 0 ? r : 0;
            dkeep[n] = opens ? 1 : 0;
        }
    }
}

// drank_off = exclusive prefix of the per-rank row counts (one CTA).
__global__ void __launch_bounds__(1024)
k_dedup_offsets(const int32_t *__restrict__ count, int32_t R, int32_t *__restrict__ drank_off)
{
    extern __shared__ int32_t sh_off[];
    block_exclusive_scan(count, R, sh_off, sh_off + R + 1);
    for (int i = threadIdx.x; i <= R; i += blockDim.x) drank_off[i] = sh_off[i];
}

// For every kept slot n of token g: dpos[n] = the row of the slot that opened its
// (token, rank) pair (dsend, from the counting sort), gidx[pos[n]] = dpos[n], and
// dtok[row] = g for the opening slot. One thread per token.
__global__ void __launch_bounds__(256)
k_dedup_finish(const int32_t *__restrict__ pos, const int32_t *__restrict__ rank_off, int32_t R, int64_t T,
               int K, const int32_t *__restrict__ dsend, int32_t *__restrict__ dpos, int32_t *__restrict__ dtok,
               int32_t *__restrict__ gidx)
{
    extern __shared__ int32_t off_sh[];
    for (int i = threadIdx.x; i <= R; i += blockDim.x) off_sh[i] = rank_off[i];
    __syncthreads();
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < T; g += (int64_t)gridDim.x * blockDim.x) {
        int32_t rk[MEP_MAX_K], row[MEP_MAX_K];
        for (int k = 0; k < K; k++) {
            const int64_t n = g * K + k;
            const int32_t p = pos[n];
            // slot_rank flagged bad rows in k_dedup_keys already; the bit is idempotent
            const int32_t r = slot_rank(pos, n, T * K, off_sh, R);
            rk[k] = r;
            int32_t u = -1;
            if (r >= 0) {
                int j = 0;
                while (rk[j] != r) j++;   // j <= k: the slot that opened the pair
                u = j == k ? dsend[n] : row[j];
                if (j == k && u >= 0) dtok[u] = (int32_t)g;
                if (u >= 0) gidx[p] = u;
            }
            row[k] = u;
            dpos[n] = u;
        }
    }
}

// dst[p, :] = src[gidx[p], :] for gidx[p] >= 0 (row_v 16-byte chunks per row), and the
// row's scale with it when scales are given. One warp per row, 4 chunks per lane in
// flight.
__global__ void __launch_bounds__(256)
k_expand_warp(const uint4 *__restrict__ src, const float *__restrict__ src_scale, int64_t src_rows,
              const int32_t *__restrict__ gidx, int64_t rows, int64_t row_v, uint4 *__restrict__ dst,
              float *__restrict__ dst_scale)
{
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; p < rows; p += nwarps) {
        const int32_t u = gidx[p];
        if (u < 0) continue;
        if (u >= src_rows) {
            if (lane == 0) flag_error(MEP_DERR_ROW_RANGE);
            continue;
        }
        if (dst_scale && lane == 0) dst_scale[p] = src_scale[u];
        const uint4 *s = src + (int64_t)u * row_v;
        uint4 *d = dst + p * row_v;
        for (int64_t c0 = lane; c0 < row_v; c0 += 32 * U) {
            uint4 v[U];
#pragma unroll
            for (int i = 0; i < U; i++)
                if (c0 + 32 * i < row_v) v[i] = ld_stream(s + c0 + 32 * i);
#pragma unroll
            for (int i = 0; i < U; i++)
                if (c0 + 32 * i < row_v) st_v4(d + c0 + 32 * i, v[i]);
        }
    }
}

// The same copy one byte at a time, for rows that are not 16-byte multiples or
// buffers that are not 16-byte aligned. One CTA per row.
__global__ void __launch_bounds__(256)
k_expand_bytes(const uint8_t *__restrict__ src, const float *__restrict__ src_scale, int64_t src_rows,
               const int32_t *__restrict__ gidx, int64_t rows, int64_t row_bytes, uint8_t *__restrict__ dst,
               float *__restrict__ dst_scale)
{
    for (int64_t p = blockIdx.x; p < rows; p += gridDim.x) {
        const int32_t u = gidx[p];
        if (u < 0) continue;
        if (u >= src_rows) {
            if (threadIdx.x == 0) flag_error(MEP_DERR_ROW_RANGE);
            continue;
        }
        if (dst_scale && threadIdx.x == 0) dst_scale[p] = src_scale[u];
        for (int64_t b = threadIdx.x; b < row_bytes; b += blockDim.x)
            dst[p * row_bytes + b] = src[(int64_t)u * row_bytes + b];
    }
}

}  // namespace mep
