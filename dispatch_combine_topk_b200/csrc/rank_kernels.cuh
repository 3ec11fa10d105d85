// Dispatch and combine across expert-parallel ranks whose receive buffers are separate
// allocations (sm_100a): the row of slot n, p = pos[n], lives in rank d = p / rows_per_rank
// at local row p mod rows_per_rank of that rank's buffer, reached through a device array
// of R base pointers. Across GPUs the pointers are peer mappings of the other ranks'
// buffers (NVLink), and the dispatch is the zero-copy exchange of MoonEP: every token row
// is stored straight into its final, expert-grouped row on the destination rank
// (twodots.gr article on MoonEP, zero-copy paragraph). The kernels only store to and load
// from those buffers with plain 16-byte accesses: no bulk copies, no multicast, no waits.
#pragma once

#include "common.cuh"

namespace mep {

// Local row of p on its rank, and the rank; -1 (and a data-error bit) when p is outside
// [-1, R * rows_per_rank).
__device__ __forceinline__ int32_t rank_of(int32_t p, int32_t R, int64_t rpr, int64_t *local)
{
    if (p < 0) {
        if (p < -1) flag_error(MEP_DERR_ROW_RANGE);
        return -1;
    }
    const int64_t d = (int64_t)p / rpr;
    if (d >= R) {
        flag_error(MEP_DERR_ROW_RANGE);
        return -1;
    }
    *local = (int64_t)p - d * rpr;
    return (int32_t)d;
}

// Base pointer of rank d's buffer from the table, or NULL (and a data-error bit) when the
// table holds NULL or a pointer without the alignment the accesses need: no access is
// ever made through such a pointer.
template <typename P>
__device__ __forceinline__ P *rank_base(P *const *table, int32_t d, uintptr_t align)
{
    P *b = table[d];
    if (!b || ((uintptr_t)b & (align - 1))) {
        flag_error(MEP_DERR_ROW_RANGE);
        return nullptr;
    }
    return b;
}

// bf16 rows, one warp per token: lane k < K finds slot k's destination row pointer, the
// warp walks the row in 16-byte chunks (4 per lane in flight) and stores each chunk to
// the K destinations. Requires H % 8 == 0 and 16-byte aligned x and buffers.
__global__ void __launch_bounds__(256)
k_dispatch_ranks_warp(const uint4 *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K, int64_t H8,
                      uint4 *const *__restrict__ recv, int32_t R, int64_t rpr)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        uint4 *mine = nullptr;
        if (lane < K) {
            int64_t local = 0;
            const int32_t d = rank_of(pos[t * K + lane], R, rpr, &local);
            uint4 *b = d >= 0 ? rank_base(recv, d, 16) : nullptr;
            if (b) mine = b + local * H8;
        }
        const uint4 *src = x + t * H8;
        for (int64_t base = 0; base < H8; base += 32 * 4) {
            const int64_t c0 = base + lane;
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; u++)
                if (c0 + 32 * u < H8) v[u] = ld_stream(src + c0 + 32 * u);
            for (int k = 0; k < K; k++) {
                uint4 *dst = (uint4 *)__shfl_sync(0xffffffffu, (unsigned long long)mine, k);
                if (!dst) continue;
#pragma unroll
                for (int u = 0; u < 4; u++)
                    if (c0 + 32 * u < H8) st_v4(dst + c0 + 32 * u, v[u]);
            }
        }
    }
}

// Per-token dynamic int8 (the codes and scale of mep_dispatch with quant 1), one CTA per
// token: amax over the row, scale = amax / 127, codes by the IEEE quotient, 8 codes per
// 8-byte store to each destination, the scale beside them. Requires H % 8 == 0, 16-byte
// aligned x and 8-byte aligned buffers.
__global__ void __launch_bounds__(256, 4)
k_dispatch_ranks_int8(const uint4 *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K, int64_t H8,
                      uint2 *const *__restrict__ recv, float *const *__restrict__ scales, int32_t R, int64_t rpr)
{
    __shared__ uint2 *s_dst[kMaxK];
    __shared__ float *s_sc[kMaxK];
    __shared__ float red[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < K) {
            int64_t local = 0;
            const int32_t d = rank_of(pos[t * K + threadIdx.x], R, rpr, &local);
            uint2 *b = d >= 0 ? rank_base(recv, d, 8) : nullptr;
            float *sb = b ? rank_base(scales, d, 4) : nullptr;
            s_dst[threadIdx.x] = sb ? b + local * H8 : nullptr;
            s_sc[threadIdx.x] = sb ? sb + local : nullptr;
        }
        const uint4 *src = x + t * H8;
        float amax = 0.0f;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            const uint4 v = src[c];
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))),
                                     fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))),
                                     fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w)))));
        }
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        float m = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); w++) m = fmaxf(m, red[w]);
        const float scale = __fdiv_rn(m, 127.0f);
        if (threadIdx.x < K && s_sc[threadIdx.x]) *s_sc[threadIdx.x] = scale;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            const uint4 v = src[c];
            uint2 q;
            q.x = q8x4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y), scale);
            q.y = q8x4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w), scale);
            for (int k = 0; k < K; k++) {
                uint2 *dst = s_dst[k];
                if (dst) dst[c] = q;
            }
        }
        __syncthreads();                                   // s_dst, s_sc and red are reused
    }
}

// bf16 combine from the ranks' buffers: out[t] = bf16(sum over kept k, ascending, of
// fl(gate * y)), fp32, no FMA (the sum of k_combine_v8). One warp per token, 16-byte
// chunks, all K loads of a chunk in flight. Requires H % 8 == 0, 16-byte alignment.
template <int KC>
__global__ void __launch_bounds__(256, 3)
k_combine_ranks_v8(const uint4 *const *__restrict__ y, const int32_t *__restrict__ pos,
                   const float *__restrict__ gates, int64_t T, int Krt, int64_t H8, int32_t R, int64_t rpr,
                   uint4 *__restrict__ out)
{
    constexpr bool kFixed = KC > 0;
    constexpr int kSlots = kFixed ? KC : 4;            // runtime K: groups of 4 slots
    const int K = kFixed ? KC : Krt;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const uint4 *mine = nullptr;
        float g_mine = 0.0f;
        if (lane < K) {
            int64_t local = 0;
            const int32_t d = rank_of(pos[t * K + lane], R, rpr, &local);
            const uint4 *b = d >= 0 ? rank_base(y, d, 16) : nullptr;
            if (b) mine = b + local * H8;
            g_mine = gates[t * K + lane];
        }
        if constexpr (kFixed) {
            // the slots' rows and gates once per token, in registers
            const uint4 *rowp[KC];
            float g[KC];
#pragma unroll
            for (int k = 0; k < KC; k++) {
                rowp[k] = (const uint4 *)__shfl_sync(0xffffffffu, (unsigned long long)mine, k);
                g[k] = __shfl_sync(0xffffffffu, g_mine, k);
            }
            for (int64_t c = lane; c < H8; c += 32) {
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; j++) acc[j] = 0.0f;
                uint4 v[KC];
#pragma unroll
                for (int k = 0; k < KC; k++) v[k] = rowp[k] ? ld_stream(rowp[k] + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < KC; k++) {
                    if (!rowp[k]) continue;
                    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        acc[2 * j] = __fadd_rn(acc[2 * j], __fmul_rn(g[k], bf16lo(w[j])));
                        acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], __fmul_rn(g[k], bf16hi(w[j])));
                    }
                }
                uint4 o;
                o.x = pack_bf16x2(acc[0], acc[1]);
                o.y = pack_bf16x2(acc[2], acc[3]);
                o.z = pack_bf16x2(acc[4], acc[5]);
                o.w = pack_bf16x2(acc[6], acc[7]);
                st_v4(out + t * H8 + c, o);
            }
        } else {
            for (int64_t base = 0; base < H8; base += 32) {
                const int64_t c = base + lane;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; j++) acc[j] = 0.0f;
#pragma unroll 1
                for (int k0 = 0; k0 < K; k0 += kSlots) {
                    const uint4 *rowp[kSlots];
                    float g[kSlots];
                    uint4 v[kSlots];
#pragma unroll
                    for (int k = 0; k < kSlots; k++) {
                        const bool in = k0 + k < K;
                        rowp[k] = in ? (const uint4 *)__shfl_sync(0xffffffffu, (unsigned long long)mine, k0 + k) : nullptr;
                        g[k] = in ? __shfl_sync(0xffffffffu, g_mine, k0 + k) : 0.0f;
                        v[k] = (rowp[k] && c < H8) ? ld_stream(rowp[k] + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int k = 0; k < kSlots; k++) {
                        if (!rowp[k]) continue;
                        const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            acc[2 * j] = __fadd_rn(acc[2 * j], __fmul_rn(g[k], bf16lo(w[j])));
                            acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], __fmul_rn(g[k], bf16hi(w[j])));
                        }
                    }
                }
                if (c < H8) {
                    uint4 o;
                    o.x = pack_bf16x2(acc[0], acc[1]);
                    o.y = pack_bf16x2(acc[2], acc[3]);
                    o.z = pack_bf16x2(acc[4], acc[5]);
                    o.w = pack_bf16x2(acc[6], acc[7]);
                    st_v4(out + t * H8 + c, o);
                }
            }
        }
    }
}

// Combine of int8 rows with per-row scales from the ranks' buffers (the sum of
// k_combine_int8_warp: dequantise to bf16, then the k-ordered fp32 sum). One warp per
// token, 16 codes per lane per slot. Requires H % 16 == 0, 16-byte alignment.
template <int KC>
__global__ void __launch_bounds__(128)
k_combine_ranks_int8(const uint4 *const *__restrict__ yq, const float *const *__restrict__ yscale,
                     const int32_t *__restrict__ pos, const float *__restrict__ gates, int64_t T, int Krt,
                     int64_t H16, int32_t R, int64_t rpr, uint4 *__restrict__ out)
{
    constexpr bool kFixed = KC > 0;
    constexpr int kSlots = kFixed ? KC : 4;            // runtime K: groups of 4 slots
    const int K = kFixed ? KC : Krt;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const uint4 *mine = nullptr;
        float g_mine = 0.0f, s_mine = 0.0f;
        if (lane < K) {
            int64_t local = 0;
            const int32_t d = rank_of(pos[t * K + lane], R, rpr, &local);
            const uint4 *b = d >= 0 ? rank_base(yq, d, 16) : nullptr;
            const float *sb = b ? rank_base(yscale, d, 4) : nullptr;
            if (sb) {
                mine = b + local * H16;
                s_mine = sb[local];
            }
            g_mine = gates[t * K + lane];
        }
        uint4 *dst = out + t * 2 * H16;
        if constexpr (kFixed) {
            // the slots' rows, gates and scales once per token, in registers
            const uint4 *rowp[KC];
            float g[KC], sc[KC];
#pragma unroll
            for (int k = 0; k < KC; k++) {
                rowp[k] = (const uint4 *)__shfl_sync(0xffffffffu, (unsigned long long)mine, k);
                g[k] = __shfl_sync(0xffffffffu, g_mine, k);
                sc[k] = __shfl_sync(0xffffffffu, s_mine, k);
            }
            for (int64_t c = lane; c < H16; c += 32) {
                float2 acc[8];
#pragma unroll
                for (int j = 0; j < 8; j++) acc[j] = make_float2(0.0f, 0.0f);
                uint4 v[KC];
#pragma unroll
                for (int k = 0; k < KC; k++) v[k] = rowp[k] ? ld_stream(rowp[k] + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < KC; k++)
                    if (rowp[k]) add_int8_x16(acc, v[k], g[k], sc[k]);
                store_bf16x16(dst + 2 * c, acc);
            }
        } else {
            for (int64_t base = 0; base < H16; base += 32) {
                const int64_t c = base + lane;
                float2 acc[8];
#pragma unroll
                for (int j = 0; j < 8; j++) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll 1
                for (int k0 = 0; k0 < K; k0 += kSlots) {
                    const uint4 *rowp[kSlots];
                    float g[kSlots], sc[kSlots];
                    uint4 v[kSlots];
#pragma unroll
                    for (int k = 0; k < kSlots; k++) {
                        const bool in = k0 + k < K;
                        rowp[k] = in ? (const uint4 *)__shfl_sync(0xffffffffu, (unsigned long long)mine, k0 + k) : nullptr;
                        g[k] = in ? __shfl_sync(0xffffffffu, g_mine, k0 + k) : 0.0f;
                        sc[k] = in ? __shfl_sync(0xffffffffu, s_mine, k0 + k) : 0.0f;
                        v[k] = (rowp[k] && c < H16) ? ld_stream(rowp[k] + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int k = 0; k < kSlots; k++)
                        if (rowp[k]) add_int8_x16(acc, v[k], g[k], sc[k]);
                }
                if (c < H16) store_bf16x16(dst + 2 * c, acc);
            }
        }
    }
}

}  // namespace mep
