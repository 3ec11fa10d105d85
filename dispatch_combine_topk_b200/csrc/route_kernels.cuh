// Mapping, dispatch, dequantisation and combine kernels (sm_100a).
//
// Dispatch and combine are HBM-bound permute-copies: dispatch reads each token row
// once and writes it K times, combine reads K rows per token and writes one. One CTA
// works on one token at a time (grid-stride over tokens, grid = a multiple of the SM
// count); its threads stride over the row in 16-byte chunks so that every warp access
// is 512 contiguous bytes. The K row indices of the token are read once into shared
// memory.
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace mep {

constexpr int kMaxK = 32;

// ------------------------------------------------------------------ mapping (a3)

// One thread per token. Mapping of aclnnMoeUpdateExpert (gitcode ops-transformer doc,
// 功能说明): instance column 1 for a single instance; otherwise local_rank_id /
// ceil(world_size / count) + 1 (by rank) or (token mod count) + 1 (by token).
// Pruning: v = sum_k fl(scale[k] * thr[k]) in fp32, ascending k, no FMA; a slot stays
// active iff the token is active and !(scale[k] < v).
__global__ void k_update_expert(const int32_t *__restrict__ ids, const int32_t *__restrict__ table,
                                const float *__restrict__ scales, const float *__restrict__ thr,
                                const uint8_t *__restrict__ active, int64_t BS, int32_t K,
                                int32_t E, int32_t F, int64_t local_rank, int64_t world_size,
                                int64_t mode, int32_t *__restrict__ out_ids,
                                uint8_t *__restrict__ out_mask)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < BS;
         i += (int64_t)gridDim.x * blockDim.x) {
        uint8_t act = 1;
        if (active) {
            act = active[i] ? 1 : 0;
            if (i > 0 && act && !active[i - 1]) flag_error(0x8);
        }
        for (int32_t k = 0; k < K; k++) {
            const int32_t e = ids[i * K + k];
            int32_t inst = -1;
            if (e < 0 || e >= E) {
                flag_error(0x1);
            } else {
                const int32_t *row = table + (int64_t)e * F;
                const int32_t c = row[0];
                if (c < 1 || c > F - 1) {
                    flag_error(0x4);
                } else {
                    int64_t col;
                    if (c == 1) col = 1;
                    else if (mode == 0) col = local_rank / ((world_size + c - 1) / c) + 1;
                    else col = (i % c) + 1;
                    const int32_t v = row[col];   // col <= c <= F-1: inside the row
                    if (v < 0 || v >= 1024) flag_error(0x4);
                    else inst = v;
                }
            }
            out_ids[i * K + k] = inst;
        }
        if (scales) {
            float v = 0.0f;
            for (int32_t k = 0; k < K; k++) v = __fadd_rn(v, __fmul_rn(scales[i * K + k], thr[k]));
            for (int32_t k = 0; k < K; k++)
                out_mask[i * K + k] = (act && !(scales[i * K + k] < v)) ? 1 : 0;
        } else {
            for (int32_t k = 0; k < K; k++) out_mask[i * K + k] = act;
        }
    }
}

// ---------------------------------------------------------------- shared helpers

// Load the K rows of token t into shared memory, replacing out-of-range rows by -1.
__device__ __forceinline__ void load_token_rows(const int32_t *__restrict__ pos, int64_t t, int K,
                                                int64_t rows, int32_t *sp)
{
    if (threadIdx.x < K) {
        int32_t p = pos[t * K + threadIdx.x];
        if (p < -1 || (int64_t)p >= rows) {
            flag_error(0x2);
            p = -1;
        }
        sp[threadIdx.x] = p;
    }
}

// ------------------------------------------------------------------ dispatch (a4)

// bf16 copy: recv[pos[t*K+k], :] = x[t, :]. V = uint4 (8 bf16 per access) when H % 8 ==
// 0 and both pointers are 16-byte aligned, else uint16_t.
template <typename V>
__global__ void __launch_bounds__(256)
k_dispatch_copy(const V *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K,
                int64_t HV, int64_t rows, V *__restrict__ recv)
{
    __shared__ int32_t sp[kMaxK];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        __syncthreads();
        const V *src = x + t * HV;
        for (int64_t c = threadIdx.x; c < HV; c += blockDim.x) {
            V v;
            if constexpr (sizeof(V) == 16) v = ld_stream(reinterpret_cast<const uint4 *>(src + c));
            else v = src[c];
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p >= 0) {
                    if constexpr (sizeof(V) == 16) st_v4(reinterpret_cast<uint4 *>(recv + (int64_t)p * HV + c), v);
                    else recv[(int64_t)p * HV + c] = v;
                }
            }
        }
        __syncthreads();
    }
}

// bf16 copy through shared memory with bulk copies (the default path).
//
// One CTA of one warp per SM, tokens strided over the CTAs. A ring of kStages row
// buffers in shared memory: lane 0 bulk-loads token rows ahead into the ring (each
// completion tracked by an mbarrier), lanes k < K each bulk-store the staged row to the
// row of slot k and wait until their stores have finished reading the stage, then the
// stage is refilled with the token kStages ahead. The row bytes travel HBM -> smem once
// and smem -> HBM K times with no register traffic; the bulk engine keeps the K stores
// of every SM in flight.
//
// Dynamic shared memory: 8*kStages (barriers) + 128*kStages (row indices), padded to
// kDispatchSmemHead, then kStages rows of row_bytes. Requires row_bytes % 16 == 0 and
// 16-byte aligned x and recv.
constexpr int kDispatchSmemHead = 2048;

template <int kStages>
__global__ void __launch_bounds__(32)
k_dispatch_bulk(const uint16_t *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K, int64_t H,
                int64_t rows, uint16_t *__restrict__ recv)
{
    extern __shared__ __align__(128) int32_t smem_i32[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(smem_i32);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    int32_t *srow = reinterpret_cast<int32_t *>(smem + 8 * kStages);   // [kStages][32]
    unsigned char *stage = smem + kDispatchSmemHead;
    const uint32_t row_bytes = (uint32_t)(H * 2);
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < kStages; s++) mbar_init(&bar[s], 1);
        mbar_fence_init();
    }
    __syncwarp();
    const int64_t n = blockIdx.x < T ? (T - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    auto token = [&](int64_t i) { return (int64_t)blockIdx.x + i * gridDim.x; };
    auto fetch = [&](int64_t i) {
        const int s = (int)(i % kStages);
        const int64_t t = token(i);
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[s], row_bytes);
            bulk_load_g2s(stage + (size_t)s * row_bytes, x + t * H, row_bytes, &bar[s]);
        }
        if (lane < K) {
            int32_t p = pos[t * K + lane];
            if (p < -1 || (int64_t)p >= rows) {
                flag_error(0x2);
                p = -1;
            }
            srow[s * 32 + lane] = p;
        }
    };
    for (int64_t i = 0; i < n && i < kStages; i++) fetch(i);
    __syncwarp();
    for (int64_t i = 0; i < n; i++) {
        const int s = (int)(i % kStages);
        const bool ok = mbar_wait_bounded(&bar[s], (uint32_t)((i / kStages) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
            // A load never completed: record it, wait (bounded) for the other loads
            // still in flight into this CTA's ring, and leave.
            if (lane == 0) {
                flag_error(0x10);
                for (int64_t j = i + 1; j < n && j < i + kStages; j++)
                    mbar_wait_bounded(&bar[j % kStages], (uint32_t)((j / kStages) & 1));
            }
            break;
        }
        if (lane < K) {
            const int32_t p = srow[s * 32 + lane];
            if (p >= 0) bulk_store_s2g(recv + (int64_t)p * H, stage + (size_t)s * row_bytes, row_bytes);
            bulk_commit();
            bulk_wait_read_all();
        }
        __syncwarp();
        if (i + kStages < n) fetch(i + kStages);
        __syncwarp();
    }
    if (lane < K) bulk_wait_all();
    __syncwarp();
}

// Quantise 8 fp32 values to int8 with the per-token scale; packed little-endian.
__device__ __forceinline__ uint32_t q8x4(float a, float b, float c, float d, float scale)
{
    auto q = [scale](float v) -> uint32_t {
        int r = 0;
        if (scale != 0.0f) {
            r = __float2int_rn(__fdiv_rn(v, scale));   // IEEE quotient, ties to even
            r = max(-127, min(127, r));
        }
        return (uint32_t)(r & 0xff);
    };
    return q(a) | (q(b) << 8) | (q(c) << 16) | (q(d) << 24);
}

// Per-token dynamic int8: one CTA per token, pass 1 reduces amax over the row, pass 2
// re-reads the row (from L1/L2) and writes the K copies of the codes and the scale.
// Needs H % 8 == 0 and 16-byte aligned x, 8-byte aligned recv.
__global__ void __launch_bounds__(256)
k_dispatch_int8(const uint4 *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K,
                int64_t H8, int64_t rows, uint2 *__restrict__ recv, float *__restrict__ recv_scale)
{
    __shared__ int32_t sp[kMaxK];
    __shared__ float red[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        const uint4 *src = x + t * H8;
        float amax = 0.0f;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            uint4 v = src[c];
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))),
                                     fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))),
                                     fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w)))));
        }
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        if (warp == 0) {
            float m = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
            for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
            if (lane == 0) red[0] = m;
        }
        __syncthreads();
        const float scale = __fdiv_rn(red[0], 127.0f);
        if (threadIdx.x < K && sp[threadIdx.x] >= 0) recv_scale[sp[threadIdx.x]] = scale;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            uint4 v = src[c];
            uint2 q;
            q.x = q8x4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y), scale);
            q.y = q8x4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w), scale);
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p >= 0) recv[(int64_t)p * H8 + c] = q;
            }
        }
        __syncthreads();
    }
}

// Scalar fallback of the int8 dispatch for any H and alignment.
__global__ void __launch_bounds__(256)
k_dispatch_int8_scalar(const uint16_t *__restrict__ x, const int32_t *__restrict__ pos, int64_t T,
                       int K, int64_t H, int64_t rows, int8_t *__restrict__ recv,
                       float *__restrict__ recv_scale)
{
    __shared__ int32_t sp[kMaxK];
    __shared__ float red[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        const uint16_t *src = x + t * H;
        float amax = 0.0f;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) amax = fmaxf(amax, fabsf(bf16lo(src[h])));
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        if (warp == 0) {
            float m = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
            for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
            if (lane == 0) red[0] = m;
        }
        __syncthreads();
        const float scale = __fdiv_rn(red[0], 127.0f);
        if (threadIdx.x < K && sp[threadIdx.x] >= 0) recv_scale[sp[threadIdx.x]] = scale;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            int r = 0;
            if (scale != 0.0f) r = max(-127, min(127, __float2int_rn(__fdiv_rn(bf16lo(src[h]), scale))));
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p >= 0) recv[(int64_t)p * H + h] = (int8_t)r;
            }
        }
        __syncthreads();
    }
}

// y[r, h] = bf16(fl(q[r, h] * scale[r])), 8 elements per thread when H % 8 == 0.
__global__ void __launch_bounds__(256)
k_dequant8(const uint2 *__restrict__ q, const float *__restrict__ scale, int64_t rows, int64_t H8,
           uint4 *__restrict__ y)
{
    const int64_t total = rows * H8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float s = scale[i / H8];
        const uint2 v = q[i];
        float f[8];
        for (int j = 0; j < 4; j++) {
            f[j] = __fmul_rn((float)(int8_t)((v.x >> (8 * j)) & 0xff), s);
            f[4 + j] = __fmul_rn((float)(int8_t)((v.y >> (8 * j)) & 0xff), s);
        }
        uint4 o;
        o.x = pack_bf16x2(f[0], f[1]);
        o.y = pack_bf16x2(f[2], f[3]);
        o.z = pack_bf16x2(f[4], f[5]);
        o.w = pack_bf16x2(f[6], f[7]);
        y[i] = o;
    }
}

__global__ void __launch_bounds__(256)
k_dequant_scalar(const int8_t *__restrict__ q, const float *__restrict__ scale, int64_t rows,
                 int64_t H, uint16_t *__restrict__ y)
{
    const int64_t total = rows * H;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn((float)q[i], scale[i / H]));
        y[i] = *reinterpret_cast<uint16_t *>(&b);
    }
}

// ------------------------------------------------------------------- combine (a5)

// out[t, :] = bf16( sum_k fl(gate[t,k] * y[pos[t,k], :]) ), fp32, ascending k, no FMA.
// All K 16-byte loads of a chunk are issued before the first add.
template <int KC>
__global__ void __launch_bounds__(256)
k_combine_v8(const uint4 *__restrict__ y, const int32_t *__restrict__ pos,
             const float *__restrict__ gates, int64_t T, int Krt, int64_t H8, int64_t rows,
             uint4 *__restrict__ out)
{
    constexpr bool kFixed = KC > 0;
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    const int K = kFixed ? KC : Krt;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; j++) acc[j] = 0.0f;
            if constexpr (kFixed) {
                uint4 v[KC];
#pragma unroll
                for (int k = 0; k < KC; k++) {
                    const int32_t p = sp[k];
                    v[k] = p >= 0 ? ld_stream(y + (int64_t)p * H8 + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int k = 0; k < KC; k++) {
                    if (sp[k] < 0) continue;
                    const float g = sg[k];
                    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        acc[2 * j] = __fadd_rn(acc[2 * j], __fmul_rn(g, bf16lo(w[j])));
                        acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], __fmul_rn(g, bf16hi(w[j])));
                    }
                }
            } else {
                for (int k = 0; k < K; k++) {
                    const int32_t p = sp[k];
                    if (p < 0) continue;
                    const uint4 vv = ld_stream(y + (int64_t)p * H8 + c);
                    const float g = sg[k];
                    const uint32_t w[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        acc[2 * j] = __fadd_rn(acc[2 * j], __fmul_rn(g, bf16lo(w[j])));
                        acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], __fmul_rn(g, bf16hi(w[j])));
                    }
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            st_v4(out + t * H8 + c, o);
        }
        __syncthreads();
    }
}

// Scalar combine for any H and alignment.
__global__ void __launch_bounds__(256)
k_combine_scalar(const uint16_t *__restrict__ y, const int32_t *__restrict__ pos,
                 const float *__restrict__ gates, int64_t T, int K, int64_t H, int64_t rows,
                 uint16_t *__restrict__ out)
{
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            float acc = 0.0f;
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p < 0) continue;
                acc = __fadd_rn(acc, __fmul_rn(sg[k], bf16lo(y[(int64_t)p * H + h])));
            }
            __nv_bfloat16 b = __float2bfloat16_rn(acc);
            out[t * H + h] = *reinterpret_cast<uint16_t *>(&b);
        }
        __syncthreads();
    }
}

}  // namespace mep
