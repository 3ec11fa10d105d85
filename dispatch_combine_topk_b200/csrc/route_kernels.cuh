// Mapping, dispatch, dequantisation and combine kernels (sm_100a).
//
// Dispatch and combine are HBM-bound permute-copies: dispatch reads each token row
// once and writes it K times, combine reads K rows per token and writes one. Rows are
// moved in 16-byte chunks so that every warp access is 512 contiguous bytes, and the K
// row indices of a token are read once per token.
#pragma once

#include "common.cuh"
#include "tma.cuh"

namespace mep {

constexpr int kMaxK = 32;

// ------------------------------------------------------------------ mapping (a3)

// One thread per slot (token g, slot k): the three loads that depend on one another
// (the id, the table row's count, the instance) are the only chain a thread waits on.
// Mapping of aclnnMoeUpdateExpert (gitcode ops-transformer doc, 功能说明): instance
// column 1 for a single instance; otherwise local_rank_id / ceil(world_size / count) + 1
// (by rank) or (token mod count) + 1 (by token).
// Pruning: v = sum_k fl(scale[k] * thr[k]) in fp32, ascending k, no FMA; a slot stays
// active iff the token is active and !(scale[k] < v).
// Rows are blocks of rows_per_rank tokens: row g belongs to rank rank0 + g / rows_per_rank
// and is that rank's token i = g % rows_per_rank (one block for a single rank).
__global__ void k_update_expert(const int32_t *__restrict__ ids, const int32_t *__restrict__ table,
                                const float *__restrict__ scales, const float *__restrict__ thr,
                                const uint8_t *__restrict__ active, int64_t rows, int64_t rows_per_rank,
                                int64_t rank0, int32_t K, int32_t E, int32_t F, int64_t world_size,
                                int64_t mode, int32_t *__restrict__ out_ids,
                                uint8_t *__restrict__ out_mask)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t slots = rows * K;
    for (int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; n < slots;
         n += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = n / K;
        const int32_t k = (int32_t)(n - g * K);
        const int64_t i = g % rows_per_rank;
        const int64_t local_rank = rank0 + g / rows_per_rank;
        uint8_t act = 1;
        if (active) {
            act = active[g] ? 1 : 0;
            if (k == 0 && i > 0 && act && !active[g - 1]) flag_error(MEP_DERR_MASK);
        }
        const int32_t e = ids[n];
        int32_t inst = -1;
        if (e < 0 || e >= E) {
            flag_error(MEP_DERR_KEY_RANGE);
        } else {
            const int32_t *row = table + (int64_t)e * F;
            const int32_t c = row[0];
            if (c < 1 || c > F - 1) {
                flag_error(MEP_DERR_TABLE);
            } else {
                int64_t col;
                if (c == 1) col = 1;
                else if (mode == 0) col = local_rank / ((world_size + c - 1) / c) + 1;
                else col = (i % c) + 1;
                const int32_t v = row[col];   // col <= c <= F-1: inside the row
                if (v < 0 || v >= 1024) flag_error(MEP_DERR_TABLE);
                else inst = v;
            }
        }
        out_ids[n] = inst;
        if (scales) {
            // the token's sum, formed alike by each of its K threads
            float v = 0.0f;
            for (int32_t j = 0; j < K; j++) v = __fadd_rn(v, __fmul_rn(scales[g * K + j], thr[j]));
            out_mask[n] = (act && !(scales[n] < v)) ? 1 : 0;
        } else {
            out_mask[n] = act;
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
            flag_error(MEP_DERR_ROW_RANGE);
            p = -1;
        }
        sp[threadIdx.x] = p;
    }
}

// ------------------------------------------------------------------ dispatch (a4)

// bf16 copy for unaligned buffers or H % 8 != 0: recv[pos[t*K+k], :] = x[t, :], one CTA
// per token, one element per access.
__global__ void __launch_bounds__(256)
k_dispatch_elem(const uint16_t *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K, int64_t H,
                int64_t rows, uint16_t *__restrict__ recv)
{
    __shared__ int32_t sp[kMaxK];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        __syncthreads();
        const uint16_t *src = x + t * H;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            const uint16_t v = src[h];
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p >= 0) recv[(int64_t)p * H + h] = v;
            }
        }
        __syncthreads();
    }
}

// bf16 copy, one warp per half token row (the default path): work item i is row half
// i % 2 of token i / 2, so the last wave of warps is half as coarse as whole rows.
//
// A warp reads its token's K row indices once (lane k holds slot k, broadcast with
// shuffles), then walks the row in 16-byte chunks, kUnroll chunks per lane in flight,
// storing each loaded chunk K times. No block barriers: a warp moves on to its next
// token as soon as its stores are issued. Launched with many more warps than fit on
// the GPU at once, so the last tokens spread over the whole machine. Measured against
// bulk copies staged through shared memory (one issuing warp per SM) this path moves
// more bytes per second on both 8 KB and 14 KB rows, since 64 warps per SM keep more
// stores in flight than one bulk-copy issuer.
// Requires H % 8 == 0 and 16-byte aligned x and recv.
constexpr int kDispatchUnroll = 4;

__global__ void __launch_bounds__(256)
k_dispatch_warp(const uint4 *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K, int64_t H8,
                int64_t rows, uint4 *__restrict__ recv)
{
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t per = (H8 + 1) / 2;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < 2 * T; it += nwarps) {
        const int64_t t = it >> 1;
        int32_t mine = -1;
        if (lane < K) {
            mine = pos[t * K + lane];
            if (mine < -1 || (int64_t)mine >= rows) {
                flag_error(MEP_DERR_ROW_RANGE);
                mine = -1;
            }
        }
        const uint4 *src = x + t * H8;
        const int64_t lo = (it & 1) * per, hi = (it & 1) ? H8 : per;
        // warp-uniform trip count: every lane reaches the shuffles below
        for (int64_t base = lo; base < hi; base += 32 * kDispatchUnroll) {
            const int64_t c0 = base + lane;
            uint4 v[kDispatchUnroll];
#pragma unroll
            for (int u = 0; u < kDispatchUnroll; u++)
                if (c0 + 32 * u < hi) v[u] = ld_stream(src + c0 + 32 * u);
            for (int k = 0; k < K; k++) {
                const int32_t p = __shfl_sync(0xffffffffu, mine, k);
                if (p < 0) continue;
                uint4 *dst = recv + (int64_t)p * H8;
#pragma unroll
                for (int u = 0; u < kDispatchUnroll; u++)
                    if (c0 + 32 * u < hi) st_v4(dst + c0 + 32 * u, v[u]);
            }
        }
    }
}

// Quantise 4 fp32 values to int8 with the per-token scale; packed little-endian:
// q = clamp(round_half_even(fl(v / scale)), -127, 127), q = 0 when scale == 0.
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

// 1 / scale for q8x4_packed: 0 when scale is 0 (every value of such a row is 0), and -1
// when 1 / scale overflows (scale below about 2.9e-39, a subnormal): such rows take the
// IEEE quotient.
__device__ __forceinline__ float quant_inv(float scale)
{
    if (scale == 0.0f) return 0.0f;
    const float inv = __frcp_rn(scale);
    return isinf(inv) ? -1.0f : inv;
}

// The codes of q8x4 for the four products v = fl(x * s) of a row whose amax gave
// scale = fl(amax / 127) (the smoothing dispatch), with inv = quant_inv(scale), packed
// into one word (lowest column in the low byte). The quotient is estimated by the exact
// product z = v * inv inside a fused multiply-add: t = fl(z + 1.5 * 2^23) holds the
// integer nearest z (half to even) in its low bits (for |z| < 2^22 the spacing of t is 1),
// whose two's-complement low byte is the code; d = fl(z - (t - 1.5 * 2^23)) is the
// distance of z to that integer (t - 1.5 * 2^23 is exact). inv is within 2^-24 of
// 1 / scale (relative; a correctly rounded reciprocal of a scale whose reciprocal is
// finite) and |v / scale| < 127.0001 (scale is within one rounding of amax / 127, also
// when it is subnormal with 1 / scale finite), so
// |z - v/scale| < 7.6e-6, and fl(v/scale) is within 3.9e-6 of v/scale: |z - fl(v/scale)|
// < 2^-16. Unless z lies within 2^-15 of a half-integer, z and the correctly rounded
// quotient therefore round to the same integer, which is in [-127, 127] without a
// clamp. When any of the four lies that close (|d| >= 0.5 - 2^-15; about 1 group in
// 4000), or the row's 1 / scale overflows, all four take the IEEE quotient of q8x4.
// Each step runs on pairs (packed f32x2, each half rounded on its own); the products v
// enter the fused steps as rounded values, as multiplicands.
__device__ __forceinline__ uint32_t q8x4_packed(const float (&x)[4], const float4 &s, float scale, float inv)
{
    const float2 kShift = make_float2(12582912.0f, 12582912.0f);
    const float2 inv2 = make_float2(inv, inv);
    const float2 v0 = mul2_rn(make_float2(x[0], x[1]), make_float2(s.x, s.y));
    const float2 v1 = mul2_rn(make_float2(x[2], x[3]), make_float2(s.z, s.w));
    const float2 t0 = fma2_rn(v0, inv2, kShift), t1 = fma2_rn(v1, inv2, kShift);
    const float2 n0 = sub2_rn(kShift, t0), n1 = sub2_rn(kShift, t1);      // minus the integers, exact
    const float2 d0 = fma2_rn(v0, inv2, n0), d1 = fma2_rn(v1, inv2, n1);
    const float dmax = fmax3(fabsf(d0.x), fabsf(d0.y), fmaxf(fabsf(d1.x), fabsf(d1.y)));
    if (inv < 0.0f || dmax >= 0.5f - 0x1p-15f) return q8x4(v0.x, v0.y, v1.x, v1.y, scale);
    return __byte_perm(__byte_perm(__float_as_uint(t0.x), __float_as_uint(t0.y), 0x0040),
                       __byte_perm(__float_as_uint(t1.x), __float_as_uint(t1.y), 0x0040), 0x5410);
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

// Bytes before the row stages in the staged kernels' shared memory (barriers, row
// indices, a reduction buffer).
constexpr int kDispatchSmemHead = 2048;

// Tokens per CTA of k_dispatch_int8_staged: a grid of CTAs for kStagedChunk consecutive
// tokens each, handed to SMs as they free up (2.6% faster than a resident grid striding
// over the tokens; 8 and 32 tokens measured slower).
constexpr int kStagedChunk = 16;

// Per-token dynamic int8 staged through shared memory (the default int8 path).
//
// kThreads threads per CTA, several CTAs per SM, kStagedChunk consecutive tokens per
// CTA. Warp 0 keeps a ring of kStages bf16 rows filled by bulk loads (mbarrier
// completion) ahead of the token being quantised. For each token all threads reduce amax over the staged row,
// quantise it into one of two int8 row buffers, and lanes k < K of warp 0 bulk-store
// the codes to the row of slot k and write the scale. The int8 buffer of token i is
// reused at token i+2, after its stores have finished reading it.
//
// Dynamic shared memory: head (barriers, row indices, reduction) kDispatchSmemHead,
// then kStages bf16 rows (2H bytes each), then 2 int8 rows (H bytes each).
// Requires H % 16 == 0 and 16-byte aligned x and recv.
template <int kStages, int kThreads>
__global__ void __launch_bounds__(kThreads)
k_dispatch_int8_staged(const uint16_t *__restrict__ x, const int32_t *__restrict__ pos, int64_t T, int K,
                       int64_t H, int64_t rows, int8_t *__restrict__ recv, float *__restrict__ recv_scale)
{
    extern __shared__ __align__(128) int32_t smem_i32[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(smem_i32);
    const uint32_t row_bytes = (uint32_t)(H * 2), q_bytes = (uint32_t)H;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
    int32_t *srow = reinterpret_cast<int32_t *>(smem + 8 * kStages);              // [kStages][32]
    float *red = reinterpret_cast<float *>(smem + 8 * kStages + 128 * kStages);   // [kThreads / 32]
    unsigned char *stage = smem + kDispatchSmemHead;
    unsigned char *qbuf = stage + (size_t)kStages * row_bytes;                    // [2][H]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        for (int s = 0; s < kStages; s++) mbar_init(&bar[s], 1);
        mbar_fence_init();
    }
    __syncthreads();
    pdl_wait();                       // the barriers' set-up above touches only this CTA's memory
    pdl_launch_dependents();
    const int64_t t_lo = (int64_t)blockIdx.x * kStagedChunk;
    const int64_t n = t_lo < T ? (T - t_lo < kStagedChunk ? T - t_lo : kStagedChunk) : 0;
    auto token = [&](int64_t i) { return t_lo + i; };
    auto fetch = [&](int64_t i) {   // warp 0 only
        const int s = (int)(i % kStages);
        const int64_t t = token(i);
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[s], row_bytes);
            bulk_load_g2s(stage + (size_t)s * row_bytes, x + t * H, row_bytes, &bar[s]);
        }
        if (lane < K) {
            int32_t p = pos[t * K + lane];
            if (p < -1 || (int64_t)p >= rows) {
                flag_error(MEP_DERR_ROW_RANGE);
                p = -1;
            }
            srow[s * 32 + lane] = p;
        }
    };
    if (warp == 0)
        for (int64_t i = 0; i < n && i < kStages; i++) fetch(i);
    __syncthreads();
    const int64_t H8 = H / 8;
    for (int64_t i = 0; i < n; i++) {
        const int s = (int)(i % kStages);
        const bool ok = mbar_wait_bounded(&bar[s], (uint32_t)((i / kStages) & 1));
        if (!__syncthreads_and(ok)) {
            // Drain every load still issued, the one that just ran out included, before
            // the CTA leaves: its shared memory may go to the next CTA on this SM. A
            // drain wait that runs out as well is recorded with its own bit.
            if (tid == 0) {
                flag_error(MEP_DERR_TIMEOUT);
                for (int64_t j = i; j < n && j < i + kStages; j++)
                    if (!mbar_wait_bounded(&bar[j % kStages], (uint32_t)((j / kStages) & 1)))
                        flag_error(MEP_DERR_DRAIN);
            }
            break;
        }
        const uint4 *row = reinterpret_cast<const uint4 *>(stage + (size_t)s * row_bytes);
        float amax = 0.0f;
        for (int64_t c = tid; c < H8; c += kThreads) {
            const uint4 v = row[c];
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))),
                                     fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))),
                                     fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w)))));
        }
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
        if (lane == 0) red[warp] = amax;
        // the int8 buffer filled below was last stored two tokens ago
        if (warp == 0 && lane < K) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncthreads();
        float m = red[0];
        for (int w = 1; w < kThreads / 32; w++) m = fmaxf(m, red[w]);
        const float scale = __fdiv_rn(m, 127.0f);
        uint2 *q = reinterpret_cast<uint2 *>(qbuf + (size_t)(i & 1) * q_bytes);
        for (int64_t c = tid; c < H8; c += kThreads) {
            const uint4 v = row[c];
            uint2 o;
            o.x = q8x4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y), scale);
            o.y = q8x4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w), scale);
            q[c] = o;
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (warp == 0) {
            if (lane < K) {
                const int32_t p = srow[s * 32 + lane];
                if (p >= 0) {
                    bulk_store_s2g(recv + (int64_t)p * H, q, q_bytes);
                    recv_scale[p] = scale;
                }
                bulk_commit();
            }
            __syncwarp();
            if (i + kStages < n) fetch(i + kStages);   // every thread is done with stage s
        }
    }
    if (warp == 0 && lane < K) bulk_wait_all();
    __syncthreads();
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

// acc[0..8) = sum over kept slots k (ascending) of fl(sg[k] * y[sp[k], chunk c]) in fp32,
// each product and sum rounded on its own. All K 16-byte loads of the chunk are issued
// before the first add (compile-time K); with KC = 0 the runtime K loop is used.
template <int KC>
__device__ __forceinline__ void combine_chunk8(const uint4 *__restrict__ y, const int32_t *sp, const float *sg,
                                               int K, int64_t H8, int64_t c, float acc[8])
{
#pragma unroll
    for (int j = 0; j < 8; j++) acc[j] = 0.0f;
    if constexpr (KC > 0) {
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
}

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
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            float acc[8];
            combine_chunk8<KC>(y, sp, sg, K, H8, c, acc);
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

// --------------------------------------------------- combine of int8 rows (f1)

// bf16 value of one dequantised code, as a float: bf16_rne(fl(q * scale)).
__device__ __forceinline__ float dequant_bf16(int32_t q, float scale)
{
    return __bfloat162float(__float2bfloat16_rn(__fmul_rn((float)q, scale)));
}

// out[t, :] = bf16( sum_k fl(gate[t,k] * bf16(fl(q[pos[t,k], :] * scale[pos[t,k]]))) ):
// exactly mep_dequantize followed by mep_combine, without writing the bf16 rows. One
// CTA per token; each thread owns 8 columns (one 8-byte load of codes per slot), all K
// loads of a chunk in flight before the first add.
template <int KC>
__global__ void __launch_bounds__(256)
k_combine_int8_v8(const uint2 *__restrict__ yq, const float *__restrict__ yscale, const int32_t *__restrict__ pos,
                  const float *__restrict__ gates, int64_t T, int Krt, int64_t H8, int64_t rows,
                  uint4 *__restrict__ out)
{
    constexpr bool kFixed = KC > 0;
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    __shared__ float ss[kMaxK];
    const int K = kFixed ? KC : Krt;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        if (threadIdx.x < K) ss[threadIdx.x] = sp[threadIdx.x] >= 0 ? yscale[sp[threadIdx.x]] : 0.0f;
        __syncthreads();
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; j++) acc[j] = 0.0f;
            // Codes to floats without the conversion unit: with the sign bit flipped a
            // code q is the byte q + 128, which a byte permute places in the mantissa of
            // 1.5 * 2^23; subtracting 1.5 * 2^23 + 128 gives q exactly. The bf16
            // rounding of fl(q * scale) is one conversion per value that leaves the
            // rounded value readable as fp32 (round_bf16), with nothing to unpack.
            auto add = [&](const uint2 &v, float g, float sc) {
                const uint32_t w[2] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u};
#pragma unroll
                for (int h = 0; h < 2; h++) {
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const float qf = __uint_as_float(__byte_perm(w[h], 0x4B400000u, 0x7650u + j)) - 12583040.0f;
                        acc[4 * h + j] = __fadd_rn(acc[4 * h + j], __fmul_rn(g, round_bf16(__fmul_rn(qf, sc))));
                    }
                }
            };
            if constexpr (kFixed) {
                uint2 v[KC];
#pragma unroll
                for (int k = 0; k < KC; k++) {
                    const int32_t p = sp[k];
                    v[k] = p >= 0 ? yq[(int64_t)p * H8 + c] : make_uint2(0, 0);
                }
#pragma unroll
                for (int k = 0; k < KC; k++)
                    if (sp[k] >= 0) add(v[k], sg[k], ss[k]);
            } else {
                for (int k = 0; k < K; k++) {
                    const int32_t p = sp[k];
                    if (p < 0) continue;
                    add(yq[(int64_t)p * H8 + c], sg[k], ss[k]);
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

// acc[j] (columns 2j, 2j+1 of a 16-column chunk) += fl(g * bf16(fl(q * sc))) for the 16
// codes in v. Codes become floats as in k_combine_int8_v8 (byte permute into 1.5 * 2^23);
// the exact bias subtraction and the code * scale product run on pairs of columns
// (packed f32x2, each half rounded on its own).
__device__ __forceinline__ void add_int8_x16(float2 (&acc)[8], const uint4 &v, float g, float sc)
{
    const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
    const float2 s2 = make_float2(sc, sc);
    const float2 nb = make_float2(-12583040.0f, -12583040.0f);
#pragma unroll
    for (int h = 0; h < 4; h++) {
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
            const float2 qb = make_float2(__uint_as_float(__byte_perm(w[h], 0x4B400000u, 0x7650u + j)),
                                          __uint_as_float(__byte_perm(w[h], 0x4B400000u, 0x7651u + j)));
            const float2 p = mul2_rn(add2_rn(qb, nb), s2);
            // the gate product is packed, the sum scalar: a packed multiply feeding a
            // packed add may be fused into one rounding, which the sum's definition (two
            // roundings) does not allow
            const float2 gy = mul2_rn(make_float2(g, g), make_float2(round_bf16(p.x), round_bf16(p.y)));
            float2 &a = acc[2 * h + j / 2];
            a.x = __fadd_rn(a.x, gy.x);
            a.y = __fadd_rn(a.y, gy.y);
        }
    }
}

__device__ __forceinline__ void store_bf16x16(uint4 *dst, const float2 (&acc)[8])
{
    uint4 o0, o1;
    o0.x = pack_bf16x2(acc[0].x, acc[0].y);
    o0.y = pack_bf16x2(acc[1].x, acc[1].y);
    o0.z = pack_bf16x2(acc[2].x, acc[2].y);
    o0.w = pack_bf16x2(acc[3].x, acc[3].y);
    o1.x = pack_bf16x2(acc[4].x, acc[4].y);
    o1.y = pack_bf16x2(acc[5].x, acc[5].y);
    o1.z = pack_bf16x2(acc[6].x, acc[6].y);
    o1.w = pack_bf16x2(acc[7].x, acc[7].y);
    st_v4(dst, o0);
    st_v4(dst + 1, o1);
}

// The combine of int8 rows for H % 16 == 0 and 16-byte aligned buffers (the same sum as
// k_combine_int8_v8, 16 codes per slot per lane), one warp per token: lane k < K holds slot k's
// row, gate and scale, which the other lanes take by shuffle once per token. There is no
// block barrier, and the slot values stay in registers across the token's column chunks.
// (Keeping them in shared memory instead allows 6 CTAs per SM instead of 5 and measured
// faster alone, but 3% slower inside the routing step, where the GPU runs at its power
// limit and the extra shared-memory reads cost more than the occupancy gains.)
constexpr int kCombineInt8Threads = 128;

template <int KC>
__global__ void __launch_bounds__(128)
k_combine_int8_warp(const uint4 *__restrict__ yq, const float *__restrict__ yscale, const int32_t *__restrict__ pos,
                    const float *__restrict__ gates, int64_t T, int Krt, int64_t H16, int64_t rows,
                    uint4 *__restrict__ out)
{
    constexpr bool kFixed = KC > 0;
    const int K = kFixed ? KC : Krt;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int32_t mine = -1;
        float g_mine = 0.0f, s_mine = 0.0f;
        if (lane < K) {
            mine = pos[t * K + lane];
            if (mine < -1 || (int64_t)mine >= rows) {
                flag_error(MEP_DERR_ROW_RANGE);
                mine = -1;
            }
            g_mine = gates[t * K + lane];
            if (mine >= 0) s_mine = yscale[mine];
        }
        uint4 *dst = out + t * 2 * H16;
        if constexpr (kFixed) {
            int32_t pk[KC];
            float gk[KC], sk[KC];
#pragma unroll
            for (int k = 0; k < KC; k++) {
                pk[k] = __shfl_sync(0xffffffffu, mine, k);
                gk[k] = __shfl_sync(0xffffffffu, g_mine, k);
                sk[k] = __shfl_sync(0xffffffffu, s_mine, k);
            }
            // every slot kept (the usual case): a loop without the per-slot tests, the rows'
            // base addresses once per token, and the output stored with plain stores, which
            // leave the compiler free to schedule around them (3% faster inside the step)
            bool all = true;
#pragma unroll
            for (int k = 0; k < KC; k++) all = all && pk[k] >= 0;
            if (all) {
                const uint4 *rp[KC];
#pragma unroll
                for (int k = 0; k < KC; k++) rp[k] = yq + (int64_t)pk[k] * H16;
                for (int64_t c = lane; c < H16; c += 32) {
                    float2 acc[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) acc[j] = make_float2(0.0f, 0.0f);
                    uint4 v[KC];
#pragma unroll
                    for (int k = 0; k < KC; k++) v[k] = ld_stream(rp[k] + c);
#pragma unroll
                    for (int k = 0; k < KC; k++) add_int8_x16(acc, v[k], gk[k], sk[k]);
                    uint4 o0, o1;
                    o0.x = pack_bf16x2(acc[0].x, acc[0].y); o0.y = pack_bf16x2(acc[1].x, acc[1].y);
                    o0.z = pack_bf16x2(acc[2].x, acc[2].y); o0.w = pack_bf16x2(acc[3].x, acc[3].y);
                    o1.x = pack_bf16x2(acc[4].x, acc[4].y); o1.y = pack_bf16x2(acc[5].x, acc[5].y);
                    o1.z = pack_bf16x2(acc[6].x, acc[6].y); o1.w = pack_bf16x2(acc[7].x, acc[7].y);
                    dst[2 * c] = o0;
                    dst[2 * c + 1] = o1;
                }
            } else {
                for (int64_t c = lane; c < H16; c += 32) {
                    float2 acc[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) acc[j] = make_float2(0.0f, 0.0f);
                    uint4 v[KC];
#pragma unroll
                    for (int k = 0; k < KC; k++)
                        v[k] = pk[k] >= 0 ? ld_stream(yq + (int64_t)pk[k] * H16 + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int k = 0; k < KC; k++)
                        if (pk[k] >= 0) add_int8_x16(acc, v[k], gk[k], sk[k]);
                    store_bf16x16(dst + 2 * c, acc);
                }
            }
        } else {
            // warp-uniform trip count: every lane reaches the shuffles
            for (int64_t base = 0; base < H16; base += 32) {
                const int64_t c = base + lane;
                float2 acc[8];
#pragma unroll
                for (int j = 0; j < 8; j++) acc[j] = make_float2(0.0f, 0.0f);
                for (int k = 0; k < K; k++) {
                    const int32_t p = __shfl_sync(0xffffffffu, mine, k);
                    const float g = __shfl_sync(0xffffffffu, g_mine, k);
                    const float sc = __shfl_sync(0xffffffffu, s_mine, k);
                    if (p >= 0 && c < H16) add_int8_x16(acc, ld_stream(yq + (int64_t)p * H16 + c), g, sc);
                }
                if (c < H16) store_bf16x16(dst + 2 * c, acc);
            }
        }
    }
}

// Element version for any H and alignment.
__global__ void __launch_bounds__(256)
k_combine_int8_scalar(const int8_t *__restrict__ yq, const float *__restrict__ yscale,
                      const int32_t *__restrict__ pos, const float *__restrict__ gates, int64_t T, int K,
                      int64_t H, int64_t rows, uint16_t *__restrict__ out)
{
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    __shared__ float ss[kMaxK];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        if (threadIdx.x < K) ss[threadIdx.x] = sp[threadIdx.x] >= 0 ? yscale[sp[threadIdx.x]] : 0.0f;
        __syncthreads();
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            float acc = 0.0f;
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p < 0) continue;
                acc = __fadd_rn(acc, __fmul_rn(sg[k], dequant_bf16(yq[(int64_t)p * H + h], ss[k])));
            }
            __nv_bfloat16 b = __float2bfloat16_rn(acc);
            out[t * H + h] = *reinterpret_cast<uint16_t *>(&b);
        }
        __syncthreads();
    }
}

// ------------------------------------------- combine + residual add + RMSNorm (f4)

// Block-wide sum of one float per thread (blockDim.x a multiple of 32, at most 1024);
// red holds 33 floats of shared memory. Every thread gets the sum. Ends with a barrier.
__device__ __forceinline__ float block_sum(float v, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float t = lane < nw ? red[lane] : 0.0f;
        for (int d = 16; d > 0; d >>= 1) t += __shfl_xor_sync(0xffffffffu, t, d);
        if (lane == 0) red[32] = t;
    }
    __syncthreads();
    return red[32];
}

// For every token: c = the combine output row (bf16, as k_combine_v8), x = fl(c + r)
// with r the residual row, x_out = bf16(x), rstd = rsqrt_rn(fl(sum x^2 / H) + eps),
// y_out = bf16(fl(fl(x * rstd) * gamma)). The fp32 row x is kept in shared memory
// (H floats) between the reduction and the second pass, column 8c + j of the row at
// xs[j * H8 + c], so that the lanes of a warp (consecutive c) touch consecutive words.
template <int KC>
__global__ void __launch_bounds__(256, 4)
k_combine_add_rmsnorm_v8(const uint4 *__restrict__ y, const int32_t *__restrict__ pos,
                         const float *__restrict__ gates, int64_t T, int Krt, int64_t H8, int64_t rows,
                         const uint4 *__restrict__ residual, const uint4 *__restrict__ gamma, float eps,
                         uint4 *__restrict__ x_out, uint4 *__restrict__ y_out, float *__restrict__ rstd_out)
{
    constexpr bool kFixed = KC > 0;
    extern __shared__ float xs[];    // [H]
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    __shared__ float red[33];
    const int K = kFixed ? KC : Krt;
    const float inv_h = 1.0f / (float)(H8 * 8);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        float ss = 0.0f;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            float acc[8];
            combine_chunk8<KC>(y, sp, sg, K, H8, c, acc);
            const uint4 r = ld_stream(residual + t * H8 + c);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
            uint32_t xo[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t cb = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);   // the combine output
                const float x0 = __fadd_rn(bf16lo(cb), bf16lo(rw[j]));
                const float x1 = __fadd_rn(bf16hi(cb), bf16hi(rw[j]));
                xs[(2 * j) * H8 + c] = x0;
                xs[(2 * j + 1) * H8 + c] = x1;
                ss = fmaf(x0, x0, ss);
                ss = fmaf(x1, x1, ss);
                xo[j] = pack_bf16x2(x0, x1);
            }
            st_v4(x_out + t * H8 + c, make_uint4(xo[0], xo[1], xo[2], xo[3]));
        }
        const float total = block_sum(ss, red);
        const float rstd = __frsqrt_rn(__fadd_rn(__fmul_rn(total, inv_h), eps));
        if (threadIdx.x == 0) rstd_out[t] = rstd;
        for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
            const uint4 gm = gamma[c];
            const uint32_t gw[4] = {gm.x, gm.y, gm.z, gm.w};
            uint32_t yo[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float y0 = __fmul_rn(__fmul_rn(xs[(2 * j) * H8 + c], rstd), bf16lo(gw[j]));
                const float y1 = __fmul_rn(__fmul_rn(xs[(2 * j + 1) * H8 + c], rstd), bf16hi(gw[j]));
                yo[j] = pack_bf16x2(y0, y1);
            }
            st_v4(y_out + t * H8 + c, make_uint4(yo[0], yo[1], yo[2], yo[3]));
        }
        __syncthreads();
    }
}

// Element version for any H and alignment (same arithmetic).
__global__ void __launch_bounds__(256)
k_combine_add_rmsnorm_scalar(const uint16_t *__restrict__ y, const int32_t *__restrict__ pos,
                             const float *__restrict__ gates, int64_t T, int K, int64_t H, int64_t rows,
                             const uint16_t *__restrict__ residual, const uint16_t *__restrict__ gamma,
                             float eps, uint16_t *__restrict__ x_out, uint16_t *__restrict__ y_out,
                             float *__restrict__ rstd_out)
{
    extern __shared__ float xs[];    // [H]
    __shared__ int32_t sp[kMaxK];
    __shared__ float sg[kMaxK];
    __shared__ float red[33];
    const float inv_h = 1.0f / (float)H;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) sg[threadIdx.x] = gates[t * K + threadIdx.x];
        __syncthreads();
        float ss = 0.0f;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            float acc = 0.0f;
            for (int k = 0; k < K; k++) {
                const int32_t p = sp[k];
                if (p < 0) continue;
                acc = __fadd_rn(acc, __fmul_rn(sg[k], bf16lo(y[(int64_t)p * H + h])));
            }
            const float cval = bf16lo(pack_bf16x2(acc, 0.0f) & 0xffffu);
            const float x = __fadd_rn(cval, bf16lo(residual[t * H + h]));
            xs[h] = x;
            ss = fmaf(x, x, ss);
            x_out[t * H + h] = (uint16_t)(pack_bf16x2(x, 0.0f) & 0xffffu);
        }
        const float total = block_sum(ss, red);
        const float rstd = __frsqrt_rn(__fadd_rn(__fmul_rn(total, inv_h), eps));
        if (threadIdx.x == 0) rstd_out[t] = rstd;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
            const float v = __fmul_rn(__fmul_rn(xs[h], rstd), bf16lo(gamma[h]));
            y_out[t * H + h] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xffffu);
        }
        __syncthreads();
    }
}

// ------------------------------------------ smooth-quantised int8 dispatch (f1)

// Block-wide max of one non-negative float per thread (every thread gets it); red holds
// 33 floats of shared memory. Ends with a barrier.
__device__ __forceinline__ float block_max(float v, float *red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int d = 16; d > 0; d >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, d));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float t = lane < nw ? red[lane] : 0.0f;
        for (int d = 16; d > 0; d >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, d));
        if (lane == 0) red[32] = t;
    }
    __syncthreads();
    return red[32];
}

// Smooth-quantised int8 dispatch, the K slots of a token taken together (any K up to
// kMaxK), one CTA of 256 threads per token, the token's row in registers: pass 1 forms, slot by slot, each thread's maximum of |fl(x * smooth[e_k])| and its warp
// maximum (every smoothing row read once; the warp maximum by redux.sync); one block
// barrier later the K scales follow from the warps' maxima; pass 2 forms each product
// again (the smoothing rows a second time, from L2) and stores the codes. Two block
// barriers per token instead of two per slot. Both passes walk the slots in a loop that
// is not unrolled, which keeps the code short and the registers at 64 (4 CTAs per SM).
// A thread takes groups of 4 columns (g = tid + 256 i): its x, its smoothing scales and
// its codes are then 8, 16 and 4 consecutive bytes, so every warp load and store of the
// three is one contiguous span (the smoothing rows, read K times per token, are the
// bulk of the traffic through L1).
template <int kGroups>
__global__ void __launch_bounds__(256)
k_dispatch_int8_smooth_k(const uint2 *__restrict__ x, const int32_t *__restrict__ ids, const int32_t *__restrict__ pos,
                         int64_t T, int K, int64_t H4, const float4 *__restrict__ smooth, int32_t n_experts, int64_t rows,
                         uint32_t *__restrict__ recv, float *__restrict__ recv_scale)
{
    __shared__ int32_t sp[kMaxK], se[kMaxK];
    __shared__ float red[8][kMaxK];                   // 256 threads = 8 warps
    __shared__ float ssc[kMaxK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h4 = (int)H4;                           // at most 256 * kGroups
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if (threadIdx.x < K) {
            int32_t p = pos[t * K + threadIdx.x];
            if (p < -1 || (int64_t)p >= rows) {
                flag_error(MEP_DERR_ROW_RANGE);
                p = -1;
            }
            int32_t e = ids[t * K + threadIdx.x];
            if (e < 0 || e >= n_experts) {
                flag_error(MEP_DERR_KEY_RANGE);
                e = -1;
            }
            sp[threadIdx.x] = p;
            se[threadIdx.x] = e;
        }
        float xr[kGroups][4];
        const uint2 *xrow = x + t * H4;
#pragma unroll
        for (int i = 0; i < kGroups; i++) {
            const int g = threadIdx.x + i * 256;
            if (g < h4) {
                const uint2 v = xrow[g];
                xr[i][0] = bf16lo(v.x);
                xr[i][1] = bf16hi(v.x);
                xr[i][2] = bf16lo(v.y);
                xr[i][3] = bf16hi(v.y);
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < K; k++) {
            float amax = 0.0f;
            const int32_t e = se[k];
            if (sp[k] >= 0 && e >= 0) {
                const float4 *srow = smooth + (int64_t)e * H4;
#pragma unroll
                for (int i = 0; i < kGroups; i++) {
                    const int g = threadIdx.x + i * 256;
                    if (g < h4) {
                        const float4 sv = srow[g];
                        const float2 v0 = mul2_rn(make_float2(xr[i][0], xr[i][1]), make_float2(sv.x, sv.y));
                        const float2 v1 = mul2_rn(make_float2(xr[i][2], xr[i][3]), make_float2(sv.z, sv.w));
                        amax = fmax3(fmax3(amax, fabsf(v0.x), fabsf(v0.y)), fabsf(v1.x), fabsf(v1.y));
                    }
                }
            }
            // warp maximum of non-negative floats (products of finite inputs): their bits order
            // like their values, so one integer reduction gives it
            amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
            if (lane == 0) red[warp][k] = amax;
        }
        __syncthreads();
        if (threadIdx.x < K) {
            float m = 0.0f;
            for (int w = 0; w < 8; w++) m = fmaxf(m, red[w][threadIdx.x]);
            const float scale = __fdiv_rn(m, 127.0f);
            ssc[threadIdx.x] = scale;
            if (sp[threadIdx.x] >= 0 && se[threadIdx.x] >= 0) recv_scale[sp[threadIdx.x]] = scale;
        }
        __syncthreads();
#pragma unroll 1
        for (int k = 0; k < K; k++) {                     // one slot at a time: a short loop body
            const int32_t p = sp[k], e = se[k];
            if (p < 0 || e < 0) continue;
            const float scale = ssc[k], inv = quant_inv(scale);
            const float4 *srow = smooth + (int64_t)e * H4;
            uint32_t *dst = recv + (int64_t)p * H4;
#pragma unroll
            for (int i = 0; i < kGroups; i++) {
                const int g = threadIdx.x + i * 256;
                if (g < h4) dst[g] = q8x4_packed(xr[i], srow[g], scale, inv);
            }
        }
        __syncthreads();                                   // sp, se, ssc and red are reused
    }
}

// Element version for any H and alignment: two passes per slot over x and the scales.
__global__ void __launch_bounds__(256)
k_dispatch_int8_smooth_scalar(const uint16_t *__restrict__ x, const int32_t *__restrict__ ids,
                              const int32_t *__restrict__ pos, int64_t T, int K, int64_t H,
                              const float *__restrict__ smooth, int32_t n_experts, int64_t rows,
                              int8_t *__restrict__ recv, float *__restrict__ recv_scale)
{
    __shared__ int32_t sp[kMaxK];
    __shared__ int32_t se[kMaxK];
    __shared__ float red[33];
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        load_token_rows(pos, t, K, rows, sp);
        if (threadIdx.x < K) {
            int32_t e = ids[t * K + threadIdx.x];
            if (e < 0 || e >= n_experts) {
                flag_error(MEP_DERR_KEY_RANGE);
                e = -1;
            }
            se[threadIdx.x] = e;
        }
        __syncthreads();
        for (int k = 0; k < K; k++) {
            const int32_t p = sp[k], e = se[k];
            if (p < 0 || e < 0) continue;
            float amax = 0.0f;
            for (int64_t h = threadIdx.x; h < H; h += blockDim.x)
                amax = fmaxf(amax, fabsf(__fmul_rn(bf16lo(x[t * H + h]), smooth[(int64_t)e * H + h])));
            amax = block_max(amax, red);
            const float scale = __fdiv_rn(amax, 127.0f);
            if (threadIdx.x == 0) recv_scale[p] = scale;
            for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
                int r = 0;
                if (scale != 0.0f) {
                    const float v = __fmul_rn(bf16lo(x[t * H + h]), smooth[(int64_t)e * H + h]);
                    r = max(-127, min(127, __float2int_rn(__fdiv_rn(v, scale))));
                }
                recv[(int64_t)p * H + h] = (int8_t)r;
            }
            __syncthreads();
        }
    }
}

// ----------------------------------- replica weight prefetch and grad reduce (f2, f3)

// One thread per rank: walk its replicas in order; a replica of an expert homed on
// another rank takes the next free slot while slots remain (weight row E + r*B + b),
// otherwise it reads the home row e; home replicas read row e.
__global__ void k_prefetch_plan(const int32_t *__restrict__ rep_count, const int32_t *__restrict__ rep_key, int32_t R,
                                int32_t E, int32_t cap, int32_t B, int32_t *__restrict__ slot_expert,
                                int32_t *__restrict__ rep_weight)
{
    const int32_t r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= R) return;
    const int32_t per_rank = E / R;
    for (int32_t b = 0; b < B; b++) slot_expert[(int64_t)r * B + b] = -1;
    for (int32_t j = 0; j < cap; j++) rep_weight[(int64_t)r * cap + j] = -1;
    int32_t n = rep_count[r];
    if (n < 0 || n > cap) {
        flag_error(MEP_DERR_KEY_RANGE);
        n = n < 0 ? 0 : cap;
    }
    int32_t used = 0;
    for (int32_t j = 0; j < n; j++) {
        const int32_t e = rep_key[(int64_t)r * cap + j];
        if (e < 0 || e >= E) {
            flag_error(MEP_DERR_KEY_RANGE);
            continue;
        }
        int32_t row = e;
        if (e / per_rank != r && used < B) {
            slot_expert[(int64_t)r * B + used] = e;
            row = E + r * B + used;
            used++;
        }
        rep_weight[(int64_t)r * cap + j] = row;
    }
}

// w_slots[s, :] = w_home[slot_expert[s], :]; blockIdx.y = slot, CTAs of a slot stride
// over its 16-byte chunks. Unused slots (-1) exit at once.
__global__ void __launch_bounds__(256)
k_prefetch_weights(const uint4 *__restrict__ w_home, const int32_t *__restrict__ slot_expert, int32_t E, int64_t D8,
                   uint4 *__restrict__ w_slots)
{
    const int32_t e = slot_expert[blockIdx.y];
    if (e < 0) return;
    if (e >= E) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(MEP_DERR_KEY_RANGE);
        return;
    }
    const uint4 *src = w_home + (int64_t)e * D8;
    uint4 *dst = w_slots + (int64_t)blockIdx.y * D8;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < D8; c += (int64_t)gridDim.x * blockDim.x)
        st_v4(dst + c, ld_stream(src + c));
}

__global__ void __launch_bounds__(256)
k_prefetch_weights_scalar(const uint16_t *__restrict__ w_home, const int32_t *__restrict__ slot_expert, int32_t E,
                          int64_t D, uint16_t *__restrict__ w_slots)
{
    const int32_t e = slot_expert[blockIdx.y];
    if (e < 0) return;
    if (e >= E) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(MEP_DERR_KEY_RANGE);
        return;
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < D; i += (int64_t)gridDim.x * blockDim.x)
        w_slots[(int64_t)blockIdx.y * D + i] = w_home[(int64_t)e * D + i];
}

// The slots holding expert e, in ascending order, compacted into list (shared memory,
// at most `max_list` entries kept). Called by every thread; returns the count.
__device__ __forceinline__ int32_t slots_of_expert(const int32_t *__restrict__ slot_expert, int32_t RB, int32_t e,
                                                   int32_t *list, int32_t max_list, int32_t *warp_cnt)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int32_t total = 0;
    for (int32_t base = 0; base < RB; base += blockDim.x) {
        const int32_t s = base + threadIdx.x;
        const bool hit = s < RB && slot_expert[s] == e;
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) warp_cnt[warp] = __popc(m);
        __syncthreads();
        int32_t before = total;
        for (int w = 0; w < warp; w++) before += warp_cnt[w];
        int32_t round_total = 0;
        for (int w = 0; w < nw; w++) round_total += warp_cnt[w];
        if (hit) {
            const int32_t at = before + __popc(m & lanemask_lt());
            if (at < max_list) list[at] = s;
        }
        total += round_total;
        __syncthreads();
    }
    return total;
}

// grad_home[e, :] += grad_slots[s, :] over e's slots in ascending order (fp32, one
// rounding per addition), then those slots are zeroed. blockIdx.y = expert; CTAs of an
// expert stride over 16-byte chunks (4 floats). Experts without a slot do nothing.
constexpr int kMaxSlotsPerExpert = 1024;
constexpr int kReduceUnroll = 4;   // 16-byte chunks per thread in flight

__global__ void __launch_bounds__(256)
k_grad_reduce(float4 *__restrict__ grad_home, float4 *__restrict__ grad_slots, const int32_t *__restrict__ slot_expert,
              int32_t RB, int64_t D4)
{
    __shared__ int32_t list[kMaxSlotsPerExpert];
    __shared__ int32_t warp_cnt[32];
    const int32_t e = blockIdx.y;
    const int32_t n = slots_of_expert(slot_expert, RB, e, list, kMaxSlotsPerExpert, warp_cnt);
    if (n == 0) return;
    const int32_t m = n < kMaxSlotsPerExpert ? n : kMaxSlotsPerExpert;
    if (n > kMaxSlotsPerExpert && blockIdx.x == 0 && threadIdx.x == 0) flag_error(MEP_DERR_KEY_RANGE);
    float4 *home = grad_home + (int64_t)e * D4;
    const int64_t step = (int64_t)gridDim.x * blockDim.x * kReduceUnroll;
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int64_t c0 = (int64_t)blockIdx.x * blockDim.x * kReduceUnroll + threadIdx.x; c0 < D4; c0 += step) {
        float4 acc[kReduceUnroll];
#pragma unroll
        for (int u = 0; u < kReduceUnroll; u++) {
            const int64_t c = c0 + (int64_t)u * blockDim.x;
            acc[u] = c < D4 ? home[c] : zero;
        }
        // all of the expert's slots are read before any is cleared, so the loads of
        // consecutive slots need not wait for stores to the same array
#pragma unroll 2
        for (int32_t i = 0; i < m; i++) {
            const float4 *slot = grad_slots + (int64_t)list[i] * D4;
            float4 v[kReduceUnroll];
#pragma unroll
            for (int u = 0; u < kReduceUnroll; u++) {
                const int64_t c = c0 + (int64_t)u * blockDim.x;
                v[u] = c < D4 ? slot[c] : zero;
            }
#pragma unroll
            for (int u = 0; u < kReduceUnroll; u++) {
                acc[u].x = __fadd_rn(acc[u].x, v[u].x);
                acc[u].y = __fadd_rn(acc[u].y, v[u].y);
                acc[u].z = __fadd_rn(acc[u].z, v[u].z);
                acc[u].w = __fadd_rn(acc[u].w, v[u].w);
            }
        }
#pragma unroll
        for (int u = 0; u < kReduceUnroll; u++) {
            const int64_t c = c0 + (int64_t)u * blockDim.x;
            if (c < D4) home[c] = acc[u];
        }
        for (int32_t i = 0; i < m; i++) {
            float4 *slot = grad_slots + (int64_t)list[i] * D4;
#pragma unroll
            for (int u = 0; u < kReduceUnroll; u++) {
                const int64_t c = c0 + (int64_t)u * blockDim.x;
                if (c < D4) slot[c] = zero;
            }
        }
    }
}

__global__ void __launch_bounds__(256)
k_grad_reduce_scalar(float *__restrict__ grad_home, float *__restrict__ grad_slots, const int32_t *__restrict__ slot_expert,
                     int32_t RB, int64_t D)
{
    __shared__ int32_t list[kMaxSlotsPerExpert];
    __shared__ int32_t warp_cnt[32];
    const int32_t e = blockIdx.y;
    const int32_t n = slots_of_expert(slot_expert, RB, e, list, kMaxSlotsPerExpert, warp_cnt);
    if (n == 0) return;
    const int32_t m = n < kMaxSlotsPerExpert ? n : kMaxSlotsPerExpert;
    if (n > kMaxSlotsPerExpert && blockIdx.x == 0 && threadIdx.x == 0) flag_error(MEP_DERR_KEY_RANGE);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < D; i += (int64_t)gridDim.x * blockDim.x) {
        float acc = grad_home[(int64_t)e * D + i];
        for (int32_t j = 0; j < m; j++) {
            const int64_t k = (int64_t)list[j] * D + i;
            acc = __fadd_rn(acc, grad_slots[k]);
            grad_slots[k] = 0.0f;
        }
        grad_home[(int64_t)e * D + i] = acc;
    }
}

// --------------------------------------------------------------- wait self-test

// Waits, with the library's bounded wait, on an mbarrier that nothing ever completes:
// the wait runs out after max_polls polls, the kernel records MEP_DERR_TIMEOUT and
// returns, exactly as a routing kernel whose bulk load never landed would.
__global__ void k_selftest_wait(int max_polls, int32_t *timed_out)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);     // one arrival expected, none ever made
        mbar_fence_init();
    }
    __syncthreads();
    const bool ok = mbar_wait_bounded(&bar, 0, max_polls);
    if (threadIdx.x == 0) {
        if (!ok) flag_error(MEP_DERR_TIMEOUT);
        *timed_out = ok ? 0 : 1;
    }
}

}  // namespace mep

