// Smooth-quantised int8 dispatch with the slots taken in expert order inside chunks of
// tokens (sm_100a).
//
// Every kept slot n of token t with expert e quantises fl(x[t, :] * smooth[e, :]) with
// its own scale (the per-expert smoothing scales of aclnnMoeDistributeDispatch, gitcode
// ops-transformer aclnnMoeUpdateExpert doc, 调用示例). Taken token by token, every slot
// reads its expert's whole smoothing row (4H bytes, twice: once for the maximum, once
// for the codes), K times the bytes of the token's own row. Here the slots are first
// sorted by expert within chunks of kSmoothChunkSlots slots (k_smooth_order, one CTA
// per chunk: a counting sort in shared memory into a caller-owned list), and a CTA then
// walks kSmoothSlotsPerCTA consecutive entries of that list: slots of a few experts,
// whose smoothing values each thread keeps in registers across the slots, and of tokens
// of one chunk, whose rows (a chunk is a few MB of x) stay in L2 while the CTAs of the
// chunk run. Per slot, the L2 reads are the token's row twice (2H bytes each) instead of
// the smoothing row twice (4H bytes each). Each CTA takes two phases over its slots with
// one barrier between them: the maxima of all its slots (no barrier per slot), then,
// after one warp has formed the slots' scales, their codes. The arithmetic per slot is
// that of k_dispatch_int8_smooth_k (the same products, maximum, scale and q8x4_packed),
// so codes and scales are identical to it.
#pragma once

#include "common.cuh"
#include "plan_kernels.cuh"
#include "route_kernels.cuh"

namespace mep {

constexpr int kSmoothChunkSlots = 2048;       // slots per chunk of tokens
constexpr int kSmoothOrderThreads = 1024;
constexpr int kSmoothSlotsPerCTA = 16;        // entries of the list per CTA (at most 32)
constexpr int kSmoothOrderMaxExperts = 6000;  // 2 (E + 2) ints of shared memory in k_smooth_order

// The sort key of slot n: its expert when the slot is kept and its id and row are in
// range, else n_experts (such slots go last in their chunk and are skipped). With
// `flag`, out-of-range ids and rows set their error bits (as k_dispatch_int8_smooth_k).
__device__ __forceinline__ int32_t smooth_key(const int32_t *__restrict__ ids, const int32_t *__restrict__ pos,
                                              int64_t n, int32_t n_experts, int64_t rows, bool flag)
{
    const int32_t p = pos[n], e = ids[n];
    bool ok = p >= 0;
    if (p < -1 || (int64_t)p >= rows) {
        if (flag) flag_error(MEP_DERR_ROW_RANGE);
        ok = false;
    }
    if (e < 0 || e >= n_experts) {
        if (flag) flag_error(MEP_DERR_KEY_RANGE);
        ok = false;
    }
    return ok ? e : n_experts;
}

// One CTA per chunk of `chunk` tokens (chunk * K slots): order[lo .. hi) = the chunk's
// slot indices sorted by smooth_key (within a key in no particular order). Dynamic
// shared memory: cnt [n_experts + 1], off [n_experts + 2].
__global__ void __launch_bounds__(kSmoothOrderThreads)
k_smooth_order(const int32_t *__restrict__ ids, const int32_t *__restrict__ pos, int64_t T, int K, int64_t chunk,
               int32_t n_experts, int64_t rows, int32_t *__restrict__ order)
{
    extern __shared__ int32_t smem[];
    __shared__ int32_t scan_scratch[33];
    int32_t *cnt = smem;
    int32_t *off = cnt + n_experts + 1;
    pdl_wait();
    pdl_launch_dependents();
    const int64_t t0 = (int64_t)blockIdx.x * chunk;
    const int64_t lo = t0 * K, hi = min(T, t0 + chunk) * K;
    for (int i = threadIdx.x; i <= n_experts; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    for (int64_t n = lo + threadIdx.x; n < hi; n += blockDim.x)
        atomicAdd(&cnt[smooth_key(ids, pos, n, n_experts, rows, true)], 1);
    __syncthreads();
    block_exclusive_scan(cnt, n_experts + 1, off, scan_scratch);
    for (int64_t n = lo + threadIdx.x; n < hi; n += blockDim.x) {
        const int32_t key = smooth_key(ids, pos, n, n_experts, rows, false);
        order[lo + atomicAdd(&off[key], 1)] = (int32_t)n;
    }
}

// The codes and scales of the slots order[i0 .. i0 + kSmoothSlotsPerCTA), i0 =
// blockIdx.x * kSmoothSlotsPerCTA, by a CTA of kSmoothThreads threads. A thread takes the
// groups of 4 columns g = tid + 256 i (i < kGroups): its x, smoothing scales and codes are
// 8, 16 and 4 consecutive bytes, contiguous over a warp, at fixed offsets from the row's
// base; with kFull (H / 4 == 256 * kGroups) every thread has all kGroups groups and the
// column tests drop out. Needs H % 4 == 0 with H / 4 <= 256 * kGroups, 8-byte aligned x,
// 16-byte aligned smooth and 4-byte aligned recv.
constexpr int kSmoothThreads = 256;
constexpr int kSmoothMaxGroups = 8;                   // H up to 8192

template <int kGroups, bool kFull>
__global__ void __launch_bounds__(kSmoothThreads, kGroups >= 7 ? 3 : 4)
k_dispatch_int8_smooth_grouped(const uint2 *__restrict__ x, const int32_t *__restrict__ ids,
                               const int32_t *__restrict__ pos, const int32_t *__restrict__ order, int64_t N, int K,
                               int64_t H4, const float4 *__restrict__ smooth, int32_t n_experts, int64_t rows,
                               uint32_t *__restrict__ recv, float *__restrict__ recv_scale)
{
    constexpr int P = kSmoothSlotsPerCTA;
    constexpr int kWarps = kSmoothThreads / 32;
    __shared__ int32_t s_tok[P], s_e[P], s_p[P];           // token, expert (-1: skipped), row
    __shared__ float red[P][kWarps];                       // per slot: the warps' maxima
    __shared__ float s_scale[P], s_inv[P];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = (int64_t)blockIdx.x * P;
    const int n_here = (int)min((int64_t)P, N - i0);
    if (threadIdx.x < P) {
        int32_t tok = 0, e = -1, p = -1;
        if ((int)threadIdx.x < n_here) {
            const int32_t n = order[i0 + threadIdx.x];
            if (n >= 0 && n < N) {                         // the list holds every slot once
                p = pos[n];
                e = ids[n];
                tok = n / K;
            }
            if (p < 0 || (int64_t)p >= rows || e < 0 || e >= n_experts) {   // flagged by k_smooth_order
                e = -1;
                p = -1;
            }
        }
        s_tok[threadIdx.x] = tok;
        s_e[threadIdx.x] = e;
        s_p[threadIdx.x] = p;
    }
    __syncthreads();
    const int h4 = (int)H4;
    float4 sv[kGroups];
    int32_t cur_e = -1;
    auto load_smooth = [&](int32_t e) {
        const float4 *srow = smooth + (int64_t)e * H4 + threadIdx.x;
#pragma unroll
        for (int i = 0; i < kGroups; i++)
            if (kFull || (int)threadIdx.x + i * kSmoothThreads < h4) sv[i] = srow[i * kSmoothThreads];
        cur_e = e;
    };
    // slot j's x row into xr (nothing for a skipped slot or j past the CTA's share)
    auto load_x = [&](int j, uint2 (&xr)[kGroups]) {
        if (j >= n_here || s_e[j] < 0) return;
        const uint2 *xrow = x + (int64_t)s_tok[j] * H4 + threadIdx.x;
#pragma unroll
        for (int i = 0; i < kGroups; i++)
            if (kFull || (int)threadIdx.x + i * kSmoothThreads < h4) xr[i] = xrow[i * kSmoothThreads];
    };
    // phase 1 body: slot j's maximum of |fl(x * smooth[e])|, per warp
    auto amax_slot = [&](int j, const uint2 (&xr)[kGroups]) {
        const int32_t e = s_e[j];
        float amax = 0.0f;
        if (e >= 0) {
            if (e != cur_e) load_smooth(e);
#pragma unroll
            for (int i = 0; i < kGroups; i++) {
                if (kFull || (int)threadIdx.x + i * kSmoothThreads < h4) {
                    const uint2 v = xr[i];
                    const float2 v0 = mul2_rn(make_float2(bf16lo(v.x), bf16hi(v.x)), make_float2(sv[i].x, sv[i].y));
                    const float2 v1 = mul2_rn(make_float2(bf16lo(v.y), bf16hi(v.y)), make_float2(sv[i].z, sv[i].w));
                    amax = fmax3(fmax3(amax, fabsf(v0.x), fabsf(v0.y)), fabsf(v1.x), fabsf(v1.y));
                }
            }
        }
        // warp maximum of non-negative floats (products of finite inputs): their bits order
        // like their values, so one integer reduction gives it
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        if (lane == 0) red[j][warp] = amax;
    };
    // phase 2 body: slot j's codes, each product formed again
    auto codes_slot = [&](int j, const uint2 (&xr)[kGroups]) {
        const int32_t e = s_e[j];
        if (e < 0) return;
        if (e != cur_e) load_smooth(e);
        const float scale = s_scale[j], inv = s_inv[j];
        uint32_t *dst = recv + (int64_t)s_p[j] * H4 + threadIdx.x;
#pragma unroll
        for (int i = 0; i < kGroups; i++) {
            if (kFull || (int)threadIdx.x + i * kSmoothThreads < h4) {
                const uint2 v = xr[i];
                const float xf[4] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y)};
                dst[i * kSmoothThreads] = q8x4_packed(xf, sv[i], scale, inv);
            }
        }
    };
    uint2 xr[kGroups];
#pragma unroll 1
    for (int j = 0; j < n_here; j++) {
        load_x(j, xr);
        amax_slot(j, xr);
    }
    __syncthreads();
    if ((int)threadIdx.x < n_here) {                   // warp 0: one slot per lane
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; w++) m = fmaxf(m, red[threadIdx.x][w]);
        const float scale = __fdiv_rn(m, 127.0f);
        s_scale[threadIdx.x] = scale;
        s_inv[threadIdx.x] = quant_inv(scale);
        if (s_e[threadIdx.x] >= 0) recv_scale[s_p[threadIdx.x]] = scale;
    }
    __syncthreads();
#pragma unroll 1
    for (int j = 0; j < n_here; j++) {
        load_x(j, xr);
        codes_slot(j, xr);
    }
}

}  // namespace mep
