// Histogram and placement-plan kernels (sm_100a).
//
// The balanced plan of MoonEP (every rank receives exactly S*K token-slots, hot experts
// spill onto temporary redundant replicas on the next ranks; twodots.gr article on
// MoonEP) orders slots by (home(e), e, src, t, k). home(e) is monotone in e and the
// flat slot index orders (src, t, k), so the order is a stable counting sort by key:
//   row(n) = off[key] + #{m < n : key(m) == key(n)}.
// The grouped plan over physical instance ids is the same sort with dropped slots
// removed. Both are done in three passes over the ids (4 bytes per slot each):
//   k_tile_count      per-tile key counts              (warp-aggregated with match.any)
//   k_scan_cols_meta  per-key prefix over tiles and hist, one CTA per 32 keys; the CTA
//                     that finishes last then writes the per-rank replica tables
//                     (cu_seqlens) and the summary counts (plan_meta)
//   k_rank            per-slot stable rank inside its tile, written as the final row
// Small plans run as one launch (k_plan_cluster, k_plan_small). The exclusive prefix of
// hist over keys (off) is small (at most 4096 keys) and is recomputed in shared memory
// by each CTA that needs it.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace mep {

constexpr int kPlanWarps = 8;                    // warps per tile CTA
constexpr int kPlanTile = kPlanWarps * 32 * 8;   // the histogram's tile: 2048 slots
// The counting sort's tile: kRounds 32-slot rounds per warp, 256 * kRounds slots.
template <int kRounds>
constexpr int sort_tile() { return kPlanWarps * 32 * kRounds; }

// Key of slot n: the id, or -1 when the slot is dropped or its id is out of range.
__device__ __forceinline__ int32_t slot_key(const int32_t *ids, const uint8_t *keep, int64_t n,
                                            int64_t N, int32_t n_keys)
{
    if (n >= N) return -1;
    if (keep && !keep[n]) return -1;
    int32_t e = ids[n];
    if (e < 0 || e >= n_keys) {
        flag_error(MEP_DERR_KEY_RANGE);
        return -1;
    }
    return e;
}

// hist[key] += count of key in this CTA's tile (global atomics, one per distinct key
// per CTA). Used by mep_histogram.
__global__ void __launch_bounds__(kPlanWarps * 32)
k_histogram(const int32_t *__restrict__ ids, int64_t N, int32_t n_keys, int32_t *__restrict__ hist)
{
    extern __shared__ int32_t sh[];
    for (int i = threadIdx.x; i < n_keys; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    for (int64_t n0 = (int64_t)blockIdx.x * kPlanTile; n0 < N; n0 += (int64_t)gridDim.x * kPlanTile) {
        for (int64_t n = n0 + threadIdx.x - lane; n < n0 + kPlanTile; n += blockDim.x) {
            int32_t key = slot_key(ids, nullptr, n + lane, N, n_keys);
            uint32_t peers = __match_any_sync(0xffffffffu, key);
            if (key >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh[key], __popc(peers));
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n_keys; i += blockDim.x)
        if (sh[i]) atomicAdd(&hist[i], sh[i]);
}

// tile_cnt[tile, key] = slots of `key` in tile `blockIdx.x` (tiles of sort_tile<kRounds>).
// zero_word, when given, is set to 0 by CTA 0 (the arrival counter of k_scan_cols_meta).
template <int kRounds>
__global__ void __launch_bounds__(kPlanWarps * 32)
k_tile_count(const int32_t *__restrict__ ids, const uint8_t *__restrict__ keep, int64_t N,
             int32_t n_keys, int32_t *__restrict__ tile_cnt, int32_t *__restrict__ zero_word)
{
    constexpr int kTile = sort_tile<kRounds>();
    extern __shared__ int32_t sh[];
    pdl_wait();
    pdl_launch_dependents();
    if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0;
    for (int i = threadIdx.x; i < n_keys; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t base = (int64_t)blockIdx.x * kTile;
    for (int64_t n = base + threadIdx.x - lane; n < base + kTile; n += blockDim.x) {
        int32_t key = slot_key(ids, keep, n + lane, N, n_keys);
        uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh[key], __popc(peers));
    }
    __syncthreads();
    int32_t *out = tile_cnt + (int64_t)blockIdx.x * n_keys;
    for (int i = threadIdx.x; i < n_keys; i += blockDim.x) out[i] = sh[i];
}

// Exclusive prefix sum of in[0..n) into out[0..n], with out[n] = the total. Called by
// every thread of the block; `scratch` holds 33 ints of shared memory. Ends with a
// block barrier.
__device__ __forceinline__ void block_exclusive_scan(const int32_t *__restrict__ in, int n, int32_t *out,
                                                     int32_t *scratch)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int32_t sum = 0;
    for (int i = lo; i < hi; i++) sum += in[i];
    int32_t inc = sum;
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += u;
    }
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int32_t w = lane < nw ? scratch[lane] : 0;
        int32_t wi = w;
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, wi, d);
            if (lane >= d) wi += u;
        }
        scratch[lane] = wi - w;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    int32_t run = scratch[warp] + inc - sum;
    for (int i = lo; i < hi; i++) {
        out[i] = run;
        run += in[i];
    }
    if (tid == 0) out[n] = scratch[32];
    __syncthreads();
}

// block_exclusive_scan of in[0..n) into out[0..n] and, in the same pass, of the flags
// in[i] > 0 into nz[0..n] (nz[i] = how many of in[0..i) are positive). scratch holds 66
// ints of shared memory. Ends with a block barrier.
__device__ __forceinline__ void block_exclusive_scan2(const int32_t *__restrict__ in, int n, int32_t *out,
                                                      int32_t *nz, int32_t *scratch)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int32_t sum = 0, cnt = 0;
    for (int i = lo; i < hi; i++) {
        const int32_t v = in[i];
        sum += v;
        cnt += v > 0 ? 1 : 0;
    }
    int32_t inc = sum, incc = cnt;
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, inc, d);
        const int32_t uc = __shfl_up_sync(0xffffffffu, incc, d);
        if (lane >= d) {
            inc += u;
            incc += uc;
        }
    }
    if (lane == 31) {
        scratch[warp] = inc;
        scratch[33 + warp] = incc;
    }
    __syncthreads();
    if (warp == 0) {
        const int32_t w = lane < nw ? scratch[lane] : 0, wc = lane < nw ? scratch[33 + lane] : 0;
        int32_t wi = w, wci = wc;
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, wi, d);
            const int32_t uc = __shfl_up_sync(0xffffffffu, wci, d);
            if (lane >= d) {
                wi += u;
                wci += uc;
            }
        }
        scratch[lane] = wi - w;
        scratch[33 + lane] = wci - wc;
        if (lane == 31) {
            scratch[32] = wi;
            scratch[65] = wci;
        }
    }
    __syncthreads();
    int32_t run = scratch[warp] + inc - sum, runc = scratch[33 + warp] + incc - cnt;
    for (int i = lo; i < hi; i++) {
        out[i] = run;
        nz[i] = runc;
        run += in[i];
        runc += in[i] > 0 ? 1 : 0;
    }
    if (tid == 0) {
        out[n] = scratch[32];
        nz[n] = scratch[65];
    }
    __syncthreads();
}

// CTA c owns keys [32c, 32c + 32), one per lane; its 32 warps split the tiles. In place:
// tile_cnt[t, key] <- sum_{t' < t} tile_cnt[t', key], and hist[key] = sum over tiles.
__device__ __forceinline__ void scan_cols(int32_t *__restrict__ tile_cnt, int32_t n_tiles, int32_t n_keys,
                                          int32_t *__restrict__ hist)
{
    __shared__ int32_t part[32][33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int seg = (n_tiles + 31) / 32;
    const int t0 = min(n_tiles, warp * seg), t1 = min(n_tiles, t0 + seg);
    const int e = blockIdx.x * 32 + lane;
    const bool ok = e < n_keys;
    int32_t s = 0;
    if (ok) {
#pragma unroll 4
        for (int t = t0; t < t1; t++) s += tile_cnt[(int64_t)t * n_keys + e];
    }
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int w = 0; w < 32; w++) {
            const int32_t v = part[w][lane];
            part[w][lane] = run;
            run += v;
        }
        if (ok) hist[e] = run;
    }
    __syncthreads();
    if (ok) {
        int32_t run = part[warp][lane];
        for (int t = t0; t < t1; t++) {
            const int64_t i = (int64_t)t * n_keys + e;
            const int32_t v = tile_cnt[i];
            tile_cnt[i] = run;
            run += v;
        }
    }
}

__global__ void __launch_bounds__(1024)
k_scan_cols(int32_t *__restrict__ tile_cnt, int32_t n_tiles, int32_t n_keys, int32_t *__restrict__ hist)
{
    pdl_wait();
    pdl_launch_dependents();
    scan_cols(tile_cnt, n_tiles, n_keys, hist);
}


// pos[n] = off[key] + (slots of key in earlier tiles) + (earlier slots of key in this
// tile), off = exclusive prefix of hist over keys, or key_base[key] when key_base is
// given (the first row of this caller's slots of each key). Each warp owns an eighth of
// the tile: it counts its sub-range per key, the CTA turns those counts into per-warp
// bases, then each warp walks its sub-range again in order, ranking equal keys with
// match.any.
// Dynamic shared memory: cnt [kPlanWarps][n_keys], off [n_keys + 1], scratch [33].
template <int kRounds>
__global__ void __launch_bounds__(kPlanWarps * 32)
k_rank(const int32_t *__restrict__ ids, const uint8_t *__restrict__ keep, int64_t N, int32_t n_keys,
       const int32_t *__restrict__ tile_base, const int32_t *__restrict__ hist,
       const int32_t *__restrict__ key_base, int32_t *__restrict__ pos)
{
    extern __shared__ int32_t cnt[];
    int32_t *key_off = cnt + kPlanWarps * n_keys;
    int32_t *scan_scratch = key_off + n_keys + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_launch_dependents();
    for (int i = threadIdx.x; i < kPlanWarps * n_keys; i += blockDim.x) cnt[i] = 0;
    if (key_base) {
        for (int i = threadIdx.x; i < n_keys; i += blockDim.x) key_off[i] = key_base[i];
        __syncthreads();
    } else {
        block_exclusive_scan(hist, n_keys, key_off, scan_scratch);
    }
    constexpr int kSub = sort_tile<kRounds>() / kPlanWarps;
    const int64_t lo = (int64_t)blockIdx.x * sort_tile<kRounds>() + warp * kSub;
    int32_t *mine = cnt + warp * n_keys;
    for (int64_t n0 = lo; n0 < lo + kSub; n0 += 32) {
        int32_t key = slot_key(ids, keep, n0 + lane, N, n_keys);
        uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) mine[key] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    const int32_t *tb = tile_base + (int64_t)blockIdx.x * n_keys;
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        int32_t run = key_off[e] + tb[e];
        for (int w = 0; w < kPlanWarps; w++) {
            int32_t v = cnt[w * n_keys + e];
            cnt[w * n_keys + e] = run;
            run += v;
        }
    }
    __syncthreads();
    const uint32_t lt = lanemask_lt();
    for (int64_t n0 = lo; n0 < lo + kSub; n0 += 32) {
        const int64_t n = n0 + lane;
        // slot_key flags out-of-range ids once more here; the bit is idempotent
        int32_t key = slot_key(ids, keep, n, N, n_keys);
        uint32_t peers = __match_any_sync(0xffffffffu, key);
        int32_t p = -1;
        if (key >= 0) p = mine[key] + __popc(peers & lt);
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) mine[key] += __popc(peers);
        __syncwarp();
        if (n < N) pos[n] = p;
    }
}

// Rank that receives row `row` (row < total rows).
__device__ __forceinline__ int32_t row_rank_balanced(int64_t row, int64_t SK) { return (int32_t)(row / SK); }

// Smallest index i in [0, n] with a[i] > x (a ascending), for a in shared memory.
__device__ __forceinline__ int32_t upper_bound_sh(const int32_t *a, int32_t n, int64_t x)
{
    int32_t lo = 0, hi = n + 1;
    while (lo < hi) {
        int32_t mid = (lo + hi) >> 1;
        if (a[mid] > x) hi = mid;
        else lo = mid + 1;
    }
    return lo;
}

// Per-rank replica tables and the summary counts, by one CTA (any multiple of 32 threads).
// smem: key_off (n_keys+1) + nz (n_keys+1) + rank_off (R+1) + e_lo (R) + count (R) ints.
__device__ __forceinline__ void plan_meta(const int32_t *__restrict__ hist, int32_t R,
                                          int32_t n_keys, int64_t SK, int32_t mode, int32_t keys_per_rank,
                                          int32_t *__restrict__ rank_off_out, int32_t *__restrict__ load_out,
                                          int32_t *__restrict__ rep_count, int32_t *__restrict__ rep_key,
                                          int32_t *__restrict__ rep_cu, int32_t *__restrict__ stats,
                                          int32_t *smem)
{
    int32_t *koff = smem;                    // n_keys + 1
    int32_t *nz = koff + (n_keys + 1);       // n_keys + 1: exclusive count of non-empty keys
    int32_t *roff = nz + (n_keys + 1);       // R + 1
    int32_t *elo = roff + (R + 1);           // R: first key on each rank
    int32_t *rcnt = elo + R;                 // R: replicas on each rank
    __shared__ int32_t s_red[8];
    __shared__ int32_t scan_scratch[66];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int32_t cap = n_keys;
    const int32_t per_rank = (mode == 0) ? n_keys / R : keys_per_rank;

    block_exclusive_scan2(hist, n_keys, koff, nz, scan_scratch);
    if (threadIdx.x < 8) s_red[threadIdx.x] = 0;
    // rank offsets
    for (int r = threadIdx.x; r <= R; r += blockDim.x) {
        int64_t ro = (mode == 0) ? (int64_t)r * SK : (int64_t)koff[min(n_keys, r * keys_per_rank)];
        roff[r] = (int32_t)ro;
        rank_off_out[r] = (int32_t)ro;
    }
    __syncthreads();
    // first key of each non-empty rank; replica counts
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        int32_t cnt = 0, first = 0;
        if (roff[r + 1] > roff[r]) {
            first = upper_bound_sh(koff, n_keys, roff[r]) - 1;
            int32_t last = upper_bound_sh(koff, n_keys, (int64_t)roff[r + 1] - 1) - 1;
            cnt = nz[last + 1] - nz[first];
            atomicAdd(&s_red[6], 1);
        }
        elo[r] = first;
        rcnt[r] = cnt;
        rep_count[r] = cnt;
        atomicMax(&s_red[1], roff[r + 1] - roff[r]);
        if (load_out) {
            int32_t l;
            if (mode == 0) l = koff[min(n_keys, (r + 1) * per_rank)] - koff[r * per_rank];
            else l = roff[r + 1] - roff[r];
            load_out[r] = l;
        }
    }
    __syncthreads();
    // one thread per key: write its replica entries on every rank it spans
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        const int32_t b = koff[e], en = koff[e + 1];
        atomicMax(&s_red[5], en - b);
        if (mode == 0 && e % per_rank == 0) {
            int32_t l = koff[min(n_keys, e + per_rank)] - b;   // home load of rank e/per_rank
            atomicMax(&s_red[0], l);
        }
        if (en <= b) continue;
        int32_t r0, r1;
        if (mode == 0) {
            r0 = row_rank_balanced(b, SK);
            r1 = row_rank_balanced((int64_t)en - 1, SK);
        } else {
            r0 = r1 = e / keys_per_rank;
        }
        const int32_t home = e / per_rank;
        int32_t pf = 0;
        for (int32_t r = r0; r <= r1; r++) {
            const int32_t j = nz[e] - nz[elo[r]];
            rep_key[(int64_t)r * cap + j] = e;
            rep_cu[(int64_t)r * (cap + 1) + j] = max(b, roff[r]) - roff[r];
            if (mode == 0 && r != home) pf++;
        }
        if (r1 > r0) atomicAdd(&s_red[2], r1 - r0);
        if (pf) atomicAdd(&s_red[3], pf);
    }
    // the rest of every rank's rows (disjoint from the entries above): no key past its
    // count, and the running row count ends at the rank's rows
    for (int r = warp; r < R; r += nwarps) {
        const int32_t c = rcnt[r];
        for (int j = c + lane; j <= cap; j += 32) {
            if (j < cap) rep_key[(int64_t)r * cap + j] = -1;
            rep_cu[(int64_t)r * (cap + 1) + j] = j == c ? roff[r + 1] - roff[r] : 0;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        stats[0] = (mode == 0) ? s_red[0] : s_red[1];
        stats[1] = s_red[1];
        stats[2] = s_red[2];
        stats[3] = s_red[3];
        stats[4] = koff[n_keys];
        stats[5] = s_red[5];
        stats[6] = s_red[6];
        stats[7] = 0;
    }
}

// k_scan_cols, then the replica tables in the CTA that finishes last: each CTA writes
// its keys' hist entries, fences them and arrives once on *arrived; the CTA whose
// arrival is the last copies hist into shared memory (through L2) and runs plan_meta.
// One launch fewer than a separate replica-table kernel; nothing waits. *arrived must be 0
// at launch (k_tile_count zeroes it).
// Dynamic shared memory: plan_meta's (2 (n_keys + 1) + (R + 1) + 2 R ints), then n_keys ints.
__global__ void __launch_bounds__(1024)
k_scan_cols_meta(int32_t *__restrict__ tile_cnt, int32_t n_tiles, int32_t n_keys, int32_t *__restrict__ hist,
                 int32_t *__restrict__ arrived, int32_t R, int64_t SK, int32_t mode, int32_t keys_per_rank,
                 int32_t *__restrict__ rank_off_out, int32_t *__restrict__ load_out,
                 int32_t *__restrict__ rep_count, int32_t *__restrict__ rep_key, int32_t *__restrict__ rep_cu,
                 int32_t *__restrict__ stats)
{
    extern __shared__ int32_t smem[];
    __shared__ int32_t s_last;
    pdl_wait();
    pdl_launch_dependents();
    scan_cols(tile_cnt, n_tiles, n_keys, hist);
    __threadfence();                                  // this CTA's hist entries before its arrival
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(arrived, 1) == (int32_t)gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    int32_t *h = smem + 2 * (n_keys + 1) + (R + 1) + 2 * R;
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) h[e] = __ldcg(hist + e);
    __syncthreads();
    plan_meta(h, R, n_keys, SK, mode, keys_per_rank, rank_off_out, load_out, rep_count, rep_key, rep_cu, stats,
              smem);
}

// The whole plan in one CTA of 1024 threads, for small problems (up to 16384 slots,
// where the four-kernel plan is bound by launch latency): the same stable counting
// sort with a single tile. Each of the 32 warps owns a contiguous sub-range of the
// slots, whose keys its lanes load at once into registers (up to kSmallPlanPerLane each,
// every load in flight together); it counts its keys, the CTA turns the counts into
// per-warp bases (after hist and its prefix over keys), each warp ranks its sub-range in
// order, then plan_meta writes the replica tables.
// Dynamic shared memory: 33 * n_keys + n_keys + 1 + 33 ints (plan_meta reuses the start,
// which n_keys >= R keeps inside the per-warp counts).
constexpr int kSmallPlanThreads = 1024;
constexpr int kSmallPlanPerLane = 16;
constexpr int64_t kSmallPlanMaxSlots = (int64_t)kSmallPlanThreads * kSmallPlanPerLane;

__global__ void __launch_bounds__(kSmallPlanThreads)
k_plan_small(const int32_t *__restrict__ ids, const uint8_t *__restrict__ keep, int64_t N, int32_t n_keys,
             int32_t R, int64_t SK, int32_t mode, int32_t keys_per_rank, int32_t *__restrict__ pos,
             int32_t *__restrict__ hist, int32_t *__restrict__ rank_off_out, int32_t *__restrict__ load_out,
             int32_t *__restrict__ rep_count, int32_t *__restrict__ rep_key, int32_t *__restrict__ rep_cu,
             int32_t *__restrict__ stats)
{
    extern __shared__ int32_t smem[];
    constexpr int kWarps = kSmallPlanThreads / 32;
    int32_t *cnt = smem;                              // [kWarps][n_keys]
    int32_t *key_off = cnt + kWarps * n_keys;         // n_keys + 1
    int32_t *scan_scratch = key_off + n_keys + 1;     // 33
    int32_t *tot = scan_scratch + 33;                 // n_keys: hist, kept for plan_meta
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_launch_dependents();
    for (int i = threadIdx.x; i < kWarps * n_keys; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    const int64_t sub = ((N + kWarps - 1) / kWarps + 31) / 32 * 32;   // <= 32 * kSmallPlanPerLane
    const int64_t lo = (int64_t)warp * sub, hi = min(N, lo + sub);
    int32_t *mine = cnt + warp * n_keys;
    // Every load first (ids and keep flags, all in flight together), then the checks:
    // key + 1 (0 for a dropped slot; keys < 4096) in 16-bit halves, two per register.
    uint32_t kp[kSmallPlanPerLane / 2];
    {
        int32_t raw[kSmallPlanPerLane];
        uint32_t kept = ~0u;                          // bit j: slot j is not dropped by keep
#pragma unroll
        for (int j = 0; j < kSmallPlanPerLane; j++) {
            const int64_t n = lo + 32 * j + lane;
            raw[j] = n < hi ? ids[n] : -1;
            if (keep && n < hi && !keep[n]) kept &= ~(1u << j);
        }
#pragma unroll
        for (int j = 0; j < kSmallPlanPerLane; j += 2) {
            int32_t k2[2];
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int64_t n = lo + 32 * (j + h) + lane;
                int32_t e = raw[j + h];
                if (n >= hi || !((kept >> (j + h)) & 1u)) {
                    e = -1;
                } else if (e < 0 || e >= n_keys) {
                    flag_error(MEP_DERR_KEY_RANGE);
                    e = -1;
                }
                k2[h] = e;
            }
            kp[j / 2] = (uint32_t)(k2[0] + 1) | ((uint32_t)(k2[1] + 1) << 16);
        }
    }
    auto key_at = [&](int j) -> int32_t { return (int32_t)((kp[j / 2] >> (16 * (j & 1))) & 0xffffu) - 1; };
#pragma unroll
    for (int j = 0; j < kSmallPlanPerLane; j++) {
        if (lo + 32 * j >= hi) break;                 // uniform over the warp
        const int32_t key = key_at(j);
        uint32_t peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) mine[key] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per key: exclusive prefix over warps (in place) and the total
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        int32_t run = 0;
        for (int w = 0; w < kWarps; w++) {
            const int32_t v = cnt[w * n_keys + e];
            cnt[w * n_keys + e] = run;
            run += v;
        }
        hist[e] = run;
        tot[e] = run;
    }
    __syncthreads();
    block_exclusive_scan(tot, n_keys, key_off, scan_scratch);
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        const int32_t b = key_off[e];
        for (int w = 0; w < kWarps; w++) cnt[w * n_keys + e] += b;
    }
    __syncthreads();
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int j = 0; j < kSmallPlanPerLane; j++) {
        if (lo + 32 * j >= hi) break;
        const int64_t n = lo + 32 * j + lane;
        const int32_t key = key_at(j);
        uint32_t peers = __match_any_sync(0xffffffffu, key);
        int32_t p = -1;
        if (key >= 0) p = mine[key] + __popc(peers & lt);
        __syncwarp();
        if (key >= 0 && lane == __ffs(peers) - 1) mine[key] += __popc(peers);
        __syncwarp();
        if (n < hi) pos[n] = p;
    }
    __syncthreads();
    plan_meta(tot, R, n_keys, SK, mode, keys_per_rank, rank_off_out, load_out, rep_count, rep_key, rep_cu, stats,
              smem);
}

// The whole plan in one cluster of kPlanClusterCTAs CTAs of 1024 threads, for small
// problems: k_plan_small's steps with the slots split over the cluster's CTAs (CTA c
// takes the c-th eighth of the slots, in order), so each warp walks at most
// kClusterPlanPerLane rounds instead of kSmallPlanPerLane. Each CTA counts its slots per
// warp and key; after a cluster barrier every CTA reads the others' per-key totals
// through distributed shared memory, forms hist and the totals of the CTAs before it,
// and ranks its slots from there. CTA 0 then writes the replica tables (plan_meta).
// Dynamic shared memory: cnt [32][n_keys], key_off [n_keys + 1], scratch [33], and
// three [n_keys] arrays: this CTA's totals, hist, the earlier CTAs' totals.
constexpr int kPlanClusterCTAs = 8;
constexpr int kClusterPlanPerLane = 2;
constexpr int64_t kClusterPlanMaxSlots = (int64_t)kPlanClusterCTAs * kSmallPlanThreads * kClusterPlanPerLane;

__global__ void __cluster_dims__(kPlanClusterCTAs, 1, 1) __launch_bounds__(kSmallPlanThreads)
k_plan_cluster(const int32_t *__restrict__ ids, const uint8_t *__restrict__ keep, int64_t N, int32_t n_keys,
               int32_t R, int64_t SK, int32_t mode, int32_t keys_per_rank, int32_t *__restrict__ pos,
               int32_t *__restrict__ hist, int32_t *__restrict__ rank_off_out, int32_t *__restrict__ load_out,
               int32_t *__restrict__ rep_count, int32_t *__restrict__ rep_key, int32_t *__restrict__ rep_cu,
               int32_t *__restrict__ stats)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t smem[];
    constexpr int kWarps = kSmallPlanThreads / 32;
    int32_t *cnt = smem;                              // [kWarps][n_keys]
    int32_t *key_off = cnt + kWarps * n_keys;         // n_keys + 1
    int32_t *scan_scratch = key_off + n_keys + 1;     // 33
    int32_t *ctot = scan_scratch + 33;                // n_keys: this CTA's slots per key
    int32_t *all = ctot + n_keys;                     // n_keys: hist (every CTA's slots)
    int32_t *pre = all + n_keys;                      // n_keys: the slots of the CTAs before this one
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kWarps * n_keys; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    const int64_t per_cta = ((N + kPlanClusterCTAs - 1) / kPlanClusterCTAs + 31) / 32 * 32;
    const int64_t c_lo = min(N, (int64_t)crank * per_cta), c_hi = min(N, c_lo + per_cta);
    const int64_t sub = ((per_cta + kWarps - 1) / kWarps + 31) / 32 * 32;   // <= 32 * kClusterPlanPerLane
    const int64_t lo = min(c_hi, c_lo + (int64_t)warp * sub), hi = min(c_hi, lo + sub);
    int32_t *mine = cnt + warp * n_keys;
    int32_t key[kClusterPlanPerLane];
#pragma unroll
    for (int j = 0; j < kClusterPlanPerLane; j++) {
        const int64_t n = lo + 32 * j + lane;
        int32_t e = n < hi ? ids[n] : -1;
        if (n < hi && keep && !keep[n]) e = -1;
        else if (n < hi && (e < 0 || e >= n_keys)) {
            flag_error(MEP_DERR_KEY_RANGE);
            e = -1;
        }
        key[j] = e;
    }
#pragma unroll
    for (int j = 0; j < kClusterPlanPerLane; j++) {
        if (lo + 32 * j >= hi) break;                 // uniform over the warp
        const uint32_t peers = __match_any_sync(0xffffffffu, key[j]);
        if (key[j] >= 0 && lane == __ffs(peers) - 1) mine[key[j]] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // per key: exclusive prefix over warps (in place) and this CTA's total
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        int32_t run = 0;
        for (int w = 0; w < kWarps; w++) {
            const int32_t v = cnt[w * n_keys + e];
            cnt[w * n_keys + e] = run;
            run += v;
        }
        ctot[e] = run;
    }
    cluster.sync();                                   // every CTA's totals are complete
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        int32_t a = 0, b = 0;
        for (int c = 0; c < kPlanClusterCTAs; c++) {
            const int32_t v = cluster.map_shared_rank(ctot, c)[e];
            a += v;
            if (c < crank) b += v;
        }
        all[e] = a;
        pre[e] = b;
        if (crank == 0) hist[e] = a;
    }
    __syncthreads();
    block_exclusive_scan(all, n_keys, key_off, scan_scratch);
    for (int e = threadIdx.x; e < n_keys; e += blockDim.x) {
        const int32_t b = key_off[e] + pre[e];
        for (int w = 0; w < kWarps; w++) cnt[w * n_keys + e] += b;
    }
    __syncthreads();
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int j = 0; j < kClusterPlanPerLane; j++) {
        if (lo + 32 * j >= hi) break;
        const int64_t n = lo + 32 * j + lane;
        const uint32_t peers = __match_any_sync(0xffffffffu, key[j]);
        int32_t p = -1;
        if (key[j] >= 0) p = mine[key[j]] + __popc(peers & lt);
        __syncwarp();
        if (key[j] >= 0 && lane == __ffs(peers) - 1) mine[key[j]] += __popc(peers);
        __syncwarp();
        if (n < hi) pos[n] = p;
    }
    cluster.sync();                                   // no CTA reads another's totals past here
    if (crank != 0) return;
    plan_meta(all, R, n_keys, SK, mode, keys_per_rank, rank_off_out, load_out, rep_count, rep_key, rep_cu, stats,
              smem);
}

// ------------------------------------------------ one rank's share of the plan (e)
//
// Each real GPU is one EP rank holding its own S tokens. With the per-rank histograms
// of all R ranks gathered (hist_all [R, E], row r = rank r's slots per expert) every
// rank knows where its slots go in the global balanced plan without seeing the others'
// ids: the plan orders slots by (e, src, t, k), so the rows of rank `rank`'s slots of
// expert e start at
//   key_base[e] = off[e] + sum_{r < rank} hist_all[r, e],   off = exclusive scan over e
//                                                             of sum_r hist_all[r, e],
// and within them follow its own slot order (k_rank with key_base). Row p lands on
// destination rank p / SK. One CTA also writes the exchange counts:
//   send_count[d] = rows this rank writes into rank d's partition,
//   recv_count[s] = rows rank s writes into this rank's partition,
// with their exclusive prefixes (R + 1 entries each), and checks that row `rank` of
// hist_all equals the histogram of this rank's ids (hist_local).
// Dynamic shared memory: off [E + 1], send [R], recv [R].
__global__ void __launch_bounds__(1024)
k_source_meta(const int32_t *__restrict__ hist_all, const int32_t *__restrict__ hist_local, int32_t R,
              int32_t E, int64_t SK, int32_t rank, int32_t *__restrict__ key_base,
              int32_t *__restrict__ send_count, int32_t *__restrict__ send_off,
              int32_t *__restrict__ recv_count, int32_t *__restrict__ recv_off)
{
    extern __shared__ int32_t smem[];
    int32_t *off = smem;                 // E + 1
    int32_t *tot = off + (E + 1);        // E (column totals, then reused)
    int32_t *snd = tot + E;              // R
    int32_t *rcv = snd + R;              // R
    __shared__ int32_t scan_scratch[33];
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        snd[r] = 0;
        rcv[r] = 0;
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t t = 0, pre = 0;
        for (int r = 0; r < R; r++) {
            const int32_t h = hist_all[(int64_t)r * E + e];
            if (r == rank) pre = t;
            t += h;
        }
        tot[e] = t;
        key_base[e] = pre;   // completed below
        if (hist_all[(int64_t)rank * E + e] != hist_local[e]) flag_error(MEP_DERR_HIST);
    }
    __syncthreads();
    block_exclusive_scan(tot, E, off, scan_scratch);
    const int64_t lo = (int64_t)rank * SK, hi = lo + SK;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int64_t b = (int64_t)off[e] + key_base[e];
        key_base[e] = (int32_t)b;
        // this rank's rows of e, split over the destination partitions they cross
        const int32_t h = hist_all[(int64_t)rank * E + e];
        for (int64_t p = b; p < b + h;) {
            const int64_t d = p / SK;
            const int64_t end = min(b + h, (d + 1) * SK);
            atomicAdd(&snd[d], (int32_t)(end - p));
            p = end;
        }
        // every source's rows of e that land in this rank's partition
        if (off[e + 1] > lo && off[e] < hi) {
            int64_t p = off[e];
            for (int r = 0; r < R; r++) {
                const int32_t hr = hist_all[(int64_t)r * E + e];
                const int64_t a = max(p, lo), z = min(p + hr, hi);
                if (z > a) atomicAdd(&rcv[r], (int32_t)(z - a));
                p += hr;
            }
        }
    }
    __syncthreads();
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        send_count[r] = snd[r];
        recv_count[r] = rcv[r];
    }
    block_exclusive_scan(snd, R, send_off, scan_scratch);
    block_exclusive_scan(rcv, R, recv_off, scan_scratch);
}

}  // namespace mep
