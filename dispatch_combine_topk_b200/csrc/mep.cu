// libmep — C ABI of MoE expert-parallel token routing on one B200 (sm_100a).
// Entry points, argument checks and launch configuration. The declarations, with the
// meaning, layout, ownership and error behaviour of every argument, are in mep.h.
//
// One translation unit on purpose: the device error word lives here and every kernel
// reaches it without relocatable device code.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <mutex>
#include <thread>

#include "mep.h"
#include "common.cuh"
#include "plan_kernels.cuh"
#include "route_kernels.cuh"
#include "dedup_kernels.cuh"
#include "rank_kernels.cuh"
#include "smooth_kernels.cuh"

namespace {

thread_local int32_t t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
// Shared memory the staged int8 dispatch may use per CTA.
constexpr int kBulkSmemMax = 200 * 1024;
// Plans of at most mep::kSmallPlanMaxSlots slots (and few enough keys for the shared
// memory below) run as one CTA: there the four-kernel plan is bound by launch latency.
constexpr int kSmallPlanSmemMax = 200 * 1024;

// ---------------------------------------------------------------- per-context state
//
// Kernel attributes (the dynamic shared-memory limits) and the device address of the
// static plan scratch belong to a CUDA context, not to a device ordinal: after
// cudaDeviceReset, or for a caller that makes its own driver context current, they
// must be set up again. The current context is identified by its driver-assigned id
// (cuCtxGetId, unique for the life of the process, also when a context is destroyed
// and another takes its handle). The two driver calls are reached through the
// runtime's entry-point query, so the library links only the CUDA runtime.

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
std::once_flag g_driver_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

void driver_entry_points()
{
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_current = (CtxGetCurrentFn)f;
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_ctx_get_id = (CtxGetIdFn)f;
    (void)cudaGetLastError();
}

// Id of the context current on this host thread; false when there is none (or the
// driver cannot say).
bool current_context_id(unsigned long long *id)
{
    std::call_once(g_driver_once, driver_entry_points);
    if (!g_ctx_get_current || !g_ctx_get_id) return false;
    CUcontext c = nullptr;
    if (g_ctx_get_current(&c) != CUDA_SUCCESS || !c) return false;
    return g_ctx_get_id(c, id) == CUDA_SUCCESS;
}

struct DeviceState {
    std::mutex m;
    std::atomic<bool> ready{false};
    std::atomic<unsigned long long> ctx_id{0};
    int sm_count = 148;
    bool cluster_plan = false;        // k_plan_cluster's cluster fits on the device
    void *plan_static_ws = nullptr;   // device address of g_plan_static_ws in ctx_id
};
DeviceState g_dev[kMaxDevices];

// Lookup of the static plan scratch's device address (defined with the array below).
cudaError_t plan_static_ws_lookup(void **addr);

// Set-up of the current device in the current context: its SM count, the kernels'
// shared-memory limits, the address of the static plan scratch. Runs again whenever
// the current context differs from the one it last ran in (several host threads may
// call at once). Without the driver's context id it runs once per device.
DeviceState &device_state(int dev)
{
    DeviceState &st = g_dev[dev];
    unsigned long long id = 0;
    const bool have = current_context_id(&id);
    if (st.ready.load(std::memory_order_acquire) && (!have || st.ctx_id.load(std::memory_order_relaxed) == id))
        return st;
    std::lock_guard<std::mutex> lock(st.m);
    if (st.ready.load(std::memory_order_relaxed) && (!have || st.ctx_id.load(std::memory_order_relaxed) == id))
        return st;
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    st.sm_count = n > 0 ? n : 148;
    const int big = 200 * 1024;
    cudaFuncSetAttribute(mep::k_rank<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_rank<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_rank<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_tile_count<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_tile_count<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_tile_count<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_histogram, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_scan_cols_meta, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_source_meta, cudaFuncAttributeMaxDynamicSharedMemorySize, big);
    cudaFuncSetAttribute(mep::k_plan_small, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallPlanSmemMax);
    cudaFuncSetAttribute(mep::k_plan_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallPlanSmemMax);
    {
        // a cluster of CTAs with the largest shared memory the plan asks for
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(mep::kPlanClusterCTAs);
        cfg.blockDim = dim3(mep::kSmallPlanThreads);
        cfg.dynamicSmemBytes = kSmallPlanSmemMax;
        cudaLaunchAttribute attr = {};
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = mep::kPlanClusterCTAs;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        st.cluster_plan = cudaOccupancyMaxActiveClusters(&clusters, mep::k_plan_cluster, &cfg) == cudaSuccess &&
                          clusters >= 1;
    }
    cudaFuncSetAttribute(mep::k_dispatch_int8_staged<4, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kBulkSmemMax);
    const int norm_smem = (int)(sizeof(float) * MEP_RMSNORM_MAX_H);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_v8<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_v8<6>, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_v8<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_v8<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_v8<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    cudaFuncSetAttribute(mep::k_combine_add_rmsnorm_scalar, cudaFuncAttributeMaxDynamicSharedMemorySize, norm_smem);
    void *ws = nullptr;
    if (plan_static_ws_lookup(&ws) != cudaSuccess) ws = nullptr;
    st.plan_static_ws = ws;
    (void)cudaGetLastError();
    // the calls above made the device's context current if none was
    unsigned long long id2 = 0;
    st.ctx_id.store(current_context_id(&id2) ? id2 : 0, std::memory_order_relaxed);
    st.ready.store(true, std::memory_order_release);
    return st;
}

// SM count of the current device (running its set-up when needed).
int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    return device_state(dev).sm_count;
}

// Whether the current device can run k_plan_cluster's cluster.
bool cluster_plan_ok()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    return device_state(dev).cluster_plan;
}

mep_status_t launched()
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        t_last_cuda_error = (int32_t)e;
        return MEP_ERR_CUDA;
    }
    return MEP_OK;
}

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Token-parallel grid: a multiple of the SM count, never more CTAs than tokens.
inline int token_grid(int64_t T, int per_sm)
{
    int64_t g = (int64_t)sm_count() * per_sm;
    if (T < g) g = T;
    return (int)(g > 0 ? g : 1);
}

// Grid of at most `want` CTAs, capped at the number the GPU holds resident at once (for
// grid-stride kernels whose CTAs should all start in the first wave).
template <typename Kernel>
int resident_grid(Kernel kernel, int threads, int64_t want)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    const int64_t g = want < cap ? want : cap;
    return (int)(g > 0 ? g : 1);
}

inline int elem_grid(int64_t total, int threads)
{
    int64_t g = (total + threads - 1) / threads;
    int64_t cap = (int64_t)sm_count() * 8;
    if (g > cap) g = cap;
    return (int)(g > 0 ? g : 1);
}

// Rounds per warp of the counting sort's tile (256 * rounds slots) for N slots: smaller
// tiles spread a small sort over all SMs, larger ones keep the per-tile scan and rank
// work low for a large one (plan times measured with CUDA events: 262,144 slots fastest
// with 512-slot tiles, 1,048,576 with 1024, 2,097,152 with 2048).
inline int sort_rounds(int64_t N) { return N <= ((int64_t)1 << 18) ? 2 : (N <= ((int64_t)1 << 20) ? 4 : 8); }
inline int64_t sort_tiles(int64_t N) { return mep::ceil_div(N, (int64_t)mep::kPlanWarps * 32 * sort_rounds(N)); }

// Launch of a kernel of the routing step with programmatic stream serialization: it may
// be scheduled before the previous kernel on the stream has finished and waits for it
// itself (pdl_wait at its start); every kernel launched this way does so.
template <typename... P, typename... A>
void launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, ((P)args)...);
}

// The plan's replica-table arguments, for a counting sort that also writes them
// (k_scan_cols_meta); arrived is one int of scratch.
struct PlanMeta {
    int32_t *arrived;
    int32_t R;
    int64_t SK;
    int32_t mode, keys_per_rank;
    int32_t *rank_off, *load, *rep_count, *rep_key, *rep_cu, *stats;
};


// Stable counting sort of N keys in [0, n_keys) (dropped: keep == 0 or out of range):
// pos[n] = base[key] + (earlier slots of key), base = the exclusive prefix of the
// histogram, or key_base when given. Writes the histogram to hist; tile_cnt holds
// sort_tiles(N) * n_keys ints of scratch.
template <int kRounds>
void counting_sort_r(const int32_t *keys, const uint8_t *keep, int64_t N, int32_t n_keys, int32_t *tile_cnt,
                     int32_t *hist, const int32_t *key_base, int32_t *pos, cudaStream_t s, const PlanMeta *meta)
{
    const int64_t tiles = mep::ceil_div(N, (int64_t)mep::sort_tile<kRounds>());
    const int threads = mep::kPlanWarps * 32;
    launch_pdl(mep::k_tile_count<kRounds>, dim3((unsigned)tiles), dim3(threads), sizeof(int32_t) * n_keys, s, keys, keep,
               N, n_keys, tile_cnt, meta ? meta->arrived : nullptr);
    if (meta) {
        const size_t meta_smem = sizeof(int32_t) * (size_t)(3 * n_keys + 2 + (meta->R + 1) + 2 * meta->R);
        launch_pdl(mep::k_scan_cols_meta, dim3((unsigned)mep::ceil_div(n_keys, 32)), dim3(1024), meta_smem, s, tile_cnt,
                   (int32_t)tiles, n_keys, hist, meta->arrived, meta->R, meta->SK, meta->mode, meta->keys_per_rank,
                   meta->rank_off, meta->load, meta->rep_count, meta->rep_key, meta->rep_cu, meta->stats);
    } else {
        launch_pdl(mep::k_scan_cols, dim3((unsigned)mep::ceil_div(n_keys, 32)), dim3(1024), 0, s, tile_cnt, (int32_t)tiles,
                   n_keys, hist);
    }
    const size_t rank_smem = sizeof(int32_t) * ((size_t)mep::kPlanWarps * n_keys + n_keys + 1 + 33);
    launch_pdl(mep::k_rank<kRounds>, dim3((unsigned)tiles), dim3(threads), rank_smem, s, keys, keep, N, n_keys,
               (const int32_t *)tile_cnt, (const int32_t *)hist, key_base, pos);
}

void counting_sort(const int32_t *keys, const uint8_t *keep, int64_t N, int32_t n_keys, int32_t *tile_cnt,
                   int32_t *hist, const int32_t *key_base, int32_t *pos, cudaStream_t s,
                   const PlanMeta *meta = nullptr)
{
    switch (sort_rounds(N)) {
    case 2: counting_sort_r<2>(keys, keep, N, n_keys, tile_cnt, hist, key_base, pos, s, meta); break;
    case 4: counting_sort_r<4>(keys, keep, N, n_keys, tile_cnt, hist, key_base, pos, s, meta); break;
    default: counting_sort_r<8>(keys, keep, N, n_keys, tile_cnt, hist, key_base, pos, s, meta); break;
    }
}

}  // namespace

extern "C" {

int32_t mep_version(void) { return (1 << 16) | 0; }

const char *mep_status_string(mep_status_t s)
{
    switch (s) {
    case MEP_OK: return "MEP_OK";
    case MEP_ERR_NULLPTR: return "MEP_ERR_NULLPTR: a required pointer is NULL";
    case MEP_ERR_DTYPE: return "MEP_ERR_DTYPE: unsupported element type or quantisation mode";
    case MEP_ERR_SHAPE: return "MEP_ERR_SHAPE: a size is outside the supported range";
    case MEP_ERR_VALUE: return "MEP_ERR_VALUE: an argument value is outside its range";
    case MEP_ERR_WORKSPACE: return "MEP_ERR_WORKSPACE: workspace NULL, too small or misaligned";
    case MEP_ERR_CUDA: return "MEP_ERR_CUDA: a CUDA call failed";
    case MEP_ERR_TIMEOUT: return "MEP_ERR_TIMEOUT: the stream's work did not finish in time";
    }
    return "unknown mep_status_t";
}

int32_t mep_last_cuda_error(void) { return t_last_cuda_error; }

mep_status_t mep_get_error(mep_stream_t stream, int32_t *code, int32_t clear)
{
    if (!code) return MEP_ERR_NULLPTR;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t word = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&word, mep::g_error_word, sizeof(int32_t), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && clear && word) {
        // clears only the bits read: a bit another stream sets meanwhile stays set
        mep::k_clear_error_bits<<<1, 1, 0, s>>>(word);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        t_last_cuda_error = (int32_t)e;
        return MEP_ERR_CUDA;
    }
    *code = word;
    return MEP_OK;
}

mep_status_t mep_histogram(const int32_t *ids, int64_t n, int32_t n_keys, int32_t *hist,
                           mep_stream_t stream)
{
    if ((!ids && n > 0) || !hist) return MEP_ERR_NULLPTR;
    if (n < 0 || n >= ((int64_t)1 << 31) || n_keys < 1 || n_keys > MEP_MAX_KEYS) return MEP_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    const int sms = sm_count();
    if (cudaMemsetAsync(hist, 0, sizeof(int32_t) * n_keys, s) != cudaSuccess) return launched();
    if (n == 0) return launched();
    int64_t tiles = mep::ceil_div(n, mep::kPlanTile);
    int grid = (int)(tiles < 2 * sms ? tiles : 2 * sms);
    mep::k_histogram<<<grid, mep::kPlanWarps * 32, sizeof(int32_t) * n_keys, s>>>(ids, n, n_keys, hist);
    return launched();
}

size_t mep_plan_workspace_size(int32_t R, int32_t n_keys, int32_t S, int32_t K)
{
    if (R < 1 || S < 1 || K < 1 || n_keys < 1) return 0;
    const int64_t N = (int64_t)R * S * K;
    // the per-tile counts, then one int: the arrival counter of k_scan_cols_meta
    return align256(sizeof(int32_t) * (size_t)sort_tiles(N) * n_keys) + 256;
}

}  // extern "C"

namespace {
// The argument checks of mep_plan, without the workspace (shared with mep_plan_static_ws).
mep_status_t plan_args(const int32_t *ids, const uint8_t *keep, int32_t R, int32_t n_keys, int32_t S, int32_t K,
                       int32_t mode, int32_t keys_per_rank, const int32_t *pos, const int32_t *hist,
                       const int32_t *rank_off, const int32_t *rep_count, const int32_t *rep_key,
                       const int32_t *rep_cu, const mep_plan_stats_t *stats)
{
    if (!ids || !pos || !hist || !rank_off || !rep_count || !rep_key || !rep_cu || !stats)
        return MEP_ERR_NULLPTR;
    if (R < 1 || S < 1 || K < 1 || K > MEP_MAX_K || n_keys < 1 || n_keys > MEP_MAX_KEYS ||
        R > MEP_MAX_KEYS)
        return MEP_ERR_SHAPE;
    const int64_t N = (int64_t)R * S * K;
    if (N >= ((int64_t)1 << 31)) return MEP_ERR_SHAPE;
    if (mode == MEP_PLAN_BALANCED) {
        if (n_keys % R != 0 || keep) return MEP_ERR_VALUE;
    } else if (mode == MEP_PLAN_GROUPED) {
        if (keys_per_rank < 1 || (int64_t)keys_per_rank * R != n_keys) return MEP_ERR_VALUE;
    } else {
        return MEP_ERR_VALUE;
    }
    return MEP_OK;
}
}  // namespace

extern "C" {

namespace {
// Whether mep_plan runs as one CTA for this shape.
bool plan_is_small(int64_t N, int32_t n_keys)
{
    const size_t small_smem = sizeof(int32_t) * (size_t)(34 * (int64_t)n_keys + 34);
    return N <= mep::kSmallPlanMaxSlots && small_smem <= (size_t)kSmallPlanSmemMax;
}
}  // namespace

int32_t mep_plan_launches(int32_t R, int32_t n_keys, int32_t S, int32_t K)
{
    if (R < 1 || S < 1 || K < 1 || n_keys < 1) return 0;
    return plan_is_small((int64_t)R * S * K, n_keys) ? 1 : 3;
}

mep_status_t mep_plan(const int32_t *ids, const uint8_t *keep, int32_t R, int32_t n_keys,
                      int32_t S, int32_t K, int32_t mode, int32_t keys_per_rank,
                      int32_t *pos, int32_t *hist, int32_t *rank_off, int32_t *load,
                      int32_t *rep_count, int32_t *rep_key, int32_t *rep_cu,
                      mep_plan_stats_t *stats, void *workspace, size_t workspace_bytes,
                      mep_stream_t stream)
{
    const mep_status_t st = plan_args(ids, keep, R, n_keys, S, K, mode, keys_per_rank, pos, hist, rank_off,
                                      rep_count, rep_key, rep_cu, stats);
    if (st != MEP_OK) return st;
    const int64_t N = (int64_t)R * S * K;
    const size_t need = mep_plan_workspace_size(R, n_keys, S, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return MEP_ERR_WORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    sm_count();
    // small problems: the whole plan in one launch instead of four, over a cluster of
    // CTAs when it fits, else in one CTA
    const size_t cluster_smem = sizeof(int32_t) * (size_t)(36 * (int64_t)n_keys + 34);
    if (N <= mep::kClusterPlanMaxSlots && cluster_smem <= (size_t)kSmallPlanSmemMax && cluster_plan_ok()) {
        launch_pdl(mep::k_plan_cluster, dim3(mep::kPlanClusterCTAs), dim3(mep::kSmallPlanThreads), cluster_smem, s, ids,
                   keep, N, n_keys, R, (int64_t)S * K, mode, keys_per_rank, pos, hist, rank_off, load, rep_count,
                   rep_key, rep_cu, (int32_t *)stats);
        return launched();
    }
    if (plan_is_small(N, n_keys)) {
        const size_t small_smem = sizeof(int32_t) * (size_t)(34 * (int64_t)n_keys + 34);
        launch_pdl(mep::k_plan_small, dim3(1), dim3(mep::kSmallPlanThreads), small_smem, s, ids, keep, N, n_keys, R,
                   (int64_t)S * K, mode, keys_per_rank, pos, hist, rank_off, load, rep_count, rep_key, rep_cu,
                   (int32_t *)stats);
        return launched();
    }
    // the sort, with the replica tables written by the last CTA of its scan
    const int64_t N_tiles = sort_tiles(N);
    PlanMeta meta;
    meta.arrived = (int32_t *)((char *)workspace + align256(sizeof(int32_t) * (size_t)N_tiles * n_keys));
    meta.R = R;
    meta.SK = (int64_t)S * K;
    meta.mode = mode;
    meta.keys_per_rank = keys_per_rank;
    meta.rank_off = rank_off;
    meta.load = load;
    meta.rep_count = rep_count;
    meta.rep_key = rep_key;
    meta.rep_cu = rep_cu;
    meta.stats = (int32_t *)stats;
    counting_sort(ids, keep, N, n_keys, (int32_t *)workspace, hist, nullptr, pos, s, &meta);
    return launched();
}

size_t mep_plan_rank_workspace_size(int32_t R, int32_t E, int32_t S, int32_t K)
{
    if (R < 1 || E < 1 || S < 1 || K < 1) return 0;
    const int64_t tiles = sort_tiles((int64_t)S * K);
    return align256(sizeof(int32_t) * (size_t)tiles * E) + 2 * align256(sizeof(int32_t) * (size_t)E);
}

mep_status_t mep_plan_rank(const int32_t *ids, const int32_t *hist_all, int32_t R, int32_t E, int32_t S,
                           int32_t K, int32_t rank, int32_t *pos, int32_t *send_count, int32_t *send_off,
                           int32_t *recv_count, int32_t *recv_off, void *workspace, size_t workspace_bytes,
                           mep_stream_t stream)
{
    if (!ids || !hist_all || !pos || !send_count || !send_off || !recv_count || !recv_off) return MEP_ERR_NULLPTR;
    if (R < 1 || S < 1 || K < 1 || K > MEP_MAX_K || E < 1 || E > MEP_MAX_KEYS || R > MEP_MAX_KEYS)
        return MEP_ERR_SHAPE;
    if ((int64_t)R * S * K >= ((int64_t)1 << 31)) return MEP_ERR_SHAPE;
    if (E % R != 0 || rank < 0 || rank >= R) return MEP_ERR_VALUE;
    const size_t need = mep_plan_rank_workspace_size(R, E, S, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return MEP_ERR_WORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    sm_count();
    const int64_t N = (int64_t)S * K;   // this rank's slots
    const int64_t tiles = sort_tiles(N);
    unsigned char *w = (unsigned char *)workspace;
    int32_t *tile_cnt = (int32_t *)w;
    w += align256(sizeof(int32_t) * (size_t)tiles * E);
    int32_t *hist_local = (int32_t *)w;
    w += align256(sizeof(int32_t) * (size_t)E);
    int32_t *key_base = (int32_t *)w;
    // the rank's own histogram first (the tile counts and their column scan), then the
    // bases from the gathered histograms, then the rows from those bases
    const int threads = mep::kPlanWarps * 32;
    const int rounds = sort_rounds(N);
    if (rounds == 2)
        mep::k_tile_count<2><<<(unsigned)tiles, threads, sizeof(int32_t) * E, s>>>(ids, nullptr, N, E, tile_cnt,
                                                                                 nullptr);
    else if (rounds == 4)
        mep::k_tile_count<4><<<(unsigned)tiles, threads, sizeof(int32_t) * E, s>>>(ids, nullptr, N, E, tile_cnt,
                                                                                 nullptr);
    else
        mep::k_tile_count<8><<<(unsigned)tiles, threads, sizeof(int32_t) * E, s>>>(ids, nullptr, N, E, tile_cnt,
                                                                                 nullptr);
    mep::k_scan_cols<<<(unsigned)mep::ceil_div(E, 32), 1024, 0, s>>>(tile_cnt, (int32_t)tiles, E, hist_local);
    const size_t meta_smem = sizeof(int32_t) * (size_t)(2 * E + 1 + 2 * R);
    mep::k_source_meta<<<1, 1024, meta_smem, s>>>(hist_all, hist_local, R, E, (int64_t)S * K, rank, key_base,
                                                  send_count, send_off, recv_count, recv_off);
    const size_t rank_smem = sizeof(int32_t) * ((size_t)mep::kPlanWarps * E + E + 1 + 33);
    if (rounds == 2)
        mep::k_rank<2><<<(unsigned)tiles, threads, rank_smem, s>>>(ids, nullptr, N, E, tile_cnt, hist_local, key_base,
                                                                   pos);
    else if (rounds == 4)
        mep::k_rank<4><<<(unsigned)tiles, threads, rank_smem, s>>>(ids, nullptr, N, E, tile_cnt, hist_local, key_base,
                                                                   pos);
    else
        mep::k_rank<8><<<(unsigned)tiles, threads, rank_smem, s>>>(ids, nullptr, N, E, tile_cnt, hist_local, key_base,
                                                                   pos);
    return launched();
}

mep_status_t mep_update_expert(const int32_t *expert_ids, const int32_t *eplb_table,
                               const float *expert_scales, const float *pruning_threshold,
                               const uint8_t *active_mask, int64_t BS, int32_t K,
                               int32_t n_experts, int32_t F, int64_t local_rank_id,
                               int64_t world_size, int64_t balance_mode,
                               int32_t *balanced_expert_ids, uint8_t *balanced_active_mask,
                               mep_stream_t stream)
{
    if (!expert_ids || !eplb_table || !balanced_expert_ids || !balanced_active_mask)
        return MEP_ERR_NULLPTR;
    if ((expert_scales == nullptr) != (pruning_threshold == nullptr)) return MEP_ERR_NULLPTR;
    if (active_mask && !expert_scales) return MEP_ERR_NULLPTR;
    if (BS < 1 || K < 1 || K > 16 || n_experts < 1 || n_experts > 1024 || K > n_experts)
        return MEP_ERR_SHAPE;
    if (world_size < 1 || F < 2 || F > world_size + 1) return MEP_ERR_SHAPE;
    if (balance_mode != 0 && balance_mode != 1) return MEP_ERR_VALUE;
    if (balance_mode == 0 && (world_size < 2 || world_size > 768)) return MEP_ERR_VALUE;
    if (balance_mode == 0 && (local_rank_id < 0 || local_rank_id >= world_size)) return MEP_ERR_VALUE;
    cudaStream_t s = (cudaStream_t)stream;
    const int threads = 256;
    int64_t g = (BS * K + threads - 1) / threads;
    int cap = sm_count() * 8;
    launch_pdl(mep::k_update_expert, dim3((unsigned)(g < cap ? g : cap)), dim3(threads), 0, s, expert_ids, eplb_table,
               expert_scales, pruning_threshold, active_mask, BS, BS, local_rank_id, K, n_experts, F, world_size,
               balance_mode, balanced_expert_ids, balanced_active_mask);
    return launched();
}

mep_status_t mep_update_expert_ranks(const int32_t *expert_ids, const int32_t *eplb_table,
                                     const float *expert_scales, const float *pruning_threshold,
                                     const uint8_t *active_mask, int64_t BS, int32_t K, int32_t n_experts,
                                     int32_t F, int64_t world_size, int64_t balance_mode,
                                     int32_t *balanced_expert_ids, uint8_t *balanced_active_mask,
                                     mep_stream_t stream)
{
    if (!expert_ids || !eplb_table || !balanced_expert_ids || !balanced_active_mask)
        return MEP_ERR_NULLPTR;
    if ((expert_scales == nullptr) != (pruning_threshold == nullptr)) return MEP_ERR_NULLPTR;
    if (active_mask && !expert_scales) return MEP_ERR_NULLPTR;
    if (BS < 1 || K < 1 || K > 16 || n_experts < 1 || n_experts > 1024 || K > n_experts)
        return MEP_ERR_SHAPE;
    if (world_size < 1 || F < 2 || F > world_size + 1) return MEP_ERR_SHAPE;
    if (balance_mode != 0 && balance_mode != 1) return MEP_ERR_VALUE;
    if (balance_mode == 0 && (world_size < 2 || world_size > 768)) return MEP_ERR_VALUE;
    if (BS * world_size * K >= ((int64_t)1 << 31)) return MEP_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    const int threads = 256;
    const int64_t rows = BS * world_size;
    int64_t g = (rows * K + threads - 1) / threads;
    int cap = sm_count() * 8;
    launch_pdl(mep::k_update_expert, dim3((unsigned)(g < cap ? g : cap)), dim3(threads), 0, s, expert_ids, eplb_table,
               expert_scales, pruning_threshold, active_mask, rows, BS, (int64_t)0, K, n_experts, F, world_size,
               balance_mode, balanced_expert_ids, balanced_active_mask);
    return launched();
}

mep_status_t mep_dispatch(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K,
                          int64_t H, int32_t quant, void *recv, float *recv_scale,
                          int64_t rows, mep_stream_t stream)
{
    if (quant != 0 && quant != 1) return MEP_ERR_DTYPE;
    if (T > 0 && (!x || !pos || (!recv && rows > 0) || (quant == 1 && !recv_scale && rows > 0)))
        return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || rows < 0 || T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = token_grid(T, 8);
    if (quant == 0) {
        if (H % 8 == 0 && aligned(x, 16) && aligned(recv, 16)) {
            // one warp per half token row, 8 warps per CTA, up to 64 CTAs per SM in waves
            const int64_t ctas = mep::ceil_div(2 * T, 8);
            const int64_t cap = (int64_t)sm_count() * 64;
            launch_pdl(mep::k_dispatch_warp, dim3((unsigned)(ctas < cap ? ctas : cap)), dim3(256), 0, s, (const uint4 *)x,
                       pos, T, K, (int64_t)(H / 8), rows, (uint4 *)recv);
        } else {
            mep::k_dispatch_elem<<<grid, 256, 0, s>>>(x, pos, T, K, H, rows, (uint16_t *)recv);
        }
    } else {
        const size_t staged_smem = (size_t)mep::kDispatchSmemHead + 4 * (size_t)H * 2 + 2 * (size_t)H;
        if (H % 16 == 0 && aligned(x, 16) && aligned(recv, 16) && staged_smem <= (size_t)kBulkSmemMax) {
            // CTAs of kStagedChunk consecutive tokens, as many as the tokens need
            launch_pdl(mep::k_dispatch_int8_staged<4, 128>, dim3((unsigned)mep::ceil_div(T, mep::kStagedChunk)),
                       dim3(128), staged_smem, s, x, pos, T, (int)K, H, rows, (int8_t *)recv, recv_scale);
        } else if (H % 8 == 0 && aligned(x, 16) && aligned(recv, 8)) {
            mep::k_dispatch_int8<<<grid, 256, 0, s>>>((const uint4 *)x, pos, T, K, H / 8, rows,
                                                      (uint2 *)recv, recv_scale);
        } else {
            mep::k_dispatch_int8_scalar<<<grid, 256, 0, s>>>(x, pos, T, K, H, rows, (int8_t *)recv,
                                                             recv_scale);
        }
    }
    return launched();
}

mep_status_t mep_dequantize(const int8_t *q, const float *scale, int64_t rows, int64_t H,
                            uint16_t *y, mep_stream_t stream)
{
    if (rows > 0 && (!q || !scale || !y)) return MEP_ERR_NULLPTR;
    if (rows < 0 || H < 1) return MEP_ERR_SHAPE;
    if (rows == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (H % 8 == 0 && aligned(q, 8) && aligned(y, 16)) {
        const int64_t total = rows * (H / 8);
        mep::k_dequant8<<<elem_grid(total, 256), 256, 0, s>>>((const uint2 *)q, scale, rows, H / 8, (uint4 *)y);
    } else {
        mep::k_dequant_scalar<<<elem_grid(rows * H, 256), 256, 0, s>>>(q, scale, rows, H, y);
    }
    return launched();
}

mep_status_t mep_combine(const uint16_t *y, int64_t rows, const int32_t *pos,
                         const float *gates, int64_t T, int32_t K, int64_t H, uint16_t *out,
                         mep_stream_t stream)
{
    if (T > 0 && (!pos || !gates || !out || (!y && rows > 0))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || rows < 0 || T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    // a CTA per token: the block scheduler balances the SMs (3% faster than a resident grid
    // striding over the tokens)
    const int grid = (int)std::min<int64_t>(T, INT32_MAX);
    if (H % 8 == 0 && aligned(y, 16) && aligned(out, 16)) {
        const uint4 *yv = (const uint4 *)y;
        uint4 *ov = (uint4 *)out;
        const int64_t H8 = H / 8;
        switch (K) {
        case 1: launch_pdl(mep::k_combine_v8<1>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        case 2: launch_pdl(mep::k_combine_v8<2>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        case 4: launch_pdl(mep::k_combine_v8<4>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        case 6: launch_pdl(mep::k_combine_v8<6>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        case 8: launch_pdl(mep::k_combine_v8<8>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        default: launch_pdl(mep::k_combine_v8<0>, dim3(grid), dim3(256), 0, s, yv, pos, gates, T, (int)K, H8, rows, ov); break;
        }
    } else {
        mep::k_combine_scalar<<<grid, 256, 0, s>>>(y, pos, gates, T, K, H, rows, out);
    }
    return launched();
}

mep_status_t mep_combine_int8(const int8_t *yq, const float *y_scale, int64_t rows, const int32_t *pos,
                              const float *gates, int64_t T, int32_t K, int64_t H, uint16_t *out,
                              mep_stream_t stream)
{
    if (T > 0 && (!pos || !gates || !out || ((!yq || !y_scale) && rows > 0))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || rows < 0 || T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = token_grid(T, 8);
    if (H % 16 == 0 && aligned(yq, 16) && aligned(out, 16)) {
        const uint4 *yv = (const uint4 *)yq;
        uint4 *ov = (uint4 *)out;
        const int64_t H16 = H / 16;
        using kernel_t = void (*)(const uint4 *, const float *, const int32_t *, const float *, int64_t, int,
                                  int64_t, int64_t, uint4 *);
        kernel_t kern;
        switch (K) {
        case 1: kern = mep::k_combine_int8_warp<1>; break;
        case 2: kern = mep::k_combine_int8_warp<2>; break;
        case 4: kern = mep::k_combine_int8_warp<4>; break;
        case 6: kern = mep::k_combine_int8_warp<6>; break;
        case 8: kern = mep::k_combine_int8_warp<8>; break;
        default: kern = mep::k_combine_int8_warp<0>; break;
        }
        // one warp per token, a CTA for every 4 tokens: the block scheduler hands CTAs to
        // SMs as they free up, which balances the SMs better than a resident grid striding
        // over the tokens (2% faster inside the step)
        const int tpb = mep::kCombineInt8Threads;
        launch_pdl(kern, dim3((unsigned)mep::ceil_div(T, tpb / 32)), dim3(tpb), 0, s, yv, y_scale,
                   pos, gates, T, (int)K, H16, rows, ov);
    } else if (H % 8 == 0 && aligned(yq, 8) && aligned(out, 16)) {
        const uint2 *yv = (const uint2 *)yq;
        uint4 *ov = (uint4 *)out;
        const int64_t H8 = H / 8;
        switch (K) {
        case 1: mep::k_combine_int8_v8<1><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        case 2: mep::k_combine_int8_v8<2><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        case 4: mep::k_combine_int8_v8<4><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        case 6: mep::k_combine_int8_v8<6><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        case 8: mep::k_combine_int8_v8<8><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        default: mep::k_combine_int8_v8<0><<<grid, 256, 0, s>>>(yv, y_scale, pos, gates, T, K, H8, rows, ov); break;
        }
    } else {
        mep::k_combine_int8_scalar<<<grid, 256, 0, s>>>(yq, y_scale, pos, gates, T, K, H, rows, out);
    }
    return launched();
}

mep_status_t mep_combine_add_rmsnorm(const uint16_t *y, int64_t rows, const int32_t *pos, const float *gates,
                                     int64_t T, int32_t K, int64_t H, const uint16_t *residual,
                                     const uint16_t *gamma, float eps, uint16_t *x_out, uint16_t *y_out,
                                     float *rstd_out, mep_stream_t stream)
{
    if (T > 0 && (!pos || !gates || !residual || !gamma || !x_out || !y_out || !rstd_out || (!y && rows > 0)))
        return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || H > MEP_RMSNORM_MAX_H || rows < 0 ||
        T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (!(eps >= 0.0f) || eps > 1.0e30f) return MEP_ERR_VALUE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = token_grid(T, 8);
    const size_t smem = sizeof(float) * (size_t)H;
    if (H % 8 == 0 && aligned(y, 16) && aligned(residual, 16) && aligned(gamma, 16) && aligned(x_out, 16) &&
        aligned(y_out, 16)) {
        const uint4 *yv = (const uint4 *)y, *rv = (const uint4 *)residual, *gv = (const uint4 *)gamma;
        uint4 *xo = (uint4 *)x_out, *yo = (uint4 *)y_out;
        const int64_t H8 = H / 8;
        switch (K) {
        case 8: mep::k_combine_add_rmsnorm_v8<8><<<grid, 256, smem, s>>>(yv, pos, gates, T, K, H8, rows, rv, gv, eps, xo, yo, rstd_out); break;
        case 6: mep::k_combine_add_rmsnorm_v8<6><<<grid, 256, smem, s>>>(yv, pos, gates, T, K, H8, rows, rv, gv, eps, xo, yo, rstd_out); break;
        case 4: mep::k_combine_add_rmsnorm_v8<4><<<grid, 256, smem, s>>>(yv, pos, gates, T, K, H8, rows, rv, gv, eps, xo, yo, rstd_out); break;
        case 2: mep::k_combine_add_rmsnorm_v8<2><<<grid, 256, smem, s>>>(yv, pos, gates, T, K, H8, rows, rv, gv, eps, xo, yo, rstd_out); break;
        default: mep::k_combine_add_rmsnorm_v8<0><<<grid, 256, smem, s>>>(yv, pos, gates, T, K, H8, rows, rv, gv, eps, xo, yo, rstd_out); break;
        }
    } else {
        mep::k_combine_add_rmsnorm_scalar<<<grid, 256, smem, s>>>(y, pos, gates, T, K, H, rows, residual, gamma, eps,
                                                                x_out, y_out, rstd_out);
    }
    return launched();
}

mep_status_t mep_prefetch_plan(const int32_t *rep_count, const int32_t *rep_key, int32_t R, int32_t E, int32_t cap,
                               int32_t B, int32_t *slot_expert, int32_t *rep_weight, mep_stream_t stream)
{
    if (!rep_count || !rep_key || !rep_weight || (B > 0 && !slot_expert)) return MEP_ERR_NULLPTR;
    if (R < 1 || E < 1 || E > MEP_MAX_KEYS || R > MEP_MAX_KEYS || cap < 1 || cap > MEP_MAX_KEYS || B < 0 ||
        (int64_t)R * B > MEP_MAX_SLOTS)
        return MEP_ERR_SHAPE;
    if (E % R != 0) return MEP_ERR_VALUE;
    mep::k_prefetch_plan<<<(unsigned)mep::ceil_div(R, 128), 128, 0, (cudaStream_t)stream>>>(
        rep_count, rep_key, R, E, cap, B, slot_expert, rep_weight);
    return launched();
}

mep_status_t mep_prefetch_weights(const uint16_t *w_home, const int32_t *slot_expert, int32_t E, int32_t R,
                                  int32_t B, int64_t D, uint16_t *w_slots, mep_stream_t stream)
{
    if ((int64_t)R * B > 0 && (!w_home || !slot_expert || !w_slots)) return MEP_ERR_NULLPTR;
    if (E < 1 || R < 1 || B < 0 || D < 1 || (int64_t)R * B > MEP_MAX_SLOTS) return MEP_ERR_SHAPE;
    if ((int64_t)R * B == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t per = (int64_t)sm_count() * 8;   // CTAs per slot, before the cap below
    if (D % 8 == 0 && aligned(w_home, 16) && aligned(w_slots, 16)) {
        const int64_t D8 = D / 8;
        int64_t gx = mep::ceil_div(D8, 256 * 4);
        if (gx > per) gx = per;
        dim3 grid((unsigned)(gx > 0 ? gx : 1), (unsigned)(R * B));
        mep::k_prefetch_weights<<<grid, 256, 0, s>>>((const uint4 *)w_home, slot_expert, E, D8, (uint4 *)w_slots);
    } else {
        int64_t gx = mep::ceil_div(D, 256 * 4);
        if (gx > per) gx = per;
        dim3 grid((unsigned)(gx > 0 ? gx : 1), (unsigned)(R * B));
        mep::k_prefetch_weights_scalar<<<grid, 256, 0, s>>>(w_home, slot_expert, E, D, w_slots);
    }
    return launched();
}

mep_status_t mep_grad_reduce(float *grad_home, float *grad_slots, const int32_t *slot_expert, int32_t E, int32_t R,
                             int32_t B, int64_t D, mep_stream_t stream)
{
    if ((int64_t)R * B > 0 && (!grad_home || !grad_slots || !slot_expert)) return MEP_ERR_NULLPTR;
    if (E < 1 || E > 65535 || R < 1 || B < 0 || D < 1 || (int64_t)R * B > MEP_MAX_SLOTS) return MEP_ERR_SHAPE;
    if ((int64_t)R * B == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int32_t RB = R * B;
    const int64_t per = (int64_t)sm_count() * 4;
    if (D % 4 == 0 && aligned(grad_home, 16) && aligned(grad_slots, 16)) {
        const int64_t D4 = D / 4;
        int64_t gx = mep::ceil_div(D4, 256 * 4 * mep::kReduceUnroll);
        if (gx > per) gx = per;
        dim3 grid((unsigned)(gx > 0 ? gx : 1), (unsigned)E);
        mep::k_grad_reduce<<<grid, 256, 0, s>>>((float4 *)grad_home, (float4 *)grad_slots, slot_expert, RB, D4);
    } else {
        int64_t gx = mep::ceil_div(D, 256 * 4);
        if (gx > per) gx = per;
        dim3 grid((unsigned)(gx > 0 ? gx : 1), (unsigned)E);
        mep::k_grad_reduce_scalar<<<grid, 256, 0, s>>>(grad_home, grad_slots, slot_expert, RB, D);
    }
    return launched();
}

mep_status_t mep_dispatch_int8_smooth(const uint16_t *x, const int32_t *ids, const int32_t *pos, int64_t T,
                                      int32_t K, int64_t H, const float *smooth, int32_t n_experts, int8_t *recv,
                                      float *recv_scale, int64_t rows, mep_stream_t stream)
{
    if (T > 0 && (!x || !ids || !pos || !smooth || (rows > 0 && (!recv || !recv_scale)))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || rows < 0 || n_experts < 1 || T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t H4 = H / 4;
    const bool vec4 = H % 4 == 0 && aligned(x, 8) && aligned(recv, 4) && aligned(smooth, 16);
    const int64_t groups = mep::ceil_div(H4, 256);
    if (vec4 && groups <= 16) {
        // the K slots of a token together, a CTA per token
        using smooth_k_t = void (*)(const uint2 *, const int32_t *, const int32_t *, int64_t, int, int64_t,
                                    const float4 *, int32_t, int64_t, uint32_t *, float *);
        const smooth_k_t fused = groups <= 8 ? mep::k_dispatch_int8_smooth_k<8> : mep::k_dispatch_int8_smooth_k<16>;
        fused<<<(unsigned)std::min<int64_t>(T, INT32_MAX), 256, 0, s>>>((const uint2 *)x, ids, pos, T, K, H4, (const float4 *)smooth,
                                                          n_experts, rows, (uint32_t *)recv, recv_scale);
    } else {
        mep::k_dispatch_int8_smooth_scalar<<<token_grid(T, 8), 256, 0, s>>>(x, ids, pos, T, K, H, smooth, n_experts,
                                                                           rows, recv, recv_scale);
    }
    return launched();
}

size_t mep_dispatch_int8_smooth_workspace_size(int64_t T, int32_t K)
{
    if (T < 0 || K < 1 || K > MEP_MAX_K || T * K >= ((int64_t)1 << 31)) return 0;
    return align256(sizeof(int32_t) * (size_t)(T * K));
}

mep_status_t mep_dispatch_int8_smooth_grouped(const uint16_t *x, const int32_t *ids, const int32_t *pos, int64_t T,
                                              int32_t K, int64_t H, const float *smooth, int32_t n_experts,
                                              int8_t *recv, float *recv_scale, int64_t rows, void *workspace,
                                              size_t workspace_bytes, mep_stream_t stream)
{
    if (T > 0 && (!x || !ids || !pos || !smooth || (rows > 0 && (!recv || !recv_scale)))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 1 || rows < 0 || n_experts < 1 || T * K >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    const size_t need = mep_dispatch_int8_smooth_workspace_size(T, K);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return MEP_ERR_WORKSPACE;
    if (T == 0) return MEP_OK;
    const int64_t H4 = H / 4;
    const bool vec4 = H % 4 == 0 && aligned(x, 8) && aligned(recv, 4) && aligned(smooth, 16);
    if (!vec4 || H4 > 256 * mep::kSmoothMaxGroups || n_experts > mep::kSmoothOrderMaxExperts)   // per-token kernels
        return mep_dispatch_int8_smooth(x, ids, pos, T, K, H, smooth, n_experts, recv, recv_scale, rows, stream);
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t N = T * K;
    int32_t *order = (int32_t *)workspace;
    const int64_t chunk = std::max<int64_t>(1, mep::kSmoothChunkSlots / K);
    launch_pdl(mep::k_smooth_order, dim3((unsigned)mep::ceil_div(T, chunk)), dim3(mep::kSmoothOrderThreads),
               sizeof(int32_t) * (2 * (size_t)n_experts + 3), s, ids, pos, T, K, chunk, n_experts, rows, order);
    // groups of 4 columns per thread: ceil(H / 4 / 256)
    using grouped_t = void (*)(const uint2 *, const int32_t *, const int32_t *, const int32_t *, int64_t, int,
                               int64_t, const float4 *, int32_t, int64_t, uint32_t *, float *);
    static const grouped_t kern[2][mep::kSmoothMaxGroups] = {
        {mep::k_dispatch_int8_smooth_grouped<1, false>, mep::k_dispatch_int8_smooth_grouped<2, false>,
         mep::k_dispatch_int8_smooth_grouped<3, false>, mep::k_dispatch_int8_smooth_grouped<4, false>,
         mep::k_dispatch_int8_smooth_grouped<5, false>, mep::k_dispatch_int8_smooth_grouped<6, false>,
         mep::k_dispatch_int8_smooth_grouped<7, false>, mep::k_dispatch_int8_smooth_grouped<8, false>},
        {mep::k_dispatch_int8_smooth_grouped<1, true>, mep::k_dispatch_int8_smooth_grouped<2, true>,
         mep::k_dispatch_int8_smooth_grouped<3, true>, mep::k_dispatch_int8_smooth_grouped<4, true>,
         mep::k_dispatch_int8_smooth_grouped<5, true>, mep::k_dispatch_int8_smooth_grouped<6, true>,
         mep::k_dispatch_int8_smooth_grouped<7, true>, mep::k_dispatch_int8_smooth_grouped<8, true>}};
    const int64_t groups = mep::ceil_div(H4, mep::kSmoothThreads);
    const bool full = H4 == groups * mep::kSmoothThreads;
    launch_pdl(kern[full][groups - 1], dim3((unsigned)mep::ceil_div(N, mep::kSmoothSlotsPerCTA)), dim3(mep::kSmoothThreads),
               0, s, (const uint2 *)x, ids, pos, (const int32_t *)order, N, (int)K, H4, (const float4 *)smooth,
               n_experts, rows, (uint32_t *)recv, recv_scale);
    return launched();
}

mep_status_t mep_stream_synchronize_timeout(mep_stream_t stream, int32_t timeout_ms)
{
    if (timeout_ms < 0) return MEP_ERR_VALUE;
    cudaStream_t s = (cudaStream_t)stream;
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaStreamQuery(s);
        if (e == cudaSuccess) return MEP_OK;
        if (e != cudaErrorNotReady) {
            t_last_cuda_error = (int32_t)e;
            return MEP_ERR_CUDA;
        }
        // "not ready" is no failure: keep it out of the error a later launch checks
        if (cudaPeekAtLastError() == cudaErrorNotReady) (void)cudaGetLastError();
        if (std::chrono::steady_clock::now() - t0 >= std::chrono::milliseconds(timeout_ms)) return MEP_ERR_TIMEOUT;
        std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
}

mep_status_t mep_selftest_bounded_wait(int32_t max_polls, int32_t *timed_out, mep_stream_t stream)
{
    if (!timed_out) return MEP_ERR_NULLPTR;
    if (max_polls < 1 || max_polls > mep::kWaitPolls) return MEP_ERR_VALUE;
    mep::k_selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>(max_polls, timed_out);
    return launched();
}

// ------------------------------------------------ f1: one row per (token, destination rank)

size_t mep_dedup_workspace_size(int32_t R, int32_t S, int32_t K)
{
    if (R < 1 || S < 1 || K < 1) return 0;
    const int64_t N = (int64_t)R * S * K;
    const int64_t tiles = sort_tiles(N);
    return align256(sizeof(int32_t) * (size_t)N) + align256((size_t)N) +
           align256(sizeof(int32_t) * (size_t)tiles * R) + align256(sizeof(int32_t) * (size_t)R);
}

mep_status_t mep_dedup_plan(const int32_t *pos, const int32_t *rank_off, int32_t R, int32_t S, int32_t K,
                            int32_t *dsend, int32_t *dpos, int32_t *drank_off, int32_t *dtok, int32_t *gidx,
                            void *workspace, size_t workspace_bytes, mep_stream_t stream)
{
    if (!pos || !rank_off || !dsend || !dpos || !drank_off || !dtok || !gidx) return MEP_ERR_NULLPTR;
    if (R < 1 || S < 1 || K < 1 || K > MEP_MAX_K || R > MEP_MAX_KEYS) return MEP_ERR_SHAPE;
    const int64_t N = (int64_t)R * S * K;
    if (N >= ((int64_t)1 << 31)) return MEP_ERR_SHAPE;
    const size_t need = mep_dedup_workspace_size(R, S, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return MEP_ERR_WORKSPACE;

    cudaStream_t s = (cudaStream_t)stream;
    const int sms = sm_count();
    const int64_t T = (int64_t)R * S;
    const int64_t tiles = sort_tiles(N);
    unsigned char *w = (unsigned char *)workspace;
    int32_t *dkey = (int32_t *)w;
    w += align256(sizeof(int32_t) * (size_t)N);
    uint8_t *dkeep = (uint8_t *)w;
    w += align256((size_t)N);
    int32_t *tile_cnt = (int32_t *)w;
    w += align256(sizeof(int32_t) * (size_t)tiles * R);
    int32_t *count = (int32_t *)w;

    if (cudaMemsetAsync(dtok, 0xff, sizeof(int32_t) * (size_t)N, s) != cudaSuccess) return launched();
    if (cudaMemsetAsync(gidx, 0xff, sizeof(int32_t) * (size_t)N, s) != cudaSuccess) return launched();
    const int64_t tg = mep::ceil_div(T, 256), tcap = (int64_t)sms * 8;
    const unsigned tgrid = (unsigned)(tg < tcap ? tg : tcap);
    const size_t off_smem = sizeof(int32_t) * (size_t)(R + 1);
    mep::k_dedup_keys<<<tgrid, 256, off_smem, s>>>(pos, rank_off, R, T, K, dkey, dkeep);
    counting_sort(dkey, dkeep, N, R, tile_cnt, count, nullptr, dsend, s);
    mep::k_dedup_offsets<<<1, 1024, sizeof(int32_t) * (size_t)(R + 1 + 33), s>>>(count, R, drank_off);
    mep::k_dedup_finish<<<tgrid, 256, off_smem, s>>>(pos, rank_off, R, T, K, dsend, dpos, dtok, gidx);
    return launched();
}

mep_status_t mep_expand(const void *src, const float *src_scale, int64_t src_rows, const int32_t *gidx,
                        int64_t rows, int64_t H, int32_t quant, void *dst, float *dst_scale, mep_stream_t stream)
{
    if (quant != 0 && quant != 1) return MEP_ERR_DTYPE;
    if (rows < 0 || src_rows < 0 || H < 1) return MEP_ERR_SHAPE;
    if (rows == 0) return MEP_OK;
    if (!gidx || !dst || (!src && src_rows > 0)) return MEP_ERR_NULLPTR;
    if (quant == 1 && (!dst_scale || (!src_scale && src_rows > 0))) return MEP_ERR_NULLPTR;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t row_bytes = quant == 1 ? H : 2 * H;
    const float *ss = quant == 1 ? src_scale : nullptr;
    float *ds = quant == 1 ? dst_scale : nullptr;
    if (row_bytes % 16 == 0 && aligned(src, 16) && aligned(dst, 16)) {
        // a CTA for every 8 rows, handed to SMs as they free up (9-12% faster than a resident
        // grid striding over the rows)
        const unsigned g = (unsigned)mep::ceil_div(rows, 8);
        mep::k_expand_warp<<<g, 256, 0, s>>>((const uint4 *)src, ss, src_rows, gidx, rows, row_bytes / 16,
                                             (uint4 *)dst, ds);
    } else {
        mep::k_expand_bytes<<<token_grid(rows, 8), 256, 0, s>>>((const uint8_t *)src, ss, src_rows, gidx, rows,
                                                              row_bytes, (uint8_t *)dst, ds);
    }
    return launched();
}

// ------------------------------------------ (e): rows in the ranks' own buffers

mep_status_t mep_dispatch_ranks(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K, int64_t H,
                                int32_t quant, void *const *recv_ptrs, float *const *scale_ptrs, int32_t R,
                                int64_t rows_per_rank, mep_stream_t stream)
{
    if (quant != 0 && quant != 1) return MEP_ERR_DTYPE;
    if (T > 0 && (!x || !pos || !recv_ptrs || (quant == 1 && !scale_ptrs))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 8 || H % 8 != 0 || R < 1 || R > MEP_MAX_KEYS ||
        rows_per_rank < 1 || T * K >= ((int64_t)1 << 31) || (int64_t)R * rows_per_rank >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T > 0 && (!aligned(x, 16) || !aligned(recv_ptrs, 8) || (quant == 1 && !aligned(scale_ptrs, 8))))
        return MEP_ERR_VALUE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (quant == 0) {
        const int64_t ctas = mep::ceil_div(T, 8);
        const int64_t cap = (int64_t)sm_count() * 16;
        mep::k_dispatch_ranks_warp<<<(int)(ctas < cap ? ctas : cap), 256, 0, s>>>(
            (const uint4 *)x, pos, T, K, H / 8, (uint4 *const *)recv_ptrs, R, rows_per_rank);
    } else {
        mep::k_dispatch_ranks_int8<<<token_grid(T, 8), 256, 0, s>>>((const uint4 *)x, pos, T, K, H / 8,
                                                                   (uint2 *const *)recv_ptrs, scale_ptrs, R,
                                                                   rows_per_rank);
    }
    return launched();
}

mep_status_t mep_combine_ranks(const void *const *y_ptrs, const float *const *scale_ptrs, int32_t quant, int32_t R,
                               int64_t rows_per_rank, const int32_t *pos, const float *gates, int64_t T, int32_t K,
                               int64_t H, uint16_t *out, mep_stream_t stream)
{
    if (quant != 0 && quant != 1) return MEP_ERR_DTYPE;
    if (T > 0 && (!y_ptrs || !pos || !gates || !out || (quant == 1 && !scale_ptrs))) return MEP_ERR_NULLPTR;
    if (T < 0 || K < 1 || K > MEP_MAX_K || H < 8 || H % (quant == 1 ? 16 : 8) != 0 || R < 1 || R > MEP_MAX_KEYS ||
        rows_per_rank < 1 || T * K >= ((int64_t)1 << 31) || (int64_t)R * rows_per_rank >= ((int64_t)1 << 31))
        return MEP_ERR_SHAPE;
    if (T > 0 && (!aligned(out, 16) || !aligned(y_ptrs, 8) || (quant == 1 && !aligned(scale_ptrs, 8))))
        return MEP_ERR_VALUE;
    if (T == 0) return MEP_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (quant == 0) {
        using kern_t = void (*)(const uint4 *const *, const int32_t *, const float *, int64_t, int, int64_t, int32_t,
                                int64_t, uint4 *);
        kern_t kern = K == 8 ? mep::k_combine_ranks_v8<8>
                    : K == 4 ? mep::k_combine_ranks_v8<4>
                    : K == 2 ? mep::k_combine_ranks_v8<2> : mep::k_combine_ranks_v8<0>;
        kern<<<resident_grid(kern, 256, mep::ceil_div(T, 8)), 256, 0, s>>>((const uint4 *const *)y_ptrs, pos, gates, T,
                                                                          K, H / 8, R, rows_per_rank, (uint4 *)out);
    } else {
        using kern_t = void (*)(const uint4 *const *, const float *const *, const int32_t *, const float *, int64_t,
                                int, int64_t, int32_t, int64_t, uint4 *);
        kern_t kern = K == 8 ? mep::k_combine_ranks_int8<8>
                    : K == 4 ? mep::k_combine_ranks_int8<4>
                    : K == 2 ? mep::k_combine_ranks_int8<2> : mep::k_combine_ranks_int8<0>;
        kern<<<resident_grid(kern, 128, mep::ceil_div(T, 4)), 128, 0, s>>>((const uint4 *const *)y_ptrs, scale_ptrs,
                                                                          pos, gates, T, K, H / 16, R, rows_per_rank,
                                                                          (uint4 *)out);
    }
    return launched();
}

// ------------------------------------------------- one round trip from host memory

mep_status_t mep_route_host(const mep_route_buffers_t *b, const int32_t *ids_h, const float *gates_h,
                            const uint16_t *x_h, uint16_t *out_h, mep_stream_t stream)
{
    if (!b || !ids_h || !gates_h || !x_h || !out_h) return MEP_ERR_NULLPTR;
    if (!b->ids || !b->gates || !b->x || !b->recv || !b->out) return MEP_ERR_NULLPTR;
    if (b->quant != 0 && b->quant != 1) return MEP_ERR_DTYPE;
    if (b->R < 1 || b->S < 1 || b->K < 1 || b->H < 1) return MEP_ERR_SHAPE;
    const int64_t T = (int64_t)b->R * b->S, N = T * b->K;
    if (N >= ((int64_t)1 << 31)) return MEP_ERR_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    auto copy = [&](void *dst, const void *src, size_t bytes, cudaMemcpyKind kind) -> mep_status_t {
        if (cudaMemcpyAsync(dst, src, bytes, kind, s) != cudaSuccess) return launched();
        return MEP_OK;
    };
    mep_status_t st;
    if ((st = copy(b->ids, ids_h, sizeof(int32_t) * (size_t)N, cudaMemcpyHostToDevice)) != MEP_OK) return st;
    if ((st = copy(b->gates, gates_h, sizeof(float) * (size_t)N, cudaMemcpyHostToDevice)) != MEP_OK) return st;
    if ((st = copy(b->x, x_h, sizeof(uint16_t) * (size_t)(T * b->H), cudaMemcpyHostToDevice)) != MEP_OK)
        return st;
    st = mep_plan(b->ids, nullptr, b->R, b->E, b->S, b->K, MEP_PLAN_BALANCED, 0, b->pos, b->hist, b->rank_off,
                  b->load, b->rep_count, b->rep_key, b->rep_cu, b->stats, b->workspace, b->workspace_bytes,
                  stream);
    if (st != MEP_OK) return st;
    st = mep_dispatch(b->x, b->pos, T, b->K, b->H, b->quant, b->recv, b->recv_scale, N, stream);
    if (st != MEP_OK) return st;
    if (b->quant == 0)
        st = mep_combine((const uint16_t *)b->recv, N, b->pos, b->gates, T, b->K, b->H, b->out, stream);
    else
        st = mep_combine_int8((const int8_t *)b->recv, b->recv_scale, N, b->pos, b->gates, T, b->K, b->H,
                              b->out, stream);
    if (st != MEP_OK) return st;
    return copy(out_h, b->out, sizeof(uint16_t) * (size_t)(T * b->H), cudaMemcpyDeviceToHost);
}

// ------------------------------------------------------------ maxvio (host only)

mep_status_t mep_maxvio(const mep_plan_stats_t *stats, int32_t S, int32_t K, int32_t n_keys,
                        double *rank_before, double *rank_after, double *expert)
{
    if (!stats) return MEP_ERR_NULLPTR;
    if (S < 1 || K < 1 || n_keys < 1) return MEP_ERR_SHAPE;
    const double mean_rank = (double)S * (double)K;
    if (rank_before) *rank_before = (double)stats->max_load / mean_rank - 1.0;
    if (rank_after) *rank_after = (double)stats->max_chunk / mean_rank - 1.0;
    if (expert)
        *expert = stats->n_kept > 0 ? (double)stats->max_hist / ((double)stats->n_kept / (double)n_keys) - 1.0
                                    : std::nan("");
    return MEP_OK;
}

}  // extern "C"


// ------------------------------------------------------------------------------------
// mep_plan with scratch compiled into the library, for callers that cannot allocate.

// The scratch: one copy on every device that loads this library, for the life of the
// process. In host code this name is only a stand-in for the symbol; the device address
// comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_plan_static_ws[MEP_PLAN_STATIC_WS_BYTES];

namespace {
// With the context that owns the address current (device_state calls it at set-up).
cudaError_t plan_static_ws_lookup(void **addr) { return cudaGetSymbolAddress(addr, g_plan_static_ws); }
}  // namespace

extern "C" mep_status_t mep_plan_static_ws(const int32_t *ids, const uint8_t *keep, int32_t R,
                                           int32_t n_keys, int32_t S, int32_t K, int32_t mode,
                                           int32_t keys_per_rank, int32_t *pos, int32_t *hist,
                                           int32_t *rank_off, int32_t *load, int32_t *rep_count,
                                           int32_t *rep_key, int32_t *rep_cu,
                                           mep_plan_stats_t *stats, mep_stream_t stream)
{
    // mep_plan's own argument checks first, then the size of the array
    const mep_status_t st = plan_args(ids, keep, R, n_keys, S, K, mode, keys_per_rank, pos, hist, rank_off,
                                      rep_count, rep_key, rep_cu, stats);
    if (st != MEP_OK) return st;
    if (mep_plan_workspace_size(R, n_keys, S, K) > (size_t)MEP_PLAN_STATIC_WS_BYTES) return MEP_ERR_WORKSPACE;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        t_last_cuda_error = (int32_t)e;
        return MEP_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return MEP_ERR_VALUE;
    // the address in the current context: looked up at the context's set-up, again
    // after a device reset or under another context
    void *ws = device_state(dev).plan_static_ws;
    if (!ws) {
        t_last_cuda_error = (int32_t)cudaErrorInvalidSymbol;
        return MEP_ERR_CUDA;
    }
    return mep_plan(ids, keep, R, n_keys, S, K, mode, keys_per_rank, pos, hist, rank_off, load,
                    rep_count, rep_key, rep_cu, stats, ws, (size_t)MEP_PLAN_STATIC_WS_BYTES, stream);
}
