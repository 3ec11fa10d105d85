/*
 * mep.h — C ABI of libmep: MoE expert-parallel token routing on one B200 (sm_100a).
 *
 * The path: a per-expert histogram of the top-K expert ids, a perfectly balanced
 * placement plan (every one of R ranks receives exactly S*K token-slots; experts that
 * straddle a rank boundary get temporary redundant replicas), the logical->physical
 * expert mapping with score-threshold pruning, and dispatch / combine of bf16 hidden
 * rows. The R expert-parallel ranks are R partitions of one GPU's memory: rank r's
 * receive buffer is rows [rank_off[r], rank_off[r+1]) of one [rows, H] array.
 *
 * Conventions for every call
 *  - Pointers named in a signature are DEVICE pointers owned by the caller unless the
 *    comment says otherwise; the library keeps no reference after the call returns
 *    and allocates no device memory. Scratch memory comes from the caller through a
 *    workspace argument whose size a *_workspace_size query returns (the two-phase
 *    "query the workspace size, then execute on a stream" pattern of the aclnn
 *    interfaces, gitcode ops-transformer aclnnMoeUpdateExpert doc, 函数原型).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and never synchronise the host, so a chain plan -> dispatch -> combine
 *    needs no host round trip (MoonEP's static shapes remove per-layer host syncs:
 *    twodots.gr article on MoonEP, static-shapes paragraph). Three calls wait:
 *    mep_get_error waits for its `stream` (and that stream only);
 *    mep_stream_synchronize_timeout waits for its `stream` with a time limit; and
 *    mep_route_host's copies are synchronous when its host buffers are pageable.
 *    No call synchronises the whole device. mep_histogram, mep_plan, mep_plan_rank,
 *    mep_dispatch_ranks, mep_combine_ranks,
 *    mep_update_expert, mep_update_expert_ranks, mep_dedup_plan, mep_dispatch,
 *    mep_expand, mep_dispatch_int8_smooth, mep_dispatch_int8_smooth_grouped,
 *    mep_dequantize, mep_combine,
 *    mep_combine_int8, mep_combine_add_rmsnorm, mep_prefetch_plan, mep_prefetch_weights
 *    and mep_grad_reduce can be captured into a CUDA graph and replayed on new inputs,
 *    once each has been called eagerly in the current context (the first call in a
 *    context sets kernel attributes).
 *  - A call first checks its arguments on the host and returns a status without
 *    launching anything when one is wrong: MEP_ERR_NULLPTR / MEP_ERR_DTYPE /
 *    MEP_ERR_SHAPE / MEP_ERR_VALUE mirror the aclnn codes 161001 (null tensor),
 *    161002 (unsupported data type) and 561002 (shape or value out of range) of the
 *    aclnnMoeUpdateExpert doc (返回值).
 *  - Errors that depend on the data (an expert id out of range, a malformed
 *    eplb_table row, an active mask with a true after a false, a row index outside
 *    the receive buffer) cannot be seen on the host. The kernels then skip the
 *    offending element (never touching memory outside the buffers) and set a bit in a
 *    sticky per-device error word that mep_get_error reads. Nothing traps.
 *  - bf16 data is passed as its 16-bit patterns (uint16_t); int8 codes as int8_t.
 *  - Receive buffers are overwritten by the next dispatch; views into them must not
 *    outlive it (the zero-copy lifetime rule of MoonEP, twodots.gr article on
 *    MoonEP, zero-copy views paragraph).
 *
 * Notation: global token g = src*S + t, slot n = g*K + k, N = R*S*K, T = R*S;
 * home(e) = e / (E/R).
 */
#ifndef MEP_H
#define MEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *mep_stream_t; /* a cudaStream_t */

typedef enum {
    MEP_OK = 0,
    MEP_ERR_NULLPTR = 1,   /* a required pointer is NULL (cf. aclnn 161001) */
    MEP_ERR_DTYPE = 2,     /* unsupported element type or quantisation mode (cf. 161002) */
    MEP_ERR_SHAPE = 3,     /* a size outside the supported range (cf. 561002) */
    MEP_ERR_VALUE = 4,     /* an argument value outside its range (cf. 561002) */
    MEP_ERR_WORKSPACE = 5, /* workspace NULL, too small or not 256-byte aligned */
    MEP_ERR_CUDA = 6,      /* a CUDA call failed; the CUDA error is in mep_last_cuda_error() */
    MEP_ERR_TIMEOUT = 7    /* mep_stream_synchronize_timeout: the work did not finish in time */
} mep_status_t;

/* Bits of the device error word (see mep_get_error). */
#define MEP_DERR_KEY_RANGE 0x1  /* an expert / instance id outside [0, n_keys) */
#define MEP_DERR_ROW_RANGE 0x2  /* a slot row outside [-1, rows) */
#define MEP_DERR_TABLE     0x4  /* eplb_table: count outside [1, F-1] or instance id outside [0, 1024) */
#define MEP_DERR_MASK      0x8  /* active_mask has a true after a false */
#define MEP_DERR_TIMEOUT   0x10 /* a bounded wait inside a kernel ran out; that kernel stopped early */
#define MEP_DERR_DRAIN     0x20 /* after such a time-out, waiting for the kernel's own copies in flight
                                   ran out as well */
#define MEP_DERR_HIST      0x40 /* mep_plan_rank: the gathered histogram row of this rank differs from
                                   the histogram of its ids (the ranks' inputs disagree) */

/* Plan modes. */
#define MEP_PLAN_BALANCED 0
#define MEP_PLAN_GROUPED  1

/* Limits. */
#define MEP_MAX_KEYS 4096   /* experts (balanced) or physical instances (grouped) */
#define MEP_MAX_K    32     /* experts per token in dispatch / combine / plan */

/* Plan summary, written by mep_plan to device memory. All counts are exact integers;
 * maxvio = max_load / (S*K) - 1 (before planning) and max_chunk / (S*K) - 1 (after)
 * follow from it on the host, in double precision (mep_maxvio). */
typedef struct {
    int32_t max_load;   /* max over ranks of the rows its home experts would receive */
    int32_t max_chunk;  /* max over ranks of the rows it receives under the plan */
    int32_t redundant;  /* sum over experts of (#ranks holding a replica - 1) */
    int32_t prefetched; /* #(rank, expert) replicas placed on a rank other than home(e) */
    int32_t n_kept;     /* slots placed (N minus dropped slots) */
    int32_t max_hist;   /* max over keys of hist (expert-level load) */
    int32_t n_ranks_used; /* ranks that receive at least one row */
    int32_t reserved;
} mep_plan_stats_t;

/*
 * maxvio of a plan (MoonEP article, maxvio paragraph: the maximum load over the mean
 * load, minus one), from the plan summary copied to host memory:
 *   rank_before = max_load / (S*K) - 1    (every expert on its home rank)
 *   rank_after  = max_chunk / (S*K) - 1   (the rows each rank receives; 0 when balanced)
 *   expert      = max_hist / (n_kept / n_keys) - 1   (NaN when n_kept is 0)
 * in double precision. Host only: no device call, no stream. Any output may be NULL.
 * Errors: NULL stats (MEP_ERR_NULLPTR); S, K or n_keys below 1 (MEP_ERR_SHAPE).
 */
mep_status_t mep_maxvio(const mep_plan_stats_t *stats, int32_t S, int32_t K, int32_t n_keys,
                        double *rank_before, double *rank_after, double *expert);

/* Library version, (major << 16) | minor. */
int32_t mep_version(void);

/* Human-readable name of a status code (static string). */
const char *mep_status_string(mep_status_t status);

/* The cudaError_t of the last call that returned MEP_ERR_CUDA on this host thread. */
int32_t mep_last_cuda_error(void);

/*
 * Reads the sticky error word of the CURRENT device into *code (a host pointer; 0 = no
 * data error since the last clear), in stream order: the read is enqueued on `stream`
 * (a stream of the current device) and the call waits for that stream only, so it sees
 * every kernel enqueued on `stream` before it. Work on other streams that has not
 * finished may set bits later. With clear != 0 the bits it returns are cleared, also in
 * stream order; a bit that work on another stream sets meanwhile stays set. The word is
 * one per device, shared by all streams: which stream's kernel set a bit cannot be told
 * apart (read it after each stream's work, or keep one stream per job).
 * (The aclnn calls report in the same two steps: the call's status on the host, then the
 * stream's result after a stream synchronisation; gitcode ops-transformer
 * aclnnMoeUpdateExpert doc, 调用示例.)
 * Errors: NULL code (MEP_ERR_NULLPTR); a failed copy or synchronisation (MEP_ERR_CUDA).
 */
mep_status_t mep_get_error(mep_stream_t stream, int32_t *code, int32_t clear);

/*
 * a1 — per-expert histogram (tokens per expert: twodots.gr article on MoonEP, "six
 * checks before trying MoonEP": measure tokens per expert and maxvio).
 *   hist[e] = #{ i in [0,n) : ids[i] == e },  e in [0, n_keys).
 * ids: int32 [n]; hist: int32 [n_keys] (overwritten). Ids outside [0, n_keys) are not
 * counted and set MEP_DERR_KEY_RANGE.
 * Errors: NULL pointer (MEP_ERR_NULLPTR); n < 0, n >= 2^31, n_keys outside
 * [1, MEP_MAX_KEYS] (MEP_ERR_SHAPE).
 */
mep_status_t mep_histogram(const int32_t *ids, int64_t n, int32_t n_keys, int32_t *hist,
                           mep_stream_t stream);

/* Bytes of workspace mep_plan needs for N = R*S*K slots and n_keys keys. */
size_t mep_plan_workspace_size(int32_t R, int32_t n_keys, int32_t S, int32_t K);

/* Kernels mep_plan launches for this shape: 1 when the whole plan runs in one launch
 * (at most 16384 slots and few enough keys for shared memory: a cluster of CTAs, or one
 * CTA), 3 otherwise (the tiled sort, whose scan also writes the replica tables); 0 for a
 * shape below 1. For launch accounting; host only. */
int32_t mep_plan_launches(int32_t R, int32_t n_keys, int32_t S, int32_t K);

/*
 * a2 — placement plan: the row of every slot in the R ranks' receive buffers.
 *
 * MEP_PLAN_BALANCED (keys = logical experts, n_keys = E, E % R == 0, keep == NULL):
 *   the perfectly balanced plan of MoonEP (twodots.gr article on MoonEP: every rank
 *   processes exactly S*K token-slots; a few temporary redundant replicas of hot
 *   experts absorb the skew). Slots are ordered by (home(e), e, src, t, k) and the
 *   ordered list is cut into R chunks of S*K rows; rank r receives rows
 *   [r*S*K, (r+1)*S*K). An expert whose rows straddle a cut has a replica on every
 *   rank it reaches. Because home(e) is monotone in e and the slot index orders
 *   (src, t, k), the row of slot n is  off[e] + #{m < n : ids[m] == e}  with off the
 *   exclusive prefix sum of hist: a stable counting sort.
 * MEP_PLAN_GROUPED (keys = physical instance ids after mep_update_expert,
 *   n_keys = R * keys_per_rank, keep optional): every kept slot goes to the rank that
 *   hosts its instance, rank = key / keys_per_rank; rows are ordered by (key, slot)
 *   and packed, rank r owning rows [rank_off[r], rank_off[r+1]); dropped slots
 *   (keep[n] == 0) get pos = -1. (Receive layout of aclnnMoeDistributeDispatch after
 *   the aclnnMoeUpdateExpert mapping, gitcode ops-transformer doc, 调用示例.)
 *
 * Inputs:  ids int32 [N] (slot n = (src*S + t)*K + k); keep uint8 [N] or NULL.
 * Outputs (all device, overwritten):
 *   pos       int32 [N]           row of every slot, -1 = dropped
 *   hist      int32 [n_keys]      slots per key (kept slots only)
 *   rank_off  int32 [R+1]         first row of every rank, rank_off[R] = n_kept
 *   load      int32 [R] or NULL   rows rank r would receive if no expert moved:
 *                                 sum of hist over its home keys
 *   rep_count int32 [R]           replicas (distinct keys) on each rank
 *   rep_key   int32 [R, n_keys]   the keys of rank r's replicas, ascending; -1 after
 *                                 rep_count[r]
 *   rep_cu    int32 [R, n_keys+1] cu_seqlens of rank r's replicas relative to
 *                                 rank_off[r] (the grouped-GEMM offsets MoonEP's
 *                                 planner produces); 0 after rep_count[r]
 *   stats     mep_plan_stats_t [1]
 * Workspace: at least mep_plan_workspace_size(R, n_keys, S, K) bytes, 256-byte aligned,
 * caller-owned scratch (no contents needed on entry); calls in flight at the same time
 * need workspaces of their own.
 * Errors: NULL pointer; R, S, K < 1, K > MEP_MAX_K, N >= 2^31, n_keys outside
 * [1, MEP_MAX_KEYS] (MEP_ERR_SHAPE); mode unknown, E % R != 0, keep given in
 * balanced mode, keys_per_rank * R != n_keys in grouped mode (MEP_ERR_VALUE);
 * workspace too small (MEP_ERR_WORKSPACE). Ids outside [0, n_keys) are dropped
 * (pos = -1) and set MEP_DERR_KEY_RANGE.
 */
mep_status_t mep_plan(const int32_t *ids, const uint8_t *keep, int32_t R, int32_t n_keys,
                      int32_t S, int32_t K, int32_t mode, int32_t keys_per_rank,
                      int32_t *pos, int32_t *hist, int32_t *rank_off, int32_t *load,
                      int32_t *rep_count, int32_t *rep_key, int32_t *rep_cu,
                      mep_plan_stats_t *stats, void *workspace, size_t workspace_bytes,
                      mep_stream_t stream);

/*
 * (e) — one expert-parallel rank's share of the balanced plan, for the layout in which
 * every GPU is one EP rank holding its own S tokens (MoonEP zero-copy dispatch: every
 * token row is written straight to its final, expert-grouped row on the destination
 * rank; twodots.gr article on MoonEP, zero-copy paragraph). Each rank computes its
 * per-expert histogram (mep_histogram of its own ids), the ranks all-gather them into
 * hist_all, and each rank then places its own slots exactly where mep_plan over the
 * ids of all ranks would: the plan orders slots by (e, src, t, k), so
 *   pos[n] = off[e] + sum_{r < rank} hist_all[r, e] + #{m < n : ids[m] == e}
 * for this rank's slot n = t*K + k with expert e, off the exclusive prefix over experts
 * of sum_r hist_all[r, e]. Row p belongs to destination rank p / (S*K), at local row
 * p mod (S*K) of its receive buffer.
 * Inputs:  ids int32 [S*K] (this rank's slots); hist_all int32 [R, E] (row r = rank r's
 *          histogram, the same on every rank); rank in [0, R).
 * Outputs (device, overwritten):
 *   pos        int32 [S*K]  global row of every slot of this rank
 *   send_count int32 [R]    rows this rank writes into rank d's partition
 *   send_off   int32 [R+1]  exclusive prefix of send_count (a send buffer packed by
 *                           destination: slots in ascending pos)
 *   recv_count int32 [R]    rows rank s writes into this rank's partition
 *   recv_off   int32 [R+1]  exclusive prefix of recv_count; recv_off[R] = S*K
 * Workspace: mep_plan_rank_workspace_size(R, E, S, K) bytes, 256-byte aligned.
 * Errors: NULL pointer; R, S, K < 1, K > MEP_MAX_K, E outside [1, MEP_MAX_KEYS],
 * R > MEP_MAX_KEYS, R*S*K >= 2^31 (MEP_ERR_SHAPE); E % R != 0, rank outside [0, R)
 * (MEP_ERR_VALUE); workspace (MEP_ERR_WORKSPACE). Data errors: ids outside [0, E)
 * (dropped, pos = -1, MEP_DERR_KEY_RANGE); row `rank` of hist_all differs from the
 * histogram of ids (MEP_DERR_HIST: the ranks' inputs disagree, the rows are not a plan).
 */
size_t mep_plan_rank_workspace_size(int32_t R, int32_t E, int32_t S, int32_t K);
mep_status_t mep_plan_rank(const int32_t *ids, const int32_t *hist_all, int32_t R, int32_t E,
                           int32_t S, int32_t K, int32_t rank, int32_t *pos, int32_t *send_count,
                           int32_t *send_off, int32_t *recv_count, int32_t *recv_off,
                           void *workspace, size_t workspace_bytes, mep_stream_t stream);

/*
 * (e) — dispatch and combine when every EP rank's receive buffer is its own allocation:
 * on several GPUs, the other ranks' buffers as peer mappings (NVLink), so that the
 * dispatch stores every token row straight into its final, expert-grouped row on the
 * destination rank (MoonEP zero-copy dispatch: twodots.gr article on MoonEP, zero-copy
 * paragraph) and the combine loads the expert outputs back from where they are. The
 * global row p = pos[n] (from mep_plan or mep_plan_rank) lives on rank
 * d = p / rows_per_rank at local row p mod rows_per_rank.
 *   mep_dispatch_ranks:  recv_ptrs[d][local, :] = x[n / K, :]      (quant 0, bf16)
 *                        or the int8 codes and scale of mep_dispatch quant 1, the scale
 *                        at scale_ptrs[d][local]
 *   mep_combine_ranks:   out[g, :] = the sum of mep_combine (quant 0) or mep_combine_int8
 *                        (quant 1) over rows y_ptrs[d][local, :] (scales scale_ptrs[d][local])
 * recv_ptrs / y_ptrs / scale_ptrs are DEVICE arrays of R pointers (8-byte aligned), each
 * a rank's buffer [rows_per_rank, H] (bf16 or int8) or its scales [rows_per_rank] fp32;
 * buffers 16-byte aligned (int8 dispatch: 8), scales 4-byte aligned. The calls only
 * store to and load from these buffers with plain 16- or 8-byte accesses; they wait on
 * nothing, so the caller orders them against the other ranks' use of the buffers
 * (a barrier between the exchange and the experts, as for any all-to-all).
 * x bf16 [T, H] 16-byte aligned; pos int32 [T*K]; gates fp32 [T*K]; out bf16 [T, H]
 * 16-byte aligned.
 * Errors: quant outside {0,1} (MEP_ERR_DTYPE); NULL pointer (MEP_ERR_NULLPTR); T < 0, K
 * outside [1, MEP_MAX_K], H not a positive multiple of 8 (combine of int8 rows: of 16),
 * R outside [1, MEP_MAX_KEYS], rows_per_rank < 1, T*K or R*rows_per_rank >= 2^31
 * (MEP_ERR_SHAPE); x, out or the pointer arrays misaligned (MEP_ERR_VALUE). Data errors:
 * a pos outside [-1, R*rows_per_rank), or a rank whose table entry is NULL or
 * misaligned, skips the slot and sets MEP_DERR_ROW_RANGE.
 */
mep_status_t mep_dispatch_ranks(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K, int64_t H,
                                int32_t quant, void *const *recv_ptrs, float *const *scale_ptrs, int32_t R,
                                int64_t rows_per_rank, mep_stream_t stream);
mep_status_t mep_combine_ranks(const void *const *y_ptrs, const float *const *scale_ptrs, int32_t quant,
                               int32_t R, int64_t rows_per_rank, const int32_t *pos, const float *gates,
                               int64_t T, int32_t K, int64_t H, uint16_t *out, mep_stream_t stream);

/*
 * a5 with int8 rows (quantised return path) — combine of per-row int8 codes with one
 * fp32 scale per row, as when the rows coming back to the token's rank are quantised
 * for the exchange (commQuantMode of aclnnMoeDistributeCombineV2, gitcode
 * ops-transformer aclnnMoeUpdateExpert doc, 调用示例):
 *   out[g, h] = bf16_rne( sum over kept k, ascending, of
 *                         fl(gates[g*K+k] * bf16_rne(fl(float(yq[p, h]) * y_scale[p]))) ),
 *   p = pos[g*K+k]
 * i.e. exactly mep_dequantize followed by mep_combine, without writing the bf16 rows:
 * it reads H bytes per kept slot instead of 2H.
 * yq int8 [rows, H]; y_scale fp32 [rows]; pos int32 [T*K]; gates fp32 [T*K];
 * out bf16 [T, H]. Errors and data errors as mep_combine.
 */
mep_status_t mep_combine_int8(const int8_t *yq, const float *y_scale, int64_t rows,
                              const int32_t *pos, const float *gates, int64_t T, int32_t K,
                              int64_t H, uint16_t *out, mep_stream_t stream);

/*
 * f1 — int8 dispatch with per-expert smoothing scales (the optional scales of shape
 * (moeExpertNum, H), fp32, that aclnnMoeDistributeDispatch takes when quantMode > 0:
 * gitcode ops-transformer aclnnMoeUpdateExpert doc, 调用示例; hiascend
 * aclnnMoeDistributeDispatchSetup doc, scalesOptional). For every kept slot n of token
 * g with expert e = ids[n] (the expert id the smoothing row belongs to):
 *   xs_h  = fl(float(x[g, h]) * smooth[e, h]),   amax = max_h |xs_h|,
 *   scale = amax / 127,   q_h = clamp(round_half_even(xs_h / scale), -127, 127)
 *   (q = 0 when amax == 0);   recv[pos[n], :] = q,   recv_scale[pos[n]] = scale.
 * Unlike mep_dispatch with quant 1, codes and scale are per slot (the smoothing depends
 * on the expert). x bf16 [T, H]; ids int32 [T*K]; pos int32 [T*K]; smooth fp32
 * [n_experts, H]; recv int8 [rows, H]; recv_scale fp32 [rows].
 * Errors: NULL pointer; T < 0, K outside [1, MEP_MAX_K], H < 1, rows < 0, n_experts < 1
 * (MEP_ERR_SHAPE). An id outside [0, n_experts) skips the slot and sets
 * MEP_DERR_KEY_RANGE; a pos outside [-1, rows) as mep_dispatch.
 */
mep_status_t mep_dispatch_int8_smooth(const uint16_t *x, const int32_t *ids, const int32_t *pos,
                                      int64_t T, int32_t K, int64_t H, const float *smooth,
                                      int32_t n_experts, int8_t *recv, float *recv_scale,
                                      int64_t rows, mep_stream_t stream);

/*
 * f1 smoothing, the same codes and scales as mep_dispatch_int8_smooth, with the slots
 * taken in expert order: a first kernel sorts the slot indices by expert within chunks
 * of about 2048 slots (the list goes into the workspace), a second quantises the slots
 * along that list, so that each smoothing row is read once for a run of slots of its
 * expert instead of twice per slot, while the chunk's token rows stay in L2.
 * Arguments as mep_dispatch_int8_smooth, plus the caller-owned workspace (no contents
 * needed on entry; calls in flight at the same time need workspaces of their own) of at
 * least mep_dispatch_int8_smooth_workspace_size(T, K) bytes, 256-byte aligned (NULL
 * allowed when that size is 0). Shapes the sorted path does not take (H % 4 != 0,
 * unaligned x / recv / smooth, H > 8192, n_experts > 6000) run the kernels of
 * mep_dispatch_int8_smooth instead, with the same results.
 * Errors: those of mep_dispatch_int8_smooth; MEP_ERR_WORKSPACE.
 */
size_t mep_dispatch_int8_smooth_workspace_size(int64_t T, int32_t K);
mep_status_t mep_dispatch_int8_smooth_grouped(const uint16_t *x, const int32_t *ids, const int32_t *pos,
                                              int64_t T, int32_t K, int64_t H, const float *smooth,
                                              int32_t n_experts, int8_t *recv, float *recv_scale,
                                              int64_t rows, void *workspace, size_t workspace_bytes,
                                              mep_stream_t stream);

/* Largest hidden size of mep_combine_add_rmsnorm (one fp32 row in shared memory). */
#define MEP_RMSNORM_MAX_H 49152

/*
 * f4 — combine fused with residual add and RMSNorm (aclnnMoeDistributeCombineAddRmsNorm:
 * residualX (BS,1,H), gamma (H,), yOut (BS,1,H), rstdOut (BS,1,1), xOut (BS,1,H);
 * gitcode ops-transformer aclnnMoeUpdateExpert doc, 调用示例). The page names the
 * arguments but not the formula; this is the plain add-then-RMSNorm reading. For every
 * token g, with c_h = the combine output of mep_combine (bf16):
 *   x_h      = fl(c_h + residual_h)                      (fp32)
 *   x_out_h  = bf16_rne(x_h)
 *   rstd     = rsqrt_rn(fl(fl(sum_h x_h^2) / H) + eps)   (fp32; the sum's order is the
 *                                                          kernel's, not fixed)
 *   y_out_h  = bf16_rne(fl(fl(x_h * rstd) * gamma_h))
 * x_out is exact (the sum c + residual rounded once to bf16); y_out and rstd carry the
 * rounding of an fp32 sum of H squares: within 1 bf16 ulp (y_out) and a relative
 * ((H+3)/2 + 2) * 2^-24 (rstd) of the exact values.
 * y bf16 [rows, H]; pos int32 [T*K]; gates fp32 [T*K]; residual bf16 [T, H]; gamma bf16
 * [H]; x_out, y_out bf16 [T, H]; rstd_out fp32 [T].
 * Errors: NULL pointer; T < 0, K outside [1, MEP_MAX_K], H outside [1, MEP_RMSNORM_MAX_H],
 * rows < 0 (MEP_ERR_SHAPE); eps negative or not finite (MEP_ERR_VALUE). Data errors as
 * mep_combine.
 */
mep_status_t mep_combine_add_rmsnorm(const uint16_t *y, int64_t rows, const int32_t *pos,
                                     const float *gates, int64_t T, int32_t K, int64_t H,
                                     const uint16_t *residual, const uint16_t *gamma, float eps,
                                     uint16_t *x_out, uint16_t *y_out, float *rstd_out,
                                     mep_stream_t stream);

/* Most prefetch slots over all ranks (R * B) of the prefetch and grad-reduce calls. */
#define MEP_MAX_SLOTS 65535

/*
 * f2 — replica weight prefetch: where every replica of the plan reads its expert's
 * weights (MoonEP memory contract; twodots.gr article on MoonEP: weights [E+B, H, H'],
 * rows 0..E-1 the ranks' own experts, rows E..E+B-1 per-rank prefetch slots; B = E/R
 * for training, 3-4 for inference; a rank with more remote experts than slots reads the
 * rest from their home rank). On one GPU the weights are one array of E + R*B rows:
 * rows [0, E) the home experts (expert e at row e, on rank e / (E/R)), rows E + r*B + b
 * rank r's slots.
 * mep_prefetch_plan walks each rank's replicas (rep_count, rep_key from mep_plan) in
 * order: a replica of an expert homed elsewhere takes the rank's next free slot while
 * slots remain (slot_expert[r, b] = e, rep_weight = E + r*B + b), otherwise it reads
 * the home row e; home replicas read row e.
 * rep_count int32 [R]; rep_key int32 [R, cap]; outputs slot_expert int32 [R, B]
 * (-1 = unused) and rep_weight int32 [R, cap] (-1 past rep_count).
 * Errors: NULL pointer; R, E or cap outside [1, MEP_MAX_KEYS], B < 0, R*B > MEP_MAX_SLOTS
 * (MEP_ERR_SHAPE); E % R != 0 (MEP_ERR_VALUE). A count or key out of range sets
 * MEP_DERR_KEY_RANGE.
 */
mep_status_t mep_prefetch_plan(const int32_t *rep_count, const int32_t *rep_key, int32_t R,
                               int32_t E, int32_t cap, int32_t B, int32_t *slot_expert,
                               int32_t *rep_weight, mep_stream_t stream);

/*
 * f2 — the prefetch copy: w_slots[s, :] = w_home[slot_expert[s], :] for every used slot
 * s of the R*B slots (unused slots are left as they are). D bf16 elements per expert
 * (H * H'). w_home bf16 [E, D]; slot_expert int32 [R*B]; w_slots bf16 [R*B, D].
 * Errors: NULL pointer; E < 1, R < 1, B < 0, D < 1, R*B > MEP_MAX_SLOTS (MEP_ERR_SHAPE).
 * A slot expert >= E is skipped and sets MEP_DERR_KEY_RANGE.
 */
mep_status_t mep_prefetch_weights(const uint16_t *w_home, const int32_t *slot_expert, int32_t E,
                                  int32_t R, int32_t B, int64_t D, uint16_t *w_slots,
                                  mep_stream_t stream);

/*
 * f3 — replica gradient reduce (MoonEP: the gradients of prefetched copies go to a
 * separate reduce buffer [R, B, H, H']; the home rank reads the slots of its experts,
 * adds them into its parameter gradient and clears them before the next microbatch).
 * For every expert e and element i, in fp32, over the slots s with slot_expert[s] == e
 * in ascending s (rank, then slot):
 *   grad_home[e, i] = (...(grad_home[e, i] + grad_slots[s0, i]) + grad_slots[s1, i]) ...
 * then those slots are set to zero. Unused slots are left as they are.
 * grad_home fp32 [E, D]; grad_slots fp32 [R*B, D]; slot_expert int32 [R*B].
 * Errors: NULL pointer; E outside [1, 65535], R < 1, B < 0, D < 1, R*B > MEP_MAX_SLOTS
 * (MEP_ERR_SHAPE). More than 1024 slots holding one expert sets MEP_DERR_KEY_RANGE
 * (only the first 1024 are added).
 */
mep_status_t mep_grad_reduce(float *grad_home, float *grad_slots, const int32_t *slot_expert,
                             int32_t E, int32_t R, int32_t B, int64_t D, mep_stream_t stream);

/*
 * Waits for the work enqueued on `stream` with a time limit: the timeout-bounded stream
 * synchronisation of the aclnnMoeUpdateExpert doc's sample (调用示例,
 * aclrtSynchronizeStreamWithTimeout(stream, 10000)). Polls the stream about every 50 us.
 * Returns MEP_OK once the work has finished; MEP_ERR_TIMEOUT when it is still running
 * after timeout_ms milliseconds (nothing is cancelled: the work keeps running, and a
 * later call may still see it finish); MEP_ERR_CUDA when the stream reports an error
 * (the CUDA error is in mep_last_cuda_error()). timeout_ms < 0 is MEP_ERR_VALUE.
 */
mep_status_t mep_stream_synchronize_timeout(mep_stream_t stream, int32_t timeout_ms);

/*
 * Diagnostic: checks the failure path of the kernels' bounded waits on this GPU.
 * Launches one CTA that waits, with the same bounded mbarrier wait the staged int8
 * dispatch uses, on a barrier that nothing ever completes. After max_polls polls
 * (1 .. 2^22; each poll backs off ~64 ns) the wait gives up, the kernel sets
 * MEP_DERR_TIMEOUT in the device error word, writes 1 to *timed_out (a device int32)
 * and returns; the context stays usable. Nothing waits without a bound, so this call
 * cannot hang. Errors: NULL timed_out (MEP_ERR_NULLPTR), max_polls out of range
 * (MEP_ERR_VALUE).
 */
mep_status_t mep_selftest_bounded_wait(int32_t max_polls, int32_t *timed_out, mep_stream_t stream);

/* Size of the scratch array compiled into libmep for mep_plan_static_ws: 4 MiB. */
#define MEP_PLAN_STATIC_WS_BYTES (4u << 20)

/*
 * mep_plan for callers that cannot allocate device memory. The paper has no
 * counterpart to this entry point; it exists for users of this library.
 *
 * Who needs it: code that must not call cudaMalloc at the point where it plans, such
 * as a program whose device memory is all owned by another allocator (a caching
 * allocator or a fixed pool that a stray cudaMalloc would overdraw or fragment), a
 * serving loop in which cudaMalloc / cudaFree could stall the device, or a plain C
 * program that links libmep and has no allocator of its own for scratch.
 *
 * Arguments, outputs and results are exactly those of mep_plan, minus the workspace:
 * the scratch is a file-scope device array of MEP_PLAN_STATIC_WS_BYTES inside libmep,
 * which every GPU that loads the library holds until the process exits. Inputs and
 * outputs are still the caller's. This call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * Set-up: the first call of the library in a CUDA context (the device's primary
 * context, or a context the caller made current) looks up the array's device address
 * with cudaGetSymbolAddress, with that context current, and keeps it for that context;
 * after cudaDeviceReset, or under another context, the next call looks it up again.
 * Make the first call in a context before any stream capture.
 * Sharing: all calls on a device use the same array, which keeps the contents of the
 * last call. The plan kernels write every scratch word before they read it, so nothing
 * has to be cleared between calls. Calls that overlap on the GPU (unordered streams)
 * race on the array and produce wrong plans: order them.
 * Limit: plans whose mep_plan_workspace_size(R, n_keys, S, K) is at most
 * MEP_PLAN_STATIC_WS_BYTES, for instance up to 2,097,152 slots with up to 1024 keys.
 * Errors: those of mep_plan; MEP_ERR_WORKSPACE for a plan larger than the array;
 * MEP_ERR_CUDA if the address lookup fails.
 */
mep_status_t mep_plan_static_ws(const int32_t *ids, const uint8_t *keep, int32_t R,
                                int32_t n_keys, int32_t S, int32_t K, int32_t mode,
                                int32_t keys_per_rank, int32_t *pos, int32_t *hist,
                                int32_t *rank_off, int32_t *load, int32_t *rep_count,
                                int32_t *rep_key, int32_t *rep_cu, mep_plan_stats_t *stats,
                                mep_stream_t stream);

/*
 * a3 — logical->physical expert mapping and score-threshold pruning
 * (aclnnMoeUpdateExpert, gitcode ops-transformer doc, 功能说明 / 参数说明).
 *
 * For slot (i, k), e = expert_ids[i,k], c = eplb_table[e, 0] (instances of e):
 *   c == 1            -> balanced_expert_ids[i,k] = eplb_table[e, 1]
 *   balance_mode 0    -> eplb_table[e, local_rank_id / ceil(world_size / c) + 1]  (by rank)
 *   balance_mode 1    -> eplb_table[e, (i mod c) + 1]                             (by token)
 * (ceil is a true ceiling; i is the token index.)
 * Pruning: v_i = sum_k fl(expert_scales[i,k] * pruning_threshold[k]) accumulated in
 * fp32 in ascending k; balanced_active_mask[i,k] = active_mask[i] &&
 * !(expert_scales[i,k] < v_i). Without scales and threshold the mask is
 * active_mask[i] broadcast over k (all 1 when active_mask is NULL too).
 *
 * expert_ids int32 [BS, K]; eplb_table int32 [n_experts, F] (column 0 = count in
 * [1, F-1], columns 1..count = distinct instance ids in [0, 1024)); expert_scales fp32
 * [BS, K] (descending within a token) or NULL; pruning_threshold fp32 [K] or NULL;
 * active_mask uint8 [BS] (every 1 before every 0) or NULL.
 * Outputs: balanced_expert_ids int32 [BS, K]; balanced_active_mask uint8 [BS, K].
 * Errors: NULL required pointer; scales without threshold or the reverse; a mask
 * without scales and threshold (MEP_ERR_NULLPTR, the doc's pairing rules);
 * BS < 1, K outside [1, 16], K > n_experts, n_experts outside [1, 1024], F outside
 * [2, world_size + 1] (MEP_ERR_SHAPE); balance_mode outside {0,1}, world_size outside
 * [2, 768] or local_rank_id outside [0, world_size) in mode 0 (MEP_ERR_VALUE).
 * The doc's BS <= 512 is a limit of the Ascend part and is not enforced.
 * Data errors: id out of range (MEP_DERR_KEY_RANGE, output -1), bad table row
 * (MEP_DERR_TABLE, output -1), mask order (MEP_DERR_MASK).
 */
mep_status_t mep_update_expert(const int32_t *expert_ids, const int32_t *eplb_table,
                               const float *expert_scales, const float *pruning_threshold,
                               const uint8_t *active_mask, int64_t BS, int32_t K,
                               int32_t n_experts, int32_t F, int64_t local_rank_id,
                               int64_t world_size, int64_t balance_mode,
                               int32_t *balanced_expert_ids, uint8_t *balanced_active_mask,
                               mep_stream_t stream);

/*
 * a3 for every simulated rank at once: the same mapping and pruning as
 * mep_update_expert, applied to the world_size ranks' tokens in one launch. Rows are
 * world_size blocks of BS tokens: row g belongs to rank r = g / BS (its local_rank_id)
 * and is that rank's token i = g % BS; the result equals world_size calls of
 * mep_update_expert, one per block.
 * expert_ids int32 [world_size*BS, K]; expert_scales fp32 [world_size*BS, K] or NULL;
 * active_mask uint8 [world_size*BS] or NULL (every 1 before every 0 within each rank's
 * block); other arguments, outputs and errors as mep_update_expert (without
 * local_rank_id).
 */
mep_status_t mep_update_expert_ranks(const int32_t *expert_ids, const int32_t *eplb_table,
                                     const float *expert_scales, const float *pruning_threshold,
                                     const uint8_t *active_mask, int64_t BS, int32_t K,
                                     int32_t n_experts, int32_t F, int64_t world_size,
                                     int64_t balance_mode, int32_t *balanced_expert_ids,
                                     uint8_t *balanced_active_mask, mep_stream_t stream);

/*
 * a4 — dispatch: every kept slot's token row written straight to its final row of the
 * receive buffer (MoonEP zero-copy dispatch: tokens land in their final,
 * expert-grouped positions; twodots.gr article on MoonEP, zero-copy paragraph).
 *   quant == 0:  recv[pos[n], :] = x[n / K, :]                  (bf16 copy)
 *   quant == 1:  per-token dynamic symmetric int8 (one fp32 scale per token, the
 *                dynamicScales output of aclnnMoeDistributeDispatch):
 *                amax = max_h |x[g,h]|, scale = amax / 127 (fp32 division),
 *                q = clamp(round_half_even(x / scale), -127, 127), q = 0 if amax == 0;
 *                recv[pos[n], :] = q (int8), recv_scale[pos[n]] = scale.
 * x bf16 [T, H]; pos int32 [T*K] (-1 = dropped); recv bf16 or int8 [rows, H];
 * recv_scale fp32 [rows] (quant == 1 only, else ignored). Rows no slot points at are
 * left untouched. For quant == 1 the row must be finite: a NaN or infinity in it leaves
 * that row's codes unspecified.
 * Errors: NULL pointer; T < 0, K outside [1, MEP_MAX_K], H < 1, rows < 0,
 * T*K >= 2^31 (MEP_ERR_SHAPE); quant outside {0,1} (MEP_ERR_DTYPE). A pos outside
 * [-1, rows) is skipped and sets MEP_DERR_ROW_RANGE.
 */
mep_status_t mep_dispatch(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K,
                          int64_t H, int32_t quant, void *recv, float *recv_scale,
                          int64_t rows, mep_stream_t stream);

/*
 * f1 — one dispatch row per (token, destination rank). The MoonEP API reference
 * (stapisi.com), section 5.2 on communication performance, names a bounds-checked
 * "dedup encoding". Reading: a token whose kept slots land on one destination rank
 * several times (several of its experts, or replicas, live there) crosses to that rank
 * once, and the rank expands it to its expert-grouped rows locally.
 *
 * From a plan (pos, rank_off of mep_plan, either mode): the destination rank of kept
 * slot n is the r with rank_off[r] <= pos[n] < rank_off[r+1]. Rank r's deduplicated
 * rows are [drank_off[r], drank_off[r+1]) and hold, in ascending global token order,
 * the tokens g with at least one kept slot on r. Outputs (device, overwritten):
 *   dsend     int32 [N]    row of the first slot of each (token, rank) pair, -1 for
 *                          every other slot: the send list (mep_dispatch(x, dsend, ...)
 *                          writes each pair's row once, bf16 or per-token int8; the
 *                          smoothing dispatch does not compose with it, its codes being
 *                          per slot)
 *   dpos      int32 [N]    row of every kept slot (shared by a pair's slots), -1 dropped
 *   drank_off int32 [R+1]  first row of every rank, drank_off[R] = the row count U
 *   dtok      int32 [N]    token of every row, -1 from U on
 *   gidx      int32 [N]    for every plan row p < rank_off[R], the row holding its token:
 *                          gidx[pos[n]] = dpos[n]; -1 elsewhere (mep_expand's index)
 * Bounds the encoding keeps: a rank's rows <= min(T, its plan rows); tokens with a kept
 * slot <= U <= kept slots.
 * Workspace: at least mep_dedup_workspace_size(R, S, K) bytes, 256-byte aligned.
 * Errors: NULL pointer; R, S, K < 1, K > MEP_MAX_K, R > MEP_MAX_KEYS, N >= 2^31
 * (MEP_ERR_SHAPE); workspace (MEP_ERR_WORKSPACE). A pos outside [-1, min(rank_off[R],
 * N)) counts as dropped and sets MEP_DERR_ROW_RANGE. rank_off must be non-decreasing
 * from 0 (as mep_plan writes it).
 */
size_t mep_dedup_workspace_size(int32_t R, int32_t S, int32_t K);
mep_status_t mep_dedup_plan(const int32_t *pos, const int32_t *rank_off, int32_t R, int32_t S, int32_t K,
                            int32_t *dsend, int32_t *dpos, int32_t *drank_off, int32_t *dtok, int32_t *gidx,
                            void *workspace, size_t workspace_bytes, mep_stream_t stream);

/*
 * f1 — expansion on the receiving rank: dst[p, :] = src[gidx[p], :] for every row p in
 * [0, rows) with gidx[p] >= 0 (other rows are left untouched); with quant == 1 also
 * dst_scale[p] = src_scale[gidx[p]]. After mep_dedup_plan and a dispatch with its send
 * list, this gives exactly the rows the plain dispatch writes.
 * quant 0: src, dst bf16 [.., H]; quant 1: int8 [.., H] with fp32 scales [..] (required).
 * src has src_rows rows; gidx int32 [rows].
 * Errors: quant outside {0,1} (MEP_ERR_DTYPE); rows, src_rows < 0, H < 1
 * (MEP_ERR_SHAPE); NULL pointer (MEP_ERR_NULLPTR). A gidx at or past src_rows is
 * skipped and sets MEP_DERR_ROW_RANGE.
 */
mep_status_t mep_expand(const void *src, const float *src_scale, int64_t src_rows, const int32_t *gidx,
                        int64_t rows, int64_t H, int32_t quant, void *dst, float *dst_scale,
                        mep_stream_t stream);

/*
 * Identity expert on int8 rows: y[r, h] = bf16_rne(fl(float(q[r,h]) * scale[r])).
 * Turns an int8 dispatch result back into bf16 rows for combine.
 * q int8 [rows, H]; scale fp32 [rows]; y bf16 [rows, H].
 * Errors: NULL pointer; rows < 0, H < 1 (MEP_ERR_SHAPE).
 */
mep_status_t mep_dequantize(const int8_t *q, const float *scale, int64_t rows, int64_t H,
                            uint16_t *y, mep_stream_t stream);

/*
 * a5 — combine: the K returned rows of every token weighted by its gates and summed
 * back in token order (aclnnMoeDistributeCombine: expandX rows weighted by
 * expertScales; gitcode ops-transformer aclnnMoeUpdateExpert doc, 调用示例).
 *   out[g, h] = bf16_rne( sum over k = 0..K-1 with pos[g*K+k] >= 0, in ascending k,
 *                         of fl(gates[g*K+k] * float(y[pos[g*K+k], h])) )
 * accumulated in fp32 starting from +0, each product and sum rounded on its own (no
 * fused multiply-add). A token with no kept slot gives a zero row.
 * y bf16 [rows, H]; pos int32 [T*K]; gates fp32 [T*K]; out bf16 [T, H].
 * Errors: NULL pointer; T < 0, K outside [1, MEP_MAX_K], H < 1, rows < 0,
 * T*K >= 2^31 (MEP_ERR_SHAPE). A pos outside [-1, rows) is treated as dropped and
 * sets MEP_DERR_ROW_RANGE.
 */
mep_status_t mep_combine(const uint16_t *y, int64_t rows, const int32_t *pos,
                         const float *gates, int64_t T, int32_t K, int64_t H, uint16_t *out,
                         mep_stream_t stream);

/*
 * One routing round trip of a batch that lives in host memory: upload, balanced plan,
 * dispatch, combine of the dispatched rows (the identity expert), download. This is the
 * composition mep_plan -> mep_dispatch -> mep_combine (or mep_combine_int8 for int8
 * rows) with its host<->device copies, all enqueued on `stream`; nothing synchronises.
 * With pinned (page-locked) host buffers the call returns at once and consecutive calls
 * on different streams with different buffer sets overlap their copies and kernels;
 * pageable host buffers make the copies synchronous. The device buffers are the
 * caller's (the call allocates nothing); they and the host buffers must not be touched
 * until the stream has passed the call.
 */
typedef struct {
    int32_t R, E, S, K;          /* ranks, experts (E % R == 0), tokens per rank, top-K */
    int64_t H;                   /* hidden size */
    int32_t quant;               /* 0: bf16 rows; 1: per-token int8 rows + scales */
    int32_t *ids;                /* [N] int32, N = R*S*K */
    float *gates;                /* [N] fp32 */
    uint16_t *x;                 /* [T, H] bf16, T = R*S */
    void *recv;                  /* [N, H] bf16 (quant 0) or int8 (quant 1) */
    float *recv_scale;           /* [N] fp32 (quant 1), else NULL */
    uint16_t *out;               /* [T, H] bf16 */
    int32_t *pos, *hist, *rank_off, *load, *rep_count, *rep_key, *rep_cu;   /* as mep_plan */
    mep_plan_stats_t *stats;
    void *workspace;             /* mep_plan_workspace_size(R, E, S, K) bytes, 256-aligned */
    size_t workspace_bytes;
} mep_route_buffers_t;

/*
 * ids_h int32 [N], gates_h fp32 [N], x_h bf16 [T, H] (host, read); out_h bf16 [T, H]
 * (host, written). Errors: NULL pointers (MEP_ERR_NULLPTR); quant outside {0,1}
 * (MEP_ERR_DTYPE); then whatever mep_plan, mep_dispatch or the combine return; a failed
 * copy (MEP_ERR_CUDA). Nothing after a failing step is enqueued.
 */
mep_status_t mep_route_host(const mep_route_buffers_t *dev, const int32_t *ids_h, const float *gates_h,
                            const uint16_t *x_h, uint16_t *out_h, mep_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MEP_H */
