/*
 * Oracle for MoE expert-parallel token routing on R simulated ranks:
 *   histogram -> perfectly balanced placement plan -> logical->physical mapping with
 *   score-threshold pruning -> dispatch (bf16 copy or per-token int8) -> combine.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, single-threaded restatement of
 * what each step computes, meant to be checked against the pages by eye. Only the
 * tests, the smoke check and the CPU-baseline leg of bench.py load it; the product
 * path never does. It shares no code, header or table with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared, no -ffast-math: every
 * float expression below is evaluated as written, one binary32 rounding per
 * operation, no fused multiply-add.
 *
 * Notation: global token g = src*S + t (src in [0,R), t in [0,S)); slot n = g*K + k;
 * N = R*S*K; home(e) = e / (E/R).
 *
 * Return codes: 0 ok, -1 invalid argument, -2 invalid data (an id, a table entry or
 * a mask outside what the method allows).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EARG (-1)
#define ORC_EDATA (-2)

/* ---------------------------------------------------------------- bf16 values */

/* bf16 -> binary32: the bf16 bits are the high half of the binary32 bits (exact). */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even (IEEE 754 default rounding
 * applied to the 16 dropped mantissa bits). NaN stays NaN (quiet bit set). */
uint16_t orc_float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;  /* tie goes to the even result */
    u = u + 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

float orc_bf16_to_float(uint16_t b) { return bf16_bits_to_float(b); }

/* ------------------------------------------------------------- a1: histogram */

/* Tokens per expert (twodots.gr article on MoonEP, "six checks before trying
 * MoonEP": measure tokens per expert and maxvio). hist[e] = #{n : ids[n] == e}.
 * Ids outside [0,E) are an error. */
int orc_histogram(const int32_t *ids, int64_t n, int32_t E, int32_t *hist)
{
    if (!ids && n > 0) return ORC_EARG;
    if (E <= 0 || !hist) return ORC_EARG;
    for (int32_t e = 0; e < E; e++) hist[e] = 0;
    for (int64_t i = 0; i < n; i++) {
        int32_t e = ids[i];
        if (e < 0 || e >= E) return ORC_EDATA;
        hist[e] += 1;
    }
    return ORC_OK;
}

/* ------------------------------------------------------ a2: placement plans */

typedef struct {
    int32_t rank;   /* home rank of the key (balanced) or physical rank (grouped) */
    int32_t key;    /* expert (balanced) or physical instance id (grouped) */
    int32_t src;
    int32_t t;
    int32_t k;
    int64_t n;      /* flat slot index */
} orc_slot;

static int cmp_slot(const void *pa, const void *pb)
{
    const orc_slot *a = (const orc_slot *)pa, *b = (const orc_slot *)pb;
    if (a->rank != b->rank) return a->rank < b->rank ? -1 : 1;
    if (a->key != b->key) return a->key < b->key ? -1 : 1;
    if (a->src != b->src) return a->src < b->src ? -1 : 1;
    if (a->t != b->t) return a->t < b->t ? -1 : 1;
    if (a->k != b->k) return a->k < b->k ? -1 : 1;
    return 0;
}

/* Walk the sorted rows, given the receiving rank of every row, and list each rank's
 * replicas: the distinct keys among its rows in row order, with cu_seqlens (row
 * offsets relative to the rank's first row). */
static void build_replica_tables(const orc_slot *sorted, const int32_t *row_rank, int64_t nrows,
                                 int32_t R, const int64_t *rank_off, int32_t cap,
                                 int32_t *rep_count, int32_t *rep_key, int32_t *rep_cu)
{
    for (int32_t r = 0; r < R; r++) {
        rep_count[r] = 0;
        for (int32_t j = 0; j <= cap; j++) rep_cu[(int64_t)r * (cap + 1) + j] = 0;
        for (int32_t j = 0; j < cap; j++) rep_key[(int64_t)r * cap + j] = -1;
    }
    int32_t prev_rank = -1, prev_key = -1;
    for (int64_t i = 0; i < nrows; i++) {
        int32_t r = row_rank[i], key = sorted[i].key;
        if (r != prev_rank || key != prev_key) {
            int32_t j = rep_count[r];
            rep_key[(int64_t)r * cap + j] = key;
            rep_cu[(int64_t)r * (cap + 1) + j] = (int32_t)(i - rank_off[r]);
            rep_count[r] = j + 1;
            prev_rank = r;
            prev_key = key;
        }
    }
    for (int32_t r = 0; r < R; r++)
        rep_cu[(int64_t)r * (cap + 1) + rep_count[r]] = (int32_t)(rank_off[r + 1] - rank_off[r]);
}

/*
 * Perfectly balanced plan (MoonEP: every rank processes exactly S*K token-slots,
 * "dynamic redundant experts"; twodots.gr article on MoonEP, core-idea and
 * redundant-experts paragraphs). The rule: order all N slots by
 * (home(e), e, src, t, k), cut the ordered list into R chunks of S*K rows, chunk r
 * is rank r's receive buffer; an expert whose rows straddle a cut gets a replica on
 * every further rank it reaches.
 *
 * Written literally: build the tuple list, sort it, the row of a slot is its index
 * in the sorted list. (Deliberately not a counting sort.)
 *
 * Outputs: pos[N] (row of every slot), hist[E], load[R] (rows each rank would get
 * if every expert stayed on its home rank), rep_count[R], rep_expert[R*cap],
 * rep_cu[R*(cap+1)], stats[8] = {max_load, max_chunk, redundant, prefetched,
 * n_kept, max_hist, 0, 0}:
 *   redundant  = sum over experts of (#ranks holding it - 1)
 *   prefetched = #(rank, expert) replicas with rank != home(expert)
 */
int orc_plan_balanced(const int32_t *ids, int32_t R, int32_t E, int32_t S, int32_t K,
                      int32_t *pos, int32_t *hist, int32_t *load, int32_t cap,
                      int32_t *rep_count, int32_t *rep_expert, int32_t *rep_cu, int64_t *stats)
{
    if (R <= 0 || E <= 0 || S <= 0 || K <= 0 || E % R != 0 || cap < E) return ORC_EARG;
    if (!ids || !pos || !hist || !load || !rep_count || !rep_expert || !rep_cu || !stats)
        return ORC_EARG;
    const int64_t N = (int64_t)R * S * K, SK = (int64_t)S * K;
    const int32_t per_rank = E / R;
    int rc = orc_histogram(ids, N, E, hist);
    if (rc != ORC_OK) return rc;

    orc_slot *sl = (orc_slot *)malloc((size_t)N * sizeof(orc_slot));
    int32_t *row_rank = (int32_t *)malloc((size_t)N * sizeof(int32_t));
    int64_t *rank_off = (int64_t *)malloc((size_t)(R + 1) * sizeof(int64_t));
    int32_t *inst = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!sl || !row_rank || !rank_off || !inst) {
        free(sl); free(row_rank); free(rank_off); free(inst);
        return ORC_EARG;
    }
    for (int32_t src = 0; src < R; src++)
        for (int32_t t = 0; t < S; t++)
            for (int32_t k = 0; k < K; k++) {
                int64_t n = ((int64_t)src * S + t) * K + k;
                int32_t e = ids[n];
                sl[n].rank = e / per_rank;
                sl[n].key = e;
                sl[n].src = src;
                sl[n].t = t;
                sl[n].k = k;
                sl[n].n = n;
            }
    qsort(sl, (size_t)N, sizeof(orc_slot), cmp_slot);
    for (int64_t i = 0; i < N; i++) {
        pos[sl[i].n] = (int32_t)i;
        row_rank[i] = (int32_t)(i / SK);   /* the cut into R chunks of S*K rows */
    }
    for (int32_t r = 0; r <= R; r++) rank_off[r] = (int64_t)r * SK;
    build_replica_tables(sl, row_rank, N, R, rank_off, cap, rep_count, rep_expert, rep_cu);

    int64_t redundant = 0, prefetched = 0, max_load = 0, max_hist = 0, max_chunk = 0;
    for (int32_t r = 0; r < R; r++) {
        load[r] = 0;
        for (int32_t j = 0; j < rep_count[r]; j++) {
            int32_t e = rep_expert[(int64_t)r * cap + j];
            inst[e] += 1;
            if (r != e / per_rank) prefetched += 1;
        }
        if (rank_off[r + 1] - rank_off[r] > max_chunk) max_chunk = rank_off[r + 1] - rank_off[r];
    }
    for (int32_t e = 0; e < E; e++) {
        load[e / per_rank] += hist[e];
        if (inst[e] > 1) redundant += inst[e] - 1;
        if (hist[e] > max_hist) max_hist = hist[e];
    }
    for (int32_t r = 0; r < R; r++)
        if (load[r] > max_load) max_load = load[r];
    stats[0] = max_load;
    stats[1] = max_chunk;
    stats[2] = redundant;
    stats[3] = prefetched;
    stats[4] = N;
    stats[5] = max_hist;
    stats[6] = 0;
    stats[7] = 0;
    free(sl); free(row_rank); free(rank_off); free(inst);
    return ORC_OK;
}

/*
 * Grouped plan over physical instance ids (the receive layout after the
 * aclnnMoeUpdateExpert mapping): every kept slot goes to the rank that hosts its
 * instance, rank = key / keys_per_rank; rows are ordered by (rank, key, src, t, k)
 * and packed, so rank r owns rows [rank_off[r], rank_off[r+1]). Dropped slots
 * (keep[n] == 0) get pos = -1. stats as in the balanced plan with load[r] = rows of
 * rank r, redundant = prefetched = 0 (no instance spans two ranks).
 */
int orc_plan_grouped(const int32_t *keys, const uint8_t *keep, int32_t R, int32_t n_keys,
                     int32_t keys_per_rank, int32_t S, int32_t K, int32_t *pos, int32_t *hist,
                     int32_t *rank_off_out, int32_t cap, int32_t *rep_count, int32_t *rep_key,
                     int32_t *rep_cu, int64_t *stats)
{
    if (R <= 0 || n_keys <= 0 || keys_per_rank <= 0 || S <= 0 || K <= 0) return ORC_EARG;
    if ((int64_t)keys_per_rank * R != n_keys || cap < n_keys) return ORC_EARG;
    if (!keys || !pos || !hist || !rank_off_out || !rep_count || !rep_key || !rep_cu || !stats)
        return ORC_EARG;
    const int64_t N = (int64_t)R * S * K;
    for (int32_t e = 0; e < n_keys; e++) hist[e] = 0;
    orc_slot *sl = (orc_slot *)malloc((size_t)(N > 0 ? N : 1) * sizeof(orc_slot));
    int32_t *row_rank = (int32_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(int32_t));
    int64_t *rank_off = (int64_t *)malloc((size_t)(R + 1) * sizeof(int64_t));
    if (!sl || !row_rank || !rank_off) {
        free(sl); free(row_rank); free(rank_off);
        return ORC_EARG;
    }
    int64_t m = 0;
    for (int32_t src = 0; src < R; src++)
        for (int32_t t = 0; t < S; t++)
            for (int32_t k = 0; k < K; k++) {
                int64_t n = ((int64_t)src * S + t) * K + k;
                pos[n] = -1;
                if (keep && !keep[n]) continue;
                int32_t key = keys[n];
                if (key < 0 || key >= n_keys) {
                    free(sl); free(row_rank); free(rank_off);
                    return ORC_EDATA;
                }
                hist[key] += 1;
                sl[m].rank = key / keys_per_rank;
                sl[m].key = key;
                sl[m].src = src;
                sl[m].t = t;
                sl[m].k = k;
                sl[m].n = n;
                m++;
            }
    qsort(sl, (size_t)m, sizeof(orc_slot), cmp_slot);
    for (int32_t r = 0; r <= R; r++) rank_off[r] = m;
    for (int64_t i = m - 1; i >= 0; i--) {
        pos[sl[i].n] = (int32_t)i;
        row_rank[i] = sl[i].rank;
        for (int32_t r = 0; r <= sl[i].rank; r++) rank_off[r] = i;
    }
    build_replica_tables(sl, row_rank, m, R, rank_off, cap, rep_count, rep_key, rep_cu);
    int64_t max_chunk = 0, max_hist = 0;
    for (int32_t r = 0; r <= R; r++) rank_off_out[r] = (int32_t)rank_off[r];
    for (int32_t r = 0; r < R; r++)
        if (rank_off[r + 1] - rank_off[r] > max_chunk) max_chunk = rank_off[r + 1] - rank_off[r];
    for (int32_t e = 0; e < n_keys; e++)
        if (hist[e] > max_hist) max_hist = hist[e];
    stats[0] = max_chunk;  /* home load == received rows: instances never move */
    stats[1] = max_chunk;
    stats[2] = 0;
    stats[3] = 0;
    stats[4] = m;
    stats[5] = max_hist;
    stats[6] = 0;
    stats[7] = 0;
    free(sl); free(row_rank); free(rank_off);
    return ORC_OK;
}

/* ------------------------------------------- a3: mapping and pruning (page 4) */

/*
 * aclnnMoeUpdateExpert (gitcode ops-transformer, "功能说明": 负载均衡 and 专家剪枝).
 *
 * Mapping of slot (i, k), e = expert_ids[i,k], c = eplb_table[e, 0]:
 *   c == 1             -> eplb_table[e, 1]
 *   balance_mode == 0  -> column local_rank_id / ceil(world_size / c) + 1   (by rank)
 *   balance_mode == 1  -> column (i mod c) + 1                              (by token)
 * ceil is a true ceiling; i is the token (row) index; in mode 1 the modulus is this
 * expert's instance count c.
 *
 * Pruning, per token i: v_i = sum over k (ascending) of fl(scale[i,k] * thr[k]),
 * accumulated in binary32; slot (i,k) stays active iff active[i] and not
 * (scale[i,k] < v_i). Without scales/threshold the mask is active[i] broadcast
 * (all true when active is NULL too).
 *
 * Argument ranges (page 4, "参数shape格式约束"): 0 < K <= 16, 0 < E <= 1024,
 * 2 <= F <= world_size + 1, world_size in [2, 768] and local_rank_id in
 * [0, world_size) for balance_mode 0. The page's BS <= 512 is a limit of that
 * hardware and is not enforced.
 * Data checks: expert id in [0,E); 1 <= c <= F-1; the chosen instance id in
 * [0, 1024) (at most 1024 instances in total); active mask has every true before
 * every false.
 */
int orc_update_expert(const int32_t *expert_ids, int64_t BS, int32_t K, const int32_t *table,
                      int32_t E, int32_t F, const float *scales, const float *thr,
                      const uint8_t *active, int64_t local_rank_id, int64_t world_size,
                      int64_t balance_mode, int32_t *out_ids, uint8_t *out_mask)
{
    if (!expert_ids || !table || !out_ids || !out_mask) return ORC_EARG;
    if (BS <= 0 || K <= 0 || K > 16 || K > E || E <= 0 || E > 1024 || F < 2) return ORC_EARG;
    if ((scales == NULL) != (thr == NULL)) return ORC_EARG;
    if (active && !scales) return ORC_EARG;
    if (balance_mode != 0 && balance_mode != 1) return ORC_EARG;
    if (world_size <= 0 || F > world_size + 1) return ORC_EARG;
    if (balance_mode == 0 && (world_size < 2 || world_size > 768)) return ORC_EARG;
    if (balance_mode == 0 && (local_rank_id < 0 || local_rank_id >= world_size)) return ORC_EARG;
    if (active)
        for (int64_t i = 1; i < BS; i++)
            if (active[i] && !active[i - 1]) return ORC_EDATA;

    for (int64_t i = 0; i < BS; i++) {
        for (int32_t k = 0; k < K; k++) {
            int32_t e = expert_ids[i * K + k];
            if (e < 0 || e >= E) return ORC_EDATA;
            const int32_t *row = table + (int64_t)e * F;
            int32_t c = row[0];
            if (c < 1 || c > F - 1) return ORC_EDATA;
            int64_t col;
            if (c == 1) {
                col = 1;
            } else if (balance_mode == 0) {
                int64_t mode_value = (world_size + c - 1) / c;   /* ceil(world_size / c) */
                col = local_rank_id / mode_value + 1;
            } else {
                col = (i % c) + 1;
            }
            if (col < 1 || col > c) return ORC_EDATA;
            int32_t inst = row[col];
            if (inst < 0 || inst >= 1024) return ORC_EDATA;
            out_ids[i * K + k] = inst;
        }
        uint8_t act = active ? (active[i] ? 1 : 0) : 1;
        if (scales) {
            float v = 0.0f;
            for (int32_t k = 0; k < K; k++) {
                float prod = scales[i * K + k] * thr[k];
                v = v + prod;
            }
            for (int32_t k = 0; k < K; k++)
                out_mask[i * K + k] = (uint8_t)(act && !(scales[i * K + k] < v));
        } else {
            for (int32_t k = 0; k < K; k++) out_mask[i * K + k] = act;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------- a4: dispatch */

/*
 * Dispatch (MoonEP zero-copy dispatch: each token row is written straight to its
 * final, expert-grouped row of the receiver; aclnnMoeDistributeDispatch: tokens sent
 * to their top-K experts). For every slot n with pos[n] >= 0:
 *   recv[pos[n], :] = x[n / K, :]
 * x is [T,H] bf16 bits, recv is [rows,H] bf16 bits. pos >= rows is an error.
 */
int orc_dispatch(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K, int64_t H,
                 int64_t rows, uint16_t *recv)
{
    if (T < 0 || K <= 0 || H <= 0 || rows < 0) return ORC_EARG;
    for (int64_t n = 0; n < T * K; n++) {
        int64_t p = pos[n];
        if (p < 0) continue;
        if (p >= rows) return ORC_EDATA;
        const uint16_t *src = x + (n / K) * H;
        uint16_t *dst = recv + p * H;
        for (int64_t h = 0; h < H; h++) dst[h] = src[h];
    }
    return ORC_OK;
}

/*
 * Per-token dynamic symmetric int8 quantisation of one bf16 row (dynamic scales,
 * one fp32 scale per token: aclnnMoeDistributeDispatch dynamicScales (TP*A,) fp32):
 *   amax  = max_h |x_h|           (x_h converted exactly to binary32)
 *   scale = amax / 127            (binary32 division)
 *   q_h   = clamp(round_half_even(x_h / scale), -127, 127),  q_h = 0 when amax == 0.
 */
void orc_quantize_row(const uint16_t *x, int64_t H, int8_t *q, float *scale_out)
{
    float amax = 0.0f;
    for (int64_t h = 0; h < H; h++) {
        float a = fabsf(bf16_bits_to_float(x[h]));
        if (a > amax) amax = a;
    }
    float scale = amax / 127.0f;
    *scale_out = scale;
    for (int64_t h = 0; h < H; h++) {
        if (scale == 0.0f) {
            q[h] = 0;
            continue;
        }
        float v = bf16_bits_to_float(x[h]) / scale;
        float r = nearbyintf(v);   /* default rounding mode: nearest, ties to even */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[h] = (int8_t)r;
    }
}

/* Dispatch with per-token int8 quantisation: every kept slot of token g receives the
 * same codes and scale, recv_q[pos[n], :] = q(x[g]), recv_scale[pos[n]] = scale(x[g]). */
int orc_dispatch_int8(const uint16_t *x, const int32_t *pos, int64_t T, int32_t K, int64_t H,
                      int64_t rows, int8_t *recv_q, float *recv_scale)
{
    if (T < 0 || K <= 0 || H <= 0 || rows < 0) return ORC_EARG;
    int8_t *q = (int8_t *)malloc((size_t)H);
    if (!q) return ORC_EARG;
    for (int64_t g = 0; g < T; g++) {
        float scale;
        orc_quantize_row(x + g * H, H, q, &scale);
        for (int32_t k = 0; k < K; k++) {
            int64_t p = pos[g * K + k];
            if (p < 0) continue;
            if (p >= rows) { free(q); return ORC_EDATA; }
            memcpy(recv_q + p * H, q, (size_t)H);
            recv_scale[p] = scale;
        }
    }
    free(q);
    return ORC_OK;
}

/* Identity expert on int8 rows: y[r, h] = bf16(fl(q[r,h] * scale[r])). */
void orc_dequantize(const int8_t *q, const float *scale, int64_t rows, int64_t H, uint16_t *y)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t h = 0; h < H; h++) {
            float v = (float)q[r * H + h] * scale[r];
            y[r * H + h] = orc_float_to_bf16(v);
        }
}

/* -------------------------------------------------------------- a5: combine */

/*
 * Combine (aclnnMoeDistributeCombine: expandX returned rows weighted by
 * expertScales and summed back into token order). For token g and column h:
 *   acc = 0; for k = 0..K-1 with pos[g*K+k] >= 0: acc = acc + fl(gate[g,k] * y[pos,h])
 *   out[g,h] = bf16(acc)
 * binary32 accumulation in ascending k; a token with no kept slot gives a zero row.
 */
int orc_combine(const uint16_t *y, int64_t rows, const int32_t *pos, const float *gates,
                int64_t T, int32_t K, int64_t H, uint16_t *out)
{
    if (T < 0 || K <= 0 || H <= 0 || rows < 0) return ORC_EARG;
    for (int64_t g = 0; g < T; g++) {
        for (int32_t k = 0; k < K; k++) {
            int64_t p = pos[g * K + k];
            if (p >= rows) return ORC_EDATA;
        }
        for (int64_t h = 0; h < H; h++) {
            float acc = 0.0f;
            for (int32_t k = 0; k < K; k++) {
                int64_t p = pos[g * K + k];
                if (p < 0) continue;
                float prod = gates[g * K + k] * bf16_bits_to_float(y[p * H + h]);
                acc = acc + prod;
            }
            out[g * H + h] = orc_float_to_bf16(acc);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------- f4: combine + residual + RMSNorm */

/* binary64 -> bf16 bits, round to nearest, ties to even, directly (no intermediate
 * binary32 rounding): the value with 8 significant bits nearest to v; below 2^-126 the
 * bf16 grid is the fixed step 2^-133. */
uint16_t orc_double_to_bf16(double v)
{
    if (v != v) return 0x7fc0u;
    if (v == 0.0) return signbit(v) ? 0x8000u : 0x0000u;
    int e;
    double m = frexp(v, &e);               /* v = m * 2^e, 0.5 <= |m| < 1 */
    double r;
    if (e - 1 >= -126) {
        r = ldexp(nearbyint(ldexp(m, 8)), e - 8);   /* 8 significant bits */
    } else {
        r = ldexp(nearbyint(ldexp(v, 133)), -133);  /* subnormal grid */
    }
    float f = (float)r;                    /* exact: r has at most 8 significant bits */
    if (fabs(r) > 3.3895313892515355e38) f = (float)(v > 0 ? INFINITY : -INFINITY);
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/*
 * Combine followed by residual add and RMSNorm (aclnnMoeDistributeCombineAddRmsNorm:
 * residualX, gamma, yOut, rstdOut, xOut; gitcode ops-transformer aclnnMoeUpdateExpert
 * doc, 调用示例). For token g, with c = the combine output row (bf16, as orc_combine):
 *   x_h      = c_h + residual_h                      (exact, binary64)
 *   x_out_h  = bf16(x_h)
 *   rstd     = 1 / sqrt( (1/H) sum_h x_h^2 + eps )   (binary64)
 *   y_h      = x_h * rstd * gamma_h                  (binary64; y_exact)
 *   y_out_h  = bf16(y_h)
 * Outputs x_out and y_out as bf16 bits, y_exact [T,H] and rstd [T] as binary64.
 */
int orc_combine_add_rmsnorm(const uint16_t *y, int64_t rows, const int32_t *pos, const float *gates,
                            int64_t T, int32_t K, int64_t H, const uint16_t *residual,
                            const uint16_t *gamma, double eps, uint16_t *x_out, uint16_t *y_out,
                            double *y_exact, double *rstd)
{
    if (T < 0 || K <= 0 || H <= 0 || rows < 0 || eps < 0) return ORC_EARG;
    uint16_t *c = (uint16_t *)malloc((size_t)(T > 0 ? T : 1) * (size_t)H * sizeof(uint16_t));
    double *x = (double *)malloc((size_t)H * sizeof(double));
    if (!c || !x) {
        free(c); free(x);
        return ORC_EARG;
    }
    int rc = orc_combine(y, rows, pos, gates, T, K, H, c);
    if (rc != ORC_OK) {
        free(c); free(x);
        return rc;
    }
    for (int64_t g = 0; g < T; g++) {
        double ss = 0.0;
        for (int64_t h = 0; h < H; h++) {
            x[h] = (double)bf16_bits_to_float(c[g * H + h]) + (double)bf16_bits_to_float(residual[g * H + h]);
            x_out[g * H + h] = orc_double_to_bf16(x[h]);
            ss += x[h] * x[h];
        }
        double r = 1.0 / sqrt(ss / (double)H + eps);
        rstd[g] = r;
        for (int64_t h = 0; h < H; h++) {
            double v = x[h] * r * (double)bf16_bits_to_float(gamma[h]);
            y_exact[g * H + h] = v;
            y_out[g * H + h] = orc_double_to_bf16(v);
        }
    }
    free(c); free(x);
    return ORC_OK;
}

/* ------------------------------- f2 / f3: replica weight prefetch and grad reduce */

/*
 * Prefetch slots (MoonEP memory contract; twodots.gr article on MoonEP: weights
 * [E+B, H, H'], rows 0..E-1 the ranks' own experts, rows E..E+B-1 per-rank prefetch
 * slots; B = E/R for training, 3-4 for inference; when a rank needs more remote experts
 * than it has slots, it reads them from the home rank).
 * Simulated layout: one weight array of E + R*B rows, rows [0, E) the home experts
 * (expert e at row e, on rank e / (E/R)), rows E + r*B + b the slots of rank r.
 * For every rank r, walk its replicas in order; a replica of an expert whose home is
 * another rank takes the next free slot (slot_expert[r][b] = e, weight row E + r*B + b)
 * while slots remain, else it reads the home row e. Home replicas read row e.
 * Outputs slot_expert [R, B] (-1 = unused) and rep_weight [R, cap] (-1 past rep_count).
 */
int orc_prefetch_plan(const int32_t *rep_count, const int32_t *rep_key, int32_t R, int32_t E, int32_t cap,
                      int32_t B, int32_t *slot_expert, int32_t *rep_weight)
{
    if (R <= 0 || E <= 0 || E % R != 0 || cap < 0 || B < 0) return ORC_EARG;
    const int32_t per_rank = E / R;
    for (int32_t r = 0; r < R; r++) {
        for (int32_t b = 0; b < B; b++) slot_expert[(int64_t)r * B + b] = -1;
        for (int32_t j = 0; j < cap; j++) rep_weight[(int64_t)r * cap + j] = -1;
        if (rep_count[r] < 0 || rep_count[r] > cap) return ORC_EDATA;
        int32_t used = 0;
        for (int32_t j = 0; j < rep_count[r]; j++) {
            int32_t e = rep_key[(int64_t)r * cap + j];
            if (e < 0 || e >= E) return ORC_EDATA;
            int32_t row;
            if (e / per_rank == r) {
                row = e;
            } else if (used < B) {
                slot_expert[(int64_t)r * B + used] = e;
                row = E + r * B + used;
                used++;
            } else {
                row = e;                    /* no slot left: read from the home rank */
            }
            rep_weight[(int64_t)r * cap + j] = row;
        }
    }
    return ORC_OK;
}

/* w_slots[r*B + b, :] = w_home[slot_expert[r][b], :] for every used slot; D elements
 * (bf16 bits) per expert. Unused slots are left as they are. */
int orc_prefetch_weights(const uint16_t *w_home, const int32_t *slot_expert, int32_t E, int32_t R, int32_t B,
                         int64_t D, uint16_t *w_slots)
{
    if (E <= 0 || R <= 0 || B < 0 || D <= 0) return ORC_EARG;
    for (int64_t s = 0; s < (int64_t)R * B; s++) {
        int32_t e = slot_expert[s];
        if (e < 0) continue;
        if (e >= E) return ORC_EDATA;
        for (int64_t i = 0; i < D; i++) w_slots[s * D + i] = w_home[(int64_t)e * D + i];
    }
    return ORC_OK;
}

/*
 * Replica gradient reduce (MoonEP: the gradients of a prefetched copy go to a separate
 * reduce buffer [R, B, H, H']; the home rank reads the slots that hold its experts, adds
 * them into its parameter gradient and clears them). For every expert e and element i,
 * in binary32, slots taken in ascending (rank, slot) order:
 *   grad_home[e][i] = (...(grad_home[e][i] + grad_slots[s0][i]) + grad_slots[s1][i]) ...
 * over the slots s with slot_expert[s] == e; then those slots are set to zero.
 */
int orc_grad_reduce(float *grad_home, float *grad_slots, const int32_t *slot_expert, int32_t E, int32_t R,
                    int32_t B, int64_t D)
{
    if (E <= 0 || R <= 0 || B < 0 || D <= 0) return ORC_EARG;
    for (int64_t s = 0; s < (int64_t)R * B; s++)
        if (slot_expert[s] >= E || slot_expert[s] < -1) return ORC_EDATA;
    for (int32_t e = 0; e < E; e++) {
        for (int64_t s = 0; s < (int64_t)R * B; s++) {
            if (slot_expert[s] != e) continue;
            for (int64_t i = 0; i < D; i++) {
                float v = grad_home[(int64_t)e * D + i] + grad_slots[s * D + i];
                grad_home[(int64_t)e * D + i] = v;
            }
        }
    }
    for (int64_t s = 0; s < (int64_t)R * B; s++) {
        if (slot_expert[s] < 0) continue;
        for (int64_t i = 0; i < D; i++) grad_slots[s * D + i] = 0.0f;
    }
    return ORC_OK;
}

/* --------------------------------------------- f1: smooth-quantised int8 dispatch */

/*
 * Dispatch with per-expert smoothing before the dynamic int8 quantisation (the
 * optional scales of shape (moeExpertNum, H), fp32, that aclnnMoeDistributeDispatch
 * takes when quantMode > 0: gitcode ops-transformer aclnnMoeUpdateExpert doc, 调用示例;
 * hiascend aclnnMoeDistributeDispatchSetup doc, scalesOptional). Reading: for every kept
 * slot n of token g with expert e = ids[n],
 *   xs_h  = fl(x_h * smooth[e, h])          (binary32)
 *   amax  = max_h |xs_h|,  scale = amax / 127,
 *   q_h   = clamp(round_half_even(xs_h / scale), -127, 127)   (q = 0 when amax == 0)
 *   recv_q[pos[n], :] = q,  recv_scale[pos[n]] = scale.
 * The codes and scale are per slot. The decisions are taken in binary32, as on the GPU.
 */
int orc_dispatch_int8_smooth(const uint16_t *x, const int32_t *ids, const int32_t *pos, int64_t T, int32_t K,
                             int64_t H, const float *smooth, int32_t n_experts, int64_t rows, int8_t *recv_q,
                             float *recv_scale)
{
    if (T < 0 || K <= 0 || H <= 0 || rows < 0 || n_experts <= 0) return ORC_EARG;
    float *xs = (float *)malloc((size_t)H * sizeof(float));
    if (!xs) return ORC_EARG;
    for (int64_t n = 0; n < T * K; n++) {
        int64_t p = pos[n];
        if (p < 0) continue;
        int32_t e = ids[n];
        if (p >= rows || e < 0 || e >= n_experts) {
            free(xs);
            return ORC_EDATA;
        }
        const uint16_t *row = x + (n / K) * H;
        float amax = 0.0f;
        for (int64_t h = 0; h < H; h++) {
            float v = bf16_bits_to_float(row[h]) * smooth[(int64_t)e * H + h];
            xs[h] = v;
            float a = fabsf(v);
            if (a > amax) amax = a;
        }
        float scale = amax / 127.0f;
        recv_scale[p] = scale;
        for (int64_t h = 0; h < H; h++) {
            int8_t q = 0;
            if (scale != 0.0f) {
                float r = nearbyintf(xs[h] / scale);
                if (r > 127.0f) r = 127.0f;
                if (r < -127.0f) r = -127.0f;
                q = (int8_t)r;
            }
            recv_q[p * H + h] = q;
        }
    }
    free(xs);
    return ORC_OK;
}

/* ------------------------------------- f1: one row per (token, destination rank) */

/* Rank that owns row p of a plan: the r with rank_off[r] <= p < rank_off[r+1]. */
static int32_t rank_of_row(const int32_t *rank_off, int32_t R, int64_t p)
{
    for (int32_t r = 0; r < R; r++)
        if (p >= rank_off[r] && p < rank_off[r + 1]) return r;
    return -1;
}

/*
 * Deduplicated dispatch encoding (the MoonEP API reference, section 5.2 on
 * communication performance, names a bounds check of a "dedup encoding"). Reading: a
 * token whose kept slots land on one destination rank several times (several of its
 * experts, or replicas, live there) crosses to that rank once. The rank's deduplicated
 * receive rows hold its tokens in ascending global token order.
 *
 * For every rank r in ascending order, for every token g in ascending order: if any
 * kept slot of g has its plan row on rank r, g takes the next deduplicated row u:
 *   dtok[u] = g;  dsend[n0] = u for the first such slot n0 (the send list);
 *   dpos[n] = u and gidx[pos[n]] = u for every such slot n.
 * drank_off[r] = the first deduplicated row of rank r, drank_off[R] = the row count.
 * Unset entries are -1. gidx has one entry per plan row (gidx_len >= rank_off[R]).
 */
int orc_dedup_plan(const int32_t *pos, int64_t N, int32_t K, const int32_t *rank_off, int32_t R,
                   int32_t *dsend, int32_t *dpos, int32_t *drank_off, int32_t *dtok, int32_t *gidx,
                   int64_t gidx_len)
{
    if (K <= 0 || N < 0 || N % K != 0 || R <= 0) return ORC_EARG;
    if (rank_off[0] != 0) return ORC_EDATA;
    for (int32_t r = 0; r < R; r++)
        if (rank_off[r + 1] < rank_off[r]) return ORC_EDATA;
    if (gidx_len < rank_off[R]) return ORC_EARG;
    for (int64_t n = 0; n < N; n++) {
        if (pos[n] < -1 || pos[n] >= rank_off[R]) return ORC_EDATA;
        dsend[n] = -1;
        dpos[n] = -1;
        dtok[n] = -1;
    }
    for (int64_t i = 0; i < gidx_len; i++) gidx[i] = -1;
    const int64_t T = N / K;
    int32_t u = 0;
    for (int32_t r = 0; r < R; r++) {
        drank_off[r] = u;
        for (int64_t g = 0; g < T; g++) {
            int64_t first = -1;
            for (int32_t k = 0; k < K; k++) {
                const int64_t n = g * K + k;
                if (pos[n] < 0 || rank_of_row(rank_off, R, pos[n]) != r) continue;
                if (first < 0) {
                    first = n;
                    dsend[n] = u;
                    dtok[u] = (int32_t)g;
                }
                dpos[n] = u;
                gidx[pos[n]] = u;
            }
            if (first >= 0) u++;
        }
    }
    drank_off[R] = u;
    return ORC_OK;
}

/*
 * Expansion on the receiving rank: dst[p, :] = src[gidx[p], :] (row_bytes bytes per
 * row) and, with scales, dst_scale[p] = src_scale[gidx[p]], for every row p with
 * gidx[p] >= 0; other rows are left as they are.
 */
int orc_expand(const uint8_t *src, const float *src_scale, int64_t src_rows, const int32_t *gidx, int64_t rows,
               int64_t row_bytes, uint8_t *dst, float *dst_scale)
{
    if (rows < 0 || row_bytes <= 0 || src_rows < 0) return ORC_EARG;
    for (int64_t p = 0; p < rows; p++) {
        const int64_t u = gidx[p];
        if (u < 0) continue;
        if (u >= src_rows) return ORC_EDATA;
        memcpy(dst + p * row_bytes, src + u * row_bytes, (size_t)row_bytes);
        if (src_scale && dst_scale) dst_scale[p] = src_scale[u];
    }
    return ORC_OK;
}
