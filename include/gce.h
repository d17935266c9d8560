/*
 * gce.h -- C ABI of the B200 (sm_100a) gradient-compression library:
 * error-feedback top-k / rand-k (Mem-SGD), PowerSGD with a warm-started Q,
 * Accordion's per-layer level switch, and the on-device aggregate of the
 * compressed payloads of W data-parallel worker replicas.
 *
 * Sources (page title, section):
 *   [MEM]  "Sparsified SGD with Memory", Method: the error-feedback update
 *            g_t = comp_k(m_t + eta*grad),  m_{t+1} = m_t + eta*grad - g_t,
 *          comp_k a k-contraction (top-k keeps the largest entries, rand-k
 *          random ones: Abstract); Key results: 0 < k <= d.
 *   [ACC]  "Accordion: Adaptive Gradient Communication via Critical Learning
 *          Regime Identification", Method: the per-layer rate of change of
 *          the gradient norm selects the low-compression level l_low inside
 *          critical regimes and the high-compression level l_high outside.
 *   [UTIL] "On the Utility of Gradient Compression in Distributed Training
 *          Systems", Method / Key results: PowerSGD (rank r) is all-reduce
 *          compatible; the encode-decode latency is what limits speedups.
 *   PowerSGD's steps are not printed on the pages; this library implements
 *   the standard single power-iteration step with a reused Q:
 *   P = M Q, orthonormalise P (modified Gram-Schmidt), Q' = M^T P,
 *   decompress P Q'^T, residual M - P Q'^T into memory.
 *
 * Conventions shared by every call:
 *   - Pointers named grad, mem, vals, idx, P, Q, out, k_or_rank, prev_norm,
 *     level, cur_norm and ws are DEVICE pointers owned by the caller; they
 *     must be 16-byte aligned.  The library never allocates during a step
 *     (only gce_table_create allocates, once).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every step call is asynchronous on that stream; a return of
 *     GCE_OK means the work was enqueued.  Host-detectable errors return a
 *     negative GCE_ERR_* before anything is enqueued; errors found on the
 *     device set bits in the workspace status word (gce_status).  No call
 *     aborts, throws or prints.
 *   - Layout: W workers' buffers are stacked.  grad and mem are
 *     [W][N] fp32; layer l of worker w starts at w*N + info.offset and is
 *     rows x cols row-major.  Sparse payloads of (w, l) are vals/idx at
 *     w*vals_per_worker + info.val_offset, k entries in ascending index
 *     (layer-local int32); an uncompressed (DENSE) layer's payload is its n
 *     values at the same place.  PowerSGD P of (w, l) is rows x r_max at
 *     w*P_per_worker + info.p_offset and Q is cols x r_max at
 *     w*Q_per_worker + info.q_offset (row stride r_max; rank r uses
 *     columns 0..r-1 and leaves the others untouched).
 *   - Inputs must be finite (NaN has no |v| order).
 *   - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef GCE_H
#define GCE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GCE_API __attribute__((visibility("default")))
#else
#define GCE_API
#endif

/* return codes */
#define GCE_OK 0
#define GCE_ERR_ARG (-1)       /* bad argument (NULL, misaligned, out of range) */
#define GCE_ERR_CUDA (-2)      /* a CUDA runtime call failed                     */
#define GCE_ERR_WORKSPACE (-3) /* ws NULL or smaller than gce_workspace_bytes   */
#define GCE_ERR_NOMEM (-4)     /* gce_table_create could not allocate           */
#define GCE_ERR_KIND (-5)      /* the table's layer kinds do not fit this call  */

/* device status bits, read with gce_status */
#define GCE_STATUS_K_RANGE 1    /* a per-layer k / rank was out of range: layer skipped   */
#define GCE_STATUS_FALLBACK 2   /* informational: an exact fallback path ran              */
#define GCE_STATUS_NONFINITE 4  /* a residual m + eta*grad was NaN or +-Inf (inputs must be
                                   finite; the step still completes, ordering such keys by
                                   their bits)                                            */
#define GCE_STATUS_WAIT_TIMEOUT 8  /* a bounded wait inside a kernel gave up (a scale that
                                      was never published): that call's results are not
                                      valid                                                 */

/* layer kinds */
#define GCE_KIND_TOPK 0
#define GCE_KIND_RANDK 1
#define GCE_KIND_POWERSGD 2
#define GCE_KIND_DENSE 3 /* sent uncompressed: payload = m + eta*grad, memory -> 0 */
#define GCE_KIND_SIGN 4  /* 1 bit per element plus one scale (signSGD with memory) */

/* operations, for gce_workspace_bytes */
#define GCE_OP_TOPK 0
#define GCE_OP_RANDK 1
#define GCE_OP_POWERSGD 2
#define GCE_OP_ACCORDION 3
#define GCE_OP_DECOMPRESS 4
#define GCE_OP_POWERSGD_DP 5
#define GCE_OP_SIGN 6

/* Accordion levels [ACC] */
#define GCE_LEVEL_LOW 0  /* l_low: less compression (critical regime) */
#define GCE_LEVEL_HIGH 1 /* l_high: more compression                 */

typedef struct gce_table gce_table;

/* One layer as the caller describes it.  cap: for TOPK / RANDK the largest k
 * any step will use (payload slots, 1 <= cap <= rows*cols); for POWERSGD the
 * largest rank r_max (1..4, <= min(rows, cols)); ignored for DENSE and SIGN.
 * A SIGN layer's payload takes 4 + ceil(n/32) slots (rounded up to a multiple
 * of 4): slot 0 the fp32 scale, slots 1-3 zero, then the packed sign words
 * (uint32 bit patterns; bit i mod 32 of word i/32 is element i's sign). */
typedef struct gce_layer_desc {
    int64_t rows;
    int64_t cols; /* 1 for a 1-D layer */
    int32_t kind;
    int32_t cap;
} gce_layer_desc;

typedef struct gce_layer_info {
    int64_t offset;     /* first element in a worker's flat buffer         */
    int64_t n;          /* rows * cols                                     */
    int64_t rows, cols;
    int32_t kind, cap;
    int64_t val_offset; /* vals/idx slot start (sparse, DENSE); -1 otherwise */
    int64_t p_offset;   /* POWERSGD only; -1 otherwise                     */
    int64_t q_offset;   /* POWERSGD only; -1 otherwise                     */
} gce_layer_info;

typedef struct gce_table_totals {
    int64_t L;
    int64_t N;               /* elements per worker                         */
    int64_t vals_per_worker; /* floats (and int32 idx slots) per worker     */
    int64_t P_per_worker;    /* floats                                      */
    int64_t Q_per_worker;    /* floats                                      */
    int32_t compressed_kind; /* TOPK / RANDK / POWERSGD, or -1 if all DENSE */
} gce_table_totals;

/*
 * Build a layer table: copies `descs` (host, L entries) and uploads the
 * device-side copy.  A table holds at most one compressed kind (TOPK, RANDK
 * or POWERSGD) plus any number of DENSE layers.  Allocates device memory
 * once; *out is owned by the caller and released with gce_table_destroy.
 * Errors: GCE_ERR_ARG (L < 1, a bad shape or cap, n > 2^31-1 per layer),
 * GCE_ERR_KIND (two compressed kinds), GCE_ERR_NOMEM / GCE_ERR_CUDA.
 */
GCE_API int gce_table_create(const gce_layer_desc* descs, int32_t L, gce_table** out);
GCE_API int gce_table_destroy(gce_table* table);
GCE_API int gce_table_get_totals(const gce_table* table, gce_table_totals* out);
GCE_API int gce_table_get_layer(const gce_table* table, int32_t l, gce_layer_info* out);

/* Bytes of device workspace an operation needs for W workers (>= 1).  The
 * caller allocates it once; its first GCE_WS_HEADER_BYTES hold the status
 * word and must be zero before first use.  The same workspace may be reused
 * by every call on the same table and W (never by two calls at once). */
#define GCE_WS_HEADER_BYTES 256
GCE_API int gce_workspace_bytes(const gce_table* table, int32_t W, int32_t op, size_t* bytes);

/*
 * Mem-SGD top-k step [MEM] for every (worker, TOPK layer), plus DENSE layers.
 *   v = fl32(mem + fl32(eta * grad))      (two roundings, no FMA)
 *   chosen set S: the k largest |v| (|v| ordered by the float's bits with
 *   the sign cleared), equal |v| -> lower index first;
 *   vals/idx <- (v_i, i) for i in S, ascending i;  mem <- v, and +0.0 on S.
 * grad [W][N] read; mem [W][N] read and written; k_or_rank: device int32[L]
 * with k per layer (1 <= k <= cap), or NULL for k = cap; entries of non-TOPK
 * layers are ignored.  vals / idx: [W][vals_per_worker].  Results are
 * bit-exact and independent of the launch configuration.
 * A layer whose k is out of range is skipped and sets GCE_STATUS_K_RANGE.
 */
GCE_API int ef_topk_step(const gce_table* table, int32_t W, const float* grad, float* mem,
                 float eta, const int32_t* k_or_rank, float* vals, int32_t* idx,
                 void* ws, size_t ws_bytes, void* stream);

/*
 * Mem-SGD rand-k step [MEM]: as ef_topk_step, but S is the k coordinates with
 * the smallest (key, index), key_i = high 32 bits of output i+1 of a
 * SplitMix64 generator (Steele, Lea, Flood 2014) whose state is derived from
 * (seed, stream 0, worker, layer, step) by successive SplitMix64 outputs; the
 * chosen values are sent unscaled (comp_k stays a k-contraction).
 */
GCE_API int ef_randk_step(const gce_table* table, int32_t W, const float* grad, float* mem,
                  float eta, const int32_t* k_or_rank, uint64_t seed, uint64_t step,
                  float* vals, int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * ef_randk_step for workers worker0 .. worker0+W-1 of a larger job (one
 * rank's share of a data-parallel job): row w of grad, mem, vals and idx
 * belongs to job-wide worker worker0 + w, whose index the generator takes,
 * so the rows are bit for bit those of an ef_randk_step over the whole job.
 * worker0 < 0 gives GCE_ERR_ARG.  ef_randk_step is this call with worker0 0.
 */
GCE_API int ef_randk_step_at(const gce_table* table, int64_t worker0, int32_t W,
                             const float* grad, float* mem, float eta,
                             const int32_t* k_or_rank, uint64_t seed, uint64_t step,
                             float* vals, int32_t* idx, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * rand-k look-ahead (on by default; the pages have no counterpart: it only
 * moves work).  The chosen set does not depend on the data, so while a step's
 * memory pass streams grad and mem, ef_randk_step also hashes the next step's
 * keys (step + 1, same seed, W, worker0 and table, with this step's k sizing
 * the band) into its workspace.  The next call with the same table,
 * workspace, seed, W, worker0 and step + 1 skips its own key pass.  Results never depend on it:
 * that call re-reads k, repairs a band the new k misses exactly, and checks a
 * tag in the workspace header, recomputing everything if another step's pass
 * is there.  Between the two calls nothing else may write the workspace.
 * Off while the stream is being captured into a graph.  on: 1 or 0; other
 * values give GCE_ERR_ARG.
 */
GCE_API int gce_set_randk_ahead(int32_t on);

/*
 * Initial (warm-start) Q for every (worker, POWERSGD layer): entries
 * (h >> 40) * 2^-23 - 1 in [-1, 1), h the SplitMix64 output c*r_max + j + 1
 * from the state of (seed, stream 1, worker, layer, step 0).  Q: [W][Q_per_worker].
 */
GCE_API int powersgd_init_q(const gce_table* table, int32_t W, uint64_t seed, float* Q,
                    void* stream);

/*
 * PowerSGD rank-r step with error feedback for every (worker, POWERSGD layer),
 * plus DENSE layers (payload to vals, memory -> 0):
 *   M = fl32(mem + fl32(eta*grad)); P = M Q (warm start); P <- orthonormal
 *   columns by modified Gram-Schmidt in column order (a zero column stays 0);
 *   Q <- M^T P; mem <- M - P Q^T; dense_out (optional) <- P Q^T.
 * k_or_rank: device int32[L] rank per layer (1 <= r <= cap) or NULL for
 * r = cap.  P [W][P_per_worker] written; Q [W][Q_per_worker] read and
 * written; vals [W][vals_per_worker] receives DENSE payloads (may be NULL if
 * the table has no DENSE layer); dense_out [W][N] or NULL.  fp32 with fp64
 * reductions; deterministic for a given table.
 */
GCE_API int powersgd_step(const gce_table* table, int32_t W, const float* grad, float* mem,
                  float eta, const int32_t* k_or_rank, float* P, float* Q, float* vals,
                  float* dense_out, void* ws, size_t ws_bytes, void* stream);

/*
 * powersgd_step with a lazy residual, for layers larger than L2: the same
 * payload (P, Q, DENSE values) bit for bit, without the pass that writes the
 * residual back.  Design of this library ([UTIL] Key results: the encode-decode
 * latency is what limits the speedup); the pages have no counterpart.
 *   lazy_rank: device int32 [W][L] (table layer order; entries of other kinds
 *   unused), owned by the caller, zero before the first call (or after
 *   gce_materialize_memory).  Entry (w, l) = 0: mem holds the residual m, as
 *   powersgd_step leaves it.  Entry r > 0: mem holds the M of the last lazy
 *   step, and the workspace that step's fp64 orthonormal P and Q' over
 *   columns 0..r-1, so that the residual is m = M - P Q'^T, each entry formed
 *   as powersgd_step forms it.
 * The step forms m on the fly while it reads mem for M = m + eta*grad, writes
 * M back to mem, and sets entry (w, l) to this step's rank (a layer skipped
 * for an out-of-range rank keeps its memory and its entry).  Memory traffic
 * per element: grad read, memory read and written, M read once more for
 * Q' = M^T P (16 B, against 24 B for powersgd_step on layers that do not stay
 * in L2).  Other arguments, the workspace (GCE_OP_POWERSGD) and errors as
 * powersgd_step, without dense_out.  Between lazy steps the memory, lazy_rank
 * and the workspace must be left as they are (the workspace carries the
 * factors); to read the memory, call gce_materialize_memory.
 */
GCE_API int powersgd_step_lazy(const gce_table* table, int32_t W, const float* grad, float* mem,
                               float eta, const int32_t* k_or_rank, float* P, float* Q,
                               float* vals, int32_t* lazy_rank, void* ws, size_t ws_bytes,
                               void* stream);

/*
 * Turns the memory that lazy steps left into the residual: for every (w, l)
 * with lazy_rank entry r > 0, mem <- M - P Q'^T over columns 0..r-1, from the
 * fp64 factors in ws (the workspace of those lazy steps) -- the residual
 * powersgd_step would have written, bit for bit; then every entry -> 0.
 * mem [W][N], lazy_rank as powersgd_step_lazy.  GCE_ERR_WORKSPACE if ws_bytes
 * is below gce_workspace_bytes(GCE_OP_POWERSGD).
 */
GCE_API int gce_materialize_memory(const gce_table* table, int32_t W, float* mem,
                                   int32_t* lazy_rank, void* ws, size_t ws_bytes, void* stream);

/*
 * Data-parallel PowerSGD step ([UTIL] Key results: PowerSGD is all-reduce
 * compatible) over the W workers of one GPU: the two all-reduces become sums
 * over the workers in worker order, the orthonormal P and the warm start Q
 * are shared, and each worker keeps its own error:
 *   M_w = fl32(mem_w + fl32(eta*grad_w));  P = sum_w M_w Q;
 *   P <- orthonormal columns (modified Gram-Schmidt, column order, fp64);
 *   Q_w = M_w^T P;  mem_w <- M_w - P Q_w^T;
 *   Q <- fl32(fl32(sum_w Q_w) * fl32(1/W))   (the workers' mean);
 * DENSE layers: vals <- fl32(fl32(sum_w M_w) * fl32(1/W)), every mem_w -> 0.
 * P Q^T (decompress_accumulate with W = 1 on P, Q, vals) is the mean of the
 * workers' decompressed updates.  grad, mem: [W][N]; P: [P_per_worker]
 * written; Q: [Q_per_worker] read and written; vals: [vals_per_worker]
 * (NULL allowed without DENSE layers).  k_or_rank as for powersgd_step.
 * ws: gce_workspace_bytes(GCE_OP_POWERSGD_DP).
 */
GCE_API int powersgd_dp_step(const gce_table* table, int32_t W, const float* grad, float* mem,
                             float eta, const int32_t* k_or_rank, float* P, float* Q,
                             float* vals, void* ws, size_t ws_bytes, void* stream);

/*
 * The data-parallel PowerSGD step cut at its two sums, for data-parallel
 * ranks that each hold some of the W workers ([UTIL] Key results: PowerSGD is
 * all-reduce compatible).  Run in this order, with the rows of every rank
 * gathered in worker order where marked; the result is powersgd_dp_step over
 * all W workers, bit for bit (the sums run over the gathered rows in worker
 * order, as that step sums them):
 *   powersgd_dp_encode(Wl workers): M_w = fl32(mem_w + fl32(eta*grad_w)) into
 *     mem; Ppart [Wl][gce_powersgd_dp_partials doubles] the fp64 partial
 *     products M_w Q of each worker (Q: the shared warm start); DENSE layers:
 *     vals [Wl][vals_per_worker] each worker's residual, memory -> 0.
 *   -- gather Ppart rows of all W workers (and the vals rows) --
 *   powersgd_dp_orthogonalize(W): P <- the orthonormal columns (modified
 *     Gram-Schmidt, fp64) of sum_w M_w Q from the W gathered Ppart rows;
 *     P [P_per_worker] fp32, and its fp64 copy kept in ws.
 *   powersgd_dp_project(Wl): Qw [Wl][Q_per_worker] <- Q_w = M_w^T P (fp32),
 *     mem_w <- M_w - P Q_w^T; reads P from ws (the same ws as
 *     powersgd_dp_orthogonalize).
 *   -- gather Qw rows of all W workers --
 *   powersgd_dp_mean(W): Q <- fl32(fl32(sum_w Q_w) * fl32(1/W)); DENSE:
 *     vals <- fl32(fl32(sum_w vals_all_w) * fl32(1/W)) from the gathered rows.
 * ws: gce_workspace_bytes(GCE_OP_POWERSGD_DP) for this rank's Wl workers, the
 * same workspace for the four calls of a step.  k_or_rank as powersgd_step
 * (the same on every rank).  Errors as powersgd_dp_step.
 */
GCE_API int gce_powersgd_dp_partials(const gce_table* table, int64_t* doubles_per_worker);
GCE_API int powersgd_dp_encode(const gce_table* table, int32_t W, const float* grad, float* mem,
                               float eta, const int32_t* k_or_rank, const float* Q, double* Ppart,
                               float* vals, void* ws, size_t ws_bytes, void* stream);
GCE_API int powersgd_dp_orthogonalize(const gce_table* table, int32_t W,
                                      const int32_t* k_or_rank, const double* Ppart, float* P,
                                      void* ws, size_t ws_bytes, void* stream);
GCE_API int powersgd_dp_project(const gce_table* table, int32_t W, float* mem,
                                const int32_t* k_or_rank, float* Qw, void* ws, size_t ws_bytes,
                                void* stream);
GCE_API int powersgd_dp_mean(const gce_table* table, int32_t W, const int32_t* k_or_rank,
                             const float* Qw, float* Q, const float* vals_all, float* vals,
                             void* stream);

/*
 * signSGD with error feedback for every (worker, SIGN layer) ([UTIL]
 * Method / Key results: sign SGD, one bit per element; [MEM] Method: the
 * memory), plus DENSE layers (payload to vals, memory -> 0):
 *   p = fl32(mem + fl32(eta*grad));  s = fl32(sum_i |p_i| / n) with the sum
 *   in fp64;  payload: s and the sign bits of p (-0 counts as negative);
 *   mem <- fl32(p - s) where p's sign bit is 0, fl32(p + s) where it is 1.
 * vals: [W][vals_per_worker] 32-bit slots laid out as gce_layer_desc states.
 * The sign bits and, for a given s, the memory are exact; s may differ from
 * a sequential fp64 sum by one fp32 rounding in rare cases (the fp64 sum's
 * order is the library's own, fixed).  ws: gce_workspace_bytes(GCE_OP_SIGN).
 * The two visits of every element (the layer scale, then the update) are
 * scheduled as gce_set_sign_ahead sets; every schedule gives the same bits.
 */
GCE_API int ef_sign_step(const gce_table* table, int32_t W, const float* grad, float* mem,
                         float eta, float* vals, void* ws, size_t ws_bytes, void* stream);

/*
 * sign SGD's majority-vote aggregate ([UTIL] Method: sign SGD is gathered,
 * not all-reduced): for every element of a SIGN layer
 *   out = scale * sign(#workers with sign bit 0 - #workers with sign bit 1),
 * 0 on a tie (the workers' scales are not used); DENSE layers are summed in
 * worker order and scaled as decompress_accumulate does.  vals as written by
 * ef_sign_step.  No workspace.
 */
GCE_API int decompress_vote(const gce_table* table, int32_t W, const float* vals, float scale,
                            float* out, void* stream);

/*
 * How ef_sign_step schedules its two visits of every element.  tiles > 0:
 * one launch in which the norm of the layer scale runs at most `tiles`
 * 8192-element tiles ahead of the memory update, so the update reads grad
 * and memory back from L2 rather than HBM (the schedule is built and cached
 * per table and W on first use, outside stream capture: that first call
 * allocates a small device array (cudaMalloc, with its implicit
 * synchronisation) kept until gce_table_destroy; while capturing before
 * that, the two passes run).  0: two passes over the whole set.  -1 (the
 * default): the tiles of grad and memory that fill 3/8 of the device's L2,
 * rounded to a multiple of 64 (768 on B200).  Every setting gives the same
 * bits.  tiles outside [-1, 2^20] gives GCE_ERR_ARG.
 */
GCE_API int gce_set_sign_ahead(int32_t tiles);

/*
 * Test of the bounded wait in the pipelined signSGD kernel.  on = 1 places
 * every memory-update tile before every norm tile and runs the kernel as one
 * block, so each update's wait for its layer scale runs out (about a second
 * per tile) and sets GCE_STATUS_WAIT_TIMEOUT; that call's results are not
 * valid.  Nothing faults or hangs.  While it is on, ef_sign_step refuses
 * (GCE_ERR_ARG) tables of more than 8 tiles of SIGN layers over all
 * workers.  0 (the default) restores the normal order.  Other values give
 * GCE_ERR_ARG.
 */
GCE_API int gce_set_sign_emit_first(int32_t on);

/*
 * The work-item order of the pipelined signSGD kernel, host only (no device
 * call; for inspection and tests).  For W workers over ncomp SIGN layers of
 * layer_tiles[l] >= 1 tiles each (8192 elements a tile, layers numbered
 * consecutively, worker-major), with the norm at most `ahead` tiles in front
 * (1 .. 2^20), or ahead = -1 for the wait test's order (every update first).
 * Writes up to cap runs to runs[4 * i ..]: (first item, lowest tile, kind:
 * 0 norm, 1 update, -1 the closing sentinel, whose first item is the item
 * count; order: 0 ascending tiles, 1 descending -- the updates of a layer of
 * more than `ahead` tiles run from its last tile down); *nruns = the number
 * of runs, sentinel included.  Bad arguments give GCE_ERR_ARG.
 */
GCE_API int gce_sign_schedule(const int32_t* layer_tiles, int32_t ncomp, int32_t W, int32_t ahead,
                              int64_t* runs, int64_t cap, int64_t* nruns);

/*
 * Accordion select [ACC] over every compressed layer of the table.
 * Sets prev_norm[l] = -1 (no earlier check) and level[l] = LOW.
 */
GCE_API int accordion_init(const gce_table* table, double* prev_norm, int32_t* level, void* stream);
/*
 * grad: device fp32 [N] (one gradient, e.g. one worker's or an aggregate).
 * If step % interval == 0 (a check step): s_l = sqrt(sum grad_i^2) per
 * compressed layer (fp64 accumulation, fixed order), cur_norm[l] = s_l,
 * rel = |prev - s_l| / prev (prev == 0: 0 if s_l == 0 else +inf),
 * level[l] = (prev < 0 || rel >= threshold) ? LOW : HIGH, prev_norm[l] = s_l.
 * Every step: k_or_rank_out[l] = the level's parameter -- for POWERSGD
 * layers the rank lvl_low / lvl_high, for TOPK / RANDK layers
 * k = max(1, floor(n * ppm / 1e6)) with ppm = lvl_low / lvl_high (parts per
 * million of the layer); DENSE and SIGN layers get 0.  lvl_low / lvl_high are host
 * values.  prev_norm, cur_norm: device double[L]; level, k_or_rank_out:
 * device int32[L].
 */
GCE_API int accordion_select(const gce_table* table, const float* grad, int64_t step,
                     int32_t interval, double threshold, int32_t lvl_low, int32_t lvl_high,
                     double* prev_norm, int32_t* level, double* cur_norm,
                     int32_t* k_or_rank_out, void* ws, size_t ws_bytes, void* stream);

/*
 * accordion_select cut in two, for data-parallel ranks that must take the
 * same decision from the norms of all their gradients ([ACC] Method: the
 * gradient norm; [UTIL] Key results: the all-reduce):
 *   accordion_sumsq: sumsq[l] = sum of grad_i^2 over each compressed layer
 *     (fp64, the fixed order accordion_select uses; 0 for DENSE layers).
 *     sumsq: device double[L].  ws as accordion_select.
 *   -- all-reduce (sum) sumsq over the ranks: the squared norm of the layer's
 *      gradients of every rank --
 *   accordion_decide: accordion_select's decision and k / rank output from
 *     s_l = sqrt(sumsq[l]) (sumsq may be NULL on steps that are not check
 *     steps).  Other arguments as accordion_select.
 * accordion_sumsq then accordion_decide on one gradient is accordion_select,
 * bit for bit.
 */
GCE_API int accordion_sumsq(const gce_table* table, const float* grad, double* sumsq, void* ws,
                            size_t ws_bytes, void* stream);
GCE_API int accordion_decide(const gce_table* table, const double* sumsq, int64_t step,
                             int32_t interval, double threshold, int32_t lvl_low,
                             int32_t lvl_high, double* prev_norm, int32_t* level,
                             double* cur_norm, int32_t* k_or_rank_out, void* stream);

/*
 * Aggregate [UTIL] of the W workers' payloads into a dense fp32 out [N]:
 *   out = scale * sum_{w = 0..W-1} decode(payload_w), summed in worker order
 *   from +0.0 with fp32 round-to-nearest adds, the product taken last.
 * decode: sparse layers scatter vals at idx (first k entries); DENSE layers
 * take their n values; POWERSGD layers P Q^T over the first r columns (each
 * entry formed with fp32 FMAs in column order).  k_or_rank as for the step
 * that produced the payloads (NULL = cap).  P/Q may be NULL when the table
 * has no POWERSGD layer, idx when it has no sparse layer.  Sparse and DENSE
 * results are bit-exact.  Sparse payloads must be in ascending index within
 * each (worker, layer), as the steps write them.  ws: workspace of
 * gce_workspace_bytes(GCE_OP_DECOMPRESS) bytes (per-tile entry ranges).
 */
GCE_API int decompress_accumulate(const gce_table* table, int32_t W, const float* vals,
                          const int32_t* idx, const int32_t* k_or_rank, const float* P,
                          const float* Q, float scale, float* out, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * Aggregate fused with the parameter update of [MEM] Method (x_{t+1} = x_t -
 * g_t, the workers' compressed updates summed): with S the worker-order sum
 * that decompress_accumulate forms,
 *   x[j] = fl(x[j] - fl(scale * S[j]))   for every j in [0, N),
 * bit for bit what decompress_accumulate into a scratch buffer followed by
 * x -= scratch would give, without the scratch buffer's write and read.
 * x: device fp32 [N], 16-byte aligned, read and written in place.  Other
 * arguments, preconditions, workspace and errors as decompress_accumulate.
 */
GCE_API int decompress_apply(const gce_table* table, int32_t W, const float* vals,
                             const int32_t* idx, const int32_t* k_or_rank, const float* P,
                             const float* Q, float scale, float* x, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * The step size of [MEM] Method for step t: eta_t = 8 / (mu (a + t)),
 * computed in double and rounded once to float into *eta (host memory).
 * GCE_ERR_ARG if eta is NULL, t < 0, mu <= 0, a + t <= 0 or the value
 * overflows float.
 */
GCE_API int gce_memsgd_eta(int64_t step, double mu, double a, float* eta);

/*
 * decompress_accumulate without a workspace (the pages have no counterpart:
 * this is a deployment variant, not part of the method).  For callers that
 * cannot allocate device memory for a workspace -- code running inside
 * another allocator such as a caching allocator's out-of-memory hook, code
 * whose device memory is reserved in full by its framework up front, or a
 * latency-critical loop that must not pay cudaMalloc's implicit device-wide
 * synchronisation.  Same arguments, results and preconditions as
 * decompress_accumulate minus ws / ws_bytes; it allocates nothing.  Its
 * scratch is a fixed 4 MiB array inside the library, reserved on every GPU
 * that loads the library until the process exits, so the table and W must
 * satisfy W x (decode spans of 1024 elements + layers) <= 1,048,576 (the
 * BERT-base table at W = 8 needs 856,088); larger ones return
 * GCE_ERR_WORKSPACE.  Every call made outside stream capture looks up the
 * current device's copy of the array (cudaGetSymbolAddress); a call made
 * while its stream is being captured reuses the address of the last call
 * outside capture on that device, so make the first call on a device before
 * any capture (a captured first call returns GCE_ERR_CUDA).  A device reset
 * (cudaDeviceReset) gives the device a new array: graphs captured before it
 * must not be replayed after it.  All calls share the one array: calls that
 * overlap on the GPU (two streams, two threads) race and must be serialised
 * by the caller.
 */
GCE_API int decompress_accumulate_noalloc(const gce_table* table, int32_t W, const float* vals,
                                          const int32_t* idx, const int32_t* k_or_rank,
                                          const float* P, const float* Q, float scale,
                                          float* out, void* stream);

/* Wait for `stream`, then read and clear the status word of workspace `ws`
 * (device pointer).  *status receives GCE_STATUS_* bits (0 = clean). */
GCE_API int gce_status(void* ws, void* stream, int32_t* status);

/* Number of kernels this library has launched since it was loaded. */
GCE_API uint64_t gce_launch_count(void);

/* Per-kernel timing.  Between gce_profile_start and gce_profile_stop every
 * launch of this library is bracketed by two CUDA events recorded on its
 * stream (at most 65536 launches are recorded).  gce_profile_stop waits for
 * those events and sums the elapsed time per kernel; gce_profile_count /
 * gce_profile_get then list (kernel name, total ms, launches).  Host-side
 * bookkeeping only; the kernels themselves are unchanged. */
GCE_API int gce_profile_start(void);
GCE_API int gce_profile_stop(void);
/* Restrict the recording to launches whose kernel name starts with
 * name_prefix (host string, copied); NULL or "" records every launch.  Fewer
 * events in the timed stream when only one kernel's time is wanted. */
GCE_API int gce_profile_only(const char* name_prefix);
GCE_API int gce_profile_count(void);
GCE_API int gce_profile_get(int32_t i, char* name, int32_t name_len, double* total_ms,
                            int64_t* launches);

/* Static description of a return code. */
GCE_API const char* gce_error_string(int code);

/* Tuning knob for the approximate pre-selection of top-k / rand-k: the safety
 * margin in standard deviations (default 6).  Results never depend on it;
 * small values only make the exact fallback run more often.  Values outside
 * (-100, 100) give GCE_ERR_ARG. */
GCE_API int gce_set_bracket_sigma(double sigma);

/*
 * Per-table settings.  gce_set_bracket_sigma, gce_set_randk_ahead,
 * gce_set_sign_ahead and gce_set_sign_emit_first set process-wide values
 * (atomically; a call reads them once, when it is made).  A table follows
 * them until one of its own options is set here; from then on calls on that
 * table use the table's value, whatever the process-wide one, so two tables
 * driven from two threads can hold different settings without sharing state.
 * Options and their values (as the process-wide setters check them):
 *   GCE_OPT_BRACKET_SIGMA    margin in standard deviations, in (-100, 100)
 *   GCE_OPT_RANDK_AHEAD      0 or 1
 *   GCE_OPT_SIGN_AHEAD       an integer in [-1, 2^20] (tiles; -1 = from L2)
 *   GCE_OPT_SIGN_EMIT_FIRST  0 or 1 (the bounded-wait test)
 * None of them changes any result.  A bad table, option or value gives
 * GCE_ERR_ARG.  gce_table_reset_option makes the table follow the
 * process-wide value again; gce_table_get_option writes the value a call on
 * the table would use now into *value (host memory).  Setting an option while
 * another thread runs a step on the same table is allowed; that step uses
 * either the old or the new value.
 */
#define GCE_OPT_BRACKET_SIGMA 0
#define GCE_OPT_RANDK_AHEAD 1
#define GCE_OPT_SIGN_AHEAD 2
#define GCE_OPT_SIGN_EMIT_FIRST 3
GCE_API int gce_table_set_option(gce_table* table, int32_t option, double value);
GCE_API int gce_table_reset_option(gce_table* table, int32_t option);
GCE_API int gce_table_get_option(const gce_table* table, int32_t option, double* value);

#ifdef __cplusplus
}
#endif
#endif /* GCE_H */
