/*
 * gce_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * gradient-compression step with error-feedback memory.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * execute this file.  Its only callers are the tests under tests/, the
 * smoke() check in __graft_entry__.py and the cpu_baseline / reference leg of
 * bench.py.  It shares no code, header, table or constant generator with the
 * CUDA library in gradient_compression_error_b200/csrc; the two are written
 * independently from the same definitions.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 *        (see oracle/build.py).  -ffp-contract=off keeps every float
 *        multiply and add separately rounded, which the Mem-SGD reading below
 *        requires.  Single-threaded; every function handles one unit
 *        (one worker's layer) and touches nothing global.
 *
 * Sources (page title, section):
 *   [MEM]  "Sparsified SGD with Memory", Method: the k-contraction operator
 *          comp_k, the memory m_t that accumulates what was not sent, and the
 *          update  g_t = comp_k(m_t + eta_t grad),
 *                  m_{t+1} = m_t + eta_t grad - g_t.
 *          Abstract / Motivation: top-k keeps the largest entries, rand-k
 *          keeps random entries.  Key results: 0 < k <= d.
 *   [ACC]  "Accordion: Adaptive Gradient Communication via Critical Learning
 *          Regime Identification", Method: per-layer gradient-norm rate of
 *          change detects critical regimes; inside one use the low-compression
 *          level l_low (e.g. higher rank / higher K), outside it the
 *          high-compression level l_high.
 *   [UTIL] "On the Utility of Gradient Compression in Distributed Training
 *          Systems", Method / Key results: PowerSGD is all-reduce compatible;
 *          payloads are summed across data-parallel workers.
 *   PowerSGD's steps are not printed on the pages (they only name it and its
 *   rank).  This oracle takes the standard single power-iteration step with a
 *   reused (warm-started) Q: P = M Q, orthonormalise P, Q' = M^T P,
 *   decompress P Q'^T, residual into memory.
 *
 * Readings where the pages are silent:
 *   - residual rounding: v = fl32(m + fl32(eta * g)), two separate roundings,
 *     no fused multiply-add;
 *   - top-k order: key = |v| taken as the float's bits with the sign cleared;
 *     larger key first, equal keys -> lower index first; the payload is
 *     emitted in ascending index; selected memory becomes +0.0f;
 *   - rand-k: uniform k-subset = the k smallest (hash key, index) pairs, the
 *     hash being SplitMix64 (Steele, Lea, Flood 2014) keyed by
 *     (seed, stream, worker, layer, step); values are not rescaled;
 *   - PowerSGD orientation: M is rows x cols row-major, P rows x r,
 *     Q cols x r (stored with row stride r_max); orthonormalisation is
 *     modified Gram-Schmidt in column order, a zero column stays zero;
 *   - Accordion: L2 norm of the raw gradient per layer at check steps, a
 *     missing previous norm (prev < 0) means "critical", rel change >= the
 *     threshold means "critical" (level LOW = l_low), else HIGH = l_high;
 *   - k from a fraction in parts per million: k = max(1, floor(n*ppm/1e6)).
 *   - signSGD with error feedback (or_ef_sign): the 1-bit payload is the
 *     float's sign bit, scaled by the layer's mean |p| (fp64 sum in index
 *     order, one rounding), so that the memory keeps p - s sign(p); the
 *     aggregate is the worker-order fp32 sum, or sign SGD's majority vote;
 *   - data-parallel PowerSGD (or_powersgd_dp): the all-reduces are sums over
 *     the workers -- P = sum_w M_w Q before orthonormalising, Q = the mean of
 *     the workers' Q_w = M_w^T P -- and each worker keeps its own error
 *     m_w = M_w - P Q_w^T; a DENSE layer sends the workers' mean residual
 *     (fp32 sum in worker order, then times fl32(1/W)).
 *
 * Pins of the generator readings (nothing on the pages fixes them; they
 * are pinned against their stated definitions by hand-worked values):
 *   or_splitmix64_output: the published SplitMix64 outputs;
 *   or_randk_base: its first fold is a published output (seed as the state,
 *   stream + 1 as the counter), the later folds a hand-worked chain
 *   (tests/golden/randk_base_hand.txt);
 *   or_q_entry: hand-worked values of the [-1, 1) mapping on published
 *   outputs (tests/golden/powersgd_init_q_hand.txt).
 * Parity unpinned: the rand-k subset distribution beyond uniformity (checked
 * statistically only).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG (-1)
#define OR_ERR_NOMEM (-2)

/* ------------------------------------------------------------------ */
/* Mem-SGD residual [MEM]: v = m + eta * g, two separate fp32 roundings. */
static float or_residual(float m, float eta, float g)
{
    float t = eta * g;   /* fl32(eta * g) */
    float v = m + t;     /* fl32(m + t)   */
    return v;
}

/* |v| ordering key: the IEEE-754 bits of v with the sign bit cleared.  For
 * finite floats this orders exactly like |v| (and +0 == -0). */
static uint32_t or_abs_key(float v)
{
    uint32_t b;
    memcpy(&b, &v, sizeof b);
    return b & 0x7FFFFFFFu;
}

typedef struct {
    uint32_t key;
    int32_t idx;
} or_pair;

/* larger key first; equal keys -> lower index first */
static int or_cmp_key_desc(const void* a, const void* b)
{
    const or_pair* x = (const or_pair*)a;
    const or_pair* y = (const or_pair*)b;
    if (x->key != y->key) return x->key > y->key ? -1 : 1;
    return x->idx < y->idx ? -1 : (x->idx > y->idx ? 1 : 0);
}

/* smaller key first; equal keys -> lower index first */
static int or_cmp_key_asc(const void* a, const void* b)
{
    const or_pair* x = (const or_pair*)a;
    const or_pair* y = (const or_pair*)b;
    if (x->key != y->key) return x->key < y->key ? -1 : 1;
    return x->idx < y->idx ? -1 : (x->idx > y->idx ? 1 : 0);
}

static int or_cmp_idx_asc(const void* a, const void* b)
{
    const or_pair* x = (const or_pair*)a;
    const or_pair* y = (const or_pair*)b;
    return x->idx < y->idx ? -1 : (x->idx > y->idx ? 1 : 0);
}

/* k from a fraction given in parts per million: max(1, floor(n*ppm/1e6)). */
int64_t or_k_from_ppm(int64_t n, int64_t ppm)
{
    int64_t k = (n * ppm) / 1000000;
    return k < 1 ? 1 : k;
}

/* Shared tail of top-k and rand-k: given v[] and the selection order already
 * applied to pairs[] (the first k pairs are the chosen set), emit the payload
 * in ascending index and write the memory update m = v - g. */
static void or_emit_selected(int64_t n, int64_t k, const float* v, or_pair* pairs,
                             float* m, float* vals, int32_t* idx)
{
    qsort(pairs, (size_t)k, sizeof(or_pair), or_cmp_idx_asc);
    for (int64_t i = 0; i < n; ++i) m[i] = v[i];          /* m_{t+1} = v - g ... */
    for (int64_t j = 0; j < k; ++j) {
        int32_t i = pairs[j].idx;
        vals[j] = v[i];                                   /* g_t,i = v_i on S   */
        idx[j] = i;
        m[i] = 0.0f;                                      /* ... = +0 on S      */
    }
}

/*
 * One Mem-SGD top-k step for one worker's layer [MEM].
 *   g[n]   gradient (read)          m[n]   memory (read, then overwritten)
 *   vals[k], idx[k]                 payload, ascending idx
 */
int or_ef_topk(int64_t n, int64_t k, float eta, const float* g, float* m,
               float* vals, int32_t* idx)
{
    if (n < 1 || k < 1 || k > n || n > INT32_MAX) return OR_ERR_ARG;
    float* v = (float*)malloc((size_t)n * sizeof(float));
    or_pair* pairs = (or_pair*)malloc((size_t)n * sizeof(or_pair));
    if (!v || !pairs) { free(v); free(pairs); return OR_ERR_NOMEM; }
    for (int64_t i = 0; i < n; ++i) {
        v[i] = or_residual(m[i], eta, g[i]);
        pairs[i].key = or_abs_key(v[i]);
        pairs[i].idx = (int32_t)i;
    }
    qsort(pairs, (size_t)n, sizeof(or_pair), or_cmp_key_desc);
    or_emit_selected(n, k, v, pairs, m, vals, idx);
    free(v);
    free(pairs);
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014): the state advances by the golden-ratio gamma
 * and each output is the state passed through the 64-bit finaliser. */
#define OR_GAMMA 0x9E3779B97F4A7C15ull

static uint64_t or_mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* The j-th output (j >= 1) of a SplitMix64 generator started at `state`. */
uint64_t or_splitmix64_output(uint64_t state, uint64_t j)
{
    return or_mix64(state + j * OR_GAMMA);
}

/* Per-unit base state: each of seed, stream, worker, layer, step is folded in
 * by taking the first SplitMix64 output from (previous + (value+1)*gamma). */
uint64_t or_randk_base(uint64_t seed, uint64_t stream, uint64_t worker,
                       uint64_t layer, uint64_t step)
{
    uint64_t h = or_splitmix64_output(seed, stream + 1);
    h = or_splitmix64_output(h, worker + 1);
    h = or_splitmix64_output(h, layer + 1);
    h = or_splitmix64_output(h, step + 1);
    return h;
}

/* rand-k key of coordinate i: high 32 bits of output i+1 from the base. */
uint32_t or_randk_key(uint64_t base, int64_t i)
{
    return (uint32_t)(or_splitmix64_output(base, (uint64_t)i + 1) >> 32);
}

/*
 * One Mem-SGD rand-k step for one worker's layer [MEM]: same update as top-k,
 * the chosen set is the k coordinates with the smallest (key, index).
 * Unscaled: g_i = v_i on the chosen set (comp_k stays a k-contraction).
 */
int or_ef_randk(int64_t n, int64_t k, float eta, const float* g, float* m,
                float* vals, int32_t* idx, uint64_t seed, uint64_t worker,
                uint64_t layer, uint64_t step)
{
    if (n < 1 || k < 1 || k > n || n > INT32_MAX) return OR_ERR_ARG;
    float* v = (float*)malloc((size_t)n * sizeof(float));
    or_pair* pairs = (or_pair*)malloc((size_t)n * sizeof(or_pair));
    if (!v || !pairs) { free(v); free(pairs); return OR_ERR_NOMEM; }
    uint64_t base = or_randk_base(seed, 0, worker, layer, step);
    for (int64_t i = 0; i < n; ++i) {
        v[i] = or_residual(m[i], eta, g[i]);
        pairs[i].key = or_randk_key(base, i);
        pairs[i].idx = (int32_t)i;
    }
    qsort(pairs, (size_t)n, sizeof(or_pair), or_cmp_key_asc);
    or_emit_selected(n, k, v, pairs, m, vals, idx);
    free(v);
    free(pairs);
    return OR_OK;
}

/* Uncompressed (1-D) layer: the payload is v itself and the memory empties. */
int or_dense(int64_t n, float eta, const float* g, float* m, float* payload)
{
    if (n < 1) return OR_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        payload[i] = or_residual(m[i], eta, g[i]);
        m[i] = 0.0f;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* One warm-start Q entry from a 64-bit generator output h: its top 24 bits,
 * read as an integer t in [0, 2^24), give x = t * 2^-23 - 1 in [-1, 1).
 * Both operations are exact in fp32 (t has 24 bits; the difference is a
 * multiple of 2^-23 below 1 in magnitude). */
float or_q_entry(uint64_t h)
{
    return (float)(h >> 40) * (1.0f / 8388608.0f) - 1.0f;
}

/* PowerSGD warm-start Q: entries uniform in [-1, 1) drawn from the hash with
 * stream 1 (or_q_entry of each output).  Q is cols x r_max, row-major;
 * element (c, j) uses counter c*r_max + j. */
int or_powersgd_init_q(int64_t cols, int64_t r_max, uint64_t seed, uint64_t worker,
                       uint64_t layer, float* Q)
{
    if (cols < 1 || r_max < 1) return OR_ERR_ARG;
    uint64_t base = or_randk_base(seed, 1, worker, layer, 0);
    for (int64_t c = 0; c < cols; ++c)
        for (int64_t j = 0; j < r_max; ++j)
            Q[c * r_max + j] =
                or_q_entry(or_splitmix64_output(base, (uint64_t)(c * r_max + j) + 1));
    return OR_OK;
}

/*
 * One PowerSGD rank-r step with error feedback for one worker's matrix.
 *   g, m      rows x cols row-major fp32; m is read and overwritten with the
 *             new residual M - P Q'^T
 *   Q         cols x r_max (row stride r_max); columns 0..r-1 are read as the
 *             warm start and overwritten with Q' = M^T P; others untouched
 *   P         rows x r_max (row stride r_max); columns 0..r-1 receive the
 *             orthonormalised P
 *   Mhat      optional rows x cols output of the decompressed P Q'^T
 * Arithmetic after M is formed runs in double and is stored as fp32.
 */
int or_powersgd(int64_t rows, int64_t cols, int64_t r, int64_t r_max, float eta,
                const float* g, float* m, float* Q, float* P, float* Mhat)
{
    if (rows < 1 || cols < 1 || r < 1 || r > r_max || r > rows || r > cols)
        return OR_ERR_ARG;
    int64_t n = rows * cols;
    double* M = (double*)malloc((size_t)n * sizeof(double));
    double* Pd = (double*)malloc((size_t)(rows * r) * sizeof(double));
    double* Qd = (double*)malloc((size_t)(cols * r) * sizeof(double));
    if (!M || !Pd || !Qd) { free(M); free(Pd); free(Qd); return OR_ERR_NOMEM; }

    /* M = m + eta*grad, formed exactly as the Mem-SGD residual */
    for (int64_t i = 0; i < n; ++i) M[i] = (double)or_residual(m[i], eta, g[i]);

    /* P = M Q */
    for (int64_t a = 0; a < rows; ++a)
        for (int64_t j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t c = 0; c < cols; ++c) s += M[a * cols + c] * (double)Q[c * r_max + j];
            Pd[a * r + j] = s;
        }

    /* modified Gram-Schmidt over the columns of P, in order 0..r-1 */
    for (int64_t j = 0; j < r; ++j) {
        for (int64_t i = 0; i < j; ++i) {
            double d = 0.0;
            for (int64_t a = 0; a < rows; ++a) d += Pd[a * r + i] * Pd[a * r + j];
            for (int64_t a = 0; a < rows; ++a) Pd[a * r + j] -= d * Pd[a * r + i];
        }
        double nn = 0.0;
        for (int64_t a = 0; a < rows; ++a) nn += Pd[a * r + j] * Pd[a * r + j];
        double nu = sqrt(nn);
        for (int64_t a = 0; a < rows; ++a) Pd[a * r + j] = nu > 0.0 ? Pd[a * r + j] / nu : 0.0;
    }

    /* Q' = M^T P */
    for (int64_t c = 0; c < cols; ++c)
        for (int64_t j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t a = 0; a < rows; ++a) s += M[a * cols + c] * Pd[a * r + j];
            Qd[c * r + j] = s;
        }

    /* decompress P Q'^T, residual into memory */
    for (int64_t a = 0; a < rows; ++a)
        for (int64_t c = 0; c < cols; ++c) {
            double s = 0.0;
            for (int64_t j = 0; j < r; ++j) s += Pd[a * r + j] * Qd[c * r + j];
            m[a * cols + c] = (float)(M[a * cols + c] - s);
            if (Mhat) Mhat[a * cols + c] = (float)s;
        }

    for (int64_t a = 0; a < rows; ++a)
        for (int64_t j = 0; j < r; ++j) P[a * r_max + j] = (float)Pd[a * r + j];
    for (int64_t c = 0; c < cols; ++c)
        for (int64_t j = 0; j < r; ++j) Q[c * r_max + j] = (float)Qd[c * r + j];

    free(M);
    free(Pd);
    free(Qd);
    return OR_OK;
}

/*
 * Data-parallel PowerSGD step for one matrix over W workers ([UTIL] Key
 * results: PowerSGD is all-reduce compatible; the all-reduces are sums over
 * the workers).  Every worker shares the warm start Q and the orthonormal P:
 *   M_w = fl32(m_w + fl32(eta*g_w))                 (the Mem-SGD residual)
 *   P   = sum_w M_w Q                               (all-reduce of P)
 *   P  <- modified Gram-Schmidt in column order
 *   Q_w = M_w^T P;  m_w <- M_w - P Q_w^T            (each worker's own error)
 *   Q   = (1/W) sum_w Q_w                           (all-reduce mean of Q)
 * so that P Q^T is the mean of the workers' decompressed updates.
 *   g, m   W x rows x cols fp32 (worker-major); m overwritten
 *   Q      cols x r_max shared warm start; columns 0..r-1 overwritten
 *   P      rows x r_max; columns 0..r-1 receive the orthonormal P
 * Arithmetic after the M_w are formed runs in double; P, Q and m are stored
 * as fp32.
 */
/* The data-parallel step in the order its two all-reduces cut it into:
 *   phase 1, each worker:  M_w = m_w + eta*grad_w (stored back in m_w, exact
 *                          in fp32), P_w = M_w Q  (fp64, rows x r);
 *   all-reduce:            P = sum_w P_w  (fp64, worker order from 0);
 *   orthonormalise P       (modified Gram-Schmidt, as or_powersgd);
 *   phase 2, each worker:  Q_w = M_w^T P (fp64), m_w = M_w - P Q_w^T;
 *   all-reduce:            Q = (float)(sum_w Q_w / W)  (fp64, worker order). */
int or_powersgd_dp_p(int64_t rows, int64_t cols, int64_t r, int64_t r_max, float eta,
                     const float* g, float* m, const float* Q, double* Pw)
{
    if (rows < 1 || cols < 1 || r < 1 || r > r_max || r > rows || r > cols) return OR_ERR_ARG;
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i) m[i] = or_residual(m[i], eta, g[i]);
    for (int64_t a = 0; a < rows; ++a)
        for (int64_t j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t c = 0; c < cols; ++c) s += (double)m[a * cols + c] * (double)Q[c * r_max + j];
            Pw[a * r + j] = s;
        }
    return OR_OK;
}

/* Modified Gram-Schmidt over the r columns of P (rows x r, fp64) in place,
 * in column order; a zero column stays zero. */
void or_mgs(int64_t rows, int64_t r, double* Pd)
{
    for (int64_t j = 0; j < r; ++j) {
        for (int64_t i = 0; i < j; ++i) {
            double d = 0.0;
            for (int64_t a = 0; a < rows; ++a) d += Pd[a * r + i] * Pd[a * r + j];
            for (int64_t a = 0; a < rows; ++a) Pd[a * r + j] -= d * Pd[a * r + i];
        }
        double nn = 0.0;
        for (int64_t a = 0; a < rows; ++a) nn += Pd[a * r + j] * Pd[a * r + j];
        double nu = sqrt(nn);
        for (int64_t a = 0; a < rows; ++a) Pd[a * r + j] = nu > 0.0 ? Pd[a * r + j] / nu : 0.0;
    }
}

/* phase 2 of one worker: m holds M_w on entry and the residual on return;
 * Qw (cols x r, fp64) receives M_w^T P. */
int or_powersgd_dp_q(int64_t rows, int64_t cols, int64_t r, const double* Pd, float* m,
                     double* Qw)
{
    if (rows < 1 || cols < 1 || r < 1 || r > rows || r > cols) return OR_ERR_ARG;
    for (int64_t c = 0; c < cols; ++c)
        for (int64_t j = 0; j < r; ++j) {
            double s = 0.0;
            for (int64_t a = 0; a < rows; ++a) s += (double)m[a * cols + c] * Pd[a * r + j];
            Qw[c * r + j] = s;
        }
    for (int64_t a = 0; a < rows; ++a)
        for (int64_t c = 0; c < cols; ++c) {
            double s = 0.0;
            for (int64_t j = 0; j < r; ++j) s += Pd[a * r + j] * Qw[c * r + j];
            m[a * cols + c] = (float)((double)m[a * cols + c] - s);
        }
    return OR_OK;
}

int or_powersgd_dp(int64_t W, int64_t rows, int64_t cols, int64_t r, int64_t r_max, float eta,
                   const float* g, float* m, float* Q, float* P)
{
    if (W < 1 || rows < 1 || cols < 1 || r < 1 || r > r_max || r > rows || r > cols)
        return OR_ERR_ARG;
    int64_t n = rows * cols;
    double* Pd = (double*)calloc((size_t)(rows * r), sizeof(double));
    double* Pw = (double*)malloc((size_t)(rows * r) * sizeof(double));
    double* Qw = (double*)malloc((size_t)(cols * r) * sizeof(double));
    double* Qsum = (double*)calloc((size_t)(cols * r), sizeof(double));
    if (!Pd || !Pw || !Qw || !Qsum) { free(Pd); free(Pw); free(Qw); free(Qsum); return OR_ERR_NOMEM; }

    /* P = sum over workers of M_w Q */
    for (int64_t w = 0; w < W; ++w) {
        or_powersgd_dp_p(rows, cols, r, r_max, eta, g + w * n, m + w * n, Q, Pw);
        for (int64_t i = 0; i < rows * r; ++i) Pd[i] += Pw[i];
    }
    or_mgs(rows, r, Pd);

    /* each worker: Q_w = M_w^T P, its residual, and the running sum of Q_w */
    for (int64_t w = 0; w < W; ++w) {
        or_powersgd_dp_q(rows, cols, r, Pd, m + w * n, Qw);
        for (int64_t i = 0; i < cols * r; ++i) Qsum[i] += Qw[i];
    }

    for (int64_t a = 0; a < rows; ++a)
        for (int64_t j = 0; j < r; ++j) P[a * r_max + j] = (float)Pd[a * r + j];
    for (int64_t c = 0; c < cols; ++c)
        for (int64_t j = 0; j < r; ++j) Q[c * r_max + j] = (float)(Qsum[c * r + j] / (double)W);

    free(Pd);
    free(Pw);
    free(Qw);
    free(Qsum);
    return OR_OK;
}

/*
 * Data-parallel uncompressed (DENSE) layer: the all-reduce mean of the
 * workers' residuals, payload = fl32(fl32(sum_w v_w) * fl32(1/W)) with the
 * sum in worker order from +0.0; every worker's memory becomes +0.0.
 *   g, m  W x n (worker-major); out n.
 */
int or_dense_dp(int64_t W, int64_t n, float eta, const float* g, float* m, float* out)
{
    if (W < 1 || n < 0) return OR_ERR_ARG;
    float inv = 1.0f / (float)W;
    for (int64_t i = 0; i < n; ++i) {
        float s = 0.0f;
        for (int64_t w = 0; w < W; ++w) {
            s = s + or_residual(m[w * n + i], eta, g[w * n + i]);
            m[w * n + i] = 0.0f;
        }
        out[i] = s * inv;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ */
/* signSGD with error feedback ([UTIL] Method / Key results evaluate sign
 * SGD, whose 1-bit payload cannot be all-reduced and is gathered; [MEM]
 * Method gives the memory).  One worker's layer of n elements:
 *   p_i   = fl32(m_i + fl32(eta * g_i))              (the Mem-SGD residual)
 *   s     = fl32( (sum_i |p_i|, in double, index order) / n )
 *   b_i   = sign bit of p_i (1 for negative, -0 included)
 *   g_i   = s with b_i's sign;  m_i <- fl32(p_i - g_i)
 * words: ceil(n/32) uint32, bit (i mod 32) of word i/32 is b_i; the unused
 * high bits of the last word are 0.  *scale receives s. */
int or_ef_sign(int64_t n, float eta, const float* g, float* m, float* scale, uint32_t* words)
{
    if (n < 1) return OR_ERR_ARG;
    double l1 = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        float p = or_residual(m[i], eta, g[i]);
        l1 += fabs((double)p);
    }
    float sc = (float)(l1 / (double)n);
    for (int64_t j = 0; j < (n + 31) / 32; ++j) words[j] = 0u;
    for (int64_t i = 0; i < n; ++i) {
        float p = or_residual(m[i], eta, g[i]);
        int neg = signbit(p) ? 1 : 0;
        if (neg) words[i / 32] |= 1u << (i % 32);
        m[i] = neg ? p + sc : p - sc;
    }
    *scale = sc;
    return OR_OK;
}

/* out[i] += (bit i set ? -scale : scale) for one worker's sign payload. */
void or_accum_sign(int64_t n, float scale, const uint32_t* words, float* out)
{
    for (int64_t i = 0; i < n; ++i) {
        int neg = (words[i / 32] >> (i % 32)) & 1u;
        out[i] = out[i] + (neg ? -scale : scale);
    }
}

/* Majority vote over W workers' sign payloads (sign SGD's aggregation):
 * out[i] = out_scale * sign(#positive - #negative), 0 on a tie. */
void or_vote_sign(int64_t W, int64_t n, int64_t words_per_worker, const uint32_t* words,
                  float out_scale, float* out)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = 0;
        for (int64_t w = 0; w < W; ++w)
            c += ((words[w * words_per_worker + i / 32] >> (i % 32)) & 1u) ? -1 : 1;
        out[i] = c > 0 ? out_scale : (c < 0 ? -out_scale : 0.0f);
    }
}

/* ------------------------------------------------------------------ */
/* Accordion [ACC]: L2 norm of one layer's raw gradient, summed in index
 * order in double. */
/* A layer's sum of squares, fp64 in index order; its square root is the
 * layer's gradient norm [ACC]. */
double or_layer_sumsq(int64_t n, const float* g)
{
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += (double)g[i] * (double)g[i];
    return s;
}

double or_layer_norm(int64_t n, const float* g)
{
    return sqrt(or_layer_sumsq(n, g));
}

/*
 * Accordion decision for one layer at a check step [ACC].
 *   s_prev < 0 means "no earlier check": the layer is treated as critical.
 *   rel = |s_prev - s_cur| / s_prev (s_prev == 0: rel = 0 if s_cur == 0,
 *   else +inf).  rel >= threshold -> LOW (0, l_low: less compression),
 *   else HIGH (1, l_high: more compression).
 */
int32_t or_accordion_decide(double s_prev, double s_cur, double threshold)
{
    if (s_prev < 0.0) return 0;
    double rel;
    if (s_prev == 0.0) rel = (s_cur == 0.0) ? 0.0 : INFINITY;
    else rel = fabs(s_prev - s_cur) / s_prev;
    return rel >= threshold ? 0 : 1;
}

/* ------------------------------------------------------------------ */
/* Decode side [UTIL]: the aggregate of the workers' payloads, summed in worker
 * order from +0.0 in fp32, then multiplied by `scale`.  These three helpers
 * add one worker's payload into one layer's slice of the dense output. */
void or_accum_sparse(int64_t k, const float* vals, const int32_t* idx, float* out)
{
    for (int64_t j = 0; j < k; ++j) out[idx[j]] = out[idx[j]] + vals[j];
}

void or_accum_dense(int64_t n, const float* payload, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = out[i] + payload[i];
}

/* out += P Q^T for one worker (P rows x r, Q cols x r, row stride r_max);
 * each entry is formed in double and rounded once before the fp32 add. */
void or_accum_lowrank(int64_t rows, int64_t cols, int64_t r, int64_t r_max,
                      const float* P, const float* Q, float* out)
{
    for (int64_t a = 0; a < rows; ++a)
        for (int64_t c = 0; c < cols; ++c) {
            double s = 0.0;
            for (int64_t j = 0; j < r; ++j) s += (double)P[a * r_max + j] * (double)Q[c * r_max + j];
            out[a * cols + c] = out[a * cols + c] + (float)s;
        }
}

void or_scale(int64_t n, float scale, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = out[i] * scale;
}
