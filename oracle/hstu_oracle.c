/*
 * CPU oracle for the HSTU transduction layer and its jagged pointwise attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library or its Python binding may
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or table with the CUDA path.
 *
 * Plain, slow and obviously correct: every function is the definition written
 * out as loops, accumulated in double precision, over host arrays.
 *
 * What it computes (sources):
 *  - "NVIDIA generative recommenders" summary, section "HSTU Architecture":
 *    softmax replaced by SiLU weighting, a relative attention bias, and an
 *    elementwise gate before the output projection.
 *  - "DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf",
 *    section "Model Architecture": projection -> pointwise attention with a
 *    bias from positional and temporal distance -> gated transformation;
 *    one causal block over a chronological sequence with the candidate
 *    appended; section "Computation Cost Analysis" (Table 7 and the text under
 *    it): only the lower triangle is evaluated, backward gives dQ, dK, dV.
 *  - The per-head formula: s_ij = q_i.k_j + rab_pos(p_i - p_j)
 *    + rab_time(bucket(t_i - t_j)); P_ij = SiLU(s_ij)/N on visible pairs, else 0;
 *    O_i = sum_j P_ij v_j; layer = f2(LayerNorm(O) * U) with
 *    [U,V,Q,K] = SiLU(f1(X)).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - bucket(dt) = min(NB-1, floor(log2(1 + max(dt, 0)))) on integer seconds,
 *    computed as bit_length(1 + dt) - 1 with integers only;
 *  - positional index = clamp(p_i - p_j, lo, hi) - lo;
 *  - the last n_t tokens of a sequence are candidates: they sit at position
 *    L - n_t, see every history token and themselves only; history tokens see
 *    j <= i;
 *  - bias tables are shared by all heads; LayerNorm is over the h*d_v features
 *    of a token with affine gamma/beta; no residual connection.
 *
 * Layouts: q,k [T,H,dqk], v,o [T,H,dv] row-major; seq_offsets int64 [B+1];
 * timestamps int64 [T]; num_targets int32 [B] or NULL.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- index functions --------------------------------------------------- */

static int bit_length_u64(uint64_t x)
{
    int n = 0;
    while (x) {
        n++;
        x >>= 1;
    }
    return n;
}

/* Temporal bucket of the pair (i, j): log2 buckets of the elapsed seconds. */
int oracle_time_bucket(int64_t t_i, int64_t t_j, int num_buckets)
{
    int64_t dt = t_i - t_j;
    if (dt < 0)
        dt = 0;
    int b = bit_length_u64((uint64_t)dt + 1u) - 1;
    return b < num_buckets - 1 ? b : num_buckets - 1;
}

/* Positional index into rab_pos for relative distance p_i - p_j. */
int oracle_pos_index(int64_t p_i, int64_t p_j, int pos_lo, int pos_hi)
{
    int64_t d = p_i - p_j;
    if (d < pos_lo)
        d = pos_lo;
    if (d > pos_hi)
        d = pos_hi;
    return (int)(d - pos_lo);
}

/*
 * Readings selected per call (set by the caller, reset after it):
 *  - g_cand_own_index: 0, the candidates of a sequence share the position
 *    L - n_t, the slot appended after the history (the DLRMv4 page, "Model
 *    Architecture": the candidate item is appended); 1, each candidate keeps its
 *    own index i as its position;
 *  - g_per_head_tables: 0, rab_pos and rab_time are shared by the heads; 1,
 *    each head h has its own tables, rab_pos[h][e] and rab_time[h][k], and its
 *    own table gradients.
 */
static int64_t g_cand_own_index = 0, g_per_head_tables = 0;

void oracle_set_variants(int64_t cand_own_index, int64_t per_head_tables)
{
    g_cand_own_index = cand_own_index;
    g_per_head_tables = per_head_tables;
}

/* Position of local token i in a sequence of length L with n_t candidates. */
static int64_t token_pos(int64_t i, int64_t L, int64_t n_t)
{
    int64_t hist = L - n_t;
    return (i < hist || g_cand_own_index) ? i : hist;
}

/* Is key j visible from query i (local indices)? */
int oracle_visible(int64_t i, int64_t j, int64_t L, int64_t n_t)
{
    int64_t hist = L - n_t;
    if (i < hist)
        return j <= i;
    return j < hist || j == i;
}

/*
 * Semi-local attention (the ULTRA-HSTU review in the pages: attention over a
 * local and a global window instead of the full causal mask).  With
 * local > 0, a pair the rule above keeps survives iff the query is less than
 * `local` positions after the key, or the key is one of the first `global`
 * tokens of the sequence.  local <= 0 keeps the full mask.
 */
int oracle_visible_sl(int64_t i, int64_t j, int64_t L, int64_t n_t, int64_t local, int64_t global)
{
    if (!oracle_visible(i, j, L, n_t))
        return 0;
    if (local <= 0)
        return 1;
    return token_pos(i, L, n_t) - token_pos(j, L, n_t) < local || j < global;
}

/* windows applied by the attention functions below (set per call by the caller) */
static int64_t g_local_window = 0, g_global_window = 0;

void oracle_set_windows(int64_t local, int64_t global)
{
    g_local_window = local;
    g_global_window = global;
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

static double silu_grad(double x)
{
    double s = 1.0 / (1.0 + exp(-x));
    return s * (1.0 + x * (1.0 - s));
}

typedef struct {
    int num_seqs, num_heads, d_qk, d_v;
    const int64_t *seq_offsets;
    const int64_t *timestamps;
    const int32_t *num_targets; /* may be NULL */
    const double *rab_pos;
    int pos_lo, pos_hi;
    const double *rab_time;
    int num_buckets;
    double inv_n;
    int64_t local_window, global_window;
} attn_args;

static int64_t seq_targets(const attn_args *a, int b)
{
    return a->num_targets ? (int64_t)a->num_targets[b] : 0;
}

/* Pre-activation score of pair (i, j) of sequence starting at row s0, head h. */
static double score(const attn_args *a, const double *q, const double *k, int64_t s0,
                    int64_t L, int64_t n_t, int h, int64_t i, int64_t j)
{
    const double *qi = q + ((s0 + i) * a->num_heads + h) * a->d_qk;
    const double *kj = k + ((s0 + j) * a->num_heads + h) * a->d_qk;
    double s = 0.0;
    for (int c = 0; c < a->d_qk; c++)
        s += qi[c] * kj[c];
    int pi = oracle_pos_index(token_pos(i, L, n_t), token_pos(j, L, n_t), a->pos_lo, a->pos_hi);
    int bt = oracle_time_bucket(a->timestamps[s0 + i], a->timestamps[s0 + j], a->num_buckets);
    /* per-head tables: head h's rows of rab_pos [H][npos] and rab_time [H][NB] */
    const int64_t hp = g_per_head_tables ? (int64_t)h * (a->pos_hi - a->pos_lo + 1) : 0;
    const int64_t ht = g_per_head_tables ? (int64_t)h * a->num_buckets : 0;
    return s + a->rab_pos[hp + pi] + a->rab_time[ht + bt];
}

/* One output row: O[s0+i, h, :] = sum over visible j of SiLU(s_ij)/N * v_j. */
static void fwd_row(const attn_args *a, const double *q, const double *k, const double *v,
                    int64_t s0, int64_t L, int64_t n_t, int h, int64_t i, double *o_row)
{
    for (int c = 0; c < a->d_v; c++)
        o_row[c] = 0.0;
    for (int64_t j = 0; j < L; j++) {
        if (!oracle_visible_sl(i, j, L, n_t, a->local_window, a->global_window))
            continue;
        double p = silu(score(a, q, k, s0, L, n_t, h, i, j)) * a->inv_n;
        const double *vj = v + ((s0 + j) * a->num_heads + h) * a->d_v;
        for (int c = 0; c < a->d_v; c++)
            o_row[c] += p * vj[c];
    }
}

static void fill_args(attn_args *a, int num_seqs, const int64_t *seq_offsets,
                      const int32_t *num_targets, int num_heads, int d_qk, int d_v,
                      const int64_t *timestamps, const double *rab_pos, int pos_lo, int pos_hi,
                      const double *rab_time, int num_buckets, double inv_n)
{
    a->num_seqs = num_seqs;
    a->seq_offsets = seq_offsets;
    a->num_targets = num_targets;
    a->num_heads = num_heads;
    a->d_qk = d_qk;
    a->d_v = d_v;
    a->timestamps = timestamps;
    a->rab_pos = rab_pos;
    a->pos_lo = pos_lo;
    a->pos_hi = pos_hi;
    a->rab_time = rab_time;
    a->num_buckets = num_buckets;
    a->inv_n = inv_n;
    a->local_window = g_local_window;
    a->global_window = g_global_window;
}

static void set_threads(int num_threads)
{
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
}

/* ---- attention forward -------------------------------------------------- */

void oracle_attn_fwd(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                     int num_heads, int d_qk, int d_v, const double *q, const double *k,
                     const double *v, const int64_t *timestamps, const double *rab_pos,
                     int pos_lo, int pos_hi, const double *rab_time, int num_buckets,
                     double inv_n, double *out, int num_threads)
{
    attn_args a;
    fill_args(&a, num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, timestamps,
              rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n);
    set_threads(num_threads);
    int64_t tasks = (int64_t)num_seqs * num_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < tasks; task++) {
        int b = (int)(task / num_heads), h = (int)(task % num_heads);
        int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0, n_t = seq_targets(&a, b);
        for (int64_t i = 0; i < L; i++)
            fwd_row(&a, q, k, v, s0, L, n_t, h, i, out + ((s0 + i) * num_heads + h) * d_v);
    }
}

/* Sequence holding global row r (seq_offsets is non-decreasing). */
static int seq_of_row(const int64_t *seq_offsets, int num_seqs, int64_t r)
{
    int b = 0;
    while (b + 1 < num_seqs && seq_offsets[b + 1] <= r)
        b++;
    return b;
}

/* Forward for selected global rows only: out_rows is [n_rows, H, dv]. */
void oracle_attn_fwd_rows(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                          int num_heads, int d_qk, int d_v, const double *q, const double *k,
                          const double *v, const int64_t *timestamps, const double *rab_pos,
                          int pos_lo, int pos_hi, const double *rab_time, int num_buckets,
                          double inv_n, int64_t n_rows, const int64_t *rows, double *out_rows,
                          int num_threads)
{
    attn_args a;
    fill_args(&a, num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, timestamps,
              rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n);
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < n_rows * num_heads; task++) {
        int64_t r = task / num_heads;
        int h = (int)(task % num_heads);
        int b = seq_of_row(seq_offsets, num_seqs, rows[r]);
        int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0, n_t = seq_targets(&a, b);
        fwd_row(&a, q, k, v, s0, L, n_t, h, rows[r] - s0, out_rows + (r * num_heads + h) * d_v);
    }
}

/* ---- visible pairs per bias entry --------------------------------------- */

/*
 * How many visible pairs of the batch land on each relative-bias entry (one
 * head): pos_counts [pos_hi - pos_lo + 1] and time_counts [num_buckets],
 * int64, overwritten.  Every pair goes through the same visibility rule (with
 * the semi-local windows local, global) and index functions as the attention.
 * When every visible pair carries the same score gradient g, the gradient of
 * rab_pos[e] is H g pos_counts[e] and that of rab_time[k] is H g time_counts[k]
 * (the tables are shared by the heads).  Sequences run in parallel, each into
 * its own count arrays, added up in sequence order.
 */
void oracle_bias_pair_counts(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                             const int64_t *timestamps, int pos_lo, int pos_hi, int num_buckets,
                             int64_t local, int64_t global, int64_t *pos_counts, int64_t *time_counts,
                             int num_threads)
{
    const int npos = pos_hi - pos_lo + 1;
    int64_t *per_pos = (int64_t *)calloc((size_t)(num_seqs > 0 ? num_seqs : 1) * npos, sizeof(int64_t));
    int64_t *per_time = (int64_t *)calloc((size_t)(num_seqs > 0 ? num_seqs : 1) * num_buckets, sizeof(int64_t));
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < num_seqs; b++) {
        const int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0;
        const int64_t n_t = num_targets ? (int64_t)num_targets[b] : 0;
        int64_t *pc = per_pos + (size_t)b * npos, *tc = per_time + (size_t)b * num_buckets;
        for (int64_t i = 0; i < L; i++)
            for (int64_t j = 0; j < L; j++) {
                if (!oracle_visible_sl(i, j, L, n_t, local, global))
                    continue;
                pc[oracle_pos_index(token_pos(i, L, n_t), token_pos(j, L, n_t), pos_lo, pos_hi)]++;
                tc[oracle_time_bucket(timestamps[s0 + i], timestamps[s0 + j], num_buckets)]++;
            }
    }
    for (int e = 0; e < npos; e++)
        pos_counts[e] = 0;
    for (int k = 0; k < num_buckets; k++)
        time_counts[k] = 0;
    for (int b = 0; b < num_seqs; b++) {
        for (int e = 0; e < npos; e++)
            pos_counts[e] += per_pos[(size_t)b * npos + e];
        for (int k = 0; k < num_buckets; k++)
            time_counts[k] += per_time[(size_t)b * num_buckets + k];
    }
    free(per_pos);
    free(per_time);
}

/* ---- attention backward ------------------------------------------------- */
/*
 * Exact derivatives of the forward above for the loss sum(O * dO):
 *   dP_ij = dO_i . v_j;  dS_ij = dP_ij * SiLU'(s_ij) / N on visible pairs;
 *   dQ_i = sum_j dS_ij k_j;  dK_j = sum_i dS_ij q_i;  dV_j = sum_i P_ij dO_i;
 *   d_rab_pos[idx(i,j)] and d_rab_time[bucket(i,j)] collect dS_ij over all
 *   pairs and heads (over the pairs of head h alone into head h's rows with
 *   per-head tables).  Gradient outputs are overwritten, not accumulated.
 */
void oracle_attn_bwd(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                     int num_heads, int d_qk, int d_v, const double *q, const double *k,
                     const double *v, const int64_t *timestamps, const double *rab_pos,
                     int pos_lo, int pos_hi, const double *rab_time, int num_buckets,
                     double inv_n, const double *dout, double *dq, double *dk, double *dv,
                     double *d_rab_pos, double *d_rab_time, int num_threads)
{
    attn_args a;
    fill_args(&a, num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, timestamps,
              rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n);
    set_threads(num_threads);
    int npos = pos_hi - pos_lo + 1;
    int64_t tasks = (int64_t)num_seqs * num_heads;
    /* one private bias-gradient pair per task, summed afterwards in task order */
    double *pos_part = (double *)calloc((size_t)(tasks > 0 ? tasks : 1) * npos, sizeof(double));
    double *time_part = (double *)calloc((size_t)(tasks > 0 ? tasks : 1) * num_buckets, sizeof(double));
    int64_t T = seq_offsets[num_seqs];
    memset(dq, 0, sizeof(double) * (size_t)T * num_heads * d_qk);
    memset(dk, 0, sizeof(double) * (size_t)T * num_heads * d_qk);
    memset(dv, 0, sizeof(double) * (size_t)T * num_heads * d_v);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < tasks; task++) {
        int b = (int)(task / num_heads), h = (int)(task % num_heads);
        int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0, n_t = seq_targets(&a, b);
        double *pp = pos_part + task * npos, *tp = time_part + task * num_buckets;
        for (int64_t i = 0; i < L; i++) {
            const double *qi = q + ((s0 + i) * num_heads + h) * d_qk;
            const double *doi = dout + ((s0 + i) * num_heads + h) * d_v;
            double *dqi = dq + ((s0 + i) * num_heads + h) * d_qk;
            for (int64_t j = 0; j < L; j++) {
                if (!oracle_visible_sl(i, j, L, n_t, a.local_window, a.global_window))
                    continue;
                const double *kj = k + ((s0 + j) * num_heads + h) * d_qk;
                const double *vj = v + ((s0 + j) * num_heads + h) * d_v;
                double *dkj = dk + ((s0 + j) * num_heads + h) * d_qk;
                double *dvj = dv + ((s0 + j) * num_heads + h) * d_v;
                double s = score(&a, q, k, s0, L, n_t, h, i, j);
                double p = silu(s) * inv_n;
                double dp = 0.0;
                for (int c = 0; c < d_v; c++)
                    dp += doi[c] * vj[c];
                double ds = dp * silu_grad(s) * inv_n;
                for (int c = 0; c < d_qk; c++) {
                    dqi[c] += ds * kj[c];
                    dkj[c] += ds * qi[c];
                }
                for (int c = 0; c < d_v; c++)
                    dvj[c] += p * doi[c];
                pp[oracle_pos_index(token_pos(i, L, n_t), token_pos(j, L, n_t), pos_lo, pos_hi)] += ds;
                tp[oracle_time_bucket(timestamps[s0 + i], timestamps[s0 + j], num_buckets)] += ds;
            }
        }
    }
    const int nh = g_per_head_tables ? num_heads : 1;
    for (int64_t e = 0; e < (int64_t)nh * npos; e++)
        d_rab_pos[e] = 0.0;
    for (int64_t e = 0; e < (int64_t)nh * num_buckets; e++)
        d_rab_time[e] = 0.0;
    for (int64_t task = 0; task < tasks; task++) {
        const int64_t h = g_per_head_tables ? task % num_heads : 0;
        for (int e = 0; e < npos; e++)
            d_rab_pos[h * npos + e] += pos_part[task * npos + e];
        for (int e = 0; e < num_buckets; e++)
            d_rab_time[h * num_buckets + e] += time_part[task * num_buckets + e];
    }
    free(pos_part);
    free(time_part);
}

/*
 * Backward for sampled rows: dq for query rows `q_rows`, dk/dv for key rows
 * `k_rows` (global token indices), each from its own sums over the pairs that
 * involve it.  Outputs are [n, H, d].
 */
void oracle_attn_bwd_rows(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                          int num_heads, int d_qk, int d_v, const double *q, const double *k,
                          const double *v, const int64_t *timestamps, const double *rab_pos,
                          int pos_lo, int pos_hi, const double *rab_time, int num_buckets,
                          double inv_n, const double *dout, int64_t n_q, const int64_t *q_rows,
                          double *dq_rows, int64_t n_k, const int64_t *k_rows, double *dk_rows,
                          double *dv_rows, int num_threads)
{
    attn_args a;
    fill_args(&a, num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, timestamps,
              rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n);
    set_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < (n_q + n_k) * num_heads; task++) {
        int64_t r = task / num_heads;
        int h = (int)(task % num_heads);
        if (r < n_q) {
            int64_t g = q_rows[r];
            int b = seq_of_row(seq_offsets, num_seqs, g);
            int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0, n_t = seq_targets(&a, b);
            int64_t i = g - s0;
            const double *doi = dout + (g * num_heads + h) * d_v;
            double *out = dq_rows + (r * num_heads + h) * d_qk;
            for (int c = 0; c < d_qk; c++)
                out[c] = 0.0;
            for (int64_t j = 0; j < L; j++) {
                if (!oracle_visible_sl(i, j, L, n_t, a.local_window, a.global_window))
                    continue;
                const double *kj = k + ((s0 + j) * num_heads + h) * d_qk;
                const double *vj = v + ((s0 + j) * num_heads + h) * d_v;
                double s = score(&a, q, k, s0, L, n_t, h, i, j);
                double dp = 0.0;
                for (int c = 0; c < d_v; c++)
                    dp += doi[c] * vj[c];
                double ds = dp * silu_grad(s) * inv_n;
                for (int c = 0; c < d_qk; c++)
                    out[c] += ds * kj[c];
            }
        } else {
            int64_t rk = r - n_q;
            int64_t g = k_rows[rk];
            int b = seq_of_row(seq_offsets, num_seqs, g);
            int64_t s0 = seq_offsets[b], L = seq_offsets[b + 1] - s0, n_t = seq_targets(&a, b);
            int64_t j = g - s0;
            const double *vj = v + (g * num_heads + h) * d_v;
            double *okk = dk_rows + (rk * num_heads + h) * d_qk;
            double *ovv = dv_rows + (rk * num_heads + h) * d_v;
            for (int c = 0; c < d_qk; c++)
                okk[c] = 0.0;
            for (int c = 0; c < d_v; c++)
                ovv[c] = 0.0;
            for (int64_t i = 0; i < L; i++) {
                if (!oracle_visible_sl(i, j, L, n_t, a.local_window, a.global_window))
                    continue;
                const double *qi = q + ((s0 + i) * num_heads + h) * d_qk;
                const double *doi = dout + ((s0 + i) * num_heads + h) * d_v;
                double s = score(&a, q, k, s0, L, n_t, h, i, j);
                double p = silu(s) * inv_n;
                double dp = 0.0;
                for (int c = 0; c < d_v; c++)
                    dp += doi[c] * vj[c];
                double ds = dp * silu_grad(s) * inv_n;
                for (int c = 0; c < d_qk; c++)
                    okk[c] += ds * qi[c];
                for (int c = 0; c < d_v; c++)
                    ovv[c] += p * doi[c];
            }
        }
    }
}

/* ---- the transduction layer --------------------------------------------- */

/* out[T, n] = act(x[T, m] w[m, n] + bias[n]); act = SiLU when `apply_silu`. */
void oracle_linear(int64_t T, int m, int n, const double *x, const double *w, const double *bias,
                   int apply_silu, double *out, int num_threads)
{
    set_threads(num_threads);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++) {
        double *o = out + t * n;
        for (int c = 0; c < n; c++)
            o[c] = 0.0;
        /* o[c] = sum_k x[t,k] w[k,c], summed over k in increasing order */
        for (int kk = 0; kk < m; kk++) {
            double xv = x[t * m + kk];
            const double *wr = w + (int64_t)kk * n;
            for (int c = 0; c < n; c++)
                o[c] += xv * wr[c];
        }
        for (int c = 0; c < n; c++) {
            o[c] += bias ? bias[c] : 0.0;
            if (apply_silu)
                o[c] = silu(o[c]);
        }
    }
}

/* G[t,:] = LayerNorm(o[t,:]; gamma, beta, eps) * u[t,:] over F features. */
void oracle_norm_gate(int64_t T, int F, const double *o, const double *u, const double *gamma,
                      const double *beta, double eps, double *g, int num_threads)
{
    set_threads(num_threads);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; t++) {
        const double *ot = o + t * F;
        double mean = 0.0, var = 0.0;
        for (int c = 0; c < F; c++)
            mean += ot[c];
        mean /= F;
        for (int c = 0; c < F; c++)
            var += (ot[c] - mean) * (ot[c] - mean);
        var /= F;
        double rstd = 1.0 / sqrt(var + eps);
        for (int c = 0; c < F; c++)
            g[t * F + c] = ((ot[c] - mean) * rstd * gamma[c] + beta[c]) * u[t * F + c];
    }
}

/*
 * One transduction layer, forward:
 *   [U | V | Q | K] = SiLU(X W1 + b1)   (column blocks in that order; each block
 *                                         is [T, H, d] with d fastest)
 *   O = attention(Q, K, V);  G = LayerNorm(O) * U;  Y = G W2 + b2.
 * With out_cat set, the output projection reads the three H dv-wide blocks
 * [U | O | G] (the 3 h d_v input width of the output-projection row of Table 7
 * on the DLRMv4 page) and W2 is [3 H dv, D]: Y = [U | O | G] W2 + b2.
 * Optional outputs uvqk [T, H(2dv+2dqk)] and o [T, H dv] (may be NULL).
 */
void oracle_layer_fwd(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                      int num_heads, int d_qk, int d_v, int d_model, const double *x,
                      const double *w1, const double *b1, const double *w2, const double *b2,
                      const double *ln_gamma, const double *ln_beta, double ln_eps,
                      const int64_t *timestamps, const double *rab_pos, int pos_lo, int pos_hi,
                      const double *rab_time, int num_buckets, double inv_n, double *y,
                      double *uvqk_out, double *o_out, int out_cat, int num_threads)
{
    int64_t T = seq_offsets[num_seqs];
    int hv = num_heads * d_v, hq = num_heads * d_qk;
    int W = 2 * hv + 2 * hq;
    double *uvqk = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * W);
    double *u = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hv);
    double *vv = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hv);
    double *qq = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hq);
    double *kk = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hq);
    double *o = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hv);
    double *g = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * hv);
    oracle_linear(T, d_model, W, x, w1, b1, 1, uvqk, num_threads);
    for (int64_t t = 0; t < T; t++) {
        memcpy(u + t * hv, uvqk + t * W, sizeof(double) * hv);
        memcpy(vv + t * hv, uvqk + t * W + hv, sizeof(double) * hv);
        memcpy(qq + t * hq, uvqk + t * W + 2 * hv, sizeof(double) * hq);
        memcpy(kk + t * hq, uvqk + t * W + 2 * hv + hq, sizeof(double) * hq);
    }
    oracle_attn_fwd(num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, qq, kk, vv,
                    timestamps, rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n, o,
                    num_threads);
    oracle_norm_gate(T, hv, o, u, ln_gamma, ln_beta, ln_eps, g, num_threads);
    if (out_cat) {
        /* the output projection reads [U | O | G], 3 h d_v wide */
        double *cat = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * 3 * hv);
        for (int64_t t = 0; t < T; t++) {
            memcpy(cat + t * 3 * hv, u + t * hv, sizeof(double) * hv);
            memcpy(cat + t * 3 * hv + hv, o + t * hv, sizeof(double) * hv);
            memcpy(cat + t * 3 * hv + 2 * hv, g + t * hv, sizeof(double) * hv);
        }
        oracle_linear(T, 3 * hv, d_model, cat, w2, b2, 0, y, num_threads);
        free(cat);
    } else {
        oracle_linear(T, hv, d_model, g, w2, b2, 0, y, num_threads);
    }
    if (uvqk_out)
        memcpy(uvqk_out, uvqk, sizeof(double) * (size_t)T * W);
    if (o_out)
        memcpy(o_out, o, sizeof(double) * (size_t)T * hv);
    free(uvqk);
    free(u);
    free(vv);
    free(qq);
    free(kk);
    free(o);
    free(g);
}

/*
 * One transduction layer, backward of the loss sum(Y * dy), by the chain rule
 * through the forward above, step by step in reverse:
 *   Z = X W1 + b1, A = SiLU(Z) = [U | V | Q | K];  O = attention(Q, K, V);
 *   xh = (O - mean) rstd, G = (xh gamma + beta) * U;  Y = G W2 + b2.
 *   dW2 = G^T dy, db2 = sum_t dy, dG = dy W2^T;
 *   dU = dG (xh gamma + beta); dL = dG U; dgamma = sum_t dL xh; dbeta = sum_t dL;
 *   dO = rstd (dL gamma - mean(dL gamma) - xh mean(dL gamma xh));
 *   (dQ, dK, dV, d_rab_pos, d_rab_time) = attention backward with dout = dO;
 *   dZ = [dU | dV | dQ | dK] * SiLU'(Z);  dW1 = X^T dZ, db1 = sum_t dZ, dX = dZ W1^T.
 * With out_cat set (Y = [U | O | G] W2 + b2): dW2 = [U | O | G]^T dy, and of
 * dcat = dy W2^T the G block is dG while the U and O blocks are added to dU and
 * dO.  Every output is overwritten.
 */
void oracle_layer_bwd(int num_seqs, const int64_t *seq_offsets, const int32_t *num_targets,
                      int num_heads, int d_qk, int d_v, int d_model, const double *x,
                      const double *w1, const double *b1, const double *w2,
                      const double *ln_gamma, const double *ln_beta, double ln_eps,
                      const int64_t *timestamps, const double *rab_pos, int pos_lo, int pos_hi,
                      const double *rab_time, int num_buckets, double inv_n, const double *dy,
                      double *dx, double *dw1, double *db1, double *dw2, double *db2,
                      double *dgamma, double *dbeta, double *d_rab_pos, double *d_rab_time,
                      int out_cat, int num_threads)
{
    int64_t T = seq_offsets[num_seqs];
    int hv = num_heads * d_v, hq = num_heads * d_qk;
    int W = 2 * hv + 2 * hq, D = d_model;
    int F = out_cat ? 3 * hv : hv; /* width of the output projection's input */
    size_t Tn = (size_t)(T > 0 ? T : 1);
    double *z = (double *)malloc(sizeof(double) * Tn * W);
    double *u = (double *)malloc(sizeof(double) * Tn * hv);
    double *vv = (double *)malloc(sizeof(double) * Tn * hv);
    double *qq = (double *)malloc(sizeof(double) * Tn * hq);
    double *kk = (double *)malloc(sizeof(double) * Tn * hq);
    double *o = (double *)malloc(sizeof(double) * Tn * hv);
    double *xh = (double *)malloc(sizeof(double) * Tn * hv);
    double *rstd = (double *)malloc(sizeof(double) * Tn);
    double *g = (double *)malloc(sizeof(double) * Tn * hv);
    double *dg = (double *)malloc(sizeof(double) * Tn * hv);
    double *cat = (double *)malloc(sizeof(double) * Tn * F);
    double *dcat = (double *)malloc(sizeof(double) * Tn * F);
    double *du = (double *)malloc(sizeof(double) * Tn * hv);
    double *dl = (double *)malloc(sizeof(double) * Tn * hv);
    double *dout = (double *)malloc(sizeof(double) * Tn * hv);
    double *dq = (double *)malloc(sizeof(double) * Tn * hq);
    double *dk = (double *)malloc(sizeof(double) * Tn * hq);
    double *dv = (double *)malloc(sizeof(double) * Tn * hv);
    double *dz = (double *)malloc(sizeof(double) * Tn * W);

    /* forward, keeping what the backward needs */
    oracle_linear(T, D, W, x, w1, b1, 0, z, num_threads);
    for (int64_t t = 0; t < T; t++) {
        for (int c = 0; c < hv; c++) {
            u[t * hv + c] = silu(z[t * W + c]);
            vv[t * hv + c] = silu(z[t * W + hv + c]);
        }
        for (int c = 0; c < hq; c++) {
            qq[t * hq + c] = silu(z[t * W + 2 * hv + c]);
            kk[t * hq + c] = silu(z[t * W + 2 * hv + hq + c]);
        }
    }
    oracle_attn_fwd(num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, qq, kk, vv,
                    timestamps, rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n, o,
                    num_threads);
    for (int64_t t = 0; t < T; t++) {
        const double *ot = o + t * hv;
        double mean = 0.0, var = 0.0;
        for (int c = 0; c < hv; c++)
            mean += ot[c];
        mean /= hv;
        for (int c = 0; c < hv; c++)
            var += (ot[c] - mean) * (ot[c] - mean);
        var /= hv;
        rstd[t] = 1.0 / sqrt(var + ln_eps);
        for (int c = 0; c < hv; c++) {
            xh[t * hv + c] = (ot[c] - mean) * rstd[t];
            g[t * hv + c] = (xh[t * hv + c] * ln_gamma[c] + ln_beta[c]) * u[t * hv + c];
        }
    }

    /* the output projection's input: G, or [U | O | G] */
    for (int64_t t = 0; t < T; t++) {
        if (out_cat) {
            memcpy(cat + t * F, u + t * hv, sizeof(double) * hv);
            memcpy(cat + t * F + hv, o + t * hv, sizeof(double) * hv);
            memcpy(cat + t * F + 2 * hv, g + t * hv, sizeof(double) * hv);
        } else {
            memcpy(cat + t * F, g + t * hv, sizeof(double) * hv);
        }
    }

    /* output projection: dW2 = cat^T dy, db2 = sum dy, dcat = dy W2^T; dG is its G block */
    for (int j = 0; j < F; j++)
        for (int c = 0; c < D; c++)
            dw2[(int64_t)j * D + c] = 0.0;
    for (int c = 0; c < D; c++)
        db2[c] = 0.0;
    for (int64_t t = 0; t < T; t++) {
        for (int c = 0; c < D; c++)
            db2[c] += dy[t * D + c];
        for (int j = 0; j < F; j++) {
            double cj = cat[t * F + j], acc = 0.0;
            for (int c = 0; c < D; c++) {
                dw2[(int64_t)j * D + c] += cj * dy[t * D + c];
                acc += dy[t * D + c] * w2[(int64_t)j * D + c];
            }
            dcat[t * F + j] = acc;
        }
        memcpy(dg + t * hv, dcat + t * F + (F - hv), sizeof(double) * hv);
    }

    /* gate and LayerNorm */
    for (int c = 0; c < hv; c++) {
        dgamma[c] = 0.0;
        dbeta[c] = 0.0;
    }
    for (int64_t t = 0; t < T; t++) {
        double m1 = 0.0, m2 = 0.0;
        for (int c = 0; c < hv; c++) {
            int64_t e = t * hv + c;
            du[e] = dg[e] * (xh[e] * ln_gamma[c] + ln_beta[c]);
            dl[e] = dg[e] * u[e];
            dgamma[c] += dl[e] * xh[e];
            dbeta[c] += dl[e];
            m1 += dl[e] * ln_gamma[c];
            m2 += dl[e] * ln_gamma[c] * xh[e];
        }
        m1 /= hv;
        m2 /= hv;
        for (int c = 0; c < hv; c++) {
            int64_t e = t * hv + c;
            dout[e] = rstd[t] * (dl[e] * ln_gamma[c] - m1 - xh[e] * m2);
        }
        if (out_cat) /* U and O also enter the projection directly */
            for (int c = 0; c < hv; c++) {
                du[t * hv + c] += dcat[t * F + c];
                dout[t * hv + c] += dcat[t * F + hv + c];
            }
    }

    /* attention */
    oracle_attn_bwd(num_seqs, seq_offsets, num_targets, num_heads, d_qk, d_v, qq, kk, vv,
                    timestamps, rab_pos, pos_lo, pos_hi, rab_time, num_buckets, inv_n, dout, dq, dk,
                    dv, d_rab_pos, d_rab_time, num_threads);

    /* projection and SiLU: dZ = [dU | dV | dQ | dK] * SiLU'(Z) */
    for (int64_t t = 0; t < T; t++) {
        for (int c = 0; c < hv; c++) {
            dz[t * W + c] = du[t * hv + c] * silu_grad(z[t * W + c]);
            dz[t * W + hv + c] = dv[t * hv + c] * silu_grad(z[t * W + hv + c]);
        }
        for (int c = 0; c < hq; c++) {
            dz[t * W + 2 * hv + c] = dq[t * hq + c] * silu_grad(z[t * W + 2 * hv + c]);
            dz[t * W + 2 * hv + hq + c] = dk[t * hq + c] * silu_grad(z[t * W + 2 * hv + hq + c]);
        }
    }
    for (int k = 0; k < D; k++)
        for (int c = 0; c < W; c++)
            dw1[(int64_t)k * W + c] = 0.0;
    for (int c = 0; c < W; c++)
        db1[c] = 0.0;
    for (int64_t t = 0; t < T; t++) {
        for (int c = 0; c < W; c++)
            db1[c] += dz[t * W + c];
        for (int k = 0; k < D; k++) {
            double xv = x[t * D + k], acc = 0.0;
            for (int c = 0; c < W; c++) {
                dw1[(int64_t)k * W + c] += xv * dz[t * W + c];
                acc += dz[t * W + c] * w1[(int64_t)k * W + c];
            }
            dx[t * D + k] = acc;
        }
    }
    free(z);
    free(u);
    free(vv);
    free(qq);
    free(kk);
    free(o);
    free(xh);
    free(rstd);
    free(g);
    free(dg);
    free(cat);
    free(dcat);
    free(du);
    free(dl);
    free(dout);
    free(dq);
    free(dk);
    free(dv);
    free(dz);
}
