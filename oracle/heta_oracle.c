/*
 * heta_oracle.c -- plain, slow, fp64 CPU oracle for the heterogeneous
 * (uncertainty-routed) attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and the two share
 * no code: no headers, helpers, tables or constants.
 *
 * Source of every definition: "Where Compute Matters: Heterogeneous Attention
 * for Efficient Video Diffusion" (HetA-DiT, arXiv 2609.31050):
 *   - dense attention ........................ §3.1.1, Eq. (2)
 *   - local attention over a 3D neighbourhood  §3.1.1, Eq. (3); §5.1 "Local
 *                                               attention neighborhood"
 *   - uncertainty per token, u_i >= 0 ......... §3.2.1, Eq. (7)
 *   - routing threshold and mask .............. §3.2.2, Eq. (11)-(12)
 *   - heterogeneous mix ....................... §3.2.2, Eq. (13)
 *   - dense fraction rho and cost model ....... §3.2.2, Eq. (14)
 *
 * Readings taken where the paper leaves a step open (each is listed again in
 * the design notes):
 *   R1 selection: exactly k = ceil(rho*N) most-uncertain tokens per sample
 *      go dense (a top-k form of the mu + c*sigma threshold of Eq. (11)).
 *      rho is read as the decimal fraction the caller states: a product
 *      rho*N within 1e-12 (relative) of an integer counts as that integer,
 *      so 0.1*30 gives 3, not the 4 a bare IEEE ceil would give.
 *   R2 ties: equal u -> the smaller token index is taken first (Eq. (12)'s
 *      strict "<" sends u == T to the dense side).  -0.0 equals +0.0.  A NaN
 *      in u is an error (status 4).
 *   R3 window: per-axis start = clamp(p - floor(w/2), 0, extent - w), so every
 *      window holds exactly M = wt*wh*ww keys (a shifted clamp at borders).
 *   R4 token order: i = (t*Hg + h)*Wg + w.
 *   R5 local softmax is normalised over the window only, with the same
 *      1/sqrt(d) scale as Eq. (2).
 *   R6 only queries are routed; keys/values are always all N tokens.
 *   R7 the uncertainty head is u = softplus(x . w + b).  The paper names it
 *      only as a "lightweight branch" with u >= 0; a linear map followed by
 *      softplus is the plainest form that satisfies Eq. (7).
 *   R10 threshold mode (the paper's own rule): mu and sigma are the mean and
 *      the population standard deviation of one sample's N uncertainties,
 *      in fp64; u == T goes dense (Eq. (12)'s strict "<").  The count then
 *      varies per sample.
 *   R11 per-block random swap: at transformer block `block`, s tokens of
 *      the dense set (a uniformly random subset) trade places with s
 *      uniformly random tokens of the local set, so the count stays k.
 *      The swap ratio r of Table 8 is read as a fraction of N (s = ceil(rN),
 *      decimal-snapped as for k), which makes r = rho fully random as the
 *      paper's "fully random selection at 20%" says.  The subsets are the s
 *      smallest (rho_i, i) of each set, rho_i = Philox4x32-10 word 0 with
 *      counter (i, b, block, 0) and key (seed low, seed high): any side can
 *      reproduce them from the seed.
 *
 * All arithmetic is IEEE fp64 on inputs that are exactly representable
 * (fp32 arrays holding bf16 values, or fp32 values), in plain loop order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_INVALID 1
#define ORACLE_NONFINITE 4

/* Number of dense tokens per sample (reading R1; rho of Eq. (14)). */
int oracle_dense_count(int N, double rho, int *k_out)
{
    if (N < 0 || !(rho >= 0.0 && rho <= 1.0) || k_out == NULL)
        return ORACLE_INVALID;
    double prod = rho * (double)N;
    double nearest = nearbyint(prod);
    double tol = 1e-12 * (prod > 1.0 ? prod : 1.0);
    *k_out = (fabs(prod - nearest) <= tol) ? (int)nearest : (int)ceil(prod);
    if (*k_out > N) *k_out = N;
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Routing: Eq. (11)-(12) in top-k form (R1, R2).                      */
/* ------------------------------------------------------------------ */

static const float *g_sort_u; /* qsort has no context pointer */

static int order_desc_then_index(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    double ua = (double)g_sort_u[a], ub = (double)g_sort_u[b];
    if (ua > ub) return -1; /* larger uncertainty first */
    if (ua < ub) return 1;
    return (a < b) ? -1 : (a > b) ? 1 : 0; /* equal: smaller index first */
}

/*
 * u: [B,N] fp32.  Writes dense_idx [B,k] and local_idx [B,N-k], each sorted
 * ascending; mask (optional) [B,N] with the paper's m_i: 1 = local, 0 = dense.
 */
int oracle_route(const float *u, int B, int N, int k,
                 int32_t *dense_idx, int32_t *local_idx, uint8_t *mask)
{
    if (B < 0 || N < 0 || k < 0 || k > N) return ORACLE_INVALID;
    for (int64_t i = 0; i < (int64_t)B * N; ++i)
        if (isnan(u[i])) return ORACLE_NONFINITE;
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    uint8_t *is_dense = (uint8_t *)malloc((size_t)(N > 0 ? N : 1));
    if (!order || !is_dense) { free(order); free(is_dense); return ORACLE_INVALID; }
    for (int b = 0; b < B; ++b) {
        const float *ub = u + (int64_t)b * N;
        for (int i = 0; i < N; ++i) order[i] = i;
        g_sort_u = ub;
        qsort(order, (size_t)N, sizeof(int32_t), order_desc_then_index);
        memset(is_dense, 0, (size_t)N);
        for (int r = 0; r < k; ++r) is_dense[order[r]] = 1;
        int nd = 0, nl = 0;
        for (int i = 0; i < N; ++i) {
            if (is_dense[i]) dense_idx[(int64_t)b * k + nd++] = i;
            else local_idx[(int64_t)b * (N - k) + nl++] = i;
            if (mask) mask[(int64_t)b * N + i] = is_dense[i] ? 0 : 1;
        }
    }
    free(order);
    free(is_dense);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Routing by the paper's own threshold rule, Eq. (11)-(12) (R10).     */
/* ------------------------------------------------------------------ */

/*
 * Per sample b: mu = (1/N) sum_i u_i and sigma = sqrt((1/N) sum_i (u_i - mu)^2)
 * (the population standard deviation, two passes), T = mu + c * sigma
 * (Eq. (11)), m_i = [u_i < T] (Eq. (12)): u_i >= T goes dense.  All in fp64,
 * summed in index order.  Writes counts[b] = |dense set|, dense_idx row b
 * (capacity N: entries 0..counts[b]-1, ascending), local_idx row b (entries
 * 0..N-counts[b]-1, ascending), thresh[b] = T (optional) and mask (optional,
 * 1 = local).  N = 0 gives empty sets; a NaN in u is status 4.
 */
int oracle_route_threshold(const float *u, int B, int N, double c, int32_t *counts,
                           int32_t *dense_idx, int32_t *local_idx, double *thresh,
                           uint8_t *mask)
{
    if (B < 0 || N < 0 || isnan(c) || isinf(c)) return ORACLE_INVALID;
    for (int64_t i = 0; i < (int64_t)B * N; ++i)
        if (isnan(u[i])) return ORACLE_NONFINITE;
    for (int b = 0; b < B; ++b) {
        const float *ub = u + (int64_t)b * N;
        double sum = 0.0;
        for (int i = 0; i < N; ++i) sum += (double)ub[i];
        const double mu = N > 0 ? sum / (double)N : 0.0;
        double sq = 0.0;
        for (int i = 0; i < N; ++i) {
            const double dev = (double)ub[i] - mu;
            sq += dev * dev;
        }
        const double sigma = N > 0 ? sqrt(sq / (double)N) : 0.0;
        const double T = mu + c * sigma;
        if (thresh) thresh[b] = T;
        int nd = 0, nl = 0;
        for (int i = 0; i < N; ++i) {
            const int local = (double)ub[i] < T;
            if (local) local_idx[(int64_t)b * N + nl++] = i;
            else dense_idx[(int64_t)b * N + nd++] = i;
            if (mask) mask[(int64_t)b * N + i] = (uint8_t)local;
        }
        counts[b] = nd;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Per-block random swap (§3.2.2 after Eq. (12); App. B Table 8), R11. */
/* ------------------------------------------------------------------ */

/*
 * Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC 2011): ten rounds
 * of two 32x32->64 multiplications (multipliers 0xD2511F53, 0xCD9E8D57) whose
 * halves are mixed with the other counter words and the key; the key is
 * advanced by the Weyl increments 0x9E3779B9, 0xBB67AE85 before every round
 * after the first.
 */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The random draw of token i of sample b at transformer block `block`. */
static uint32_t swap_draw(int i, int b, int block, uint64_t seed)
{
    const uint32_t ctr[4] = {(uint32_t)i, (uint32_t)b, (uint32_t)block, 0u};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[0];
}

static const uint32_t *g_sort_draw; /* qsort has no context pointer */

static int order_draw_then_index(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    if (g_sort_draw[a] < g_sort_draw[b]) return -1;
    if (g_sort_draw[a] > g_sort_draw[b]) return 1;
    return (a < b) ? -1 : (a > b) ? 1 : 0;
}

/*
 * One block's swap, per sample b: every token i draws rho_i (above); of the
 * dense set D (dense_idx row b, k entries) the s tokens with the smallest
 * (rho_i, i) go local, and of its complement the s tokens with the smallest
 * (rho_i, i) go dense.  Writes the new sets, ascending, to dense_out [B,k]
 * and local_out [B,N-k].  Requires 0 <= s <= min(k, N-k) and a valid
 * dense_idx (distinct ids in [0,N)); otherwise status 1.
 */
int oracle_route_swap(const int32_t *dense_idx, int B, int N, int k, int s, uint64_t seed,
                      int block, int32_t *dense_out, int32_t *local_out)
{
    if (B < 0 || N < 0 || k < 0 || k > N || s < 0 || s > k || s > N - k)
        return ORACLE_INVALID;
    uint8_t *dense = (uint8_t *)malloc((size_t)(N > 0 ? N : 1));
    uint32_t *draw = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(N > 0 ? N : 1));
    int32_t *gd = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    int32_t *gl = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N - k > 0 ? N - k : 1));
    int rc = ORACLE_OK;
    if (!dense || !draw || !gd || !gl) rc = ORACLE_INVALID;
    for (int b = 0; b < B && rc == ORACLE_OK; ++b) {
        memset(dense, 0, (size_t)N);
        for (int j = 0; j < k; ++j) {
            const int32_t t = dense_idx[(int64_t)b * k + j];
            if (t < 0 || t >= N || dense[t]) { rc = ORACLE_INVALID; break; }
            dense[t] = 1;
        }
        if (rc != ORACLE_OK) break;
        int nd = 0, nl = 0;
        for (int i = 0; i < N; ++i) {
            draw[i] = swap_draw(i, b, block, seed);
            if (dense[i]) gd[nd++] = i;
            else gl[nl++] = i;
        }
        g_sort_draw = draw;
        qsort(gd, (size_t)nd, sizeof(int32_t), order_draw_then_index);
        qsort(gl, (size_t)nl, sizeof(int32_t), order_draw_then_index);
        for (int j = 0; j < s; ++j) {
            dense[gd[j]] = 0;
            dense[gl[j]] = 1;
        }
        nd = nl = 0;
        for (int i = 0; i < N; ++i) {
            if (dense[i]) dense_out[(int64_t)b * k + nd++] = i;
            else local_out[(int64_t)b * (N - k) + nl++] = i;
        }
    }
    free(dense);
    free(draw);
    free(gd);
    free(gl);
    return rc;
}

/* ------------------------------------------------------------------ */
/* 3D neighbourhood: Eq. (3) with reading R3/R4.                       */
/* ------------------------------------------------------------------ */

/* Start of the width-`width` run along one axis that holds position p. */
int oracle_window_start(int p, int extent, int width)
{
    int s = p - width / 2;
    if (s > extent - width) s = extent - width;
    if (s < 0) s = 0;
    return s;
}

/* Enumerates the keys of token i's window in ascending token order.
 * Returns the number written (always wt*wh*ww for valid sizes). */
int oracle_window(int Tg, int Hg, int Wg, int wt, int wh, int ww, int i,
                  int32_t *keys_out)
{
    int t = i / (Hg * Wg), h = (i / Wg) % Hg, w = i % Wg;
    int st = oracle_window_start(t, Tg, wt);
    int sh = oracle_window_start(h, Hg, wh);
    int sw = oracle_window_start(w, Wg, ww);
    int n = 0;
    for (int a = st; a < st + wt; ++a)
        for (int c = sh; c < sh + wh; ++c)
            for (int e = sw; e < sw + ww; ++e)
                keys_out[n++] = (a * Hg + c) * Wg + e;
    return n;
}

/* ------------------------------------------------------------------ */
/* Attention for a list of output rows: Eq. (2), (3) and (13).         */
/* ------------------------------------------------------------------ */

/* softmax(scale * q . k_j) weighted sum of v_j over the key list J. */
static void attend_one_row(const float *q, const float *Kh, const float *Vh,
                           int d, double scale, const int32_t *J, int nJ,
                           double *s /* [nJ] scratch */, double *acc /* [d] */,
                           double *out)
{
    double m = -INFINITY;
    for (int j = 0; j < nJ; ++j) {
        const float *kj = Kh + (int64_t)J[j] * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += (double)q[c] * (double)kj[c];
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double den = 0.0;
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    for (int j = 0; j < nJ; ++j) {
        double p = exp(s[j] - m);
        den += p;
        const float *vj = Vh + (int64_t)J[j] * d;
        for (int c = 0; c < d; ++c) acc[c] += p * (double)vj[c];
    }
    for (int c = 0; c < d; ++c) out[c] = acc[c] / den;
}

/*
 * Q,K,V: [B,H,N,d] fp32 (values exactly representable; read as fp64).
 * dense_idx: [B,k] -- the dense set D_b of each sample (any order).
 * rows: flat row ids r = (b*H + h)*N + i, nrows of them; out: [nrows, d].
 * A row whose token is in D_b attends over all N keys (Eq. (2)); every other
 * row over its clamped window (Eq. (3)); Eq. (13) picks one per row.
 */
int oracle_attention_rows(const float *Q, const float *K, const float *V,
                          int B, int H, int N, int d,
                          int Tg, int Hg, int Wg, int wt, int wh, int ww,
                          double scale, const int32_t *dense_idx, int k,
                          const int64_t *rows, int64_t nrows, double *out,
                          int nthreads)
{
    if (B < 0 || H < 0 || N < 0 || d <= 0 || k < 0 || k > N) return ORACLE_INVALID;
    if ((int64_t)Tg * Hg * Wg != N) return ORACLE_INVALID;
    if (wt < 1 || wh < 1 || ww < 1 || wt > Tg || wh > Hg || ww > Wg) return ORACLE_INVALID;
    const int M = wt * wh * ww;

    uint8_t *dense_flag = (uint8_t *)calloc((size_t)B * (size_t)(N > 0 ? N : 1), 1);
    int32_t *all_keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!dense_flag || !all_keys) { free(dense_flag); free(all_keys); return ORACLE_INVALID; }
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < k; ++r) {
            int32_t i = dense_idx[(int64_t)b * k + r];
            if (i < 0 || i >= N) { free(dense_flag); free(all_keys); return ORACLE_INVALID; }
            dense_flag[(int64_t)b * N + i] = 1;
        }
    for (int j = 0; j < N; ++j) all_keys[j] = j;

    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(N > M ? N : M));
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        int32_t *win = (int32_t *)malloc(sizeof(int32_t) * (size_t)M);
        if (!s || !acc || !win) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t row = rows[r];
                if (row < 0 || row >= (int64_t)B * H * N) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                int64_t bh = row / N;
                int i = (int)(row % N);
                int b = (int)(bh / H);
                const float *q = Q + row * d;
                const float *Kh = K + bh * (int64_t)N * d;
                const float *Vh = V + bh * (int64_t)N * d;
                if (dense_flag[(int64_t)b * N + i]) {
                    attend_one_row(q, Kh, Vh, d, scale, all_keys, N, s, acc, out + r * d);
                } else {
                    int n = oracle_window(Tg, Hg, Wg, wt, wh, ww, i, win);
                    attend_one_row(q, Kh, Vh, d, scale, win, n, s, acc, out + r * d);
                }
            }
        }
        free(s);
        free(acc);
        free(win);
    }
    free(dense_flag);
    free(all_keys);
    return bad ? ORACLE_INVALID : ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Uncertainty head: Eq. (7) with reading R7.                          */
/* ------------------------------------------------------------------ */

static double softplus(double z)
{
    /* log(1 + e^z), written so that neither branch overflows */
    return (z > 0.0) ? z + log1p(exp(-z)) : log1p(exp(z));
}

/* X: [B,N,C] fp32 (exact bf16 values), w: [C], u_out: [B*N] fp64. */
int oracle_uncertainty(const float *X, const float *w, double bias,
                       int B, int N, int C, double *u_out, int nthreads)
{
    if (B < 0 || N < 0 || C <= 0) return ORACLE_INVALID;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)B * N; ++r) {
        const float *x = X + r * C;
        double z = 0.0;
        for (int c = 0; c < C; ++c) z += (double)x[c] * (double)w[c];
        u_out[r] = softplus(z + bias);
    }
    return ORACLE_OK;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
