/*
 * Engram conditional-memory oracle: a plain, slow, fp64 CPU restatement of the
 * Engram n-gram hash, the table-row gather and the Engram gate (forward and
 * backward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, no
 * header and no constant with the CUDA library; the product path never calls
 * it and must fail loudly when its own CUDA extension is missing.
 *
 * Source of every definition: the page "DeepSeek 开源 TileKernels：用 Python
 * 写出逼近硬件极限的 GPU 内核" (zhichai.net/topic/177618722), section
 * "5. Engram — 条件记忆门控":
 *   - engram_hash: an n-gram hash combining XOR and multiplication over the
 *     token sequence, mapped to embedding-table indices; 2 n-gram layers, up
 *     to 3-grams, 8 embedding tables per layer;
 *   - the gate formula
 *       gate   = sigmoid(signed_sqrt(dot(RMSNorm(x, wh), RMSNorm(k, we)) * scalar))
 *       output = hidden_states + gate * v
 *     with signed_sqrt(x) = sign(x) * sqrt(|x|) and scalar = 1/sqrt(hidden_size);
 *   - engram_gate_bwd and engram_grad_w_reduce: the backward of that formula
 *     and the reduction of the weight gradients over tokens.
 *
 * Readings where the page is silent (each is listed with its reason in the
 * design notes):
 *   - hash of layer l at token s of sequence b:
 *       h = XOR_{i=0}^{n_l-1} (u64(tok[b, s-i]) * m[l][i])  (wrapping u64),
 *     tok[b, s-i] = pad_id when s-i < 0 (history never crosses a sequence);
 *   - idx[l][j] = h mod P[l][j], unsigned 64-bit, one prime P per table;
 *   - RMSNorm(x, w)_j = x_j * (mean(x^2) + eps)^(-1/2) * w_j;
 *   - hidden_states is the same tensor x;
 *   - in the derivative of signed_sqrt, |s| is clamped to at least 1e-6:
 *       d signed_sqrt(s) / ds = 1 / (2 sqrt(max(|s|, 1e-6)));
 *   - the gate is an output only: no gradient flows into it from outside.
 *
 * Arithmetic: every floating-point step is in double.  The gate functions take
 * double inputs (a caller holding bf16 data widens it exactly first, which also
 * lets finite differences perturb the inputs); the gather copies bf16 bit
 * patterns.  Outputs are double; rounding them to bf16 is left to the caller.
 * Loops run in the formula's order.  OpenMP only splits independent tokens (or,
 * for the weight gradients, independent columns whose sums over tokens stay in
 * token order), so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* engram_hash: n-gram hash, then one index per embedding table.            */
/* tokens[B*S]; multipliers[L*n_max] (row l holds m[l][0..n_max-1]);         */
/* ngram_n[L] (n of layer l, <= n_max); table_sizes[L*J] (table (l,j) at    */
/* l*J+j); idx_out[B*S*L*J], laid out [b][s][l][j].                          */
/* ------------------------------------------------------------------------ */
void oracle_engram_hash(const int64_t *tokens, int64_t B, int64_t S,
                        const uint64_t *multipliers, const int32_t *ngram_n,
                        int32_t L, int32_t n_max, const int64_t *table_sizes,
                        int32_t J, int64_t pad_id, int64_t *idx_out)
{
    int64_t T = B * S;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        int64_t b = t / S;
        int64_t s = t % S;
        for (int32_t l = 0; l < L; ++l) {
            uint64_t h = 0;
            for (int32_t i = 0; i < ngram_n[l]; ++i) {
                int64_t tok = (s - i >= 0) ? tokens[b * S + (s - i)] : pad_id;
                h ^= (uint64_t)tok * multipliers[(int64_t)l * n_max + i];
            }
            for (int32_t j = 0; j < J; ++j) {
                uint64_t P = (uint64_t)table_sizes[(int64_t)l * J + j];
                idx_out[(t * L + l) * J + j] = (int64_t)(h % P);
            }
        }
    }
}

/* First row of each table in the concatenated tables (at most 256 tables). */
static void table_first_rows(const int64_t *table_sizes, int32_t ntab, int64_t *first_row)
{
    int64_t acc = 0;
    for (int32_t q = 0; q < ntab && q < 256; ++q) {
        first_row[q] = acc;
        acc += table_sizes[q];
    }
}

/* ------------------------------------------------------------------------ */
/* Table-row gather.  tables holds the L*J tables one after another, table  */
/* (l,j) with table_sizes[l*J+j] rows of D bf16 values.  rows_out[T*L*J*D]  */
/* is laid out [t][l][j][D].                                                */
/* ------------------------------------------------------------------------ */
void oracle_engram_gather(const int64_t *idx, int64_t T, int32_t L, int32_t J,
                          const int64_t *table_sizes, const uint16_t *tables,
                          int32_t D, uint16_t *rows_out)
{
    int32_t ntab = L * J;
    int64_t first_row[256];
    table_first_rows(table_sizes, ntab, first_row);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t q = 0; q < ntab; ++q) {
            int64_t r = idx[t * ntab + q];
            const uint16_t *src = tables + (first_row[q] + r) * D;
            uint16_t *dst = rows_out + (t * ntab + q) * D;
            for (int32_t c = 0; c < D; ++c) dst[c] = src[c];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Gate forward, one token at a time, in the formula's own steps.           */
/* x, k, v [T*H]; wh, we [H]; out [T*H] and gate [T] in double.              */
/* ------------------------------------------------------------------------ */
static double signed_sqrt(double s)
{
    if (s > 0) return sqrt(s);
    if (s < 0) return -sqrt(-s);
    return 0.0;
}

static double sigmoid(double u) { return 1.0 / (1.0 + exp(-u)); }

/* 1 / sqrt(mean(z^2) + eps) over one row of H values. */
static double rms_inverse(const double *z, int32_t H, double eps)
{
    double ss = 0.0;
    for (int32_t j = 0; j < H; ++j) ss += z[j] * z[j];
    return 1.0 / sqrt(ss / (double)H + eps);
}

/* dot(RMSNorm(x, wh), RMSNorm(k, we)) for one token, with rx, rk returned. */
static double normed_dot(const double *x, const double *k, const double *wh,
                         const double *we, int32_t H, double eps, double *rx_out,
                         double *rk_out)
{
    double rx = rms_inverse(x, H, eps);
    double rk = rms_inverse(k, H, eps);
    double dot = 0.0;
    for (int32_t j = 0; j < H; ++j) {
        double a = x[j] * rx * wh[j];
        double b = k[j] * rk * we[j];
        dot += a * b;
    }
    *rx_out = rx;
    *rk_out = rk;
    return dot;
}

void oracle_engram_gate_fwd(const double *x, const double *k, const double *v,
                            const double *wh, const double *we, int64_t T,
                            int32_t H, double eps, double scalar, double *out,
                            double *gate)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *xt = x + t * H, *kt = k + t * H, *vt = v + t * H;
        double rx, rk;
        double dot = normed_dot(xt, kt, wh, we, H, eps, &rx, &rk);
        double g = sigmoid(signed_sqrt(dot * scalar));
        gate[t] = g;
        for (int32_t j = 0; j < H; ++j) out[t * H + j] = xt[j] + g * vt[j];
    }
}

/* ------------------------------------------------------------------------ */
/* Gate backward.  grad_out [T*H] is dL/d(output).  The chain rule is taken  */
/* back through the forward's own steps:                                     */
/*   output = x + gate*v         -> dv = gate*g, dgate = sum_j g_j v_j,      */
/*                                  and g flows into x unchanged;            */
/*   gate = sigmoid(u)           -> du = dgate * gate * (1 - gate);          */
/*   u = signed_sqrt(s)          -> ds = du / (2 sqrt(max(|s|, 1e-6)));      */
/*   s = dot * scalar            -> ddot = ds * scalar;                      */
/*   dot = sum_j a_j b_j         -> da_j = ddot*b_j, db_j = ddot*a_j;        */
/*   a_j = x_j * rx * wh_j with rx = (sum_i x_i^2 / H + eps)^(-1/2)          */
/*                               -> dx_j += rx*wh_j*da_j                     */
/*                                  - rx^3 x_j/H * sum_i x_i wh_i da_i,      */
/*                                  dwh_j += sum over tokens of da_j*x_j*rx; */
/*   b_j likewise with k, rk, we.                                            */
/* dx, dk, dv [T*H] (each may be NULL to skip it); dwh, dwe [H] (overwritten; */
/* both NULL to skip the sums over tokens).  stats [T*4] receives, per token, rx, rk, s and ddot (also used as the     */
/* workspace of the weight-gradient pass).                                   */
/* ------------------------------------------------------------------------ */
void oracle_engram_gate_bwd(const double *grad_out, const double *x,
                            const double *k, const double *v, const double *wh,
                            const double *we, int64_t T, int32_t H, double eps,
                            double scalar, double *dx, double *dk, double *dv,
                            double *dwh, double *dwe, double *stats)
{
    /* Per-token part: everything except the sums over tokens. */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *xt = x + t * H, *kt = k + t * H, *vt = v + t * H;
        const double *gt = grad_out + t * H;
        double rx, rk;
        double dot = normed_dot(xt, kt, wh, we, H, eps, &rx, &rk);
        double s = dot * scalar;
        double gate = sigmoid(signed_sqrt(s));

        double dgate = 0.0;
        for (int32_t j = 0; j < H; ++j) dgate += gt[j] * vt[j];
        double du = dgate * gate * (1.0 - gate);
        double abs_s = fabs(s);
        double ds = du / (2.0 * sqrt(abs_s > 1e-6 ? abs_s : 1e-6));
        double ddot = ds * scalar;

        /* cx = sum_i x_i wh_i da_i and ck = sum_i k_i we_i db_i */
        double cx = 0.0, ck = 0.0;
        for (int32_t j = 0; j < H; ++j) {
            double a = xt[j] * rx * wh[j], b = kt[j] * rk * we[j];
            double da = ddot * b, db = ddot * a;
            cx += xt[j] * wh[j] * da;
            ck += kt[j] * we[j] * db;
        }
        for (int32_t j = 0; j < H; ++j) {
            double a = xt[j] * rx * wh[j], b = kt[j] * rk * we[j];
            double da = ddot * b, db = ddot * a;
            if (dx) dx[t * H + j] = gt[j] + rx * wh[j] * da - rx * rx * rx * xt[j] * cx / (double)H;
            if (dk) dk[t * H + j] = rk * we[j] * db - rk * rk * rk * kt[j] * ck / (double)H;
            if (dv) dv[t * H + j] = gate * gt[j];
        }
        stats[4 * t + 0] = rx;
        stats[4 * t + 1] = rk;
        stats[4 * t + 2] = s;
        stats[4 * t + 3] = ddot;
    }

    /* Weight gradients: dwh_j = sum_t da_tj x_tj rx_t and
     * dwe_j = sum_t db_tj k_tj rk_t.  Each column's sum runs over t = 0..T-1
     * in order; columns are split into blocks only so that one pass over the
     * tokens serves a block of columns. */
    if (!dwh || !dwe) return;
    enum { CB = 32 };
    int32_t nblk = (H + CB - 1) / CB;
#pragma omp parallel for schedule(static)
    for (int32_t blk = 0; blk < nblk; ++blk) {
        int32_t j0 = blk * CB;
        int32_t j1 = j0 + CB < H ? j0 + CB : H;
        double sh[CB], se[CB];
        for (int32_t j = j0; j < j1; ++j) sh[j - j0] = se[j - j0] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double rx = stats[4 * t + 0], rk = stats[4 * t + 1];
            double ddot = stats[4 * t + 3];
            for (int32_t j = j0; j < j1; ++j) {
                double xj = x[t * H + j], kj = k[t * H + j];
                double a = xj * rx * wh[j], b = kj * rk * we[j];
                sh[j - j0] += (ddot * b) * xj * rx;
                se[j - j0] += (ddot * a) * kj * rk;
            }
        }
        for (int32_t j = j0; j < j1; ++j) {
            dwh[j] = sh[j - j0];
            dwe[j] = se[j - j0];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Gather backward: the gradient reaching a gathered row is added to the     */
/* table row it was read from, so a row read several times receives the sum */
/* of their gradients (the transpose of the gather above).                   */
/* idx [T*L*J] local rows as from oracle_engram_hash; d_rows [T*L*J*D];      */
/* d_tables receives the global rows [row_lo, row_hi) of the concatenated    */
/* tables, (row_hi - row_lo) * D doubles, overwritten:                       */
/*   d_tables[r - row_lo][c] = sum over (t, l, j) with                      */
/*        first_row(l, j) + idx[t][l][j] == r  of  d_rows[t][l][j][c],      */
/* summed in (t, l, j) order.                                                */
/* ------------------------------------------------------------------------ */
void oracle_engram_gather_bwd(const int64_t *idx, int64_t T, int32_t L, int32_t J,
                              const int64_t *table_sizes, const double *d_rows, int32_t D,
                              int64_t row_lo, int64_t row_hi, double *d_tables)
{
    int32_t ntab = L * J;
    int64_t first_row[256];
    table_first_rows(table_sizes, ntab, first_row);
    for (int64_t i = 0; i < (row_hi - row_lo) * D; ++i) d_tables[i] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t q = 0; q < ntab; ++q) {
            int64_t r = first_row[q] + idx[t * ntab + q];
            if (r < row_lo || r >= row_hi) continue;
            const double *src = d_rows + (t * ntab + q) * D;
            double *dst = d_tables + (r - row_lo) * D;
            for (int32_t c = 0; c < D; ++c) dst[c] += src[c];
        }
    }
}
