/*
 * Plain fp64 CPU oracle for the FLARE / FLARE++ mixer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline of the benchmark may load this code.  It shares nothing with the
 * CUDA library: no header, no helper, no table.
 *
 * What it computes (FLARE++ paper, arXiv 2608.11519, section "Method"):
 *   - per-head projections  K_h = X W_{K,h}  (the C x C matrix W split into H
 *     column blocks of width D = C/H; section "Full self-attention" gives the
 *     head split, "FLARE: fixed-query latent routing" and "FLARE++: dynamic
 *     token routing" (eq. 7, eq. 9) give the K, V, K~, V~ projections);
 *   - the encoder  Z_h = SDPA(Q_h, K_h, V_h) = softmax_n(Q_h K_h^T / sqrt(D)) V_h
 *     (eq. 5; with seeds Q~ it is the query synthesis of eq. 8, with Q(X) it
 *     is eq. 10);
 *   - the decoder  Y_h = SDPA(K_h, Q_h, Z_h) = softmax_m(K_h Q_h^T / sqrt(D)) Z_h
 *     (eq. 6 / eq. 11).
 * The softmax is evaluated as written: the maximum over the row is taken
 * first, then exp(a - max) is summed, in fp64, in ascending index order.  No
 * blocking, no online rescaling, no fusion.
 *
 * Key padding (the pages are silent; the reading used here): lengths[b] = L
 * means tokens n < L are valid.  Masked tokens are not keys of the encoder,
 * and the decoder writes zero rows for them.
 *
 * Layouts (all row-major, double):
 *   X [B][N][C], W [C][C] (K = X @ W), K/V/Y [B][H][N][D],
 *   queries Q [G][M][D] with G = H (shared over the batch, q_per_batch = 0)
 *   or G = B*H (one set per sample, q_per_batch = 1), Z [B][H][M][D].
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

static long valid_len(const int32_t *lengths, long b, long N)
{
    if (!lengths) return N;
    long L = lengths[b];
    if (L < 0) L = 0;
    if (L > N) L = N;
    return L;
}

/* out[b][h][n][d] = sum_c X[b][n][c] * W[c][h*D + d] */
void flare_oracle_project(const double *X, const double *W, double *out,
                          long B, long N, long C, long H, long D)
{
    long bn;
#pragma omp parallel for schedule(static)
    for (bn = 0; bn < B * N; ++bn) {
        long b = bn / N, n = bn % N;
        const double *x = X + bn * C;
        for (long h = 0; h < H; ++h) {
            for (long d = 0; d < D; ++d) {
                double s = 0.0;
                for (long c = 0; c < C; ++c) s += x[c] * W[c * C + h * D + d];
                out[((b * H + h) * N + n) * D + d] = s;
            }
        }
    }
}

static double dot(const double *a, const double *b, long D)
{
    double s = 0.0;
    for (long d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/*
 * Encoder: for every (b, h, m)
 *   a_n   = scale * <Q[g][m], K[b][h][n]>           for n < L_b
 *   mu    = max_n a_n
 *   w_n   = exp(a_n - mu)
 *   Z     = sum_n w_n V[b][h][n] / sum_n w_n
 *   lse   = mu + log(sum_n w_n)        (the row log-normaliser; may be NULL)
 * A row with no valid token gets Z = 0 and lse = -inf.
 */
void flare_oracle_encode(const double *Q, int q_per_batch, const double *K,
                         const double *V, const int32_t *lengths, double scale,
                         long B, long H, long N, long M, long D,
                         double *Z, double *lse)
{
    long r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < B * H * M; ++r) {
        long b = r / (H * M), h = (r / M) % H, m = r % M;
        long g = q_per_batch ? b * H + h : h;
        const double *q = Q + (g * M + m) * D;
        const double *Kh = K + (b * H + h) * N * D;
        const double *Vh = V + (b * H + h) * N * D;
        double *z = Z + ((b * H + h) * M + m) * D;
        long L = valid_len(lengths, b, N);
        for (long d = 0; d < D; ++d) z[d] = 0.0;
        if (L == 0) {
            if (lse) lse[(b * H + h) * M + m] = -INFINITY;
            continue;
        }
        double mu = -INFINITY;
        for (long n = 0; n < L; ++n) {
            double a = scale * dot(q, Kh + n * D, D);
            if (a > mu) mu = a;
        }
        double den = 0.0;
        for (long n = 0; n < L; ++n) {
            double w = exp(scale * dot(q, Kh + n * D, D) - mu);
            den += w;
            for (long d = 0; d < D; ++d) z[d] += w * Vh[n * D + d];
        }
        for (long d = 0; d < D; ++d) z[d] /= den;
        if (lse) lse[(b * H + h) * M + m] = mu + log(den);
    }
}

/*
 * Decoder: for every (b, h) and every token n listed in rows[0..nrows)
 * (all n in [0, N) when rows == NULL):
 *   c_m = scale * <K[b][h][n], Q[g][m]>,  nu = max_m c_m,  p_m = exp(c_m - nu)
 *   Y   = sum_m p_m Z[b][h][m] / sum_m p_m          for n <  L_b
 *   Y   = 0                                         for n >= L_b
 * Output Y[b][h][i][d] for the i-th listed token.
 */
void flare_oracle_decode(const double *K, const double *Q, int q_per_batch,
                         const double *Z, const int32_t *lengths, double scale,
                         long B, long H, long N, long M, long D,
                         const int64_t *rows, long nrows, double *Y)
{
    long cnt = rows ? nrows : N;
    long r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < B * H * cnt; ++r) {
        long b = r / (H * cnt), h = (r / cnt) % H, i = r % cnt;
        long n = rows ? (long)rows[i] : i;
        long g = q_per_batch ? b * H + h : h;
        const double *k = K + ((b * H + h) * N + n) * D;
        const double *Qg = Q + g * M * D;
        const double *Zh = Z + (b * H + h) * M * D;
        double *y = Y + ((b * H + h) * cnt + i) * D;
        long L = valid_len(lengths, b, N);
        for (long d = 0; d < D; ++d) y[d] = 0.0;
        if (n >= L) continue;
        double nu = -INFINITY;
        for (long m = 0; m < M; ++m) {
            double c = scale * dot(k, Qg + m * D, D);
            if (c > nu) nu = c;
        }
        double den = 0.0;
        for (long m = 0; m < M; ++m) {
            double p = exp(scale * dot(k, Qg + m * D, D) - nu);
            den += p;
            for (long d = 0; d < D; ++d) y[d] += p * Zh[m * D + d];
        }
        for (long d = 0; d < D; ++d) y[d] /= den;
    }
}

int flare_oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
