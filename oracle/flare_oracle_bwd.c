/*
 * Plain fp64 CPU oracle for the FLARE / FLARE++ mixer backward (gradients).
 *
 * TEST INFRASTRUCTURE ONLY, like flare_oracle.c: only the tests, the smoke
 * check and the CPU baseline of the benchmark may load it, and it shares
 * nothing with the CUDA library.
 *
 * The backward equations of the full paper (eq. 13-40) are named, not
 * printed (review of the FLARE++ paper, referee report, "significance").
 * Every step of the mixer is one SDPA call (FLARE++ paper, arXiv 2608.11519,
 * section "FLARE++: dynamic token routing", eq. 8, 10, 11), so the gradients
 * here are the textbook SDPA backward, written out per call.  For
 * O = softmax_rows(s Qa Ka^T) Va with upstream gradient dO, and
 * P[r][k] the softmax weights:
 *     dVa[k]  += sum_r P[r][k] dO[r]
 *     dP[r][k] = <dO[r], Va[k]>
 *     delta_r  = sum_k P[r][k] dP[r][k]  ( = <dO[r], O[r]> )
 *     dS[r][k] = P[r][k] (dP[r][k] - delta_r)
 *     dQa[r]  += s sum_k dS[r][k] Ka[k]
 *     dKa[k]  += s sum_r dS[r][k] Qa[r]
 * The encoder is this call with rows = latents and keys = valid tokens; the
 * decoder is it with rows = valid tokens and keys = latents.  The softmax
 * weights are recomputed as in the forward (maximum first, then exp, fp64,
 * ascending index order).  Outputs are accumulated (+=), so the two uses of
 * the keys K (encoder and decoder) add up in the caller's buffer.
 *
 * Queries shared over the batch (q_per_batch = 0) receive the sum over the
 * batch of their per-sample gradients, added in ascending b.
 *
 * Layouts as in flare_oracle.c: Q/dQ [G][M][D], K/V/dK/dV/dY [B][H][N][D],
 * Z/dZ [B][H][M][D], X/dX [B][N][C], W/dW [C][C].
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static long valid_len_bwd(const int32_t *lengths, long b, long N)
{
    if (!lengths) return N;
    long L = lengths[b];
    if (L < 0) L = 0;
    if (L > N) L = N;
    return L;
}

static double dot_bwd(const double *a, const double *b, long D)
{
    double s = 0.0;
    for (long d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* Adds the per-(b,h) query gradients tmp [B][H][M][D] into dQ [G][M][D]. */
static void fold_query_grads(const double *tmp, int q_per_batch, long B, long H, long M, long D,
                             double *dQ)
{
    const long per = M * D;
    for (long b = 0; b < B; ++b)
        for (long h = 0; h < H; ++h) {
            const long g = q_per_batch ? b * H + h : h;
            const double *src = tmp + (b * H + h) * per;
            double *dst = dQ + g * per;
            for (long i = 0; i < per; ++i) dst[i] += src[i];
        }
}

/*
 * Encoder backward.  Forward, per (b, h, m):
 *   a_n = scale <Q[g][m], K[n]>, A_n = softmax_n(a)  (n < L_b),  Z[m] = sum_n A_n V[n]
 * Given dZ, accumulates dQ (into [G][M][D]), dK and dV ([B][H][N][D]).
 */
void flare_oracle_encode_bwd(const double *Q, int q_per_batch, const double *K, const double *V,
                             const int32_t *lengths, double scale, long B, long H, long N, long M,
                             long D, const double *dZ, double *dQ, double *dK, double *dV)
{
    double *tmp = (double *)calloc((size_t)(B * H * M * D), sizeof(double));
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < B * H; ++bh) {
        long b = bh / H, h = bh % H;
        long g = q_per_batch ? b * H + h : h;
        long L = valid_len_bwd(lengths, b, N);
        const double *Kh = K + bh * N * D, *Vh = V + bh * N * D;
        double *dKh = dK + bh * N * D, *dVh = dV + bh * N * D;
        double *A = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
        double *z = (double *)malloc((size_t)D * sizeof(double));
        for (long m = 0; m < M && L > 0; ++m) {
            const double *q = Q + (g * M + m) * D;
            const double *dz = dZ + (bh * M + m) * D;
            double *dq = tmp + (bh * M + m) * D;
            double mu = -INFINITY;
            for (long n = 0; n < L; ++n) {
                A[n] = scale * dot_bwd(q, Kh + n * D, D);
                if (A[n] > mu) mu = A[n];
            }
            double den = 0.0;
            for (long n = 0; n < L; ++n) {
                A[n] = exp(A[n] - mu);
                den += A[n];
            }
            for (long d = 0; d < D; ++d) z[d] = 0.0;
            for (long n = 0; n < L; ++n) {
                A[n] /= den;
                for (long d = 0; d < D; ++d) z[d] += A[n] * Vh[n * D + d];
            }
            const double gamma = dot_bwd(dz, z, D);
            for (long n = 0; n < L; ++n) {
                const double dS = A[n] * (dot_bwd(dz, Vh + n * D, D) - gamma);
                for (long d = 0; d < D; ++d) {
                    dVh[n * D + d] += A[n] * dz[d];
                    dKh[n * D + d] += scale * dS * q[d];
                    dq[d] += scale * dS * Kh[n * D + d];
                }
            }
        }
        free(A);
        free(z);
    }
    fold_query_grads(tmp, q_per_batch, B, H, M, D, dQ);
    free(tmp);
}

/*
 * Decoder backward.  Forward, per (b, h) and valid token n < L_b:
 *   c_m = scale <K[n], Q[g][m]>, P_m = softmax_m(c),  Y[n] = sum_m P_m Z[m]
 * (Y[n] = 0 for masked tokens, which therefore get no gradient).
 * Given dY, accumulates dK ([B][H][N][D]), dQ ([G][M][D]) and dZ ([B][H][M][D]).
 */
void flare_oracle_decode_bwd(const double *K, const double *Q, int q_per_batch, const double *Z,
                             const int32_t *lengths, double scale, long B, long H, long N, long M,
                             long D, const double *dY, double *dK, double *dQ, double *dZ)
{
    double *tmp = (double *)calloc((size_t)(B * H * M * D), sizeof(double));
    long bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < B * H; ++bh) {
        long b = bh / H, h = bh % H;
        long g = q_per_batch ? b * H + h : h;
        long L = valid_len_bwd(lengths, b, N);
        const double *Qg = Q + g * M * D, *Zh = Z + bh * M * D;
        double *dZh = dZ + bh * M * D, *dq = tmp + bh * M * D;
        double *P = (double *)malloc((size_t)M * sizeof(double));
        double *y = (double *)malloc((size_t)D * sizeof(double));
        for (long n = 0; n < L; ++n) {
            const double *k = K + (bh * N + n) * D;
            const double *dy = dY + (bh * N + n) * D;
            double *dk = dK + (bh * N + n) * D;
            double nu = -INFINITY;
            for (long m = 0; m < M; ++m) {
                P[m] = scale * dot_bwd(k, Qg + m * D, D);
                if (P[m] > nu) nu = P[m];
            }
            double den = 0.0;
            for (long m = 0; m < M; ++m) {
                P[m] = exp(P[m] - nu);
                den += P[m];
            }
            for (long d = 0; d < D; ++d) y[d] = 0.0;
            for (long m = 0; m < M; ++m) {
                P[m] /= den;
                for (long d = 0; d < D; ++d) y[d] += P[m] * Zh[m * D + d];
            }
            const double delta = dot_bwd(dy, y, D);
            for (long m = 0; m < M; ++m) {
                const double dS = P[m] * (dot_bwd(dy, Zh + m * D, D) - delta);
                for (long d = 0; d < D; ++d) {
                    dZh[m * D + d] += P[m] * dy[d];
                    dk[d] += scale * dS * Qg[m * D + d];
                    dq[m * D + d] += scale * dS * k[d];
                }
            }
        }
        free(P);
        free(y);
    }
    fold_query_grads(tmp, q_per_batch, B, H, M, D, dQ);
    free(tmp);
}

/*
 * Projection backward.  Forward: out[b][h][n][d] = sum_c X[b][n][c] W[c][h*D + d].
 * Given dOut, accumulates
 *   dX[b][n][c]    += sum_{h,d} dOut[b][h][n][d] W[c][h*D + d]
 *   dW[c][h*D + d] += sum_{b,n} X[b][n][c] dOut[b][h][n][d]   (ascending b, n)
 */
void flare_oracle_project_bwd(const double *X, const double *W, const double *dOut, long B, long N,
                              long C, long H, long D, double *dX, double *dW)
{
    long i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < B * N; ++i) {
        long b = i / N, n = i % N;
        for (long c = 0; c < C; ++c) {
            double s = 0.0;
            for (long h = 0; h < H; ++h)
                for (long d = 0; d < D; ++d)
                    s += dOut[((b * H + h) * N + n) * D + d] * W[c * C + h * D + d];
            dX[i * C + c] += s;
        }
    }
#pragma omp parallel for schedule(static)
    for (i = 0; i < C; ++i) {
        for (long h = 0; h < H; ++h)
            for (long d = 0; d < D; ++d) {
                double s = 0.0;
                for (long b = 0; b < B; ++b)
                    for (long n = 0; n < N; ++n)
                        s += X[(b * N + n) * C + i] * dOut[((b * H + h) * N + n) * D + d];
                dW[i * C + h * D + d] += s;
            }
    }
}
