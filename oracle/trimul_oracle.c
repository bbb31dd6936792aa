/*
 * Triangle multiplicative update -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The product path never calls it, and
 * it shares no code, header or constant with the CUDA library.
 *
 * What it computes, for batch element b, residues i, j and pair mask m_ij
 * (all arrays row-major, pair tensors channel-last [B, N, N, C], linear weights
 * [out, in] with y = x W^T + bias, every bias optional = 0):
 *
 *   1. zhat_ij = LayerNorm over c_z of z_ij (mean, biased variance, eps inside
 *      the square root, per-channel gamma and beta).
 *      ("RFProteina architecture" page, section "Triangle multiplication on
 *      SM90": K1's input LayerNorm.)
 *   2. a_ij = m_ij * sigmoid(zhat_ij W_ag^T + b_ag) (.) (zhat_ij W_ap^T + b_ap),
 *      b_ij the same with (W_bg, b_bg, W_bp, b_bp); c_h channels each.
 *      (Same page, section "Dual-GEMM gates", the one-input "x_x" gate that
 *      reads the normalized pair tensor and applies the pair mask.)
 *   3. outgoing: x_ij = sum_k a_ik (.) b_jk ;  incoming: x_ij = sum_k a_ki (.) b_kj,
 *      k = 0 .. N-1 in ascending order, one fp64 accumulator per channel.
 *      (Same page, K2: the contraction, one direction at a time; "Inside the
 *      velocity network": outgoing then incoming triangle multiplication.)
 *   4. out_ij = m_ij * sigmoid(zhat_ij W_g^T + b_g)
 *                    (.) (LayerNorm over c_h of x_ij) W_o^T + b_o)
 *      (Same page, section "Dual-GEMM gates", the two-input "x0_x1" gate with
 *      x0 the normalized input pair tensor and x1 the contracted hidden tensor;
 *      K3 applies the output LayerNorm.)
 *
 * sigmoid(v) = 1 / (1 + exp(-v)) in double precision. No blocking, fusion or
 * reordering beyond the definitions above. OpenMP only splits independent
 * rows across threads; every sum runs in the stated order on one thread.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OUTGOING 0
#define ORACLE_INCOMING 1

typedef struct {
    const double *ln_in_g, *ln_in_b;
    const double *w_ag, *b_ag, *w_ap, *b_ap;
    const double *w_bg, *b_bg, *w_bp, *b_bp;
    const double *w_g, *b_g;
    const double *ln_out_g, *ln_out_b;
    const double *w_o, *b_o;
} oracle_weights_t;

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double logistic(double v) { return 1.0 / (1.0 + exp(-v)); }

/* y[r, :] = LayerNorm(x[r, :]) over C channels. gamma/beta may be NULL (1 / 0). */
int oracle_layernorm(int64_t rows, int64_t C, const double *x, const double *gamma,
                     const double *beta, double eps, double *y) {
    if (rows < 0 || C <= 0 || !x || !y) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * C;
        double *yr = y + r * C;
        double mean = 0.0;
        for (int64_t c = 0; c < C; ++c) mean += xr[c];
        mean /= (double)C;
        double var = 0.0;
        for (int64_t c = 0; c < C; ++c) {
            double d = xr[c] - mean;
            var += d * d;
        }
        var /= (double)C;
        double rstd = 1.0 / sqrt(var + eps);
        for (int64_t c = 0; c < C; ++c) {
            double g = gamma ? gamma[c] : 1.0;
            double bb = beta ? beta[c] : 0.0;
            yr[c] = (xr[c] - mean) * rstd * g + bb;
        }
    }
    return 0;
}

/* y[r, o] = sum_i x[r, i] W[o, i] + bias[o], i ascending. */
int oracle_linear(int64_t rows, int64_t c_in, int64_t c_out, const double *x, const double *W,
                  const double *bias, double *y) {
    if (rows < 0 || c_in <= 0 || c_out <= 0 || !x || !W || !y) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * c_in;
        for (int64_t o = 0; o < c_out; ++o) {
            const double *wo = W + o * c_in;
            double s = 0.0;
            for (int64_t i = 0; i < c_in; ++i) s += xr[i] * wo[i];
            y[r * c_out + o] = s + (bias ? bias[o] : 0.0);
        }
    }
    return 0;
}

/* Step 2: y[r, :] = m_r * sigmoid(xhat W_g^T + b_g) (.) (xhat W_p^T + b_p). mask NULL = 1. */
int oracle_gated_projection(int64_t rows, int64_t c_in, int64_t c_out, const double *xhat,
                            const double *mask, const double *Wg, const double *bg,
                            const double *Wp, const double *bp, double *y) {
    if (rows < 0 || c_in <= 0 || c_out <= 0 || !xhat || !Wg || !Wp || !y) return -1;
    double *g = (double *)malloc(sizeof(double) * (size_t)(rows * c_out + 1));
    if (!g) return -2;
    oracle_linear(rows, c_in, c_out, xhat, Wg, bg, g);
    oracle_linear(rows, c_in, c_out, xhat, Wp, bp, y);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double m = mask ? mask[r] : 1.0;
        for (int64_t o = 0; o < c_out; ++o) {
            int64_t t = r * c_out + o;
            y[t] = m * logistic(g[t]) * y[t];
        }
    }
    free(g);
    return 0;
}

/* Step 3 on [B, N, N, C] tensors a, b -> x.
 * outgoing: x[b,i,j,c] = sum_k a[b,i,k,c] * b[b,j,k,c]
 * incoming: x[b,i,j,c] = sum_k a[b,k,i,c] * b[b,k,j,c]
 * Each output element has its own accumulator and sees k in ascending order. */
int oracle_contract(int64_t B, int64_t N, int64_t C, const double *a, const double *bm,
                    int direction, double *x) {
    if (B < 0 || N < 0 || C <= 0 || !a || !bm || !x) return -1;
    if (direction != ORACLE_OUTGOING && direction != ORACLE_INCOMING) return -1;
    const int64_t row = N * C, plane = N * N * C;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bb = 0; bb < B; ++bb) {
        for (int64_t i = 0; i < N; ++i) {
            double *xi = x + bb * plane + i * row;
            memset(xi, 0, sizeof(double) * (size_t)row);
            if (direction == ORACLE_OUTGOING) {
                const double *ai = a + bb * plane + i * row;          /* a[b, i, :, :] */
                for (int64_t j = 0; j < N; ++j) {
                    const double *bj = bm + bb * plane + j * row;     /* b[b, j, :, :] */
                    double *xij = xi + j * C;
                    for (int64_t k = 0; k < N; ++k)
                        for (int64_t c = 0; c < C; ++c) xij[c] += ai[k * C + c] * bj[k * C + c];
                }
            } else {
                for (int64_t k = 0; k < N; ++k) {
                    const double *aki = a + bb * plane + k * row + i * C;  /* a[b, k, i, :] */
                    const double *bk = bm + bb * plane + k * row;          /* b[b, k, :, :] */
                    for (int64_t j = 0; j < N; ++j)
                        for (int64_t c = 0; c < C; ++c) xi[j * C + c] += aki[c] * bk[j * C + c];
                }
            }
        }
    }
    return 0;
}

/* Step 4: out[r, :] = m_r * sigmoid(zhat W_g^T + b_g) (.) (LayerNorm_{c_h}(x) W_o^T + b_o). */
int oracle_output_gate(int64_t rows, int64_t c_z, int64_t c_h, const double *zhat,
                       const double *x, const double *mask, const double *Wg, const double *bg,
                       const double *ln_out_g, const double *ln_out_b, double eps,
                       const double *Wo, const double *bo, double *out) {
    if (rows < 0 || c_z <= 0 || c_h <= 0 || !zhat || !x || !Wg || !Wo || !out) return -1;
    double *xn = (double *)malloc(sizeof(double) * (size_t)(rows * c_h + 1));
    double *g = (double *)malloc(sizeof(double) * (size_t)(rows * c_z + 1));
    if (!xn || !g) { free(xn); free(g); return -2; }
    oracle_layernorm(rows, c_h, x, ln_out_g, ln_out_b, eps, xn);
    oracle_linear(rows, c_h, c_z, xn, Wo, bo, out);
    oracle_linear(rows, c_z, c_z, zhat, Wg, bg, g);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double m = mask ? mask[r] : 1.0;
        for (int64_t o = 0; o < c_z; ++o) {
            int64_t t = r * c_z + o;
            out[t] = m * logistic(g[t]) * out[t];
        }
    }
    free(xn);
    free(g);
    return 0;
}

/* Steps 1-4 on the whole problem. out is [B, N, N, c_z]. mask NULL = all ones.
 * Optional hooks a_out/b_out/x_out ([B, N, N, c_h]) receive the intermediates. */
int oracle_trimul_ex(int64_t B, int64_t N, int64_t c_z, int64_t c_h, const double *z,
                     const double *mask, const oracle_weights_t *w, int direction, double eps,
                     double *out, double *a_out, double *b_out, double *x_out) {
    if (B < 0 || N < 0 || c_z <= 0 || c_h <= 0 || !z || !w || !out) return -1;
    if (!w->w_ag || !w->w_ap || !w->w_bg || !w->w_bp || !w->w_g || !w->w_o) return -1;
    const int64_t P = B * N * N;
    if (P == 0) return 0;
    double *zhat = (double *)malloc(sizeof(double) * (size_t)(P * c_z));
    double *a = a_out ? a_out : (double *)malloc(sizeof(double) * (size_t)(P * c_h));
    double *bm = b_out ? b_out : (double *)malloc(sizeof(double) * (size_t)(P * c_h));
    double *x = x_out ? x_out : (double *)malloc(sizeof(double) * (size_t)(P * c_h));
    int rc = 0;
    if (!zhat || !a || !bm || !x) { rc = -2; goto done; }
    oracle_layernorm(P, c_z, z, w->ln_in_g, w->ln_in_b, eps, zhat);
    oracle_gated_projection(P, c_z, c_h, zhat, mask, w->w_ag, w->b_ag, w->w_ap, w->b_ap, a);
    oracle_gated_projection(P, c_z, c_h, zhat, mask, w->w_bg, w->b_bg, w->w_bp, w->b_bp, bm);
    rc = oracle_contract(B, N, c_h, a, bm, direction, x);
    if (rc) goto done;
    rc = oracle_output_gate(P, c_z, c_h, zhat, x, mask, w->w_g, w->b_g, w->ln_out_g,
                            w->ln_out_b, eps, w->w_o, w->b_o, out);
done:
    free(zhat);
    if (!a_out) free(a);
    if (!b_out) free(bm);
    if (!x_out) free(x);
    return rc;
}

int oracle_trimul(int64_t B, int64_t N, int64_t c_z, int64_t c_h, const double *z,
                  const double *mask, const oracle_weights_t *w, int direction, double eps,
                  double *out) {
    return oracle_trimul_ex(B, N, c_z, c_h, z, mask, w, direction, eps, out, NULL, NULL, NULL);
}

/* Steps 1-4 for the nI x nJ entries (I[p], J[q]) of every batch element only.
 * out is [B, nI, nJ, c_z]. Outgoing needs a on rows I and b on rows J; incoming
 * needs a on columns I and b on columns J. The per-entry arithmetic, including
 * the order of the k sum, is the same as in the full computation. */
int oracle_trimul_sampled(int64_t B, int64_t N, int64_t c_z, int64_t c_h, const double *z,
                          const double *mask, const oracle_weights_t *w, int direction,
                          double eps, const int64_t *I, int64_t nI, const int64_t *J,
                          int64_t nJ, double *out) {
    if (B < 0 || N <= 0 || c_z <= 0 || c_h <= 0 || !z || !w || !out || !I || !J) return -1;
    if (direction != ORACLE_OUTGOING && direction != ORACLE_INCOMING) return -1;
    for (int64_t p = 0; p < nI; ++p) if (I[p] < 0 || I[p] >= N) return -1;
    for (int64_t q = 0; q < nJ; ++q) if (J[q] < 0 || J[q] >= N) return -1;
    const int64_t nmax = nI > nJ ? nI : nJ;
    double *zg = (double *)malloc(sizeof(double) * (size_t)(nmax * N * c_z));
    double *zh = (double *)malloc(sizeof(double) * (size_t)(nmax * N * c_z));
    double *mg = (double *)malloc(sizeof(double) * (size_t)(nmax * N));
    double *as = (double *)malloc(sizeof(double) * (size_t)(nI * N * c_h));
    double *bs = (double *)malloc(sizeof(double) * (size_t)(nJ * N * c_h));
    double *xs = (double *)malloc(sizeof(double) * (size_t)(nI * nJ * c_h));
    double *zs = (double *)malloc(sizeof(double) * (size_t)(nI * nJ * c_z));
    double *zsh = (double *)malloc(sizeof(double) * (size_t)(nI * nJ * c_z));
    double *ms = (double *)malloc(sizeof(double) * (size_t)(nI * nJ));
    int rc = 0;
    if (!zg || !zh || !mg || !as || !bs || !xs || !zs || !zsh || !ms) { rc = -2; goto done; }
    for (int64_t bb = 0; bb < B; ++bb) {
        const double *zb = z + bb * N * N * c_z;
        const double *mb = mask ? mask + bb * N * N : NULL;
        /* gather the lines of pairs that feed a (index set I) and b (index set J) */
        for (int side = 0; side < 2; ++side) {
            const int64_t *S = side == 0 ? I : J;
            const int64_t nS = side == 0 ? nI : nJ;
            for (int64_t p = 0; p < nS; ++p) {
                for (int64_t k = 0; k < N; ++k) {
                    /* outgoing: pair (S[p], k); incoming: pair (k, S[p]) */
                    int64_t pr = direction == ORACLE_OUTGOING ? S[p] * N + k : k * N + S[p];
                    memcpy(zg + (p * N + k) * c_z, zb + pr * c_z, sizeof(double) * (size_t)c_z);
                    mg[p * N + k] = mb ? mb[pr] : 1.0;
                }
            }
            oracle_layernorm(nS * N, c_z, zg, w->ln_in_g, w->ln_in_b, eps, zh);
            if (side == 0)
                oracle_gated_projection(nS * N, c_z, c_h, zh, mg, w->w_ag, w->b_ag, w->w_ap, w->b_ap, as);
            else
                oracle_gated_projection(nS * N, c_z, c_h, zh, mg, w->w_bg, w->b_bg, w->w_bp, w->b_bp, bs);
        }
        /* x at (I[p], J[q]): sum over k ascending of as[p, k] * bs[q, k] */
#pragma omp parallel for collapse(2) schedule(static)
        for (int64_t p = 0; p < nI; ++p) {
            for (int64_t q = 0; q < nJ; ++q) {
                double *xpq = xs + (p * nJ + q) * c_h;
                for (int64_t c = 0; c < c_h; ++c) xpq[c] = 0.0;
                for (int64_t k = 0; k < N; ++k)
                    for (int64_t c = 0; c < c_h; ++c)
                        xpq[c] += as[(p * N + k) * c_h + c] * bs[(q * N + k) * c_h + c];
            }
        }
        for (int64_t p = 0; p < nI; ++p)
            for (int64_t q = 0; q < nJ; ++q) {
                int64_t pr = I[p] * N + J[q];
                memcpy(zs + (p * nJ + q) * c_z, zb + pr * c_z, sizeof(double) * (size_t)c_z);
                ms[p * nJ + q] = mb ? mb[pr] : 1.0;
            }
        oracle_layernorm(nI * nJ, c_z, zs, w->ln_in_g, w->ln_in_b, eps, zsh);
        rc = oracle_output_gate(nI * nJ, c_z, c_h, zsh, xs, ms, w->w_g, w->b_g, w->ln_out_g,
                                w->ln_out_b, eps, w->w_o, w->b_o, out + bb * nI * nJ * c_z);
        if (rc) goto done;
    }
done:
    free(zg); free(zh); free(mg); free(as); free(bs); free(xs); free(zs); free(zsh); free(ms);
    return rc;
}
