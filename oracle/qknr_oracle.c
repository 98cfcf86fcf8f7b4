/*
 * CPU oracle for the fused per-head QK-RMSNorm + rotate-half RoPE,
 * forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. This file is compiled into a separate shared
 * object that only the test suite, the package's smoke check and the bench's
 * CPU-baseline leg load. The CUDA library never links, includes or calls it,
 * and it shares no code with the CUDA path.
 *
 * Plain C, fp64 throughout, one row at a time, in the order the method is
 * stated. No blocking, fusion or reordering: a reader should be able to check
 * each line against the definition below.
 *
 * Sources for the method:
 *  - Chronicals (arXiv 2601.02609), abstract, contribution (1): Q and K go
 *    through RMSNorm and RoPE in one fused pass ("QK-RoPE").
 *  - "QK-Normed MLA: QK normalization without full key caching", abstract:
 *    the statistic kept per (token, head) is one inverse-RMS scalar.
 *  - "Fractional Rotation, Full Potential? Investigating Performance and
 *    Convergence of Partial RoPE", abstract: only the first fraction of each
 *    head's dimensions is rotated; the rest pass through.
 *  - The pages print no formula. The formula written out here is the plain
 *    reading of the benchmark spec: RMSNorm over the head dimension D with
 *    eps inside the root and a learned per-dim weight gamma, then
 *    rotate-half RoPE over the first R dims with inverse frequency
 *    theta^(-2i/R).
 *
 * Forward, per row x (one token, one head), position m:
 *   ms      = (1/D) * sum_d x_d^2
 *   r       = 1 / sqrt(ms + eps)                     (saved inverse RMS)
 *   n_d     = x_d * r * gamma_d                      for all d < D
 *   w_i     = theta^(-2i/R)                          for i < R/2
 *   y_i     = n_i * cos(m w_i) - n_{i+R/2} * sin(m w_i)
 *   y_{i+R/2} = n_{i+R/2} * cos(m w_i) + n_i * sin(m w_i)
 *   y_d     = n_d                                    for R <= d < D
 * Backward, given dy = dL/dy for the row:
 *   g       = transpose(rotation) applied to dy      (dL/dn)
 *   dgamma_d += g_d * x_d * r                        (summed over the tensor's rows)
 *   h_d     = g_d * gamma_d
 *   dx_d    = r * h_d - r^3 * x_d * (1/D) * sum_e h_e x_e
 * Mean-centred variant (QK-LayerNorm: "Nyonic Technical Report", abstract,
 * names QK-LayerNorm with rotary embeddings; weight only, no bias):
 *   mu      = (1/D) * sum_d x_d
 *   r       = 1 / sqrt((1/D) * sum_d (x_d - mu)^2 + eps)    (saved)
 *   n_d     = (x_d - mu) * r * gamma_d, then the same rotation
 *   backward: xh = (x - mu) r, dgamma += g xh, h = g gamma,
 *   dx_d    = r * (h_d - (1/D) sum_e h_e - xh_d (1/D) sum_e h_e xh_e)
 * Layerwise variant ("SwiftQK: Fast and Communication-Efficient Tensor
 * Parallelism for Query-Key Normalization", abstract: the normalisation
 * factor depends on the full hidden vector): per token, over all H heads,
 *   r_t     = 1 / sqrt((1/(H D)) * sum_{h,d} x[h,d]^2 + eps)   (saved)
 *   n[h,d]  = x[h,d] * r_t * gamma[h*D + d]   (gamma over the full hidden),
 *   then the same rotation on every head row; backward, per token:
 *   xh = x r_t, dgamma[h*D + d] += g xh, hh = g gamma,
 *   dx = r_t * (hh - xh * (1/(H D)) * sum_{h,d} hh xh)
 * Rotation alone (no normalisation), forward or inverse:
 *   y = R(m) x, or y = R(m)^T x = R(-m) x, which strips RoPE from a rotated
 *   row (the cross-model KV cache transfer abstract on the papers listing:
 *   keys have RoPE stripped before mapping so the fit is position-free).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Inverse frequency of rotary pair i over a rotary span of R dims. */
double oracle_inv_freq(int i, int R, double theta)
{
    return pow(theta, -2.0 * (double)i / (double)R);
}

/* Inverse RMS of one row: 1 / sqrt(mean(x^2) + eps). */
double oracle_rstd(const double *x, int D, double eps)
{
    double ms = 0.0;
    for (int d = 0; d < D; ++d)
        ms += x[d] * x[d];
    ms /= (double)D;
    return 1.0 / sqrt(ms + eps);
}

/* Forward of one row. y and x may not overlap. */
void oracle_fwd_row(const double *x, const double *gamma, int D, int R,
                    double theta, double eps, int64_t m,
                    double *y, double *rstd)
{
    double r = oracle_rstd(x, D, eps);
    double *n = (double *)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d)
        n[d] = x[d] * r * gamma[d];
    for (int d = 0; d < D; ++d)
        y[d] = n[d];
    int half = R / 2;
    for (int i = 0; i < half; ++i) {
        double phi = (double)m * oracle_inv_freq(i, R, theta);
        double c = cos(phi), s = sin(phi);
        y[i] = n[i] * c - n[i + half] * s;
        y[i + half] = n[i + half] * c + n[i] * s;
    }
    free(n);
    *rstd = r;
}

/*
 * Backward of one row. dx is written; dgamma (length D) is accumulated into,
 * so the caller zeroes it once per tensor.
 */
void oracle_bwd_row(const double *x, const double *gamma, const double *dy,
                    int D, int R, double theta, double eps, int64_t m,
                    double *dx, double *dgamma)
{
    double r = oracle_rstd(x, D, eps);
    double *g = (double *)malloc(sizeof(double) * (size_t)D);
    double *h = (double *)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d)
        g[d] = dy[d];
    int half = R / 2;
    for (int i = 0; i < half; ++i) {
        double phi = (double)m * oracle_inv_freq(i, R, theta);
        double c = cos(phi), s = sin(phi);
        g[i] = dy[i] * c + dy[i + half] * s;
        g[i + half] = -dy[i] * s + dy[i + half] * c;
    }
    for (int d = 0; d < D; ++d)
        dgamma[d] += g[d] * x[d] * r;
    for (int d = 0; d < D; ++d)
        h[d] = g[d] * gamma[d];
    double dot = 0.0;
    for (int e = 0; e < D; ++e)
        dot += h[e] * x[e];
    for (int d = 0; d < D; ++d)
        dx[d] = r * h[d] - r * r * r * x[d] * dot / (double)D;
    free(g);
    free(h);
}

/*
 * Forward over T tokens. q [T,Hq,D], k [T,Hkv,D] contiguous (T = B*S, or any
 * run of consecutive tokens); m [T] holds each token's position. Outputs use
 * the same indexing; rstd_q [T,Hq], rstd_k [T,Hkv].
 */
void oracle_fwd(const double *q, const double *k,
                const double *gamma_q, const double *gamma_k,
                const int64_t *m, int64_t T, int Hq, int Hkv, int D, int R,
                double theta, double eps,
                double *q_out, double *k_out, double *rstd_q, double *rstd_k)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < Hq; ++h) {
            int64_t row = t * Hq + h;
            oracle_fwd_row(q + row * D, gamma_q, D, R, theta, eps, m[t],
                           q_out + row * D, rstd_q + row);
        }
        for (int h = 0; h < Hkv; ++h) {
            int64_t row = t * Hkv + h;
            oracle_fwd_row(k + row * D, gamma_k, D, R, theta, eps, m[t],
                           k_out + row * D, rstd_k + row);
        }
    }
}

/*
 * Backward over T tokens (layout as oracle_fwd). dgamma_q / dgamma_k are
 * accumulated into: zero them before the first run of tokens.
 */
void oracle_bwd(const double *q, const double *k,
                const double *gamma_q, const double *gamma_k,
                const int64_t *m, const double *dq_out, const double *dk_out,
                int64_t T, int Hq, int Hkv, int D, int R, double theta,
                double eps,
                double *dq, double *dk, double *dgamma_q, double *dgamma_k)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < Hq; ++h) {
            int64_t row = t * Hq + h;
            oracle_bwd_row(q + row * D, gamma_q, dq_out + row * D, D, R,
                           theta, eps, m[t], dq + row * D, dgamma_q);
        }
        for (int h = 0; h < Hkv; ++h) {
            int64_t row = t * Hkv + h;
            oracle_bwd_row(k + row * D, gamma_k, dk_out + row * D, D, R,
                           theta, eps, m[t], dk + row * D, dgamma_k);
        }
    }
}

/*
 * Independent rows, each with its own position (used to check sampled rows
 * of full-size problems). x, y, dy, dx: [n, D]; m: [n]; rstd: [n].
 * dgamma_rows: [n, D], each row's own contribution g * x * r (not summed).
 */
void oracle_fwd_rows(const double *x, const double *gamma, const int64_t *m,
                     int64_t n, int D, int R, double theta, double eps,
                     double *y, double *rstd)
{
    for (int64_t j = 0; j < n; ++j)
        oracle_fwd_row(x + j * D, gamma, D, R, theta, eps, m[j], y + j * D,
                       rstd + j);
}

void oracle_bwd_rows(const double *x, const double *gamma, const double *dy,
                     const int64_t *m, int64_t n, int D, int R, double theta,
                     double eps, double *dx, double *dgamma_rows)
{
    for (int64_t j = 0; j < n; ++j) {
        memset(dgamma_rows + j * D, 0, sizeof(double) * (size_t)D);
        oracle_bwd_row(x + j * D, gamma, dy + j * D, D, R, theta, eps, m[j],
                       dx + j * D, dgamma_rows + j * D);
    }
}

/*
 * Rotation alone, rows x [n, D] at positions m [n]: y = R(m) x, or with
 * inverse != 0 the transpose R(m)^T x (sine negated). Dims >= R copy through.
 */
void oracle_rope_rows(const double *x, const int64_t *m, int64_t n, int D,
                      int R, double theta, int inverse, double *y)
{
    int half = R / 2;
    for (int64_t j = 0; j < n; ++j) {
        const double *xr = x + j * D;
        double *yr = y + j * D;
        for (int d = 0; d < D; ++d)
            yr[d] = xr[d];
        for (int i = 0; i < half; ++i) {
            double phi = (double)m[j] * oracle_inv_freq(i, R, theta);
            double c = cos(phi), s = sin(phi);
            if (inverse)
                s = -s;
            yr[i] = xr[i] * c - xr[i + half] * s;
            yr[i + half] = xr[i + half] * c + xr[i] * s;
        }
    }
}

/* Mean of one row. */
double oracle_mean(const double *x, int D)
{
    double s = 0.0;
    for (int d = 0; d < D; ++d)
        s += x[d];
    return s / (double)D;
}

/* Inverse standard deviation of one row about its mean: 1 / sqrt(var + eps). */
double oracle_ln_rstd(const double *x, int D, double eps)
{
    double mu = oracle_mean(x, D);
    double var = 0.0;
    for (int d = 0; d < D; ++d)
        var += (x[d] - mu) * (x[d] - mu);
    var /= (double)D;
    return 1.0 / sqrt(var + eps);
}

/* Mean-centred forward of rows x [n, D] at positions m [n]. */
void oracle_ln_fwd_rows(const double *x, const double *gamma, const int64_t *m,
                        int64_t n, int D, int R, double theta, double eps,
                        double *y, double *rstd)
{
    int half = R / 2;
    double *nr = (double *)malloc(sizeof(double) * (size_t)D);
    for (int64_t j = 0; j < n; ++j) {
        const double *xr = x + j * D;
        double *yr = y + j * D;
        double mu = oracle_mean(xr, D);
        double r = oracle_ln_rstd(xr, D, eps);
        for (int d = 0; d < D; ++d)
            nr[d] = (xr[d] - mu) * r * gamma[d];
        for (int d = 0; d < D; ++d)
            yr[d] = nr[d];
        for (int i = 0; i < half; ++i) {
            double phi = (double)m[j] * oracle_inv_freq(i, R, theta);
            double c = cos(phi), s = sin(phi);
            yr[i] = nr[i] * c - nr[i + half] * s;
            yr[i + half] = nr[i + half] * c + nr[i] * s;
        }
        rstd[j] = r;
    }
    free(nr);
}

/*
 * Mean-centred backward of rows: dx [n, D]; dgamma_rows [n, D] holds each
 * row's own term g * xh (not summed).
 */
void oracle_ln_bwd_rows(const double *x, const double *gamma, const double *dy,
                        const int64_t *m, int64_t n, int D, int R,
                        double theta, double eps, double *dx,
                        double *dgamma_rows)
{
    int half = R / 2;
    double *g = (double *)malloc(sizeof(double) * (size_t)D);
    double *h = (double *)malloc(sizeof(double) * (size_t)D);
    double *xh = (double *)malloc(sizeof(double) * (size_t)D);
    for (int64_t j = 0; j < n; ++j) {
        const double *xr = x + j * D, *dyr = dy + j * D;
        double mu = oracle_mean(xr, D);
        double r = oracle_ln_rstd(xr, D, eps);
        for (int d = 0; d < D; ++d)
            g[d] = dyr[d];
        for (int i = 0; i < half; ++i) {
            double phi = (double)m[j] * oracle_inv_freq(i, R, theta);
            double c = cos(phi), s = sin(phi);
            g[i] = dyr[i] * c + dyr[i + half] * s;
            g[i + half] = -dyr[i] * s + dyr[i + half] * c;
        }
        for (int d = 0; d < D; ++d)
            xh[d] = (xr[d] - mu) * r;
        for (int d = 0; d < D; ++d)
            dgamma_rows[j * D + d] = g[d] * xh[d];
        for (int d = 0; d < D; ++d)
            h[d] = g[d] * gamma[d];
        double mean_h = 0.0, mean_hx = 0.0;
        for (int e = 0; e < D; ++e) {
            mean_h += h[e];
            mean_hx += h[e] * xh[e];
        }
        mean_h /= (double)D;
        mean_hx /= (double)D;
        for (int d = 0; d < D; ++d)
            dx[j * D + d] = r * (h[d] - mean_h - xh[d] * mean_hx);
    }
    free(g);
    free(h);
    free(xh);
}

/*
 * Layerwise forward: x [T, H, D] (one tensor), gamma [H*D], m [T]; y like x,
 * rstd [T] (one statistic per token over its whole hidden vector).
 */
void oracle_lw_fwd(const double *x, const double *gamma, const int64_t *m,
                   int64_t T, int H, int D, int R, double theta, double eps,
                   double *y, double *rstd)
{
    int half = R / 2;
    int64_t HD = (int64_t)H * D;
    for (int64_t t = 0; t < T; ++t) {
        const double *xt = x + t * HD;
        double *yt = y + t * HD;
        double ss = 0.0;
        for (int64_t e = 0; e < HD; ++e)
            ss += xt[e] * xt[e];
        double r = 1.0 / sqrt(ss / (double)HD + eps);
        rstd[t] = r;
        for (int h = 0; h < H; ++h) {
            const double *xr = xt + (int64_t)h * D;
            double *yr = yt + (int64_t)h * D;
            for (int d = 0; d < D; ++d)
                yr[d] = xr[d] * r * gamma[h * D + d];
            for (int i = 0; i < half; ++i) {
                double phi = (double)m[t] * oracle_inv_freq(i, R, theta);
                double c = cos(phi), s = sin(phi);
                double a = yr[i], b = yr[i + half];
                yr[i] = a * c - b * s;
                yr[i + half] = b * c + a * s;
            }
        }
    }
}

/* Layerwise backward: dx like x; dgamma [H*D] accumulated into. */
void oracle_lw_bwd(const double *x, const double *gamma, const double *dy,
                   const int64_t *m, int64_t T, int H, int D, int R,
                   double theta, double eps, double *dx, double *dgamma)
{
    int half = R / 2;
    int64_t HD = (int64_t)H * D;
    double *g = (double *)malloc(sizeof(double) * (size_t)HD);
    for (int64_t t = 0; t < T; ++t) {
        const double *xt = x + t * HD, *dyt = dy + t * HD;
        double ss = 0.0;
        for (int64_t e = 0; e < HD; ++e)
            ss += xt[e] * xt[e];
        double r = 1.0 / sqrt(ss / (double)HD + eps);
        for (int h = 0; h < H; ++h) {
            const double *dr = dyt + (int64_t)h * D;
            double *gr = g + (int64_t)h * D;
            for (int d = 0; d < D; ++d)
                gr[d] = dr[d];
            for (int i = 0; i < half; ++i) {
                double phi = (double)m[t] * oracle_inv_freq(i, R, theta);
                double c = cos(phi), s = sin(phi);
                gr[i] = dr[i] * c + dr[i + half] * s;
                gr[i + half] = -dr[i] * s + dr[i + half] * c;
            }
        }
        double dot = 0.0;
        for (int64_t e = 0; e < HD; ++e) {
            dgamma[e] += g[e] * xt[e] * r;
            dot += g[e] * gamma[e] * xt[e] * r;
        }
        for (int64_t e = 0; e < HD; ++e)
            dx[t * HD + e] = r * (g[e] * gamma[e] - xt[e] * r * dot / (double)HD);
    }
    free(g);
}
