/*
 * CPU oracle for the calibration that produces the decode path's tables --
 * TEST INFRASTRUCTURE ONLY (see stepq_oracle.h): loaded by the tests and the
 * benchmark's CPU leg, never by the product path.
 *
 * The pages describe an offline calibration that fixes, once for all
 * requests, (1) each unit's width from its quantisation distortion at the
 * candidate widths and its mean log retention, under an average bit budget
 * with the riskiest few units kept as FP16 pivots, and (2) a per-key-row
 * impact score, the expected squared weight of the row's error in the readout
 * ([P2] ai.info, "Methodology in Plain English"; [P4] ai-papers.net,
 * "STEPQuantの仕組み"; [P5] ai-trend.me, "방법").  Units are whole heads for
 * Gated-DeltaNet and key rows for KDA ([P4], [P5]).
 *
 * Readings taken where the pages leave a step open (each restated below):
 *   - impact score rho_i = mean over the calibration requests and steps of
 *     q_i^2: the readout o = S^T q weighs an error in key row i by q_i;
 *   - lifetime weight w_u = 1 / (1 - abar_u^2), abar_u = exp(mean log alpha_u):
 *     the summed squared decay sum_t abar^(2t) of an error written once;
 *   - distortion D_u(b) = sum over sampled fp32 rollout states of
 *     sum_(rows i of u) rho_i sum_j (S_ij - r_i c_j code_ij)^2, every row of
 *     the head fitted and quantised at width b;
 *   - allocation: every unit starts at the narrowest width; the n_piv units
 *     of largest risk w_u D_u(narrowest) become pivots (16 bits, counted in the
 *     budget); then the upgrade to the next candidate width with the largest
 *     w_u (D_u(b) - D_u(b')) / (b' - b) that still fits the remaining budget
 *     and lowers the objective is applied, until none is left; ties go to the
 *     lower unit index.
 */
#include "stepq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

void oracle_calib_accumulate(int kda, int batch, int heads, int dk, const float *q, const float *alpha,
                             double *acc_q2, double *acc_loga)
{
    for (int h = 0; h < heads; h++)
        for (int i = 0; i < dk; i++) {
            double s = 0.0;
            for (int b = 0; b < batch; b++) {
                const double x = (double)q[((size_t)b * heads + h) * dk + i];
                s += x * x;
            }
            acc_q2[(size_t)h * dk + i] += s;
        }
    if (kda) {
        for (int h = 0; h < heads; h++)
            for (int i = 0; i < dk; i++) {
                double s = 0.0;
                for (int b = 0; b < batch; b++) s += log((double)alpha[((size_t)b * heads + h) * dk + i]);
                acc_loga[(size_t)h * dk + i] += s;
            }
    } else {
        for (int h = 0; h < heads; h++) {
            double s = 0.0;
            for (int b = 0; b < batch; b++) s += log((double)alpha[(size_t)b * heads + h]);
            acc_loga[h] += s;
        }
    }
}

void oracle_calib_rho(int heads, int dk, double n_samples, const double *acc_q2, float *rho)
{
    for (int u = 0; u < heads * dk; u++) {
        double m = acc_q2[u] / n_samples;
        if (m < ORACLE_CALIB_RHO_FLOOR) m = ORACLE_CALIB_RHO_FLOOR;
        rho[u] = (float)m;
    }
}

void oracle_calib_row_error(int dk, int dv, const float *S, int b, const float *rho, int ls_iters, float *r,
                            float *c, double *err)
{
    uint8_t *bits = (uint8_t *)malloc((size_t)dk);
    int32_t *code = (int32_t *)malloc(sizeof(int32_t) * (size_t)dk * dv);
    float *piv = (float *)malloc(sizeof(float) * (size_t)dk * dv);
    memset(bits, b, (size_t)dk);
    oracle_fit_quantise_f32(dk, dv, S, bits, rho, ls_iters, ORACLE_PIVOT_FP16, r, c, code, piv, NULL, NULL);
    for (int i = 0; i < dk; i++) {
        double e = 0.0;
        for (int j = 0; j < dv; j++) {
            const double d = (double)S[(size_t)i * dv + j] - (double)r[i] * (double)c[j] * (double)code[(size_t)i * dv + j];
            e += d * d;
        }
        err[i] = e;
    }
    free(bits);
    free(code);
    free(piv);
}

double oracle_calib_weight(double mean_log_alpha)
{
    const double a = exp(mean_log_alpha);
    double g = 1.0 - a * a;
    if (g < ORACLE_CALIB_GAP_FLOOR) g = ORACLE_CALIB_GAP_FLOOR;
    return 1.0 / g;
}

int oracle_calib_allocate(int n, const double *weight, const double *D, int nc, const int *choices,
                          double avg_bits, int n_piv, uint8_t *bits)
{
    int *k = (int *)malloc(sizeof(int) * (size_t)n);  /* index into choices; -1 = pivot */
    for (int u = 0; u < n; u++) k[u] = 0;
    /* pivots: the n_piv largest risks w_u D_u(narrowest), ties to the lower index */
    for (int p = 0; p < n_piv && p < n; p++) {
        int best = -1;
        double br = 0.0;
        for (int u = 0; u < n; u++) {
            if (k[u] < 0) continue;
            const double risk = weight[u] * D[(size_t)u * nc];
            if (best < 0 || risk > br) {
                best = u;
                br = risk;
            }
        }
        k[best] = -1;
    }
    long long used = 0;
    for (int u = 0; u < n; u++) used += (k[u] < 0) ? ORACLE_PIVOT_BITS : choices[0];
    long long remaining = llround(avg_bits * n) - used;
    const int status = (remaining < 0) ? -1 : 0;
    for (;;) {
        int best = -1;
        double bg = 0.0;
        for (int u = 0; u < n; u++) {
            if (k[u] < 0 || k[u] + 1 >= nc) continue;
            const int cost = choices[k[u] + 1] - choices[k[u]];
            if (cost > remaining) continue;
            const double g = weight[u] * (D[(size_t)u * nc + k[u]] - D[(size_t)u * nc + k[u] + 1]) / cost;
            if (!(g > 0.0)) continue;
            if (best < 0 || g > bg) {
                best = u;
                bg = g;
            }
        }
        if (best < 0) break;
        remaining -= choices[k[best] + 1] - choices[k[best]];
        k[best]++;
    }
    for (int u = 0; u < n; u++) bits[u] = (uint8_t)((k[u] < 0) ? ORACLE_PIVOT_BITS : choices[k[u]]);
    free(k);
    return status;
}

int oracle_calib_bits(int kda, int heads, int dk, double n_samples, const double *acc_loga, const float *rho,
                      const double *err, int nc, const int *choices, double avg_bits, double pivot_frac,
                      uint8_t *bits)
{
    const int n = kda ? heads * dk : heads;
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    double *D = (double *)malloc(sizeof(double) * (size_t)n * nc);
    for (int u = 0; u < n; u++) w[u] = oracle_calib_weight(acc_loga[u] / n_samples);
    for (int h = 0; h < heads; h++)
        for (int x = 0; x < nc; x++) {
            const double *e = err + ((size_t)h * nc + x) * dk;
            if (kda) {
                for (int i = 0; i < dk; i++) D[((size_t)h * dk + i) * nc + x] = (double)rho[h * dk + i] * e[i];
            } else {
                double s = 0.0;
                for (int i = 0; i < dk; i++) s += (double)rho[h * dk + i] * e[i];
                D[(size_t)h * nc + x] = s;
            }
        }
    const int n_piv = (pivot_frac > 0.0) ? (int)ceil(pivot_frac * n - 1e-9) : 0;
    uint8_t *ub = (uint8_t *)malloc((size_t)n);
    const int status = oracle_calib_allocate(n, w, D, nc, choices, avg_bits, n_piv, ub);
    for (int h = 0; h < heads; h++)
        for (int i = 0; i < dk; i++) bits[h * dk + i] = kda ? ub[h * dk + i] : ub[h];
    free(w);
    free(D);
    free(ub);
    return status;
}
