/*
 * CPU oracle for the STEPQuant packed-state gated Delta-rule decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it, and it shares no code
 * with that path.
 *
 * Plain, slow, scalar nested loops written for a reader who checks them against
 * the pages describing the method:
 *   [P1] ai-feeds.com summary (Chinese), sections "方法" (method) and
 *        "核心洞察" (insights);
 *   [P2] ai.info summary "STEPQuant: When and Where Errors Matter in
 *        Delta-Rule Recurrent State Quantization", sections "Key
 *        Contributions", "Main Findings", "Methodology in Plain English";
 *   [P4] ai-papers.net article, section "STEPQuantの仕組み" (mechanism);
 *   [P5] ai-trend.me review, sections "방법" (method), "핵심 용어" (terms).
 *
 * Each function is compiled twice: with REAL = float (suffix _f32, the
 * parity mode: every stored or element-wise quantity is fp32, sums are
 * accumulated in fp64 and rounded once) and REAL = double (suffix _f64, for
 * the invariant checks).
 *
 * Readings taken where the pages are silent (each restated at its function):
 *   - state S is [dk x dv], key rows i, value columns j;
 *   - update: S' = diag(alpha) S; v_old = S'^T k; S = S' + beta k (v - v_old)^T;
 *     readout o = S^T q on the updated, unquantised state;
 *   - stored form S_ij = r_i * c_j * code_ij, symmetric codes in [-Q_b, Q_b],
 *     Q_b = 2^(b-1) - 1, kept offset-binary (u = code + 2^(b-1), never 0);
 *   - row scale r_i = rms_i * max(rho_i, rho_max / 4)^(-1/2) / Q_(b_i)
 *     (rms_i -> 1 if zero; rho_max the largest weight of the state's quantised rows);
 *   - column scale: init c_j = max_i |S_ij| / (r_i Q_(b_i)) (-> 1 if zero),
 *     then ls_iters rounds of impact-weighted least squares for fixed codes,
 *     weights rho_i r_i^2 on p_ij = S_ij / r_i;
 *   - rounding half-to-even everywhere; pivot rows stored as IEEE binary16.
 */
#ifndef STEPQ_ORACLE_H
#define STEPQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_PIVOT_BITS 16

/* pivot storage: fp16 (the method), or exact REAL (debug: lets an all-pivot
 * state be compared bit for bit with an unquantised recursion) */
#define ORACLE_PIVOT_FP16 0
#define ORACLE_PIVOT_EXACT 1

/* ---- type-generic per-item functions (one (request, head) state) ---------- */

/* Fit row and column scales to S and quantise it.
 *   S      [dk*dv] row-major state to store.
 *   bits   [dk] row widths: 2..8, or 16 for an FP16 pivot row.
 *   rho    [dk] row-impact weights (> 0).
 * Outputs: r [dk] (0 on pivot rows), c [dv] (0 if every row is a pivot),
 *   code [dk*dv] signed codes (0 on pivot rows), piv [dk*dv] pivot values
 *   (0 on quantised rows).
 * Optional diagnostics (NULL to skip): tpre [dk*dv] the final pre-round values
 *   p_ij / c_j; lsgap [dv] per column, the smallest relative distance of a
 *   least-squares rounding decision from a rounding boundary (+inf if none). */
void oracle_fit_quantise_f32(int dk, int dv, const float *S, const uint8_t *bits,
                             const float *rho, int ls_iters, int pivot_mode,
                             float *r, float *c, int32_t *code, float *piv,
                             float *tpre, float *lsgap);
void oracle_fit_quantise_f64(int dk, int dv, const double *S, const uint8_t *bits,
                             const float *rho, int ls_iters, int pivot_mode,
                             double *r, double *c, int32_t *code, double *piv,
                             double *tpre, double *lsgap);
/* Fit variants for the ablations (stepq_oracle_core.inc states each):
 * ORACLE_SCALE_DUAL (the method), _ROW (row scales only), _COL (column scales
 * only), _HEAD (one scale per state).  Outputs as oracle_fit_quantise_f32. */
#define ORACLE_SCALE_DUAL 0
#define ORACLE_SCALE_ROW 1
#define ORACLE_SCALE_COL 2
#define ORACLE_SCALE_HEAD 3
void oracle_fit_quantise_mode_f32(int mode, int dk, int dv, const float *S, const uint8_t *bits,
                                  const float *rho, int ls_iters, int pivot_mode, float *r, float *c,
                                  int32_t *code, float *piv, float *tpre);
void oracle_fit_quantise_mode_f64(int mode, int dk, int dv, const double *S, const uint8_t *bits,
                                  const float *rho, int ls_iters, int pivot_mode, double *r, double *c,
                                  int32_t *code, double *piv, double *tpre);

/* Quantise S with given scales (final step of the fit, exposed for checks). */
void oracle_quantise_f32(int dk, int dv, const float *S, const uint8_t *bits, const float *r,
                         const float *c, int32_t *code, float *tpre);
void oracle_quantise_f64(int dk, int dv, const double *S, const uint8_t *bits, const double *r,
                         const double *c, int32_t *code, double *tpre);

/* Dequantise: S_ij = (r_i * c_j) * code_ij on quantised rows, piv_ij on pivot rows. */
void oracle_dequant_f32(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                        const int32_t *code, const float *piv, float *S);
void oracle_dequant_f64(int dk, int dv, const uint8_t *bits, const double *r, const double *c,
                        const int32_t *code, const double *piv, double *S);

/* Gated Delta-rule update in place, then readout:
 *   S'_ij = alpha_i S_ij; v_old_j = sum_i S'_ij k_i;
 *   S_ij = S'_ij + (beta k_i)(v_j - v_old_j); o_j = sum_i S_ij q_i.
 * alpha [dk] (Gated-DeltaNet passes one value repeated over the rows). */
void oracle_update_f32(int dk, int dv, float *S, const float *alpha, const float *q,
                       const float *k, const float *v, float beta, float *o);
void oracle_update_f64(int dk, int dv, double *S, const double *alpha, const double *q,
                       const double *k, const double *v, double beta, double *o);

/* Weighted reconstruction error of one column j under scales r, c and codes:
 * sum over quantised rows of rho_i (S_ij - r_i c_j code_ij)^2. */
double oracle_column_error_f64(int dk, int dv, int j, const double *S, const uint8_t *bits,
                               const float *rho, const double *r, double cj,
                               const int32_t *code);

/* ---- IEEE binary16 (round to nearest, ties to even) ----------------------- */
uint16_t oracle_to_fp16(double x);
double oracle_from_fp16(uint16_t h);

/* ---- packed byte format (the pool) ---------------------------------------- *
 * item = r[dk] fp32 | c[dv] fp32 | slab 0 | ... | slab dv/16 - 1; slab s holds
 * value columns 16s..16s+15 as NS = 4 dk/16 streams.  Stream l covers key rows
 * 16 (l % (dk/16)) .. +15 and columns 16s + 4 (l / (dk/16)) .. +3: row by row,
 * column by column, an F_p-bit field per element (offset-binary code
 * u = code + 2^(F_p - 1), or the 16 binary16 bits on a pivot row),
 * little-endian, zero-padded to W = ceil(4 sum_p F_p / 32) words; F_p, the
 * field width of position p (row 16 g + p of any group g), is the widest row
 * at that position over the groups.  Word m of stream l sits at word
 * m * NS + l of the slab.  Storage rows: key order when the head has one
 * width; otherwise the key rows sorted by width (widest first, ties by
 * index), the j-th stored as row 16 (j % (dk/16)) + j / (dk/16); r[] is
 * stored in storage order.  Requires dk % 16 == 0, dk <= 1024 and
 * dv % 16 == 0. */
size_t oracle_item_bytes(int dk, int dv, const uint8_t *bits);
void oracle_pack_item(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                      const int32_t *code, const float *piv, uint8_t *item);
void oracle_unpack_item(int dk, int dv, const uint8_t *bits, const uint8_t *item,
                        float *r, float *c, int32_t *code, float *piv);

/* ---- batched drivers over "slots" (a slot = one (request, head) state) ---- *
 * slot_head[s] gives the head of slot s; bits/rho are per-head tables
 * [H*dk].  The pool holds the slots' items back to back in slot order.
 * alpha is [n*dk] when kda != 0, else [n]. */
size_t oracle_pool_bytes(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits);
void oracle_pack_pool(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                      const float *rho, int ls_iters, const float *S, uint8_t *pool);
void oracle_unpack_pool(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                        const uint8_t *pool, float *S);
/* One decode step over every slot: dequantise, update, read out, refit,
 * requantise, repack.  Optional diagnostics as in oracle_fit_quantise_f32
 * (tpre [n*dk*dv], lsgap [n*dv]); S_new [n*dk*dv] receives the updated
 * unquantised state. */
void oracle_decode_step(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                        const float *rho, int ls_iters, int kda, uint8_t *pool,
                        const float *q, const float *k, const float *v, const float *alpha,
                        const float *beta, float *out, float *S_new, float *tpre, float *lsgap);
/* oracle_pack_pool and oracle_decode_step with a fit variant (ORACLE_SCALE_*);
 * mode ORACLE_SCALE_DUAL is the two functions above. */
void oracle_pack_pool_mode(int mode, int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                           const float *rho, int ls_iters, const float *S, uint8_t *pool);
void oracle_decode_step_mode(int mode, int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                             const float *rho, int ls_iters, int kda, uint8_t *pool, const float *q,
                             const float *k, const float *v, const float *alpha, const float *beta,
                             float *out, float *S_new, float *tpre);
/* Unquantised fp32 recursion over slots (the fp32-state baseline). */
void oracle_fp32_step(int n, int dk, int dv, int kda, float *S, const float *q, const float *k,
                      const float *v, const float *alpha, const float *beta, float *out);
/* Unquantised fp64 recursion over slots. */
void oracle_fp64_step(int n, int dk, int dv, int kda, double *S, const double *q,
                      const double *k, const double *v, const double *alpha,
                      const double *beta, double *out);

/* ---- calibration of the tables (stepq_oracle_calib.c) --------------------- *
 * The offline step before the decode path: impact scores rho and row widths
 * from a synthetic calibration rollout.  Units: heads (Gated-DeltaNet) or key
 * rows (KDA). */
#define ORACLE_CALIB_RHO_FLOOR 1e-30  /* rho of a row whose query weight is always 0 */
#define ORACLE_CALIB_GAP_FLOOR 1e-12  /* 1 - abar^2 floor: a unit that never decays */

/* One step's inputs into the running sums: acc_q2[h*dk+i] += sum_b q[b,h,i]^2
 * (fp64, batch order); acc_loga[u] += sum_b log alpha[b,u], u = h for
 * Gated-DeltaNet (alpha [batch*heads]) or h*dk+i for KDA (alpha
 * [batch*heads*dk]).  q is [batch*heads*dk]. */
void oracle_calib_accumulate(int kda, int batch, int heads, int dk, const float *q, const float *alpha,
                             double *acc_q2, double *acc_loga);
/* rho[u] = fp32(max(acc_q2[u] / n_samples, ORACLE_CALIB_RHO_FLOOR)), u < heads*dk. */
void oracle_calib_rho(int heads, int dk, double n_samples, const double *acc_q2, float *rho);
/* S [dk*dv] fitted and quantised with every row at width b (fp32 parity
 * mode): r [dk], c [dv] and err[i] = sum_j (S_ij - r_i c_j code_ij)^2 in fp64. */
void oracle_calib_row_error(int dk, int dv, const float *S, int b, const float *rho, int ls_iters, float *r,
                            float *c, double *err);
/* Lifetime weight 1 / (1 - exp(m)^2) of a unit with mean log retention m. */
double oracle_calib_weight(double mean_log_alpha);
/* Greedy lifetime-weighted allocation: D [n*nc] distortion of unit u at
 * choices[x] (ascending); writes bits [n] (16 = pivot).  Returns -1 (bits
 * still written, with no upgrade) when the pivots and the narrowest width
 * alone exceed the budget round(avg_bits * n), else 0. */
int oracle_calib_allocate(int n, const double *weight, const double *D, int nc, const int *choices,
                          double avg_bits, int n_piv, uint8_t *bits);
/* Widths of every row, bits [heads*dk], from the sums: weights from acc_loga
 * (n_samples terms per unit), distortions from err [heads][nc][dk] (the
 * per-row errors summed over the sampled states) weighted by rho [heads*dk];
 * n_piv = ceil(pivot_frac * units).  Returns as oracle_calib_allocate. */
int oracle_calib_bits(int kda, int heads, int dk, double n_samples, const double *acc_loga, const float *rho,
                      const double *err, int nc, const int *choices, double avg_bits, double pivot_frac,
                      uint8_t *bits);

#ifdef __cplusplus
}
#endif
#endif
