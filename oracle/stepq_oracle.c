/*
 * CPU oracle for the STEPQuant packed-state decode step -- TEST INFRASTRUCTURE
 * ONLY (see stepq_oracle.h): loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (oracle/build.py).
 */
#include "stepq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- IEEE binary16, round to nearest even, written from the format's
 * definition: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;
 * normal numbers span [2^-14, 65504], subnormals are multiples of 2^-24. */
uint16_t oracle_to_fp16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return 0x7E00u;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7C00u;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);          /* a in [2^(e-1), 2^e) */
    int ex = e - 1;
    if (ex < -14) ex = -14; /* the subnormal range shares the quantum 2^-24 */
    double quantum = ldexp(1.0, ex - 10);
    double y = nearbyint(a / quantum) * quantum; /* exact scaling, ties to even */
    if (y > 65504.0) return sign | 0x7C00u;
    if (y < ldexp(1.0, -14)) return sign | (uint16_t)(y / ldexp(1.0, -24));
    frexp(y, &e);
    int E = e - 1; /* y in [2^E, 2^(E+1)) */
    uint16_t frac = (uint16_t)((y / ldexp(1.0, E) - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | frac;
}

double oracle_from_fp16(uint16_t h)
{
    int s = (h >> 15) & 1, E = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (E == 0) v = ldexp((double)f, -24);
    else if (E == 31) v = f ? NAN : INFINITY;
    else v = ldexp(1.0 + f / 1024.0, E - 15);
    return s ? -v : v;
}

#define REAL float
#define SFX(name) name##_f32
#include "stepq_oracle_core.inc"
#undef REAL
#undef SFX

#define REAL double
#define SFX(name) name##_f64
#include "stepq_oracle_core.inc"
#undef REAL
#undef SFX

double oracle_column_error_f64(int dk, int dv, int j, const double *S, const uint8_t *bits,
                               const float *rho, const double *r, double cj,
                               const int32_t *code)
{
    double e = 0.0;
    for (int i = 0; i < dk; i++) {
        if (bits[i] == ORACLE_PIVOT_BITS) continue;
        double d = S[i * dv + j] - r[i] * cj * (double)code[i * dv + j];
        e += (double)rho[i] * d * d;
    }
    return e;
}

/* ---- the packed byte format ---------------------------------------------- *
 * item = r[dk] fp32 | c[dv] fp32 | slab 0 | ... | slab dv/16 - 1.
 * Slab s holds value columns 16s .. 16s+15 of every key row as NS = 4 dk/16
 * streams.  Stream l covers the key rows of row group l % (dk/16) (rows
 * 16 (l % (dk/16)) .. +15) and the value columns 16s + 4 (l / (dk/16)) .. +3:
 * its codes are taken row by row, and within a row column by column, as
 * fields concatenated into one little-endian bit stream that is zero-padded
 * to W 32-bit words.  Word m of stream l is stored at word m * NS + l of the
 * slab.
 *
 * Storage rows.  "Row" above means a storage row.  If every key row of the
 * head has the same width, storage row s is key row s.  Otherwise the key
 * rows are sorted by width, widest first (a pivot row counts 16), ties by key
 * index, and the j-th of them is stored as storage row 16 (j % RG) + j / RG:
 * the rows are dealt to the RG row groups in turn, so every group receives
 * rows of nearly the same widths.  The row scales r[] of the header are
 * stored in storage order.
 *
 * Field widths.  The fields of storage row 16 g + p (position p of group g)
 * are F_p bits wide, F_p = the largest width at position p over all row
 * groups; a row narrower than its field is stored in the wider field.  A
 * quantised row's field holds the offset-binary code u = code + 2^(F_p - 1),
 * a pivot row's field (F_p = 16 then) the binary16 bits of the element.  Every
 * stream of a head therefore has the same layout, and W = ceil(4 sum_p F_p /
 * 32).  For a head of one width b, F_p = b and W = 2b. */

enum { GROUP_ROWS = 16, GROUP_COLS = 4, SLAB_COLS = 16 };

static int field_bits(int b) { return b; } /* a pivot row's field is its 16 binary16 bits */

/* key_of[s] = the key row stored as storage row s (rule above). */
static void storage_rows(int dk, const uint8_t *bits, int *key_of)
{
    int uniform = 1;
    for (int i = 1; i < dk; i++) uniform &= bits[i] == bits[0];
    if (uniform || dk < GROUP_ROWS) {
        for (int s = 0; s < dk; s++) key_of[s] = s;
        return;
    }
    const int RG = dk / GROUP_ROWS;
    int j = 0;
    for (int b = 16; b >= 1; b--) /* widths from widest down; key order within a width */
        for (int i = 0; i < dk; i++)
            if (bits[i] == b) {
                key_of[GROUP_ROWS * (j % RG) + j / RG] = i;
                j++;
            }
}

/* fw[p] = F_p, the field width of position p (rule above), p < 16. */
static void position_widths(int dk, const uint8_t *bits, const int *key_of, int *fw)
{
    for (int p = 0; p < GROUP_ROWS; p++) {
        fw[p] = 0;
        for (int g = 0; g < dk / GROUP_ROWS; g++) {
            const int b = field_bits(bits[key_of[g * GROUP_ROWS + p]]);
            if (b > fw[p]) fw[p] = b;
        }
    }
}

static size_t stream_words(int dk, const uint8_t *bits)
{
    int key_of[1024], fw[GROUP_ROWS];
    storage_rows(dk, bits, key_of);
    position_widths(dk, bits, key_of, fw);
    size_t nbits = 0;
    for (int p = 0; p < GROUP_ROWS; p++) nbits += (size_t)GROUP_COLS * fw[p];
    return (nbits + 31) / 32;
}

size_t oracle_item_bytes(int dk, int dv, const uint8_t *bits)
{
    const size_t NS = (size_t)GROUP_COLS * (dk / GROUP_ROWS);
    return 4 * (size_t)dk + 4 * (size_t)dv + 4 * stream_words(dk, bits) * NS * (size_t)(dv / SLAB_COLS);
}

static void put_f32(uint8_t *dst, float x) { memcpy(dst, &x, 4); } /* host is little-endian */
static float get_f32(const uint8_t *src) { float x; memcpy(&x, src, 4); return x; }

/* bit t of word index wi (little-endian 32-bit words) */
static void set_bit(uint8_t *words, size_t wi, int t) { words[4 * wi + t / 8] |= (uint8_t)(1u << (t % 8)); }
static int get_bit(const uint8_t *words, size_t wi, int t) { return (words[4 * wi + t / 8] >> (t % 8)) & 1; }

void oracle_pack_item(int dk, int dv, const uint8_t *bits, const float *r, const float *c,
                      const int32_t *code, const float *piv, uint8_t *item)
{
    uint8_t *p = item;
    const int RG = dk / GROUP_ROWS, NS = GROUP_COLS * RG;
    const size_t W = stream_words(dk, bits);
    int key_of[1024], fw[GROUP_ROWS];
    storage_rows(dk, bits, key_of);
    position_widths(dk, bits, key_of, fw);
    for (int s = 0; s < dk; s++, p += 4) put_f32(p, r[key_of[s]]);
    for (int j = 0; j < dv; j++, p += 4) put_f32(p, c[j]);
    for (int sl = 0; sl < dv / SLAB_COLS; sl++) {
        memset(p, 0, 4 * W * NS);
        for (int l = 0; l < NS; l++) {
            const int g = l % RG, cg = l / RG;
            size_t pos = 0; /* bit position in stream l */
            for (int rr = 0; rr < GROUP_ROWS; rr++) {
                const int i = key_of[g * GROUP_ROWS + rr], b = bits[i], F = fw[rr];
                for (int kk = 0; kk < GROUP_COLS; kk++) {
                    const int j = sl * SLAB_COLS + cg * GROUP_COLS + kk;
                    const uint32_t u = (b == ORACLE_PIVOT_BITS)
                                           ? oracle_to_fp16((double)piv[i * dv + j])
                                           : (uint32_t)(code[i * dv + j] + (1 << (F - 1)));
                    for (int t = 0; t < F; t++, pos++)
                        if ((u >> t) & 1u) set_bit(p, (pos / 32) * NS + l, (int)(pos % 32));
                }
            }
        }
        p += 4 * W * NS;
    }
}

void oracle_unpack_item(int dk, int dv, const uint8_t *bits, const uint8_t *item,
                        float *r, float *c, int32_t *code, float *piv)
{
    const uint8_t *p = item;
    const int RG = dk / GROUP_ROWS, NS = GROUP_COLS * RG;
    const size_t W = stream_words(dk, bits);
    int key_of[1024], fw[GROUP_ROWS];
    storage_rows(dk, bits, key_of);
    position_widths(dk, bits, key_of, fw);
    for (int s = 0; s < dk; s++, p += 4) r[key_of[s]] = get_f32(p);
    for (int j = 0; j < dv; j++, p += 4) c[j] = get_f32(p);
    for (int sl = 0; sl < dv / SLAB_COLS; sl++) {
        for (int l = 0; l < NS; l++) {
            const int g = l % RG, cg = l / RG;
            size_t pos = 0;
            for (int rr = 0; rr < GROUP_ROWS; rr++) {
                const int i = key_of[g * GROUP_ROWS + rr], b = bits[i], F = fw[rr];
                for (int kk = 0; kk < GROUP_COLS; kk++) {
                    const int j = sl * SLAB_COLS + cg * GROUP_COLS + kk;
                    uint32_t u = 0;
                    for (int t = 0; t < F; t++, pos++)
                        u |= (uint32_t)get_bit(p, (pos / 32) * NS + l, (int)(pos % 32)) << t;
                    if (b == ORACLE_PIVOT_BITS) {
                        piv[i * dv + j] = (float)oracle_from_fp16((uint16_t)u);
                        code[i * dv + j] = 0;
                    } else {
                        code[i * dv + j] = (int32_t)u - (1 << (F - 1));
                        piv[i * dv + j] = 0;
                    }
                }
            }
        }
        p += 4 * W * NS;
    }
}

/* ---- batched drivers ------------------------------------------------------ */

size_t oracle_pool_bytes(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits)
{
    size_t tot = 0;
    for (int s = 0; s < n; s++) tot += oracle_item_bytes(dk, dv, bits + (size_t)slot_head[s] * dk);
    return tot;
}

typedef struct {
    float *r, *c, *piv, *S, *arow;
    int32_t *code;
} scratch_t;

static scratch_t scratch_new(int dk, int dv)
{
    scratch_t w;
    w.r = (float *)malloc(sizeof(float) * dk);
    w.c = (float *)malloc(sizeof(float) * dv);
    w.piv = (float *)malloc(sizeof(float) * (size_t)dk * dv);
    w.S = (float *)malloc(sizeof(float) * (size_t)dk * dv);
    w.arow = (float *)malloc(sizeof(float) * dk);
    w.code = (int32_t *)malloc(sizeof(int32_t) * (size_t)dk * dv);
    return w;
}

static void scratch_free(scratch_t *w)
{
    free(w->r); free(w->c); free(w->piv); free(w->S); free(w->arow); free(w->code);
}

void oracle_pack_pool(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                      const float *rho, int ls_iters, const float *S, uint8_t *pool)
{
    scratch_t w = scratch_new(dk, dv);
    size_t off = 0;
    for (int s = 0; s < n; s++) {
        const uint8_t *bh = bits + (size_t)slot_head[s] * dk;
        const float *rh = rho + (size_t)slot_head[s] * dk;
        oracle_fit_quantise_f32(dk, dv, S + (size_t)s * dk * dv, bh, rh, ls_iters,
                                ORACLE_PIVOT_FP16, w.r, w.c, w.code, w.piv, NULL, NULL);
        oracle_pack_item(dk, dv, bh, w.r, w.c, w.code, w.piv, pool + off);
        off += oracle_item_bytes(dk, dv, bh);
    }
    scratch_free(&w);
}

void oracle_unpack_pool(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                        const uint8_t *pool, float *S)
{
    scratch_t w = scratch_new(dk, dv);
    size_t off = 0;
    for (int s = 0; s < n; s++) {
        const uint8_t *bh = bits + (size_t)slot_head[s] * dk;
        oracle_unpack_item(dk, dv, bh, pool + off, w.r, w.c, w.code, w.piv);
        oracle_dequant_f32(dk, dv, bh, w.r, w.c, w.code, w.piv, S + (size_t)s * dk * dv);
        off += oracle_item_bytes(dk, dv, bh);
    }
    scratch_free(&w);
}

void oracle_decode_step(int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                        const float *rho, int ls_iters, int kda, uint8_t *pool,
                        const float *q, const float *k, const float *v, const float *alpha,
                        const float *beta, float *out, float *S_new, float *tpre, float *lsgap)
{
    scratch_t w = scratch_new(dk, dv);
    size_t off = 0;
    for (int s = 0; s < n; s++) {
        const uint8_t *bh = bits + (size_t)slot_head[s] * dk;
        const float *rh = rho + (size_t)slot_head[s] * dk;
        /* reconstruct the stored state */
        oracle_unpack_item(dk, dv, bh, pool + off, w.r, w.c, w.code, w.piv);
        oracle_dequant_f32(dk, dv, bh, w.r, w.c, w.code, w.piv, w.S);
        /* gated Delta update + readout */
        for (int i = 0; i < dk; i++) w.arow[i] = kda ? alpha[(size_t)s * dk + i] : alpha[s];
        oracle_update_f32(dk, dv, w.S, w.arow, q + (size_t)s * dk, k + (size_t)s * dk,
                          v + (size_t)s * dv, beta[s], out + (size_t)s * dv);
        if (S_new) memcpy(S_new + (size_t)s * dk * dv, w.S, sizeof(float) * (size_t)dk * dv);
        /* refit, requantise, write back */
        oracle_fit_quantise_f32(dk, dv, w.S, bh, rh, ls_iters, ORACLE_PIVOT_FP16, w.r, w.c,
                                w.code, w.piv, tpre ? tpre + (size_t)s * dk * dv : NULL,
                                lsgap ? lsgap + (size_t)s * dv : NULL);
        oracle_pack_item(dk, dv, bh, w.r, w.c, w.code, w.piv, pool + off);
        off += oracle_item_bytes(dk, dv, bh);
    }
    scratch_free(&w);
}

void oracle_pack_pool_mode(int mode, int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                           const float *rho, int ls_iters, const float *S, uint8_t *pool)
{
    scratch_t w = scratch_new(dk, dv);
    size_t off = 0;
    for (int s = 0; s < n; s++) {
        const uint8_t *bh = bits + (size_t)slot_head[s] * dk;
        const float *rh = rho + (size_t)slot_head[s] * dk;
        oracle_fit_quantise_mode_f32(mode, dk, dv, S + (size_t)s * dk * dv, bh, rh, ls_iters, ORACLE_PIVOT_FP16,
                                     w.r, w.c, w.code, w.piv, NULL);
        oracle_pack_item(dk, dv, bh, w.r, w.c, w.code, w.piv, pool + off);
        off += oracle_item_bytes(dk, dv, bh);
    }
    scratch_free(&w);
}

void oracle_decode_step_mode(int mode, int n, const int32_t *slot_head, int dk, int dv, const uint8_t *bits,
                             const float *rho, int ls_iters, int kda, uint8_t *pool, const float *q,
                             const float *k, const float *v, const float *alpha, const float *beta,
                             float *out, float *S_new, float *tpre)
{
    scratch_t w = scratch_new(dk, dv);
    size_t off = 0;
    for (int s = 0; s < n; s++) {
        const uint8_t *bh = bits + (size_t)slot_head[s] * dk;
        const float *rh = rho + (size_t)slot_head[s] * dk;
        oracle_unpack_item(dk, dv, bh, pool + off, w.r, w.c, w.code, w.piv);
        oracle_dequant_f32(dk, dv, bh, w.r, w.c, w.code, w.piv, w.S);
        for (int i = 0; i < dk; i++) w.arow[i] = kda ? alpha[(size_t)s * dk + i] : alpha[s];
        oracle_update_f32(dk, dv, w.S, w.arow, q + (size_t)s * dk, k + (size_t)s * dk,
                          v + (size_t)s * dv, beta[s], out + (size_t)s * dv);
        if (S_new) memcpy(S_new + (size_t)s * dk * dv, w.S, sizeof(float) * (size_t)dk * dv);
        oracle_fit_quantise_mode_f32(mode, dk, dv, w.S, bh, rh, ls_iters, ORACLE_PIVOT_FP16, w.r, w.c,
                                     w.code, w.piv, tpre ? tpre + (size_t)s * dk * dv : NULL);
        oracle_pack_item(dk, dv, bh, w.r, w.c, w.code, w.piv, pool + off);
        off += oracle_item_bytes(dk, dv, bh);
    }
    scratch_free(&w);
}

void oracle_fp32_step(int n, int dk, int dv, int kda, float *S, const float *q, const float *k,
                      const float *v, const float *alpha, const float *beta, float *out)
{
    float *arow = (float *)malloc(sizeof(float) * dk);
    for (int s = 0; s < n; s++) {
        for (int i = 0; i < dk; i++) arow[i] = kda ? alpha[(size_t)s * dk + i] : alpha[s];
        oracle_update_f32(dk, dv, S + (size_t)s * dk * dv, arow, q + (size_t)s * dk,
                          k + (size_t)s * dk, v + (size_t)s * dv, beta[s], out + (size_t)s * dv);
    }
    free(arow);
}

void oracle_fp64_step(int n, int dk, int dv, int kda, double *S, const double *q,
                      const double *k, const double *v, const double *alpha,
                      const double *beta, double *out)
{
    double *arow = (double *)malloc(sizeof(double) * dk);
    for (int s = 0; s < n; s++) {
        for (int i = 0; i < dk; i++) arow[i] = kda ? alpha[(size_t)s * dk + i] : alpha[s];
        oracle_update_f64(dk, dv, S + (size_t)s * dk * dv, arow, q + (size_t)s * dk,
                          k + (size_t)s * dk, v + (size_t)s * dv, beta[s], out + (size_t)s * dv);
    }
    free(arow);
}
