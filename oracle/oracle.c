/*
 * oracle.c -- plain, slow CPU restatement of block-scaled weight quantization with a
 * searched E4M3 block scale.
 *
 * TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the benchmark's CPU
 * baseline are its only callers. It shares no code, header, table or constant with the
 * CUDA library, and the library never calls it.
 *
 * Sources (page title, section):
 *  - "Is Finer Better? The Limits of Microscaling Formats in LLMs", sec. 2.1
 *    (Microscaling formats): s = Q_scale(xmax / C), q_i = Q_elem(x_i / s), x^ = s * q.
 *    Appendix F.3: the smallest positive E4M3 value 2^-9 (subnormals included); a block
 *    whose scale rounds to zero has every element rounded to zero.
 *  - qwantize "Results", section "INT8 (FP8 E4M3 scales)": symmetric INT8 in [-127, 127],
 *    the per-block amax stored as E4M3, effective scale amax_fp8 / 127 divided in float32;
 *    the bounded search around the naive amax snap.
 *  - qwantize "Results", sections "NVFP4 (FP8 E4M3 scales)" and "Correctness notes":
 *    naive / SSE-optimal / H-optimal; FP4 decisions at the 0.75, 1.75, 3.5 boundaries;
 *    section "Exotic Scales": the E2M1 codebook {0, 0.5, 1, 1.5, 2, 3, 4, 6} and the count
 *    of 126 positive E4M3 values.
 *  - qwantize "Results", section "MXFP4 (UE8M0 power-of-2 scales)": E2M1 elements with a
 *    power-of-two block scale; sections "GPTQ Quantization" (the NVINT4 rows) and "Larger
 *    blocks": INT4 elements, symmetric 0..7, with an E4M3 block scale; section "Exotic
 *    Scales": the unsigned 8-bit scale formats UE4M4 (4 exponent bits, bias 7, 4 mantissa
 *    bits, max 496) and UE5M3 (5 exponent bits, bias 15, 3 mantissa bits, max 122880),
 *    every code finite, 255 positive values each.
 *  - "Is Finer Better? ...", sec. 2.1: the OCP microscaling scale E8M0, 2^-127 .. 2^127.
 *  - "quantization_algorithms.txt", section 1 (Activation-weighted scale search): the
 *    diagonal objective sum_ij h_j (w_ij - s Q(w_ij / s))^2 with h_j = E[x_j^2]; a
 *    logarithmic grid of tile scales; section 2: nearest-E4M3 projection by binary search
 *    in a sorted float32 table of the finite E4M3 values.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - every rounding onto a grid is round-to-nearest, ties to the even code, saturating at
 *    the largest finite value; the division w / s is IEEE float32 (C float division);
 *  - the block error of one candidate is accumulated in double, in element order, as
 *    e += c_j * (d * d) with d = (double)w - (double)fl32(s * q);
 *  - candidate ties go to the lowest candidate index (the smallest scale);
 *  - a naive scale that rounds to E4M3 code 0 gives all-zero magnitudes (sign bits kept);
 *    the search never picks code 0; a window around code 0 is [1, w]. The same holds for
 *    the other scale formats whose code 0 is zero (UE4M4, UE5M3);
 *  - the naive UE8M0 (MXFP4) scale is the OCP rule 2^(floor(log2 amax) - 2), 2 being the
 *    largest E2M1 exponent, clamped to the E8M0 range (code 0 for amax = 0); the naive
 *    scale of every other grid is the grid's nearest value to amax / qmax (qmax = 6 for
 *    E2M1, 7 for INT4, 1 for the INT8 stored amax);
 *  - INT4 codes are two's-complement nibbles in [-7, 7], element 2i in the low nibble.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared oracle.c -lm
 * (no fused multiply-add: every product and sum above is a separately rounded step).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------------------
 * Number formats, decoded from their bit fields.
 * ---------------------------------------------------------------------------------- */

/* E4M3 ("FN": no infinities; S.1111.111 is NaN): 4 exponent bits with bias 7, 3 mantissa
 * bits. Exponent field 0 encodes subnormals m/8 * 2^-6, otherwise (1 + m/8) * 2^(e-7). */
double orc_e4m3_value(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* E2M1: 2 exponent bits with bias 1, 1 mantissa bit. Exponent field 0 encodes m * 0.5. */
double orc_e2m1_value(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + (double)m / 2.0, e - 1);
    return s ? -v : v;
}

/* UE4M4 (unsigned, every code finite): 4 exponent bits with bias 7, 4 mantissa bits.
 * Exponent field 0 encodes m/16 * 2^-6, otherwise (1 + m/16) * 2^(e-7). */
double orc_ue4m4_value(int code)
{
    int e = (code >> 4) & 15, m = code & 15;
    if (e == 0) return ldexp((double)m / 16.0, -6);
    return ldexp(1.0 + (double)m / 16.0, e - 7);
}

/* UE5M3 (unsigned, every code finite): 5 exponent bits with bias 15, 3 mantissa bits.
 * Exponent field 0 encodes m/8 * 2^-14, otherwise (1 + m/8) * 2^(e-15). */
double orc_ue5m3_value(int code)
{
    int e = (code >> 3) & 31, m = code & 7;
    if (e == 0) return ldexp((double)m / 8.0, -14);
    return ldexp(1.0 + (double)m / 8.0, e - 15);
}

/* UE8M0: the power of two 2^(code - 127); code 255 is NaN. */
double orc_ue8m0_value(int code)
{
    if ((code & 255) == 255) return NAN;
    return ldexp(1.0, (code & 255) - 127);
}

/* Sorted tables of the non-negative grid values; the table index is the magnitude code
 * (for every format here the codes of positive values increase with the value). */
static float T_E4M3[127];   /* codes 0x00 .. 0x7E: 0, 2^-9, ..., 448 */
static float T_E2M1[8];     /* codes 0 .. 7: 0, 0.5, ..., 6 */
static float T_INT[128];    /* 0 .. 127 (its first 8 entries are the INT4 magnitudes) */
static float T_UE4M4[256];  /* 0, 2^-10, ..., 496 */
static float T_UE5M3[256];  /* 0, 2^-17, ..., 122880 */
static float T_UE8M0[255];  /* 2^-127, ..., 2^127 */

__attribute__((constructor)) static void orc_init_tables(void)
{
    for (int c = 0; c < 127; ++c) T_E4M3[c] = (float)orc_e4m3_value(c);
    for (int c = 0; c < 8; ++c) T_E2M1[c] = (float)orc_e2m1_value(c);
    for (int c = 0; c < 128; ++c) T_INT[c] = (float)c;
    for (int c = 0; c < 256; ++c) T_UE4M4[c] = (float)orc_ue4m4_value(c);
    for (int c = 0; c < 256; ++c) T_UE5M3[c] = (float)orc_ue5m3_value(c);
    for (int c = 0; c < 255; ++c) T_UE8M0[c] = (float)orc_ue8m0_value(c);
}

/* The block-scale grids: table, number of codes, first candidate code of a search. */
enum { ORC_S_E4M3 = 0, ORC_S_UE4M4 = 1, ORC_S_UE5M3 = 2, ORC_S_UE8M0 = 3 };
typedef struct { const float *tab; int n; int first; } scale_grid;

static int grid_of(int sfmt, scale_grid *g)
{
    switch (sfmt) {
    case ORC_S_E4M3: *g = (scale_grid){T_E4M3, 127, 1}; return 0;
    case ORC_S_UE4M4: *g = (scale_grid){T_UE4M4, 256, 1}; return 0;
    case ORC_S_UE5M3: *g = (scale_grid){T_UE5M3, 256, 1}; return 0;
    case ORC_S_UE8M0: *g = (scale_grid){T_UE8M0, 255, 0}; return 0;
    default: return -1;
    }
}

/* Copy of a scale grid's table (out holds 256 floats); returns the number of codes. */
int orc_scale_table(int sfmt, float *out)
{
    scale_grid g;
    if (grid_of(sfmt, &g)) return -1;
    memcpy(out, g.tab, sizeof(float) * (size_t)g.n);
    return g.n;
}

/* Copies of the tables, for the self-tests. */
void orc_e4m3_table(float *out127) { memcpy(out127, T_E4M3, sizeof T_E4M3); }
void orc_e2m1_table(float *out8) { memcpy(out8, T_E2M1, sizeof T_E2M1); }

/* Index of the table value nearest to z >= 0 (tab ascending, tab[0] == 0). Equidistant
 * values go to the even index; z at or above the last value (and +inf) saturates to the
 * last index; zero and NaN give 0. */
static int nearest_rne(const float *tab, int n, float z)
{
    if (!(z > 0.0f)) return 0;
    if (z >= tab[n - 1]) return n - 1;
    int lo = 0, hi = n - 1;            /* tab[lo] <= z < tab[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (tab[mid] <= z) lo = mid; else hi = mid;
    }
    double dlo = (double)z - (double)tab[lo];
    double dhi = (double)tab[hi] - (double)z;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo % 2 == 0) ? lo : hi;
}

/* Round-to-nearest-even onto the non-negative E4M3 grid with saturation: the code. */
int orc_e4m3_rne_code(float x) { return nearest_rne(T_E4M3, 127, x); }
/* Round-to-nearest-even onto the E2M1 magnitudes with saturation at 6: the code 0..7. */
int orc_e2m1_rne_code(float x) { return nearest_rne(T_E2M1, 8, x); }
/* Round-to-nearest-even onto 0..127. */
int orc_int127_rne(float x) { return nearest_rne(T_INT, 128, x); }

/* ----------------------------------------------------------------------------------
 * Element access.
 * ---------------------------------------------------------------------------------- */

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_NVFP4 = 0, ORC_INT8 = 1, ORC_E4M3 = 2, ORC_INT4 = 3 };
enum { ORC_NAIVE = 0, ORC_SSE = 1, ORC_HOPT = 2 };

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static float elem(const void *base, int dtype, int64_t ld, int64_t i, int64_t j)
{
    if (dtype == ORC_BF16) return bf16_to_float(((const uint16_t *)base)[i * ld + j]);
    return ((const float *)base)[i * ld + j];
}

/* ----------------------------------------------------------------------------------
 * h_j = E[x_j^2] over the rows of X ("quantization_algorithms.txt", section 1).
 * The sum of squares is taken in double, then divided by R and rounded to float once.
 * ---------------------------------------------------------------------------------- */
void orc_act_sqsum(const void *X, int dtype, int64_t rows, int64_t cols, int64_t ld,
                   int64_t row0, int64_t row1, double *colsum)
{
    for (int64_t j = 0; j < cols; ++j) colsum[j] = 0.0;
    for (int64_t r = row0; r < row1 && r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j) {
            double x = (double)elem(X, dtype, ld, r, j);
            colsum[j] += x * x;
        }
}

void orc_act_sqmean(const void *X, int dtype, int64_t rows, int64_t cols, int64_t ld,
                    float *h)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(cols > 0 ? cols : 1));
    orc_act_sqsum(X, dtype, rows, cols, ld, 0, rows, s);
    for (int64_t j = 0; j < cols; ++j) h[j] = rows > 0 ? (float)(s[j] / (double)rows) : 0.0f;
    free(s);
}

/* ----------------------------------------------------------------------------------
 * One-dimensional blocks (NVFP4 and INT8): B contiguous weights of one row share one
 * E4M3 scale byte.
 * ---------------------------------------------------------------------------------- */

/* The magnitude code of element w at candidate scale code c of grid sfmt, and its
 * dequantised value fl32(scale * q) (without sign). NVFP4 (E2M1 elements): scale = the
 * grid value, q = E2M1 nearest of fl32(|w| / scale). INT4: q = nearest integer in [0, 7]
 * of fl32(|w| / scale). INT8 (E4M3 grid only): scale = fl32(E4M3(c) / 127), q = nearest
 * integer in [0, 127] of fl32(|w| / scale). A zero scale (a naive snap to zero) gives
 * q = 0. */
static int project(int fmt, int sfmt, int c, float w, float *wq_abs)
{
    float a = fabsf(w);
    scale_grid g;
    if (grid_of(sfmt, &g)) { *wq_abs = NAN; return 0; }
    if (g.tab[c] == 0.0f) { *wq_abs = 0.0f; return 0; }
    if (fmt == ORC_NVFP4) {
        float s = g.tab[c];
        float z = a / s;
        int q = nearest_rne(T_E2M1, 8, z);
        *wq_abs = s * T_E2M1[q];
        return q;
    } else if (fmt == ORC_INT4) {
        float s = g.tab[c];
        float z = a / s;
        int q = nearest_rne(T_INT, 8, z);
        *wq_abs = (float)q * s;
        return q;
    } else {
        float s = T_E4M3[c] / 127.0f;
        float z = a / s;
        int q = nearest_rne(T_INT, 128, z);
        *wq_abs = (float)q * s;
        return q;
    }
}

/* Exported for the exhaustive projection self-tests. */
int orc_project(int fmt, int sfmt, int c, float w, float *wq_abs)
{
    return project(fmt, sfmt, c, w, wq_abs);
}

void orc_project_many(int fmt, int sfmt, int c, const float *w, int64_t count, uint8_t *q,
                      float *wq_abs)
{
    for (int64_t i = 0; i < count; ++i) q[i] = (uint8_t)project(fmt, sfmt, c, w[i], &wq_abs[i]);
}

/* Block error at candidate c: sum_j c_j (w_j - wq_j)^2 in double, element order. */
static double block_error(int fmt, int sfmt, int c, const float *w, const float *cw, int B)
{
    double e = 0.0;
    for (int j = 0; j < B; ++j) {
        float wq_abs;
        project(fmt, sfmt, c, w[j], &wq_abs);
        float wq = copysignf(wq_abs, w[j]);
        double d = (double)w[j] - (double)wq;
        e += (double)cw[j] * (d * d);
    }
    return e;
}

/* Naive snap. NVFP4 on E4M3: E4M3(fl32(amax / 6)); INT8: E4M3(amax) (the stored amax);
 * UE8M0: 2^(floor(log2 amax) - 2) (OCP), clamped to codes 0 .. 254; every other grid:
 * its nearest value to fl32(amax / qmax), qmax = 6 (E2M1) or 7 (INT4). */
static int naive_code(int fmt, int sfmt, float amax)
{
    scale_grid g;
    if (fmt == ORC_INT8) return nearest_rne(T_E4M3, 127, amax);
    if (fmt == ORC_NVFP4 && sfmt == ORC_S_E4M3) return nearest_rne(T_E4M3, 127, amax / 6.0f);
    if (sfmt == ORC_S_UE8M0) {
        if (!(amax > 0.0f)) return 0;
        int ex;
        frexp((double)amax, &ex);           /* amax = f 2^ex, 0.5 <= f < 1 */
        int c = (ex - 1) - 2 + 127;
        return c < 0 ? 0 : (c > 254 ? 254 : c);
    }
    if (grid_of(sfmt, &g)) return -1;
    float qmax = (fmt == ORC_NVFP4) ? 6.0f : 7.0f;
    return nearest_rne(g.tab, g.n, amax / qmax);
}

int orc_naive_code(int fmt, int sfmt, float amax) { return naive_code(fmt, sfmt, amax); }

/* Candidate codes of one block: every candidate of the grid, or the window of codes
 * [c0 - window, c0 + window] clipped to them ([1, max(window, 1)] for a zero naive scale). */
static void candidate_range(const scale_grid *g, int c0, int window, int *lo, int *hi)
{
    const int cmax = g->n - 1;
    *lo = g->first;
    *hi = cmax;
    if (window >= 0) {
        *lo = c0 - window < g->first ? g->first : c0 - window;
        *hi = c0 + window > cmax ? cmax : c0 + window;
        if (g->tab[c0] == 0.0f) { *lo = 1; *hi = window < 1 ? 1 : window; }
    }
}

/* Running smallest and second-smallest candidate error; equal errors keep the earlier
 * (lower) code. */
static void keep_best(double e, int c, double *e1, double *e2, int *cbest)
{
    if (e < *e1) { *e2 = *e1; *e1 = e; *cbest = c; }
    else if (e < *e2) *e2 = e;
}

/* Codes of row i's block starting at column j0 at scale code c (layouts as below). */
static void emit_block(int fmt, int sfmt, int c, const float *w, int B, uint8_t *codes,
                       int64_t i, int64_t j0, int64_t k)
{
    for (int j = 0; j < B; ++j) {
        float wq_abs;
        int q = project(fmt, sfmt, c, w[j], &wq_abs);
        int neg = signbit(w[j]) ? 1 : 0;
        if (fmt == ORC_NVFP4 || fmt == ORC_INT4) {
            uint8_t nib = (fmt == ORC_NVFP4) ? (uint8_t)((neg << 3) | q)
                                             : (uint8_t)((neg ? -q : q) & 15);
            uint8_t *p = &codes[i * (k / 2) + (j0 + j) / 2];
            if (((j0 + j) & 1) == 0) *p = (uint8_t)((*p & 0xF0) | nib);
            else *p = (uint8_t)((*p & 0x0F) | (nib << 4));
        } else {
            int v = neg ? -q : q;
            ((int8_t *)codes)[i * k + j0 + j] = (int8_t)v;
        }
    }
}

/* The quantizer's pick for one block of B weights w with error weights cw: the naive
 * code in naive mode, else the candidate of smallest error, the lowest code on equal
 * errors. e1 / e2: the smallest and second-smallest candidate errors (NaN in naive mode);
 * naive: the naive code. */
static int search_block(int fmt, int sfmt, int mode, int window, const scale_grid *g,
                        const float *w, const float *cw, int B, double *e1, double *e2,
                        int *naive)
{
    float amax = 0.0f;
    for (int j = 0; j < B; ++j)
        if (fabsf(w[j]) > amax) amax = fabsf(w[j]);
    int c0 = naive_code(fmt, sfmt, amax);
    int cbest = c0;
    *e1 = NAN;
    *e2 = NAN;
    if (mode != ORC_NAIVE) {
        int lo, hi;
        candidate_range(g, c0, window, &lo, &hi);
        *e1 = INFINITY; *e2 = INFINITY; cbest = lo;
        for (int c = lo; c <= hi; ++c)
            keep_best(block_error(fmt, sfmt, c, w, cw, B), c, e1, e2, &cbest);
    }
    *naive = c0;
    return cbest;
}

/*
 * Quantize rows [row0, row1) of W [n, k] (leading dimension ld) in blocks of B along k.
 * fmt: ORC_NVFP4 (E2M1 elements), ORC_INT4 or ORC_INT8; sfmt: the scale grid
 * (ORC_S_E4M3 for all three; UE4M4, UE5M3 or UE8M0 for E2M1 elements; UE4M4 or UE5M3 for
 * INT4). mode: ORC_NAIVE, ORC_SSE or ORC_HOPT (h required).
 * window < 0: every candidate code of the grid (E4M3 1..126, UE4M4 / UE5M3 1..255, UE8M0
 * 0..254); otherwise codes [c0-window, c0+window] clipped to that range, c0 the naive code.
 * Outputs (row-major, all n rows addressable): codes -- NVFP4 [n][k/2] with element 2i in
 * the low nibble, nibble = sign << 3 | E2M1 code; INT4 [n][k/2], same nibble order, the
 * nibble the two's complement of the signed code; INT8 [n][k] two's complement.
 * scales [n][k/B] scale codes. Optional (may be NULL): best / second [n][k/B] -- the
 * smallest and the second-smallest candidate error (second = +inf with one candidate;
 * both NaN in naive mode), naive [n][k/B] the naive code.
 * Returns 0, or -1 on bad arguments.
 */
int orc_quantize_blocks(const void *W, int dtype, int64_t n, int64_t k, int64_t ld,
                        const float *h, int fmt, int sfmt, int mode, int B, int window,
                        int64_t row0, int64_t row1, uint8_t *codes, uint8_t *scales,
                        double *best, double *second, int32_t *naive)
{
    scale_grid g;
    if (B <= 0 || k % B != 0 || grid_of(sfmt, &g)) return -1;
    if (fmt != ORC_NVFP4 && fmt != ORC_INT8 && fmt != ORC_INT4) return -1;
    if (fmt == ORC_INT8 && sfmt != ORC_S_E4M3) return -1;
    if (fmt == ORC_INT4 && sfmt == ORC_S_UE8M0) return -1;
    if (mode == ORC_HOPT && h == NULL) return -1;
    int64_t kb = k / B;
    float *w = (float *)malloc(sizeof(float) * (size_t)B);
    float *cw = (float *)malloc(sizeof(float) * (size_t)B);
    for (int64_t i = row0; i < row1 && i < n; ++i) {
        for (int64_t b = 0; b < kb; ++b) {
            int64_t j0 = b * B;
            for (int j = 0; j < B; ++j) {
                w[j] = elem(W, dtype, ld, i, j0 + j);
                cw[j] = (mode == ORC_HOPT) ? h[j0 + j] : 1.0f;
            }
            double e1, e2;
            int c0;
            int cbest = search_block(fmt, sfmt, mode, window, &g, w, cw, B, &e1, &e2, &c0);
            scales[i * kb + b] = (uint8_t)cbest;
            if (best) best[i * kb + b] = e1;
            if (second) second[i * kb + b] = e2;
            if (naive) naive[i * kb + b] = c0;
            emit_block(fmt, sfmt, cbest, w, B, codes, i, j0, k);
        }
    }
    free(w);
    free(cw);
    return 0;
}

/* ----------------------------------------------------------------------------------
 * GPTQ with the block quantizer as its inner step (qwantize "Results", "GPTQ
 * Quantization": the GPTQ block is the quantization block; after a block is quantised its
 * error is compensated in all remaining columns by one product of the block's residuals
 * with the block's rows of the inverse-Hessian factor). The algorithm is Frantar et al.
 * 2022, Algorithm 1, in its Cholesky form. When the sweep reaches a block, its scale is the
 * quantizer's pick (naive / SSE / H-optimal, as orc_quantize_blocks) for the block's
 * CURRENT weights -- GPTQ fixes a group's quantization grid at the moment the group is
 * reached -- and the block's columns are then quantised one after another at that scale.
 * Rows are independent; for row i, with the block visited at sweep position t being
 * perm[t] (t itself when perm is NULL) and p = t B + j the sweep position of column
 * col = b B + j:
 *   for j = 0 .. B-1:
 *     q = project(w at p, the block's scale), wq = +-fl32(s q) (the sign of w),
 *     err_j = (w - wq) / U[p][p],
 *     w at position p' -= err_j * U[p][p'] for the block's later positions p'
 *       (product, then difference: the in-block update of the algorithm);
 *   then for every position p' after the block (the block's product "err @ U[block, rest]"):
 *     acc = 0; for j = 0 .. B-1: acc = fma(err_j, U[t B + j][p'], acc);  w at p' -= acc.
 * Every step is one IEEE float32 operation (fma rounded once). U [k][k] (float32, upper
 * triangular) is the upper Cholesky factor of the damped H^-1 with H's rows and columns in
 * sweep order. codes / scales: the layouts of orc_quantize_blocks; rows [row0, row1).
 * ---------------------------------------------------------------------------------- */
int orc_gptq_blocks(const void *W, int dtype, int64_t n, int64_t k, int64_t ld,
                    const float *h, int fmt, int sfmt, int mode, int B, int window,
                    const float *U, const int32_t *perm, int64_t row0, int64_t row1,
                    uint8_t *codes, uint8_t *scales)
{
    scale_grid g;
    if (B <= 0 || B > 256 || k % B != 0 || U == NULL || grid_of(sfmt, &g)) return -1;
    if (fmt != ORC_NVFP4 && fmt != ORC_INT8 && fmt != ORC_INT4) return -1;
    if (fmt == ORC_INT8 && sfmt != ORC_S_E4M3) return -1;
    if (fmt == ORC_INT4 && sfmt == ORC_S_UE8M0) return -1;
    if (mode == ORC_HOPT && h == NULL) return -1;
    int64_t kb = k / B;
    int64_t *col = (int64_t *)malloc(sizeof(int64_t) * (size_t)k);   /* position -> column */
    for (int64_t t = 0; t < kb; ++t) {
        int64_t b = perm ? perm[t] : t;
        if (b < 0 || b >= kb) { free(col); return -1; }
        for (int j = 0; j < B; ++j) col[t * B + j] = b * B + j;
    }
    float *w = (float *)malloc(sizeof(float) * (size_t)k);
    float *cw = (float *)malloc(sizeof(float) * (size_t)B);
    float *err = (float *)malloc(sizeof(float) * (size_t)B);
    for (int64_t i = row0; i < row1 && i < n; ++i) {
        for (int64_t j = 0; j < k; ++j) w[j] = elem(W, dtype, ld, i, j);
        for (int64_t t = 0; t < kb; ++t) {
            int64_t j0 = col[t * B];                 /* the block's first column */
            for (int j = 0; j < B; ++j) cw[j] = (mode == ORC_HOPT) ? h[j0 + j] : 1.0f;
            double e1, e2;
            int c0;
            int c = search_block(fmt, sfmt, mode, window, &g, &w[j0], cw, B, &e1, &e2, &c0);
            scales[i * kb + j0 / B] = (uint8_t)c;
            for (int j = 0; j < B; ++j) {            /* the block's columns, in order */
                int64_t p = t * B + j;
                float wv = w[j0 + j];
                float wq_abs;
                project(fmt, sfmt, c, wv, &wq_abs);
                emit_block(fmt, sfmt, c, &w[j0 + j], 1, codes, i, j0 + j, k);
                float wq = copysignf(wq_abs, wv);
                err[j] = (wv - wq) / U[p * k + p];
                for (int j2 = j + 1; j2 < B; ++j2) {
                    float prod = err[j] * U[p * k + t * B + j2];
                    w[j0 + j2] = w[j0 + j2] - prod;
                }
            }
            for (int64_t p2 = (t + 1) * B; p2 < k; ++p2) {   /* the rest: one product */
                float acc = 0.0f;
                for (int j = 0; j < B; ++j) acc = fmaf(err[j], U[(t * B + j) * k + p2], acc);
                w[col[p2]] = w[col[p2]] - acc;
            }
        }
    }
    free(w);
    free(cw);
    free(err);
    free(col);
    return 0;
}

/* ----------------------------------------------------------------------------------
 * Block-Hessian objective ("quantization_algorithms.txt", section 1: the scale minimising
 * || X_b (W_b - s Q(W_b / s))^T ||_F^2 over the block's calibration inputs X_b; the
 * diagonal h_j = E[x_j^2] is its cheap approximation). For one row's block of B weights
 * the objective is R * d^T G d with G = X_b^T X_b / R, the block's B x B Gram matrix.
 * G is kept in float32 as fl32(sum_r x_ri x_rj / R) (the sum in double, rows ascending,
 * then divided and rounded once, exactly as h), so diag(G) is h bit for bit.
 * ---------------------------------------------------------------------------------- */

/* G[b][i][j] for every column block b = 0 .. cols/B - 1 (row-major [cols/B][B][B]). */
int orc_block_gram(const void *X, int dtype, int64_t rows, int64_t cols, int64_t ld, int B,
                   float *G)
{
    if (B <= 0 || cols % B != 0) return -1;
    double *acc = (double *)malloc(sizeof(double) * (size_t)B * (size_t)B);
    for (int64_t b = 0; b < cols / B; ++b) {
        for (int t = 0; t < B * B; ++t) acc[t] = 0.0;
        for (int64_t r = 0; r < rows; ++r)
            for (int i = 0; i < B; ++i) {
                double xi = (double)elem(X, dtype, ld, r, b * B + i);
                for (int j = 0; j < B; ++j)
                    acc[i * B + j] += xi * (double)elem(X, dtype, ld, r, b * B + j);
            }
        for (int t = 0; t < B * B; ++t)
            G[b * B * B + t] = rows > 0 ? (float)(acc[t] / (double)rows) : 0.0f;
    }
    free(acc);
    return 0;
}

/* d^T G d of one block at candidate c, in double, in the order
 * e += G_ij * (d_i * d_j) for i ascending, j ascending (d_i = w_i - fl32(s q_i)). */
static double block_error_gram(int fmt, int sfmt, int c, const float *w, const float *Gb, int B)
{
    double *d = (double *)malloc(sizeof(double) * (size_t)B);
    for (int j = 0; j < B; ++j) {
        float wq_abs;
        project(fmt, sfmt, c, w[j], &wq_abs);
        d[j] = (double)w[j] - (double)copysignf(wq_abs, w[j]);
    }
    double e = 0.0;
    for (int i = 0; i < B; ++i)
        for (int j = 0; j < B; ++j)
            e += (double)Gb[i * B + j] * (d[i] * d[j]);
    free(d);
    return e;
}

/*
 * Block-Hessian H-optimal search: as orc_quantize_blocks in SSE / H mode, with the
 * candidate error d^T G_b d (G from orc_block_gram, [k/B][B][B] float). Same outputs,
 * candidates, window and tie rule.
 */
int orc_quantize_blocks_gram(const void *W, int dtype, int64_t n, int64_t k, int64_t ld,
                             const float *G, int fmt, int sfmt, int B, int window,
                             int64_t row0, int64_t row1, uint8_t *codes, uint8_t *scales,
                             double *best, double *second, int32_t *naive)
{
    scale_grid g;
    if (B <= 0 || k % B != 0 || grid_of(sfmt, &g) || G == NULL) return -1;
    if (fmt != ORC_NVFP4 && fmt != ORC_INT8 && fmt != ORC_INT4) return -1;
    if (fmt == ORC_INT8 && sfmt != ORC_S_E4M3) return -1;
    if (fmt == ORC_INT4 && sfmt == ORC_S_UE8M0) return -1;
    int64_t kb = k / B;
    float *w = (float *)malloc(sizeof(float) * (size_t)B);
    for (int64_t i = row0; i < row1 && i < n; ++i) {
        for (int64_t b = 0; b < kb; ++b) {
            int64_t j0 = b * B;
            const float *Gb = G + b * B * B;
            float amax = 0.0f;
            for (int j = 0; j < B; ++j) {
                w[j] = elem(W, dtype, ld, i, j0 + j);
                if (fabsf(w[j]) > amax) amax = fabsf(w[j]);
            }
            int c0 = naive_code(fmt, sfmt, amax);
            int lo, hi, cbest;
            candidate_range(&g, c0, window, &lo, &hi);
            double e1 = INFINITY, e2 = INFINITY;
            cbest = lo;
            for (int c = lo; c <= hi; ++c)
                keep_best(block_error_gram(fmt, sfmt, c, w, Gb, B), c, &e1, &e2, &cbest);
            scales[i * kb + b] = (uint8_t)cbest;
            if (best) best[i * kb + b] = e1;
            if (second) second[i * kb + b] = e2;
            if (naive) naive[i * kb + b] = c0;
            emit_block(fmt, sfmt, cbest, w, B, codes, i, j0, k);
        }
    }
    free(w);
    return 0;
}

/* ----------------------------------------------------------------------------------
 * E4M3 elements on T x T tiles with one float32 scale per tile, searched on a
 * logarithmic grid ("quantization_algorithms.txt", section 1).
 * base = fl32(amax_tile / 448); grid g_p = fl32(2^(lo + (hi - lo) p / (P - 1))),
 * p = 0..P-1 (computed in double, rounded once); candidate s_p = fl32(base * g_p).
 * Naive mode: s = base. A tile whose scale is 0 gets zero magnitudes (sign bits kept);
 * a candidate scale that underflows to 0 is skipped.
 * ---------------------------------------------------------------------------------- */

static int e4m3_elem_code(float a, float s, float *wq_abs)
{
    if (s == 0.0f) { *wq_abs = 0.0f; return 0; }
    float z = a / s;
    int q = nearest_rne(T_E4M3, 127, z);
    *wq_abs = s * T_E4M3[q];
    return q;
}

int orc_project_e4m3(float w, float s, float *wq_abs) { return e4m3_elem_code(fabsf(w), s, wq_abs); }

void orc_project_e4m3_many(float s, const float *w, int64_t count, uint8_t *q, float *wq_abs)
{
    for (int64_t i = 0; i < count; ++i) q[i] = (uint8_t)e4m3_elem_code(fabsf(w[i]), s, &wq_abs[i]);
}

void orc_log_grid(int P, double lo, double hi, float *g)
{
    for (int p = 0; p < P; ++p)
        g[p] = (float)exp2(lo + (hi - lo) * (double)p / (double)(P - 1));
}

/*
 * Tiles of T rows x T columns; tile rows [trow0, trow1). codes [n][k] bytes
 * (sign << 7 | E4M3 code), scales [n/T][k/T] float. best / second / grid_index optional:
 * [n/T][k/T] (grid_index -1 in naive mode).
 */
int orc_quantize_tiles(const void *W, int dtype, int64_t n, int64_t k, int64_t ld,
                       const float *h, int mode, int T, int P, double lo, double hi,
                       int64_t trow0, int64_t trow1, uint8_t *codes, float *scales,
                       double *best, double *second, int32_t *grid_index)
{
    if (T <= 0 || n % T != 0 || k % T != 0 || P < 2 || P > 4096) return -1;
    if (mode == ORC_HOPT && h == NULL) return -1;
    int64_t tn = n / T, tk = k / T;
    float *g = (float *)malloc(sizeof(float) * (size_t)P);
    orc_log_grid(P, lo, hi, g);
    for (int64_t ti = trow0; ti < trow1 && ti < tn; ++ti) {
        for (int64_t tj = 0; tj < tk; ++tj) {
            int64_t i0 = ti * T, j0 = tj * T;
            float amax = 0.0f;
            for (int64_t i = 0; i < T; ++i)
                for (int64_t j = 0; j < T; ++j) {
                    float a = fabsf(elem(W, dtype, ld, i0 + i, j0 + j));
                    if (a > amax) amax = a;
                }
            float base = amax / 448.0f;
            float s = base;
            int pbest = -1;
            double e1 = NAN, e2 = NAN;
            if (mode != ORC_NAIVE && base > 0.0f) {
                e1 = INFINITY; e2 = INFINITY;
                for (int p = 0; p < P; ++p) {
                    float sp = base * g[p];
                    if (sp == 0.0f) continue;
                    double e = 0.0;
                    for (int64_t i = 0; i < T; ++i)
                        for (int64_t j = 0; j < T; ++j) {
                            float w = elem(W, dtype, ld, i0 + i, j0 + j);
                            float wq_abs;
                            e4m3_elem_code(fabsf(w), sp, &wq_abs);
                            float wq = copysignf(wq_abs, w);
                            double d = (double)w - (double)wq;
                            double c = (mode == ORC_HOPT) ? (double)h[j0 + j] : 1.0;
                            e += c * (d * d);
                        }
                    if (e < e1) { e2 = e1; e1 = e; pbest = p; }
                    else if (e < e2) e2 = e;
                }
                s = pbest >= 0 ? base * g[pbest] : 0.0f;
            }
            scales[ti * tk + tj] = s;
            if (best) best[ti * tk + tj] = e1;
            if (second) second[ti * tk + tj] = e2;
            if (grid_index) grid_index[ti * tk + tj] = pbest;
            for (int64_t i = 0; i < T; ++i)
                for (int64_t j = 0; j < T; ++j) {
                    float w = elem(W, dtype, ld, i0 + i, j0 + j);
                    float wq_abs;
                    int q = e4m3_elem_code(fabsf(w), s, &wq_abs);
                    codes[(i0 + i) * k + j0 + j] = (uint8_t)((signbit(w) ? 0x80 : 0) | q);
                }
        }
    }
    free(g);
    return 0;
}

/* ----------------------------------------------------------------------------------
 * FP8-GPTQ on 64 x 64 tiles ("quantization_algorithms.txt", section 1, "For a 64x64 tile
 * scheme": fix or search the tile scale, H = X^T X + lambda I over the tile's 64 input
 * dimensions, quantise the columns sequentially to E4M3, propagate each quantisation
 * residual through H^-1). The propagation is GPTQ's (Frantar et al. 2022) in its Cholesky
 * form: with U the upper Cholesky factor of H^-1 (H^-1 = U^T U), after column i
 *     err_r = (w_ri - q_ri) / U_ii,   w_rj -= err_r * U_ij   for j > i,
 * every step a separately rounded float32 operation (division, product, difference).
 * U [k/64][64][64] (float32, upper triangular; computed by the Python front end from the
 * Gram blocks) and the tile scales [n/64][k/64] are inputs. codes as orc_quantize_tiles;
 * W_prop (optional) receives the propagated weights at the moment each column was
 * quantised.
 * ---------------------------------------------------------------------------------- */
int orc_gptq_tiles(const void *W, int dtype, int64_t n, int64_t k, int64_t ld, const float *U,
                   const float *scales, uint8_t *codes, float *W_prop)
{
    const int T = 64;
    if (n % T != 0 || k % T != 0 || U == NULL || scales == NULL) return -1;
    int64_t tn = n / T, tk = k / T;
    float *w = (float *)malloc(sizeof(float) * T * T);
    for (int64_t ti = 0; ti < tn; ++ti)
        for (int64_t tj = 0; tj < tk; ++tj) {
            const float *Ub = U + tj * T * T;
            float s = scales[ti * tk + tj];
            for (int i = 0; i < T; ++i)
                for (int j = 0; j < T; ++j)
                    w[i * T + j] = elem(W, dtype, ld, ti * T + i, tj * T + j);
            for (int c = 0; c < T; ++c) {            /* column c, every row r of the tile */
                for (int r = 0; r < T; ++r) {
                    float wv = w[r * T + c];
                    float wq_abs;
                    int q = e4m3_elem_code(fabsf(wv), s, &wq_abs);
                    float wq = copysignf(wq_abs, wv);
                    codes[(ti * T + r) * k + tj * T + c] = (uint8_t)((signbit(wv) ? 0x80 : 0) | q);
                    if (W_prop) W_prop[(ti * T + r) * k + tj * T + c] = wv;
                    float err = (wv - wq) / Ub[c * T + c];
                    for (int j = c + 1; j < T; ++j) {
                        float prod = err * Ub[c * T + j];
                        w[r * T + j] = w[r * T + j] - prod;
                    }
                }
            }
        }
    free(w);
    return 0;
}

/* ----------------------------------------------------------------------------------
 * Dequantisation and error metrics (qwantize "Results": weight error
 * ||Q(W) - W||_F / ||W||_F; the h-weighted error is the diagonal objective itself).
 * ---------------------------------------------------------------------------------- */

/* W^ [n][k] float from codes and scales. fmt / sfmt as above; B the block (tile edge for
 * E4M3 elements, whose scales are floats). */
int orc_dequant(const uint8_t *codes, const void *scales, int fmt, int sfmt, int B, int64_t n,
                int64_t k, float *out)
{
    scale_grid g;
    if (B <= 0 || k % B != 0 || grid_of(sfmt, &g)) return -1;
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < k; ++j) {
            float v;
            if (fmt == ORC_NVFP4 || fmt == ORC_INT4) {
                uint8_t byte = codes[i * (k / 2) + j / 2];
                int nib = (j & 1) ? (byte >> 4) : (byte & 15);
                int sc = ((const uint8_t *)scales)[i * (k / B) + j / B];
                float s = sc < g.n ? g.tab[sc] : NAN;
                if (fmt == ORC_NVFP4) {
                    v = s * T_E2M1[nib & 7];
                    if (nib & 8) v = -v;
                } else {
                    int q = (nib & 8) ? 16 - nib : nib;       /* magnitude of the signed nibble */
                    v = (float)q * s;
                    if (nib & 8) v = -v;
                }
            } else if (fmt == ORC_INT8) {
                int q = ((const int8_t *)codes)[i * k + j];
                float s = T_E4M3[((const uint8_t *)scales)[i * (k / B) + j / B]] / 127.0f;
                v = (float)(q < 0 ? -q : q) * s;
                if (q < 0) v = -v;
            } else {
                uint8_t c = codes[i * k + j];
                float s = ((const float *)scales)[(i / B) * (k / B) + j / B];
                v = s * T_E4M3[c & 0x7F];
                if (c & 0x80) v = -v;
            }
            out[i * k + j] = v;
        }
    return 0;
}

/* Block-scale bytes [n][kb] rearranged into the tile layout that sm_100 block-scaled tensor
 * core instructions read (not on the pages; an interface requirement of the hardware):
 * 128-row x 4-column tiles of 512 bytes, tiles ordered by row tile then column tile; inside
 * a tile, row m and column c sit at byte (m % 32) * 16 + (m / 32) * 4 + c. Rows are padded to
 * a multiple of 128 and columns to a multiple of 4 with zero bytes. out: ceil(n/128) * 128 *
 * ceil(kb/4) * 4 bytes. */
void orc_swizzle_scales(const uint8_t *in, int64_t n, int64_t kb, uint8_t *out)
{
    int64_t rt = (n + 127) / 128, ct = (kb + 3) / 4;
    memset(out, 0, (size_t)(rt * 128 * ct * 4));
    for (int64_t m = 0; m < n; ++m)
        for (int64_t c = 0; c < kb; ++c) {
            int64_t tile = (m / 128) * ct + c / 4;
            int64_t mm = m % 128, cc = c % 4;
            out[tile * 512 + (mm % 32) * 16 + (mm / 32) * 4 + cc] = in[m * kb + c];
        }
}

/* sums[0] = sum (w - w^)^2, sums[1] = sum w^2, sums[2] = sum h_j (w - w^)^2,
 * sums[3] = sum h_j w^2 (both 0 when h is NULL); doubles, row-major order. */
void orc_error_sums(const void *W, int dtype, int64_t n, int64_t k, int64_t ld,
                    const float *What, const float *h, double *sums)
{
    double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < k; ++j) {
            double w = (double)elem(W, dtype, ld, i, j);
            double d = w - (double)What[i * k + j];
            s0 += d * d;
            s1 += w * w;
            if (h) {
                s2 += (double)h[j] * (d * d);
                s3 += (double)h[j] * (w * w);
            }
        }
    sums[0] = s0; sums[1] = s1; sums[2] = s2; sums[3] = s3;
}
