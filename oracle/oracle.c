/*
 * oracle.c -- plain, slow, fp64 CPU oracle of the dense-and-sparse quantized
 * matrix-vector product
 *
 *     y[b][i] = sum_j x[b][j] * What[i][j],   What = W_dense + W_sparse
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  It shares no code,
 * header, table or helper with the CUDA library; it is compiled on its own
 * with gcc and knows nothing of the packed device layout.
 *
 * Sources it restates:
 *  - SqueezeLLM page, "Dense-and-Sparse decomposition": W = W_dense + W_sparse,
 *    the sparse part being the outliers kept in fp16.
 *  - SpQR page, "Diagramme de la matrice sparse vs dense": the dense part has
 *    holes at the outlier positions; the sparse part is CSR with fp16 values.
 *  - SpQR page, "Le format de stockage sparse": values / col_idx / row_ptr
 *    (row i owns entries row_ptr[i] .. row_ptr[i+1]-1).
 *  - SpQR page, "Quantification d'un modele" (wbits 3, groupsize 16): the
 *    dense part is uniform codes over groups of 16 inputs.  The decode
 *    formula is not printed; it is read as w = scale * (q - zero), with the
 *    fp16 scale and the integral fp16 zero of the weight's group.
 *  - SqueezeLLM page, "Sensitivity-based non-uniform quantization": the dense
 *    part is codes into a non-uniform table of bins; read as one fp16 table
 *    of 2^bits centroids per output row, w = table[row][q].
 *  - BPDQ page, "1. Formulation de la Grille Variable": the dense part is
 *    What = REP(C_0) + sum_{i=1..k} REP(C_i) (.) B_i, with k bit planes
 *    B_i in {0,1} and scalar coefficients C_0..C_k per group along the input
 *    dimension.  Read as: groups of 32 * 2^k inputs, fp16 coefficients, a
 *    weight's k plane bits held in one code q with b_i = bit (i-1) of q, and
 *    the sum C_0 + sum_i C_i b_i evaluated exactly and rounded once to fp16.
 *  - Huffman-encoded PTQ (gist.science 2507.18553, the HPTQ bullet): inliers
 *    and outliers on one unconstrained integer grid, the integers Huffman
 *    coded.  Read as: an fp16 scale per group of 16 inputs and a signed
 *    integer q per weight (|q| <= 8191), w = scale * q rounded once to fp16;
 *    the Huffman code is storage, so the oracle reads the integers directly.
 *  - SINQ page, "Mise a l'echelle sur deux axes": a vector of scales for the
 *    rows and another for the columns around the quantized matrix.  Read as:
 *    the dense weight is r_i * c_j * Wd_ij with fp16 r and c and Wd the
 *    decoded dense weight above (the product is exact in fp64 and is not
 *    rounded); the outliers, taken from the unscaled matrix, are added
 *    unscaled.
 *
 * Precision.  A decoded dense weight is an fp16 value: a table entry is
 * copied bit for bit; an affine weight is scale*(q-zero) evaluated exactly in
 * fp64 (an 11-bit significand times a small integer) and rounded once to
 * fp16, nearest-even.  Everything after decoding is fp64: the outlier is
 * added to the decoded weight, and y_ref, together with the error scale
 * bound[b][i] = sum_j |What[i][j]| * |x[b][j]|, is a plain ascending-j sum.
 *
 * Pins (tests/test_oracle.py): fp16 conversions against numpy on every
 * binary16 pattern and on ties; the SpQR CSR worked example; table decode
 * returning the table; affine decode against hand-computed values; the
 * product against exact rational arithmetic; degenerate cases.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_LUT 0
#define ORACLE_AFFINE 1
#define ORACLE_BITPLANE 2
#define ORACLE_INTGRID 3
#define ORACLE_GROUP 16

/* IEEE 754 binary16 -> real value: sign, 5-bit biased exponent (bias 15),
 * 10-bit fraction; exponent 0 encodes subnormals m * 2^-24. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* Real value -> nearest binary16, ties to the even significand; values at or
 * beyond 65520 become infinity; results below 2^-14 are subnormal. */
uint16_t oracle_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    int e2, E;
    double m, fl, r;
    uint64_t n;
    if (isnan(v))
        return 0x7E00;
    if (isinf(v))
        return sign | 0x7C00;
    if (a == 0.0)
        return sign;
    frexp(a, &e2);          /* a in [2^(e2-1), 2^e2) */
    E = e2 - 1;             /* binade of a */
    if (E < -14)
        E = -14;            /* subnormal binade shares the quantum 2^-24 */
    m = ldexp(a, 10 - E);   /* a in units of the quantum 2^(E-10); exact */
    fl = floor(m);
    r = m - fl;
    n = (uint64_t)fl;
    if (r > 0.5 || (r == 0.5 && (n & 1)))
        n += 1;
    if (n == 2048) {        /* rounded up into the next binade */
        n = 1024;
        E += 1;
    }
    if (E > 15)
        return sign | 0x7C00;
    if (n < 1024)           /* only reachable in the subnormal binade */
        return sign | (uint16_t)n;
    return sign | (uint16_t)(((E + 15) << 10) | (int)(n - 1024));
}

void oracle_half_to_double_n(const uint16_t *h, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_half_to_double(h[i]);
}

void oracle_double_to_half_n(const double *v, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        out[i] = oracle_double_to_half(v[i]);
}

/* Decoded dense weight of row i, column j, as an fp16 bit pattern.
 * codes: one uint8 code per weight; INTGRID mode: one int16 integer.
 * table: LUT mode rows x 2^bits centroids; AFFINE and INTGRID modes rows x
 * cols/16 scales; BITPLANE mode rows x cols/(32*2^bits) x (bits+1)
 * coefficients C_0..C_k.
 * zeros: AFFINE mode rows x cols/16 integral zeros (unused otherwise). */
uint16_t oracle_decode_one(int64_t i, int64_t j, int cols, int bits, int mode,
                           const uint8_t *codes, const uint16_t *table,
                           const uint16_t *zeros)
{
    if (mode == ORACLE_INTGRID) {
        int qi = ((const int16_t *)codes)[i * (int64_t)cols + j];
        double scale = oracle_half_to_double(table[i * (int64_t)(cols / ORACLE_GROUP) + j / ORACLE_GROUP]);
        return oracle_double_to_half(scale * (double)qi);
    }
    int q = codes[i * (int64_t)cols + j];
    if (mode == ORACLE_LUT)
        return table[i * ((int64_t)1 << bits) + q];
    if (mode == ORACLE_BITPLANE) {
        /* C_0 + sum over the planes whose bit is set; fp16 terms of at most
         * 11 significant bits between 2^-24 and 2^16 sum exactly in fp64 */
        int64_t gsize = (int64_t)32 << bits;
        const uint16_t *c = table + (i * (cols / gsize) + j / gsize) * (bits + 1);
        double w = oracle_half_to_double(c[0]);
        for (int p = 1; p <= bits; p++)
            if ((q >> (p - 1)) & 1)
                w += oracle_half_to_double(c[p]);
        return oracle_double_to_half(w);
    }
    {
        int64_t g = i * (int64_t)(cols / ORACLE_GROUP) + j / ORACLE_GROUP;
        double scale = oracle_half_to_double(table[g]);
        double zero = oracle_half_to_double(zeros[g]);
        return oracle_double_to_half(scale * ((double)q - zero));
    }
}

/* W_dense: rows x cols fp16 bit patterns (holes decode from their codes). */
void oracle_decode(int rows, int cols, int bits, int mode, const uint8_t *codes,
                   const uint16_t *table, const uint16_t *zeros, uint16_t *wd)
{
    for (int64_t i = 0; i < rows; i++)
        for (int64_t j = 0; j < cols; j++)
            wd[i * cols + j] =
                oracle_decode_one(i, j, cols, bits, mode, codes, table, zeros);
}

/* What row i in fp64: decoded dense weights (times r_i * c_j when the row
 * and column scales are given, NULL meaning none), then each CSR entry of the
 * row added to the weight at its column. */
void oracle_weight_row_two_axis(int64_t i, int cols, int bits, int mode,
                                const uint8_t *codes, const uint16_t *table,
                                const uint16_t *zeros, const int32_t *row_ptr,
                                const int32_t *col_idx, const uint16_t *values,
                                const uint16_t *rscale, const uint16_t *cscale,
                                double *wrow)
{
    double r = rscale ? oracle_half_to_double(rscale[i]) : 1.0;
    for (int64_t j = 0; j < cols; j++) {
        double c = cscale ? oracle_half_to_double(cscale[j]) : 1.0;
        wrow[j] = r * c * oracle_half_to_double(
            oracle_decode_one(i, j, cols, bits, mode, codes, table, zeros));
    }
    for (int64_t k = row_ptr[i]; k < row_ptr[i + 1]; k++)
        wrow[col_idx[k]] += oracle_half_to_double(values[k]);
}

void oracle_weight_row(int64_t i, int cols, int bits, int mode,
                       const uint8_t *codes, const uint16_t *table,
                       const uint16_t *zeros, const int32_t *row_ptr,
                       const int32_t *col_idx, const uint16_t *values,
                       double *wrow)
{
    oracle_weight_row_two_axis(i, cols, bits, mode, codes, table, zeros, row_ptr,
                               col_idx, values, NULL, NULL, wrow);
}

/* What: rows x cols fp64 (row and column scales may be NULL). */
void oracle_materialize_two_axis(int rows, int cols, int bits, int mode,
                                 const uint8_t *codes, const uint16_t *table,
                                 const uint16_t *zeros, const int32_t *row_ptr,
                                 const int32_t *col_idx, const uint16_t *values,
                                 const uint16_t *rscale, const uint16_t *cscale,
                                 double *w)
{
    for (int64_t i = 0; i < rows; i++)
        oracle_weight_row_two_axis(i, cols, bits, mode, codes, table, zeros,
                                   row_ptr, col_idx, values, rscale, cscale,
                                   w + i * cols);
}

void oracle_materialize(int rows, int cols, int bits, int mode,
                        const uint8_t *codes, const uint16_t *table,
                        const uint16_t *zeros, const int32_t *row_ptr,
                        const int32_t *col_idx, const uint16_t *values,
                        double *w)
{
    oracle_materialize_two_axis(rows, cols, bits, mode, codes, table, zeros,
                                row_ptr, col_idx, values, NULL, NULL, w);
}

/* y_ref and bound for the listed output rows only (all rows when
 * row_list == NULL, n_list == rows).  x: batch x cols fp16; y_ref and bound:
 * batch x n_list fp64, column t holding row row_list[t].  Row and column
 * scales may be NULL. */
int oracle_gemv_rows_two_axis(int rows, int cols, int bits, int mode,
                              const uint8_t *codes, const uint16_t *table,
                              const uint16_t *zeros, const int32_t *row_ptr,
                              const int32_t *col_idx, const uint16_t *values,
                              const uint16_t *rscale, const uint16_t *cscale,
                              int batch, const uint16_t *x,
                              const int32_t *row_list, int n_list,
                              double *y_ref, double *bound)
{
    double *wrow = (double *)malloc(sizeof(double) * (cols > 0 ? cols : 1));
    double *xd = (double *)malloc(sizeof(double) * ((int64_t)batch * cols + 1));
    if (!wrow || !xd) {
        free(wrow);
        free(xd);
        return -1;
    }
    for (int64_t t = 0; t < (int64_t)batch * cols; t++)
        xd[t] = oracle_half_to_double(x[t]);
    for (int t = 0; t < n_list; t++) {
        int64_t i = row_list ? row_list[t] : t;
        oracle_weight_row_two_axis(i, cols, bits, mode, codes, table, zeros,
                                   row_ptr, col_idx, values, rscale, cscale,
                                   wrow);
        for (int b = 0; b < batch; b++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t j = 0; j < cols; j++) {
                acc += wrow[j] * xd[(int64_t)b * cols + j];
                mag += fabs(wrow[j]) * fabs(xd[(int64_t)b * cols + j]);
            }
            y_ref[(int64_t)b * n_list + t] = acc;
            bound[(int64_t)b * n_list + t] = mag;
        }
    }
    (void)rows;
    free(wrow);
    free(xd);
    return 0;
}

int oracle_gemv_rows(int rows, int cols, int bits, int mode,
                     const uint8_t *codes, const uint16_t *table,
                     const uint16_t *zeros, const int32_t *row_ptr,
                     const int32_t *col_idx, const uint16_t *values, int batch,
                     const uint16_t *x, const int32_t *row_list, int n_list,
                     double *y_ref, double *bound)
{
    return oracle_gemv_rows_two_axis(rows, cols, bits, mode, codes, table,
                                     zeros, row_ptr, col_idx, values, NULL,
                                     NULL, batch, x, row_list, n_list, y_ref,
                                     bound);
}

/* Full product: y_ref, bound are batch x rows. */
int oracle_gemv(int rows, int cols, int bits, int mode, const uint8_t *codes,
                const uint16_t *table, const uint16_t *zeros,
                const int32_t *row_ptr, const int32_t *col_idx,
                const uint16_t *values, int batch, const uint16_t *x,
                double *y_ref, double *bound)
{
    return oracle_gemv_rows(rows, cols, bits, mode, codes, table, zeros,
                            row_ptr, col_idx, values, batch, x, NULL, rows,
                            y_ref, bound);
}

/* ------------------------------------------------------------------------
 * The decomposition before the product (SqueezeLLM page, "Dense-and-Sparse
 * decomposition"; SpQR page, "Diagramme de la matrice sparse vs dense" and
 * "Quantification d'un modele"): from the weights w (fp32, rows x cols) the
 * nnz largest |w| of the whole matrix become fp16 outliers in CSR (equal |w|:
 * the lower row-major index first); the other weights form the dense part,
 * the outlier positions being holes that count as 0, quantized
 *  - AFFINE: per group of 16 inputs, over the range [min, max] of its dense
 *    weights widened to contain 0: scale = fp16((max - min) / (2^b - 1));
 *    when that scale is not a positive finite number the group gets scale 1
 *    and zero 0; zero = rint(-min / scale), clipped to [0, 2^b - 1];
 *    q = rint(w / scale) + zero, clipped the same way (rint: nearest, ties to
 *    even; the arithmetic in fp64 on the fp16 scale);
 *  - LUT: per row, the centroids are the fp16 roundings of the odd quantiles
 *    (2k+1)/2^(b+1) of the row's dense (non-hole) weights, a quantile being
 *    the linear interpolation x[lo] + t (x[lo+1] - x[lo]) at position
 *    (n-1) p of the sorted values (0 when the row has none); each weight, a
 *    hole counting as 0, takes the nearest centroid, the lower index on a tie.
 * ---------------------------------------------------------------------- */

struct oracle_item {
    float a;
    int64_t i;
};

static int oracle_cmp_outlier(const void *pa, const void *pb)
{
    const struct oracle_item *a = (const struct oracle_item *)pa;
    const struct oracle_item *b = (const struct oracle_item *)pb;
    if (a->a != b->a)
        return a->a > b->a ? -1 : 1;
    return a->i < b->i ? -1 : (a->i > b->i ? 1 : 0);
}

static int oracle_cmp_double(const void *pa, const void *pb)
{
    double a = *(const double *)pa, b = *(const double *)pb;
    return a < b ? -1 : (a > b ? 1 : 0);
}

int oracle_decompose(int rows, int cols, int bits, int mode, int64_t nnz,
                     const float *w, uint8_t *codes, uint16_t *table,
                     uint16_t *zeros, int32_t *row_ptr, int32_t *col_idx,
                     uint16_t *values)
{
    int64_t n = (int64_t)rows * cols, k = 0;
    int K = 1 << bits, qmax = K - 1;
    struct oracle_item *it = (struct oracle_item *)malloc(sizeof(*it) * (n > 0 ? n : 1));
    uint8_t *hole = (uint8_t *)calloc(n > 0 ? n : 1, 1);
    double *sorted = (double *)malloc(sizeof(double) * (cols > 0 ? cols : 1));
    if (!it || !hole || !sorted || nnz < 0 || nnz > n) {
        free(it);
        free(hole);
        free(sorted);
        return -1;
    }
    /* outliers: the nnz largest |w| */
    for (int64_t t = 0; t < n; t++) {
        it[t].a = fabsf(w[t]);
        it[t].i = t;
    }
    qsort(it, (size_t)n, sizeof(*it), oracle_cmp_outlier);
    for (int64_t t = 0; t < nnz; t++)
        hole[it[t].i] = 1;
    /* CSR, row by row, columns ascending */
    row_ptr[0] = 0;
    for (int64_t i = 0; i < rows; i++) {
        for (int64_t j = 0; j < cols; j++)
            if (hole[i * cols + j]) {
                col_idx[k] = (int32_t)j;
                values[k] = oracle_double_to_half((double)w[i * cols + j]);
                k++;
            }
        row_ptr[i + 1] = (int32_t)k;
    }
    /* dense part */
    if (mode == ORACLE_AFFINE) {
        int64_t G = cols / ORACLE_GROUP;
        for (int64_t i = 0; i < rows; i++)
            for (int64_t g = 0; g < G; g++) {
                double mn = 0.0, mx = 0.0, sv, z;
                uint16_t s16;
                for (int c = 0; c < ORACLE_GROUP; c++) {
                    int64_t t = i * cols + g * ORACLE_GROUP + c;
                    double v = hole[t] ? 0.0 : (double)w[t];
                    if (v < mn) mn = v;
                    if (v > mx) mx = v;
                }
                s16 = oracle_double_to_half((mx - mn) / qmax);
                sv = oracle_half_to_double(s16);
                if (isfinite(sv) && sv > 0.0) {
                    z = rint(-mn / sv);
                    z = z < 0.0 ? 0.0 : (z > qmax ? qmax : z);
                } else {
                    s16 = 0x3C00;
                    sv = 1.0;
                    z = 0.0;
                }
                table[i * G + g] = s16;
                zeros[i * G + g] = oracle_double_to_half(z);
                for (int c = 0; c < ORACLE_GROUP; c++) {
                    int64_t t = i * cols + g * ORACLE_GROUP + c;
                    double v = hole[t] ? 0.0 : (double)w[t];
                    double q = rint(v / sv) + z;
                    codes[t] = (uint8_t)(q < 0.0 ? 0 : (q > qmax ? qmax : q));
                }
            }
    } else {
        for (int64_t i = 0; i < rows; i++) {
            int64_t m = 0;
            double cent[16];
            for (int64_t j = 0; j < cols; j++)
                if (!hole[i * cols + j])
                    sorted[m++] = (double)w[i * cols + j];
            qsort(sorted, (size_t)m, sizeof(double), oracle_cmp_double);
            for (int q = 0; q < K; q++) {
                double c = 0.0;
                if (m > 0) {
                    double p = (2.0 * q + 1.0) / (2.0 * K);
                    double h = (double)(m - 1) * p;
                    int64_t lo = (int64_t)floor(h);
                    int64_t hi = lo + 1 < m ? lo + 1 : m - 1;
                    c = sorted[lo] + (h - (double)lo) * (sorted[hi] - sorted[lo]);
                }
                table[i * K + q] = oracle_double_to_half(c);
                cent[q] = oracle_half_to_double(table[i * K + q]);
            }
            for (int64_t j = 0; j < cols; j++) {
                int64_t t = i * cols + j;
                double v = hole[t] ? 0.0 : (double)w[t];
                int best = 0;
                double bd = fabs(v - cent[0]);
                for (int q = 1; q < K; q++)
                    if (fabs(v - cent[q]) < bd) {
                        bd = fabs(v - cent[q]);
                        best = q;
                    }
                codes[t] = (uint8_t)best;
            }
        }
    }
    free(it);
    free(hole);
    free(sorted);
    return 0;
}
