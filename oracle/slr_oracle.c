/*
 * slr_oracle.c -- CPU oracle for the 2:4-sparse + low-rank linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The product
 * path (the CUDA library under sparse_rank_linear_02_b200/) never calls it,
 * and the two share no code, header, table or helper.
 *
 * What it computes, and where the pages define it:
 *
 *   1. The 2:4 projection of a dense weight W (d_out x d_in).
 *      "HASSLE-free" (arXiv 2502.00899), section 4.1.1: with an identity
 *      Hessian the optimal sparse update is hard-thresholding, i.e. keep the
 *      entries of largest magnitude.  The 3BASiL summary page ("Splitting each
 *      weight matrix into two parts" / "A three-block ADMM ..." paragraphs)
 *      defines 2:4 as at most two nonzeros in every four weights.  Readings
 *      taken where the pages are silent: groups are the aligned runs of four
 *      along d_in; the magnitude key is the bf16 bit pattern with the sign bit
 *      cleared; ties go to the lower index; exactly two positions are kept per
 *      group (they may hold zeros); kept values are stored in ascending index
 *      order; metadata byte j of a row holds group 2j in its low nibble and
 *      group 2j+1 in its high nibble, nibble = idx0 | idx1 << 2.
 *
 *   1b. The activation-aware 2:4 projection.  HASSLE-free, section 4.1.2:
 *      with a diagonal Hessian the optimal sparse update is a scaled
 *      hard-thresholding (the Wanda-style score |w_ij| * s_j, s_j the norm of
 *      input column j, s_j^2 the Hessian diagonal).  The score of a weight is
 *      the single-precision product |w| * |s| (round to nearest); any NaN
 *      product scores 0x7FFFFFFF; keys are compared as unsigned integers
 *      (the bits of a non-negative float), ties go to the lower index, and the
 *      packed format is the one above.  The column norms s_j = ||X[:, j]||_2
 *      are computed in fp64.
 *
 *   1c. The 2:8 projection (the "2:8 plus rank-64" configuration of the
 *      3BASiL summary page, "Faster compression and gains that survive LoRA"
 *      and "Weigh the gap reduction against the configuration"): at most two
 *      nonzeros in every aligned run of eight weights along d_in, kept by the
 *      same hard-thresholding rule (largest magnitude keys, ties to the lower
 *      index).  Packed densely: two values per group of eight in ascending
 *      index order, and one metadata byte per group, idx0 | idx1 << 3.  Every
 *      2:8 matrix is also a 2:4 matrix (each half-group of four holds at most
 *      two nonzeros), so the forward of a 2:8 layer is the forward of its
 *      2:4 packing (oracle_pack_2to4 of the unpacked matrix).
 *
 *   2. The forward pass.  LoSparse (arXiv 2306.11222), section 3 and
 *      section 3.2: the compressed layer replaces X*W by the sum of a sparse
 *      term and a low-rank term, run in parallel.  In the d_out x d_in
 *      convention used here, W' = S + U*V and Y = X * W'^T.  The oracle forms
 *      each row of W' densely in fp64 (no rounding) and takes the dot products
 *      in fp64, exactly as that definition reads.  It also returns the
 *      per-element magnitude bound  B = |X| * |W'|^T  used by the acceptance
 *      test  |Y_gpu - Y| <= 1e-2 * B + 1e-3.
 *
 * Parity pins for every function here live in tests/test_oracle.py (brute
 * force over all groups of a small alphabet, invariants, pack/unpack round
 * trips, a hand-derived fixture, the algebraic identity with exact small
 * integers, and numpy fp64 cross-checks).
 *
 * Inputs are raw bf16 bit patterns (uint16_t).  Widening bf16 to double is
 * exact.  OpenMP only splits independent output rows across threads; the
 * arithmetic of each output element is a single sequential loop.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Number of metadata bytes per row: one nibble per group of four, two nibbles
 * per byte, rounded up. */
int64_t oracle_meta_row_bytes(int64_t d_in)
{
    int64_t groups = d_in / 4;
    return (groups + 1) / 2;
}

/* Choose the two kept positions of one group of four bf16 values.
 * Each position p gets a rank: the number of positions q that come before it
 * in the order (magnitude key descending, index ascending).  The two positions
 * of rank 0 and 1 are kept; they are reported in ascending index order. */
static void choose_two(const uint16_t w[4], int *idx0, int *idx1)
{
    int kept[2];
    int n = 0;
    for (int p = 0; p < 4; ++p) {
        unsigned kp = w[p] & 0x7FFFu;
        int rank = 0;
        for (int q = 0; q < 4; ++q) {
            unsigned kq = w[q] & 0x7FFFu;
            if (kq > kp || (kq == kp && q < p)) ++rank;
        }
        if (rank < 2) kept[n++] = p;
    }
    /* p runs upward, so kept[0] < kept[1]. */
    *idx0 = kept[0];
    *idx1 = kept[1];
}

/* 2:4 projection and packing.
 *   W    : d_out rows, row stride ldw elements (ldw >= d_in), bf16 bits.
 *   vals : d_out x (d_in/2) bf16 bits, dense rows.
 *   meta : d_out x oracle_meta_row_bytes(d_in) bytes, dense rows.
 * Returns 0, or -1 when d_in is not a multiple of 4 or ldw < d_in. */
int oracle_pack_2to4(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                     uint16_t *vals, uint8_t *meta)
{
    if (d_in % 4 != 0 || ldw < d_in || d_out < 0) return -1;
    int64_t groups = d_in / 4;
    int64_t mrow = oracle_meta_row_bytes(d_in);
    for (int64_t i = 0; i < d_out; ++i) {
        memset(meta + i * mrow, 0, (size_t)mrow);
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t *w = W + i * ldw + 4 * g;
            int a, b;
            choose_two(w, &a, &b);
            vals[i * (d_in / 2) + 2 * g + 0] = w[a];
            vals[i * (d_in / 2) + 2 * g + 1] = w[b];
            unsigned nib = (unsigned)a | ((unsigned)b << 2);
            meta[i * mrow + g / 2] |= (uint8_t)(nib << (4 * (g % 2)));
        }
    }
    return 0;
}

/* Score key of one weight under the activation-aware projection: the bits
 * of the float product |w| * |s| (IEEE single, round to nearest, one multiply;
 * both factors are non-negative, so the sign bit is clear and the bits order
 * like the values); a NaN product scores 0x7FFFFFFF. */
static uint32_t scaled_key(uint16_t w, float s)
{
    uint32_t u = ((uint32_t)(w & 0x7FFFu)) << 16;
    float aw;
    memcpy(&aw, &u, sizeof aw);
    volatile float prod = aw * fabsf(s);
    if (isnan(prod)) return 0x7FFFFFFFu;
    float pf = prod;
    uint32_t k;
    memcpy(&k, &pf, sizeof k);
    return k;
}

/* As choose_two, on the scaled keys of the four positions. */
static void choose_two_keys(const uint32_t key[4], int *idx0, int *idx1)
{
    int kept[2];
    int n = 0;
    for (int p = 0; p < 4; ++p) {
        int rank = 0;
        for (int q = 0; q < 4; ++q)
            if (key[q] > key[p] || (key[q] == key[p] && q < p)) ++rank;
        if (rank < 2) kept[n++] = p;
    }
    *idx0 = kept[0];
    *idx1 = kept[1];
}

/* Activation-aware 2:4 projection and packing: as oracle_pack_2to4, with the
 * weights of column j ranked by the scaled key of (w_ij, scale[j]).
 *   scale : d_in floats. */
int oracle_pack_2to4_scaled(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw, const float *scale,
                            uint16_t *vals, uint8_t *meta)
{
    if (d_in % 4 != 0 || ldw < d_in || d_out < 0) return -1;
    int64_t groups = d_in / 4;
    int64_t mrow = oracle_meta_row_bytes(d_in);
    for (int64_t i = 0; i < d_out; ++i) {
        memset(meta + i * mrow, 0, (size_t)mrow);
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t *w = W + i * ldw + 4 * g;
            uint32_t key[4];
            for (int p = 0; p < 4; ++p) key[p] = scaled_key(w[p], scale[4 * g + p]);
            int a, b;
            choose_two_keys(key, &a, &b);
            vals[i * (d_in / 2) + 2 * g + 0] = w[a];
            vals[i * (d_in / 2) + 2 * g + 1] = w[b];
            unsigned nib = (unsigned)a | ((unsigned)b << 2);
            meta[i * mrow + g / 2] |= (uint8_t)(nib << (4 * (g % 2)));
        }
    }
    return 0;
}

/* 2:8 projection and packing.
 *   W    : d_out rows, row stride ldw elements (ldw >= d_in), bf16 bits.
 *   vals : d_out x (d_in/4) bf16 bits: the two kept values of group g (columns
 *          8g..8g+7) at 2g, 2g+1, lower index first.
 *   meta : d_out x (d_in/8) bytes: byte g = idx0 | idx1 << 3, idx0 < idx1.
 * The two kept positions of a group are those whose magnitude key (bf16 bits
 * without the sign) is beaten by fewer than two others, where q beats p when
 * its key is larger, or equal with q < p.
 * Returns 0, or -1 when d_in is not a multiple of 8 or ldw < d_in. */
int oracle_pack_2to8(const uint16_t *W, int64_t d_out, int64_t d_in, int64_t ldw,
                     uint16_t *vals, uint8_t *meta)
{
    if (d_in % 8 != 0 || ldw < d_in || d_out < 0) return -1;
    int64_t groups = d_in / 8;
    for (int64_t i = 0; i < d_out; ++i) {
        for (int64_t g = 0; g < groups; ++g) {
            const uint16_t *w = W + i * ldw + 8 * g;
            int kept[2];
            int n = 0;
            for (int p = 0; p < 8; ++p) {
                unsigned kp = w[p] & 0x7FFFu;
                int beaten = 0;
                for (int q = 0; q < 8; ++q) {
                    unsigned kq = w[q] & 0x7FFFu;
                    if (kq > kp || (kq == kp && q < p)) ++beaten;
                }
                if (beaten < 2) kept[n++] = p;
            }
            vals[i * (d_in / 4) + 2 * g + 0] = w[kept[0]];
            vals[i * (d_in / 4) + 2 * g + 1] = w[kept[1]];
            meta[i * groups + g] = (uint8_t)(kept[0] | (kept[1] << 3));
        }
    }
    return 0;
}

/* Expand a 2:8 packing back to the dense d_out x d_in matrix (+0.0 at the
 * positions that were not kept). */
int oracle_unpack_2to8(const uint16_t *vals, const uint8_t *meta, int64_t d_out, int64_t d_in, uint16_t *S)
{
    if (d_in % 8 != 0 || d_out < 0) return -1;
    int64_t groups = d_in / 8;
    for (int64_t i = 0; i < d_out; ++i) {
        for (int64_t j = 0; j < d_in; ++j) S[i * d_in + j] = 0;
        for (int64_t g = 0; g < groups; ++g) {
            unsigned byte = meta[i * groups + g];
            int a = (int)(byte & 7u), b = (int)((byte >> 3) & 7u);
            S[i * d_in + 8 * g + a] = vals[i * (d_in / 4) + 2 * g + 0];
            S[i * d_in + 8 * g + b] = vals[i * (d_in / 4) + 2 * g + 1];
        }
    }
    return 0;
}

/* Column norms of X (M x d_in, bf16 bits): out[j] = sqrt(sum_m X[m][j]^2) in
 * fp64, the sum taken in row order. */
int oracle_column_norms(const uint16_t *X, int64_t M, int64_t d_in, double *out)
{
    if (M < 0 || d_in < 0) return -1;
    for (int64_t j = 0; j < d_in; ++j) {
        double acc = 0.0;
        for (int64_t m = 0; m < M; ++m) {
            double x = bf16_bits_to_double(X[m * d_in + j]);
            acc += x * x;
        }
        out[j] = sqrt(acc);
    }
    return 0;
}

/* Expand packed (vals, meta) back to a dense d_out x d_in bf16 matrix; the
 * positions that were not kept hold +0.0 (bits 0x0000). */
int oracle_unpack_2to4(const uint16_t *vals, const uint8_t *meta, int64_t d_out,
                       int64_t d_in, uint16_t *S)
{
    if (d_in % 4 != 0 || d_out < 0) return -1;
    int64_t groups = d_in / 4;
    int64_t mrow = oracle_meta_row_bytes(d_in);
    for (int64_t i = 0; i < d_out; ++i) {
        for (int64_t j = 0; j < d_in; ++j) S[i * d_in + j] = 0;
        for (int64_t g = 0; g < groups; ++g) {
            unsigned nib = (meta[i * mrow + g / 2] >> (4 * (g % 2))) & 0xFu;
            int a = (int)(nib & 3u), b = (int)(nib >> 2);
            S[i * d_in + 4 * g + a] = vals[i * (d_in / 2) + 2 * g + 0];
            S[i * d_in + 4 * g + b] = vals[i * (d_in / 2) + 2 * g + 1];
        }
    }
    return 0;
}

/* One row of the dense fp64 matrix W' = S + U*V, for output row i.
 * S is given packed; U is d_out x r, V is r x d_in (row-major bf16 bits). */
static void dense_row(const uint16_t *vals, const uint8_t *meta, const uint16_t *U,
                      const uint16_t *V, int64_t d_in, int64_t r, int64_t i,
                      double *row)
{
    int64_t groups = d_in / 4;
    int64_t mrow = oracle_meta_row_bytes(d_in);
    for (int64_t j = 0; j < d_in; ++j) row[j] = 0.0;
    for (int64_t g = 0; g < groups; ++g) {
        unsigned nib = (meta[i * mrow + g / 2] >> (4 * (g % 2))) & 0xFu;
        int a = (int)(nib & 3u), b = (int)(nib >> 2);
        row[4 * g + a] = bf16_bits_to_double(vals[i * (d_in / 2) + 2 * g + 0]);
        row[4 * g + b] = bf16_bits_to_double(vals[i * (d_in / 2) + 2 * g + 1]);
    }
    for (int64_t j = 0; j < d_in; ++j) {
        double lr = 0.0;
        for (int64_t k = 0; k < r; ++k)
            lr += bf16_bits_to_double(U[i * r + k]) * bf16_bits_to_double(V[k * d_in + j]);
        row[j] += lr;
    }
}

/* Forward pass in fp64:  Y[m, i] = sum_j X[m, j] * W'[i, j],
 *                        B[m, i] = sum_j |X[m, j]| * |W'[i, j]|.
 * rows      : the n_rows indices of X (tokens) to evaluate, or NULL for all M.
 * outs      : the n_outs output indices i to evaluate, or NULL for all d_out.
 * Y, Bound  : n_rows x n_outs doubles (entry [t, o] is token rows[t], output
 *             outs[o]); Bound may be NULL.
 * r may be 0 (no low-rank term; U and V are then ignored). */
int oracle_forward(const uint16_t *X, int64_t M, const uint16_t *vals, const uint8_t *meta,
                   int64_t d_out, int64_t d_in, const uint16_t *U, const uint16_t *V,
                   int64_t r, const int64_t *rows, int64_t n_rows, const int64_t *outs,
                   int64_t n_outs, double *Y, double *Bound, int nthreads)
{
    if (d_in % 4 != 0 || d_out < 0 || M < 0 || r < 0) return -1;
    if (rows == NULL) n_rows = M;
    if (outs == NULL) n_outs = d_out;
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t m = rows ? rows[t] : t;
        if (m < 0 || m >= M) return -1;
    }
    for (int64_t o = 0; o < n_outs; ++o) {
        int64_t i = outs ? outs[o] : o;
        if (i < 0 || i >= d_out) return -1;
    }
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * (size_t)(d_in > 0 ? d_in : 1));
        double *xr = (double *)malloc(sizeof(double) * (size_t)(d_in > 0 ? d_in : 1));
        if (row == NULL || xr == NULL) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t o = 0; o < n_outs; ++o) {
                int64_t i = outs ? outs[o] : o;
                dense_row(vals, meta, U, V, d_in, r, i, row);
                for (int64_t t = 0; t < n_rows; ++t) {
                    int64_t m = rows ? rows[t] : t;
                    for (int64_t j = 0; j < d_in; ++j) xr[j] = bf16_bits_to_double(X[m * d_in + j]);
                    double acc = 0.0, bound = 0.0;
                    for (int64_t j = 0; j < d_in; ++j) {
                        acc += xr[j] * row[j];
                        bound += fabs(xr[j]) * fabs(row[j]);
                    }
                    Y[t * n_outs + o] = acc;
                    if (Bound) Bound[t * n_outs + o] = bound;
                }
            }
        }
        free(row);
        free(xr);
    }
    return failed ? -2 : 0;
}

/* Low-rank projection alone, T = X * V^T in fp64 (n_rows x r).  Used by the
 * tests to check a kernel's intermediate, and by nothing else. */
int oracle_lowrank_project(const uint16_t *X, int64_t M, const uint16_t *V, int64_t d_in,
                           int64_t r, double *T)
{
    if (M < 0 || r < 0 || d_in < 0) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < r; ++k) {
            double acc = 0.0;
            for (int64_t j = 0; j < d_in; ++j)
                acc += bf16_bits_to_double(X[m * d_in + j]) * bf16_bits_to_double(V[k * d_in + j]);
            T[m * r + k] = acc;
        }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
