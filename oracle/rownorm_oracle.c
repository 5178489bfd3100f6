/*
 * Row-normalization ORACLE: plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. This file is built and called by the test suite,
 * by the entry module's smoke check and by the CPU-baseline leg of the
 * benchmark. The product library never links, loads or calls it, and it
 * shares no code, header, constant or helper with the CUDA path.
 *
 * What it computes (one row at a time, every sum in fp64, plain sequential
 * order, no blocking or reordering):
 *
 *   RMSNorm   -- "Fused transformer kernels on Emily", Part 1 (the composed
 *                RMSNorm written with Nx primitives) and "Emily.Fast",
 *                `rms_norm/3`:
 *                  y_j = x_j / sqrt( (1/D) * sum_i x_i^2 + eps ) * w_j
 *
 *   LayerNorm -- "Emily.Fast", `layer_norm/4`:
 *                  mu      = (1/D) * sum_i x_i
 *                  var     = (1/D) * sum_i (x_i - mu)^2
 *                  y_j     = (x_j - mu) / sqrt(var + eps) * w_j + b_j
 *                The page names the statistic "Welford-style" mean and
 *                variance; that is a way of computing the same population
 *                mean and variance, so the oracle writes out the definition.
 *
 *   Dual q/k head RMSNorm -- "norm_fusion.rs" (mlx_c_rust compile module),
 *                `build_dual_head_norm_graph` / `apply_compiled_dual_head_norm`:
 *                the RMSNorm of the query rows with the query weight, and the
 *                RMSNorm of the key rows with the key weight, one eps shared,
 *                returned queries first, keys second.
 *
 *   Residual add + RMSNorm -- the elementwise-producer fusion that
 *                "norm_fusion.rs" (module doc comment) leaves composed until
 *                a kernel pins the summation order. The composed path adds
 *                the residual, stores the sum in the tensor's type, then
 *                normalizes what it stored:
 *                  h_j = round_T(x_j + r_j)
 *                  y_j = h_j / sqrt( (1/D) * sum_i h_i^2 + eps ) * w_j
 *
 *   Gated RMSNorm -- "norm_fusion.rs" (module doc comment): the output RMS
 *                normalization chained into the SwiGLU epilogue, i.e. the
 *                normalized row times the SiLU of the gate:
 *                  y_j = x_j / sqrt( (1/D) * sum_i x_i^2 + eps ) * w_j
 *                        * silu(z_j),   silu(t) = t / (1 + exp(-t))
 *
 *   Dual q/k head RMSNorm + RoPE -- the dual head norm above, each normalized
 *                head row then rotated as "Emily.Fast", `rope/3` and
 *                `rope_with_freqs/4` describe: with pos = offset + token
 *                (token = row / heads) and, for plane i < dims/2,
 *                  theta_i = pos * scale * f_i,
 *                  f_i = base^(-2i/dims), or the given inverse frequency,
 *                the plane (a, b) = (i, i + dims/2) (split-half) or
 *                (2i, 2i + 1) (traditional) becomes
 *                  y_a = n_a cos theta_i - n_b sin theta_i
 *                  y_b = n_b cos theta_i + n_a sin theta_i
 *                and columns from dims on are n unchanged.
 *
 * Readings where the pages are silent (each is listed in the design doc):
 *   - the variance divisor is D (population variance);
 *   - eps travels as a binary32 value (norm_fusion.rs keeps it as f32 bits)
 *     and is promoted exactly to fp64 here;
 *   - a null weight means all ones, a null bias all zeros;
 *   - round_T is round-to-nearest-even to the storage type (binary32, or
 *     bfloat16: the upper 16 bits of the binary32 value, rounded on the
 *     16 bits dropped).
 *
 * Inputs are [rows, dim] views whose last axis is contiguous and whose rows
 * start row_stride elements apart. Element type 0 = binary32, 1 = bfloat16
 * (raw 16-bit patterns). Every input element is decoded exactly to fp64.
 * Outputs are dense [rows, dim] fp64 arrays.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* bfloat16 is, by its definition, the upper 16 bits of an IEEE binary32
 * value; placing the pattern there and widening is exact. */
static double decode_element(const void *base, int dtype, int64_t index) {
    if (dtype == ORACLE_F32) {
        float f;
        memcpy(&f, (const char *)base + 4 * index, 4);
        return (double)f;
    }
    uint16_t half;
    memcpy(&half, (const char *)base + 2 * index, 2);
    uint32_t bits = (uint32_t)half << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

static int check_view(const void *x, int dtype, int64_t rows, int64_t dim,
                      int64_t row_stride) {
    if (x == NULL && rows > 0) return 1;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return 2;
    if (rows < 0 || dim < 1 || row_stride < dim) return 3;
    return 0;
}

/* One RMSNorm row, exactly in the order the composed formula states. */
static void rms_norm_row(const void *x, int dtype, int64_t row, int64_t dim,
                         int64_t row_stride, const void *w, double eps,
                         double *y_row) {
    const int64_t first = row * row_stride;
    double sum_sq = 0.0;
    for (int64_t i = 0; i < dim; ++i) {
        double v = decode_element(x, dtype, first + i);
        sum_sq += v * v;
    }
    double mean_sq = sum_sq / (double)dim;
    double rms = sqrt(mean_sq + eps);
    for (int64_t j = 0; j < dim; ++j) {
        double v = decode_element(x, dtype, first + j);
        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;
        y_row[j] = v / rms * weight;
    }
}

/* One LayerNorm row: population mean, population variance, then affine. */
static void layer_norm_row(const void *x, int dtype, int64_t row, int64_t dim,
                           int64_t row_stride, const void *w, const void *b,
                           double eps, double *y_row) {
    const int64_t first = row * row_stride;
    double sum = 0.0;
    for (int64_t i = 0; i < dim; ++i) sum += decode_element(x, dtype, first + i);
    double mean = sum / (double)dim;
    double sum_dev_sq = 0.0;
    for (int64_t i = 0; i < dim; ++i) {
        double dev = decode_element(x, dtype, first + i) - mean;
        sum_dev_sq += dev * dev;
    }
    double var = sum_dev_sq / (double)dim;
    double denom = sqrt(var + eps);
    for (int64_t j = 0; j < dim; ++j) {
        double v = decode_element(x, dtype, first + j);
        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;
        double bias = (b != NULL) ? decode_element(b, dtype, j) : 0.0;
        y_row[j] = (v - mean) / denom * weight + bias;
    }
}

/* Rows are independent; nthreads > 1 only spreads whole rows over threads
 * and leaves every row's arithmetic exactly as above. */
int oracle_rms_norm(const void *x, int dtype, int64_t rows, int64_t dim,
                    int64_t row_stride, const void *w, float eps, double *y,
                    int nthreads) {
    int status = check_view(x, dtype, rows, dim, row_stride);
    if (status) return status;
    if (rows > 0 && y == NULL) return 1;
    const double eps64 = (double)eps;
    (void)nthreads;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r)
        rms_norm_row(x, dtype, r, dim, row_stride, w, eps64, y + r * dim);
    return 0;
}

int oracle_layer_norm(const void *x, int dtype, int64_t rows, int64_t dim,
                      int64_t row_stride, const void *w, const void *b,
                      float eps, double *y, int nthreads) {
    int status = check_view(x, dtype, rows, dim, row_stride);
    if (status) return status;
    if (rows > 0 && y == NULL) return 1;
    const double eps64 = (double)eps;
    (void)nthreads;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t r = 0; r < rows; ++r)
        layer_norm_row(x, dtype, r, dim, row_stride, w, b, eps64, y + r * dim);
    return 0;
}

/* Queries first, keys second; both with the one shared eps. */
int oracle_dual_head_rms_norm(const void *q, int64_t q_rows, int64_t q_dim,
                              int64_t q_stride, const void *k, int64_t k_rows,
                              int64_t k_dim, int64_t k_stride, int dtype,
                              const void *wq, const void *wk, float eps,
                              double *yq, double *yk, int nthreads) {
    int status = oracle_rms_norm(q, dtype, q_rows, q_dim, q_stride, wq, eps, yq,
                                 nthreads);
    if (status) return status;
    return oracle_rms_norm(k, dtype, k_rows, k_dim, k_stride, wk, eps, yk,
                           nthreads);
}

/* x + r as the composed path stores it: rounded to nearest, ties to even,
 * to the storage type. (double)->(float) rounds to nearest-even (the C
 * default rounding mode); for two binary32 or two bfloat16 operands the
 * binary32 value is the exact sum rounded once, and bfloat16 rounding then
 * acts on the 16 low bits the narrower format drops. */
static double store_round(double s, int dtype) {
    float f = (float)s;
    if (dtype == ORACLE_F32) return (double)f;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {
        /* infinity keeps its pattern; NaN stays NaN (quiet bit set) */
        if (u & 0x007fffffu) u |= 0x00400000u;
        u &= 0xffff0000u;
    } else {
        const uint32_t dropped = u & 0xffffu;
        const uint32_t kept_lsb = (u >> 16) & 1u;
        u &= 0xffff0000u;
        if (dropped > 0x8000u || (dropped == 0x8000u && kept_lsb)) u += 0x10000u;
    }
    memcpy(&f, &u, 4);
    return (double)f;
}

/* One residual-add + RMSNorm row: the stored sum, then RMSNorm of it. */
static void add_rms_norm_row(const void *x, const void *r, int dtype, int64_t row,
                             int64_t dim, int64_t x_stride, int64_t r_stride,
                             const void *w, double eps, double *y_row,
                             double *h_row) {
    for (int64_t i = 0; i < dim; ++i) {
        double s = decode_element(x, dtype, row * x_stride + i) +
                   decode_element(r, dtype, row * r_stride + i);
        h_row[i] = store_round(s, dtype);
    }
    double sum_h2 = 0.0;
    for (int64_t i = 0; i < dim; ++i) sum_h2 += h_row[i] * h_row[i];
    double mean_h2 = sum_h2 / (double)dim;
    double rms_h = sqrt(mean_h2 + eps);
    for (int64_t j = 0; j < dim; ++j) {
        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;
        y_row[j] = h_row[j] / rms_h * weight;
    }
}

/* One gated RMSNorm row: RMSNorm, weight, then times silu of the gate. */
static void gated_rms_norm_row(const void *x, const void *z, int dtype, int64_t row,
                               int64_t dim, int64_t x_stride, int64_t z_stride,
                               const void *w, double eps, double *y_row) {
    double sum_x2 = 0.0;
    for (int64_t i = 0; i < dim; ++i) {
        double xv = decode_element(x, dtype, row * x_stride + i);
        sum_x2 += xv * xv;
    }
    double mean_x2 = sum_x2 / (double)dim;
    double rms_x = sqrt(mean_x2 + eps);
    for (int64_t j = 0; j < dim; ++j) {
        double xv = decode_element(x, dtype, row * x_stride + j);
        double weight = (w != NULL) ? decode_element(w, dtype, j) : 1.0;
        double gate = decode_element(z, dtype, row * z_stride + j);
        double silu = gate / (1.0 + exp(-gate));
        y_row[j] = xv / rms_x * weight * silu;
    }
}

int oracle_add_rms_norm(const void *x, const void *r, int dtype, int64_t rows,
                        int64_t dim, int64_t x_stride, int64_t r_stride,
                        const void *w, float eps, double *y, double *h,
                        int nthreads) {
    int status = check_view(x, dtype, rows, dim, x_stride);
    if (!status) status = check_view(r, dtype, rows, dim, r_stride);
    if (status) return status;
    if (rows > 0 && (y == NULL || h == NULL)) return 1;
    const double eps64 = (double)eps;
    (void)nthreads;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < rows; ++i)
        add_rms_norm_row(x, r, dtype, i, dim, x_stride, r_stride, w, eps64,
                         y + i * dim, h + i * dim);
    return 0;
}

int oracle_gated_rms_norm(const void *x, const void *z, int dtype, int64_t rows,
                          int64_t dim, int64_t x_stride, int64_t z_stride,
                          const void *w, float eps, double *y, int nthreads) {
    int status = check_view(x, dtype, rows, dim, x_stride);
    if (!status) status = check_view(z, dtype, rows, dim, z_stride);
    if (status) return status;
    if (rows > 0 && y == NULL) return 1;
    const double eps64 = (double)eps;
    (void)nthreads;
#pragma omp parallel for schedule(static) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < rows; ++i)
        gated_rms_norm_row(x, z, dtype, i, dim, x_stride, z_stride, w, eps64,
                           y + i * dim);
    return 0;
}

/* RMSNorm of one row into n_row (fp64), then RoPE of its first dims columns
 * at position pos, into y_row. */
static void rms_rope_row(const void *x, int dtype, int64_t row, int64_t dim,
                         int64_t row_stride, const void *w, double eps, double pos,
                         int64_t dims, int traditional, double base, double scale,
                         const float *inv_freq, double *n_row, double *y_row) {
    rms_norm_row(x, dtype, row, dim, row_stride, w, eps, n_row);
    for (int64_t j = 0; j < dim; ++j) y_row[j] = n_row[j];
    const int64_t half = dims / 2;
    for (int64_t i = 0; i < half; ++i) {
        double f = (inv_freq != NULL) ? (double)inv_freq[i]
                                      : pow(base, -2.0 * (double)i / (double)dims);
        double theta = pos * scale * f;
        double c = cos(theta), s = sin(theta);
        int64_t a = traditional ? 2 * i : i;
        int64_t b = traditional ? 2 * i + 1 : i + half;
        y_row[a] = n_row[a] * c - n_row[b] * s;
        y_row[b] = n_row[b] * c + n_row[a] * s;
    }
}

static int rms_rope_rows(const void *x, int dtype, int64_t rows, int64_t dim,
                         int64_t stride, const void *w, double eps, int64_t heads,
                         int64_t offset, int64_t dims, int traditional, double base,
                         double scale, const float *inv_freq, double *y, int nthreads) {
    int status = check_view(x, dtype, rows, dim, stride);
    if (status) return status;
    if (rows > 0 && y == NULL) return 1;
    if (heads < 1 || rows % heads != 0 || dims < 0 || dims % 2 != 0 || dims > dim) return 3;
    (void)nthreads;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *n_row = (double *)malloc((size_t)dim * sizeof(double));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            double pos = (double)(offset + r / heads);
            rms_rope_row(x, dtype, r, dim, stride, w, eps, pos, dims, traditional, base,
                         scale, inv_freq, n_row, y + r * dim);
        }
        free(n_row);
    }
    return 0;
}

/* Queries first, keys second; one eps, one position schedule. */
int oracle_dual_head_rms_norm_rope(const void *q, int64_t q_rows, int64_t q_dim,
                                   int64_t q_stride, const void *k, int64_t k_rows,
                                   int64_t k_dim, int64_t k_stride, int dtype,
                                   const void *wq, const void *wk, float eps,
                                   int64_t heads_q, int64_t heads_k, int64_t offset,
                                   int64_t dims, int traditional, float base, float scale,
                                   const float *inv_freq, double *yq, double *yk,
                                   int nthreads) {
    if (heads_q < 1 || heads_k < 1 || q_rows / heads_q != k_rows / heads_k) return 3;
    int status = rms_rope_rows(q, dtype, q_rows, q_dim, q_stride, wq, (double)eps, heads_q,
                               offset, dims, traditional, (double)base, (double)scale,
                               inv_freq, yq, nthreads);
    if (status) return status;
    return rms_rope_rows(k, dtype, k_rows, k_dim, k_stride, wk, (double)eps, heads_k,
                         offset, dims, traditional, (double)base, (double)scale, inv_freq,
                         yk, nthreads);
}

/* Exposed so the test suite can pin the element decoding on its own. */
void oracle_decode(const void *src, int dtype, int64_t n, double *dst) {
    for (int64_t i = 0; i < n; ++i) dst[i] = decode_element(src, dtype, i);
}
