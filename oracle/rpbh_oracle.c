/*
 * Oracle: OrbitQuant RPBH weight path and its Lloyd-Max codebook (page "orbit_quant.py").
 * TEST INFRASTRUCTURE ONLY.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include "wq_oracle.h"

/* ---- gaussian_lloyd_max ------------------------------------------------------------------ */

/* libm has no inverse error function: solve erf(y) = t by bisection on [-7, 7] (erf is strictly
 * increasing) until the bracket stops shrinking, which leaves |y - erfinv(t)| at the last ulp. */
double or_erfinv(double t) {
    if (t <= -1.0) return -INFINITY;
    if (t >= 1.0) return INFINITY;
    double lo = -7.0, hi = 7.0;
    for (int it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (erf(mid) < t)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

void or_gaussian_lloyd_max_f64(int bits, int iters, double *c) {
    const int L = 1 << bits;
    const double sqrt_2pi = sqrt(2.0 * 3.141592653589793); /* math.sqrt(2.0 * math.pi) */
    /* init at the gaussian quantile midpoints: q = (k + 0.5) / L, c = sqrt(2) * erfinv(2q - 1) */
    for (int k = 0; k < L; ++k) {
        double q = ((double)k + 0.5) / (double)L;
        c[k] = sqrt(2.0) * or_erfinv(2.0 * q - 1.0);
    }
    double *lo = (double *)malloc(sizeof(double) * (size_t)L);
    double *hi = (double *)malloc(sizeof(double) * (size_t)L);
    for (int it = 0; it < iters; ++it) {
        /* edges = (c[:-1] + c[1:]) / 2; lo = [-inf, edges]; hi = [edges, inf] */
        lo[0] = -INFINITY;
        hi[L - 1] = INFINITY;
        for (int k = 0; k + 1 < L; ++k) {
            double e = (c[k] + c[k + 1]) / 2.0;
            hi[k] = e;
            lo[k + 1] = e;
        }
        /* c = (phi(lo) - phi(hi)) / (Phi(hi) - Phi(lo)) */
        for (int k = 0; k < L; ++k) {
            double phi_lo = exp(-lo[k] * lo[k] / 2.0) / sqrt_2pi;
            double phi_hi = exp(-hi[k] * hi[k] / 2.0) / sqrt_2pi;
            double cdf_lo = 0.5 * (1.0 + erf(lo[k] / sqrt(2.0)));
            double cdf_hi = 0.5 * (1.0 + erf(hi[k] / sqrt(2.0)));
            c[k] = (phi_lo - phi_hi) / (cdf_hi - cdf_lo);
        }
    }
    free(lo);
    free(hi);
}

void or_gaussian_lloyd_max(int bits, int iters, float *out) {
    double c[16];
    or_gaussian_lloyd_max_f64(bits, iters, c);
    for (int k = 0; k < (1 << bits); ++k) out[k] = (float)c[k];
}

/* ---- rotation ---------------------------------------------------------------------------- */

int64_t or_hadamard_block_size(int64_t d) { return d & (-d); }

/* x * h ** -0.5: the Python double is applied to the fp32 tensor as fp32. */
float or_rpbh_fwht_post(int64_t h) { return (float)pow((double)h, -0.5); }

/* gaussian_lloyd_max(bits) * d ** -0.5, both fp32. */
void or_rpbh_codebook(int bits, int64_t d, float *out) {
    float c[16];
    or_gaussian_lloyd_max(bits, 200, c);
    const float s = (float)pow((double)d, -0.5);
    for (int k = 0; k < (1 << bits); ++k) out[k] = c[k] * s;
}

void or_rpbh_forward(const float *x, int64_t rows, int64_t d, const int32_t *perm,
                     const int8_t *signs, int64_t h, float *y) {
    const float post = or_rpbh_fwht_post(h);
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * d;
        float *yr = y + r * d;
        /* index_select(x, -1, perm) * signs */
        for (int64_t j = 0; j < d; ++j) yr[j] = xr[perm[j]] * (float)signs[j];
        /* _fwht on each contiguous h-block */
        for (int64_t b = 0; b < d; b += h) or_fwht(yr + b, h, post);
    }
}

void or_rpbh_inverse(const float *y, int64_t rows, int64_t d, const int32_t *inv_perm,
                     const int8_t *signs, int64_t h, float *out) {
    const float post = or_rpbh_fwht_post(h);
    float *z = (float *)malloc(sizeof(float) * (size_t)d);
    for (int64_t r = 0; r < rows; ++r) {
        memcpy(z, y + r * d, sizeof(float) * (size_t)d);
        for (int64_t b = 0; b < d; b += h) or_fwht(z + b, h, post);
        for (int64_t j = 0; j < d; ++j) z[j] = z[j] * (float)signs[j];
        /* index_select(z, -1, inv_perm) */
        for (int64_t i = 0; i < d; ++i) out[r * d + i] = z[inv_perm[i]];
    }
    free(z);
}

/* ---- bitstream --------------------------------------------------------------------------- */

int64_t or_packed_bytes(int64_t numel, int bits) { return (numel + 7) / 8 * bits; }

/* pack_codes: code k contributes its bits MSB first at stream positions bits*k ...; stream
 * position p is bit (7 - p % 8) of byte p / 8; the tail is zero padded to 8 codes. */
void or_pack_codes(const uint8_t *codes, int64_t numel, int bits, uint8_t *out) {
    const int64_t nbytes = or_packed_bytes(numel, bits);
    memset(out, 0, (size_t)nbytes);
    for (int64_t k = 0; k < numel; ++k) {
        for (int b = 0; b < bits; ++b) {
            int bit = (codes[k] >> (bits - 1 - b)) & 1;
            int64_t p = k * bits + b;
            if (bit) out[p / 8] |= (uint8_t)(1u << (7 - p % 8));
        }
    }
}

void or_unpack_codes(const uint8_t *packed, int64_t numel, int bits, uint8_t *codes) {
    for (int64_t k = 0; k < numel; ++k) {
        int v = 0;
        for (int b = 0; b < bits; ++b) {
            int64_t p = k * bits + b;
            v = (v << 1) | ((packed[p / 8] >> (7 - p % 8)) & 1);
        }
        codes[k] = (uint8_t)v;
    }
}

/* ---- _quantize_rows ---------------------------------------------------------------------- */

void or_rpbh_quantize(const void *w, int w_is_bf16, int64_t rows, int64_t d,
                      const int32_t *perm, const int8_t *signs, int64_t h,
                      const float *codebook, int bits, uint8_t *packed, float *row_norms,
                      uint8_t *codes_out, float *unit_out) {
    const int L = 1 << bits;
    float edges[15];
    /* edges = (codebook[:-1] + codebook[1:]) / 2 in fp32 */
    for (int k = 0; k + 1 < L; ++k) edges[k] = (codebook[k] + codebook[k + 1]) / 2.0f;

    float *xr = (float *)malloc(sizeof(float) * (size_t)d);
    float *yr = (float *)malloc(sizeof(float) * (size_t)d);
    uint8_t *codes = (uint8_t *)malloc((size_t)(rows * d > 0 ? rows * d : 1));
    for (int64_t r = 0; r < rows; ++r) {
        /* weight_fp32 (bf16 widening is exact) */
        for (int64_t j = 0; j < d; ++j)
            xr[j] = w_is_bf16 ? or_bf16_to_f32(((const uint16_t *)w)[r * d + j])
                              : ((const float *)w)[r * d + j];
        or_rpbh_forward(xr, 1, d, perm, signs, h, yr);
        /* row_norms = w_rot.norm(dim=1): order not given; double, index order, one rounding */
        double ss = 0.0;
        for (int64_t j = 0; j < d; ++j) ss += (double)yr[j] * (double)yr[j];
        const float rho = (float)sqrt(ss);
        row_norms[r] = rho;
        /* unit = w_rot / (row_norms + 1e-10) */
        const float den = rho + 1e-10f;
        for (int64_t j = 0; j < d; ++j) {
            const float u = yr[j] / den;
            /* bucketize(unit, edges), right=False: the number of edges strictly below u */
            uint8_t c = 0;
            for (int k = 0; k + 1 < L; ++k)
                if (edges[k] < u) ++c;
            codes[r * d + j] = c;
            if (unit_out) unit_out[r * d + j] = u;
        }
    }
    or_pack_codes(codes, rows * d, bits, packed);
    if (codes_out) memcpy(codes_out, codes, (size_t)(rows * d));
    free(codes);
    free(xr);
    free(yr);
}

/* ---- _dequantize_rotated / dequantize ---------------------------------------------------- */

void or_rpbh_dequantize_rotated(const uint8_t *packed, const float *row_norms, int64_t rows,
                                int64_t d, int bits, const float *codebook, void *out,
                                int out_is_bf16) {
    uint8_t *codes = (uint8_t *)malloc((size_t)(rows * d > 0 ? rows * d : 1));
    or_unpack_codes(packed, rows * d, bits, codes);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < d; ++j) {
            const uint8_t c = codes[r * d + j];
            if (out_is_bf16) {
                /* codebook.to(bf16)[codes] * row_norms.to(bf16): a bf16 product, one rounding */
                const float cb = or_bf16_to_f32(or_f32_to_bf16(codebook[c]));
                const float rb = or_bf16_to_f32(or_f32_to_bf16(row_norms[r]));
                ((uint16_t *)out)[r * d + j] = or_f32_to_bf16(cb * rb);
            } else {
                ((float *)out)[r * d + j] = codebook[c] * row_norms[r];
            }
        }
    }
    free(codes);
}

void or_rpbh_dequantize(const uint8_t *packed, const float *row_norms, int64_t rows, int64_t d,
                        int bits, const float *codebook, const int32_t *inv_perm,
                        const int8_t *signs, int64_t h, float *out) {
    float *w = (float *)malloc(sizeof(float) * (size_t)(rows * d > 0 ? rows * d : 1));
    or_rpbh_dequantize_rotated(packed, row_norms, rows, d, bits, codebook, w, 0);
    or_rpbh_inverse(w, rows, d, inv_perm, signs, h, out);
    free(w);
}

void or_rpbh_rotate_bf16(const uint16_t *x_bits, int64_t rows, int64_t d, const int32_t *perm,
                         const int8_t *signs, int64_t h, uint16_t *out_bits) {
    float *xr = (float *)malloc(sizeof(float) * (size_t)d);
    float *yr = (float *)malloc(sizeof(float) * (size_t)d);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < d; ++j) xr[j] = or_bf16_to_f32(x_bits[r * d + j]);
        or_rpbh_forward(xr, 1, d, perm, signs, h, yr);
        for (int64_t j = 0; j < d; ++j) out_bits[r * d + j] = or_f32_to_bf16(yr[j]);
    }
    free(xr);
    free(yr);
}
