/*
 * Oracle: TQ3 codec (page "tq3_core.py", ComfyUI-TurboQuant). TEST INFRASTRUCTURE ONLY.
 *
 * Every function follows the page's steps in order, one fp32 IEEE operation at a time.
 */
#include <math.h>
#include <string.h>
#include "wq_oracle.h"

/* TQ3_CENTROIDS and TQ3_BOUNDARIES as printed on the page (decimal literals rounded to fp32,
 * which is what torch.tensor(..., dtype=float32) does). */
static const float k_centroids[8] = {-0.9816f, -0.6168f, -0.3479f, -0.1129f,
                                     0.1129f, 0.3479f, 0.6168f, 0.9816f};
static const float k_boundaries[7] = {-0.7992f, -0.4824f, -0.2304f, 0.0f,
                                      0.2304f, 0.4824f, 0.7992f};

void or_tq3_tables(float *centroids, float *boundaries) {
    memcpy(centroids, k_centroids, sizeof k_centroids);
    memcpy(boundaries, k_boundaries, sizeof k_boundaries);
}

float or_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint16_t or_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
    /* round to nearest, ties to even, on the 16 discarded bits */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* _fwht_inplace / _fwht: butterflies on (i, i + h) inside 2h-blocks, h ascending, then scale. */
void or_fwht(float *v, int64_t n, float post) {
    for (int64_t h = 1; h < n; h *= 2) {
        for (int64_t blk = 0; blk < n; blk += 2 * h) {
            for (int64_t i = blk; i < blk + h; ++i) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
    for (int64_t i = 0; i < n; ++i) v[i] = v[i] * post;
}

/* x.mul_(1.0 / math.sqrt(n)): the Python double scalar is applied to an fp32 tensor as fp32. */
float or_tq3_fwht_post(int64_t n) { return (float)(1.0 / sqrt((double)n)); }

/* searchsorted(TQ3_BOUNDARIES, xs), right=False: the number of boundaries strictly below xs. */
uint8_t or_tq3_bucketize(float xs) {
    uint8_t idx = 0;
    for (int j = 0; j < 7; ++j)
        if (k_boundaries[j] < xs) ++idx;
    return idx;
}

/* _pack_3bit: 16 groups of 8 indices; index i of a group goes to bits 3i..3i+2 of a 24-bit
 * word, written as 3 little-endian bytes. */
void or_tq3_pack(const uint8_t *idx, int64_t n_vec, uint8_t *packed) {
    for (int64_t v = 0; v < n_vec; ++v) {
        const uint8_t *in = idx + v * 128;
        uint8_t *out = packed + v * 48;
        for (int g = 0; g < 16; ++g) {
            uint32_t bits = 0;
            for (int i = 0; i < 8; ++i) bits |= (uint32_t)in[g * 8 + i] << (i * 3);
            out[g * 3 + 0] = (uint8_t)(bits & 0xffu);
            out[g * 3 + 1] = (uint8_t)((bits >> 8) & 0xffu);
            out[g * 3 + 2] = (uint8_t)((bits >> 16) & 0xffu);
        }
    }
}

/* _unpack_3bit: inverse of the above. */
void or_tq3_unpack(const uint8_t *packed, int64_t n_vec, uint8_t *idx) {
    for (int64_t v = 0; v < n_vec; ++v) {
        const uint8_t *in = packed + v * 48;
        uint8_t *out = idx + v * 128;
        for (int g = 0; g < 16; ++g) {
            uint32_t bits = (uint32_t)in[g * 3] | ((uint32_t)in[g * 3 + 1] << 8) |
                            ((uint32_t)in[g * 3 + 2] << 16);
            for (int i = 0; i < 8; ++i) out[g * 8 + i] = (uint8_t)((bits >> (i * 3)) & 7u);
        }
    }
}

/* Steps 1-5 of tq3_quantize for one vector: fills xs[128], idx[128], *norm, *scale. */
static void encode_one(const float *x, const float *signs, float *xs, uint8_t *idx, float *norm,
                       float *scale) {
    float y[128];
    /* Step 1: torch.norm(xb, dim=-1).clamp(min=1e-8); the reduction order is not given by the
     * page: sum of squares in double, in index order, then sqrt, then one rounding to fp32. */
    double ss = 0.0;
    for (int i = 0; i < 128; ++i) ss += (double)x[i] * (double)x[i];
    float n = (float)sqrt(ss);
    if (n < 1e-8f) n = 1e-8f;
    /* xn = xb / norms */
    for (int i = 0; i < 128; ++i) y[i] = x[i] / n;
    /* Steps 2+3: signs first, then the normalised FWHT. */
    for (int i = 0; i < 128; ++i) y[i] = y[i] * signs[i];
    or_fwht(y, 128, or_tq3_fwht_post(128));
    /* Step 4: absmax scale, clamp(min=1e-8), xs = xh / scales. */
    float s = 0.0f;
    for (int i = 0; i < 128; ++i) {
        float a = fabsf(y[i]);
        if (a > s) s = a;
    }
    if (s < 1e-8f) s = 1e-8f;
    for (int i = 0; i < 128; ++i) xs[i] = y[i] / s;
    /* Step 5: indices against TQ3_BOUNDARIES. */
    for (int i = 0; i < 128; ++i) idx[i] = or_tq3_bucketize(xs[i]);
    *norm = n;
    *scale = s;
}

static void load_vec(const void *x, int x_is_bf16, int64_t v, float *out) {
    /* x.float(): bf16 -> fp32 is exact. */
    if (x_is_bf16) {
        const uint16_t *b = (const uint16_t *)x + v * 128;
        for (int i = 0; i < 128; ++i) out[i] = or_bf16_to_f32(b[i]);
    } else {
        memcpy(out, (const float *)x + v * 128, 128 * sizeof(float));
    }
}

void or_tq3_encode(const void *x, int x_is_bf16, int64_t n_vec, const float *signs,
                   uint8_t *packed, float *norms, float *scales) {
    float xv[128], xs[128];
    uint8_t idx[128];
    for (int64_t v = 0; v < n_vec; ++v) {
        load_vec(x, x_is_bf16, v, xv);
        encode_one(xv, signs, xs, idx, &norms[v], &scales[v]);
        /* Step 6: pack */
        or_tq3_pack(idx, 1, packed + v * 48);
    }
}

void or_tq3_encode_debug(const void *x, int x_is_bf16, int64_t n_vec, const float *signs,
                         float *xs, uint8_t *idx, float *norms, float *scales) {
    float xv[128];
    for (int64_t v = 0; v < n_vec; ++v) {
        load_vec(x, x_is_bf16, v, xv);
        encode_one(xv, signs, xs + v * 128, idx + v * 128, &norms[v], &scales[v]);
    }
}

/* tq3_dequantize: unpack, centroids[idx], * scale, FWHT, * signs, * norm. */
void or_tq3_decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec,
                   const float *signs, void *out, int out_is_bf16) {
    uint8_t idx[128];
    float y[128];
    const float post = or_tq3_fwht_post(128);
    for (int64_t v = 0; v < n_vec; ++v) {
        or_tq3_unpack(packed + v * 48, 1, idx);
        for (int i = 0; i < 128; ++i) y[i] = k_centroids[idx[i]];
        for (int i = 0; i < 128; ++i) y[i] = y[i] * scales[v];
        or_fwht(y, 128, post);
        for (int i = 0; i < 128; ++i) y[i] = y[i] * signs[i];
        for (int i = 0; i < 128; ++i) y[i] = y[i] * norms[v];
        if (out_is_bf16) {
            uint16_t *o = (uint16_t *)out + v * 128;
            for (int i = 0; i < 128; ++i) o[i] = or_f32_to_bf16(y[i]);
        } else {
            memcpy((float *)out + v * 128, y, sizeof y);
        }
    }
}

/* tq3_memory_bytes: 56 bytes per 128-block, fp16 original. */
int64_t or_tq3_memory_bytes(const int64_t *shape, int ndim, int64_t *original_bytes) {
    if (ndim <= 0) return -1;
    if (shape[ndim - 1] <= 0 || shape[ndim - 1] % 128 != 0) return -1;
    int64_t total = 1;
    for (int i = 0; i < ndim; ++i) {
        if (shape[i] <= 0) return -1;
        total *= shape[i];
    }
    int64_t D = shape[ndim - 1];
    int64_t num_blocks = D / 128;
    int64_t num_vectors = total / D;
    *original_bytes = total * 2;
    return num_vectors * num_blocks * 56;
}

void or_hadamard_dense(int64_t n, int8_t *H) {
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < n; ++j) {
            uint64_t m = (uint64_t)(i & j);
            int pc = 0;
            while (m) {
                pc += (int)(m & 1u);
                m >>= 1;
            }
            H[i * n + j] = (int8_t)((pc & 1) ? -1 : 1);
        }
}

int or_nearest_centroid(float v, const float *c, int L) {
    int best = 0;
    double bd = fabs((double)v - (double)c[0]);
    for (int k = 1; k < L; ++k) {
        double dk = fabs((double)v - (double)c[k]);
        if (dk < bd) {
            bd = dk;
            best = k;
        }
    }
    return best;
}
