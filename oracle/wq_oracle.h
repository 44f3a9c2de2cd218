/*
 * Reference oracle for the TQ3 KV codec and the OrbitQuant RPBH weight path.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, single-threaded C99 restatement of what the
 * source pages compute, written to be checked by eye against them. Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it; the library under test never does, and
 * the two share no code, headers, tables or helpers.
 *
 * Sources (page title, then the part of the page each function follows):
 *   "tq3_core.py" (ComfyUI-TurboQuant)  -- module docstring (format, algorithm), TQ3_CENTROIDS,
 *       TQ3_BOUNDARIES, _generate_sign_flips, _fwht_inplace, _quantize_to_indices, _pack_3bit,
 *       _unpack_3bit, tq3_quantize, tq3_dequantize, tq3_memory_bytes.
 *   "orbit_quant.py" (OrbitQuant weight-only backend) -- gaussian_lloyd_max, hadamard_block_size,
 *       _fwht, rpbh_forward, rpbh_inverse, pack_codes, unpack_codes, _quantize_rows,
 *       OrbitQuantizer.quantize_, _dequantize_rotated, dequantize, forward.
 *
 * Precision: the pages compute in fp32 (x.float(), weight_fp32); every fp32 step here is one IEEE
 * single-precision operation in the order the page writes it. The pages leave the reduction order
 * of the two L2 norms open; here both are summed in double in index order and the double square
 * root is rounded once to fp32. The Lloyd-Max iteration runs in double as on the page.
 * Built with -ffp-contract=off and no -march, so no multiply-add is ever fused.
 *
 * Parity pins: every function is pinned by a test in tests/test_oracle_pins.py against values the
 * pages print, closed forms or brute force. None is "parity unpinned".
 */
#ifndef WQ_ORACLE_H
#define WQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar helpers ---------------------------------------------------------------------- */
float    or_bf16_to_f32(uint16_t b);            /* exact widening */
uint16_t or_f32_to_bf16(float f);               /* round to nearest even (torch .to(bfloat16)) */

/* Normalised FWHT of one block of n = 2^k floats, in place: stages h = 1, 2, ..., n/2 of
 * (a, b) -> (a + b, a - b) on positions (i, i + h) inside each 2h-block, then every element is
 * multiplied by the fp32 scalar `post` (tq3_core.py _fwht_inplace; orbit_quant.py _fwht). */
void or_fwht(float *v, int64_t n, float post);
/* The two post-multipliers the pages use: 1.0/math.sqrt(n) and h ** -0.5, each cast to fp32. */
float or_tq3_fwht_post(int64_t n);
float or_rpbh_fwht_post(int64_t h);

/* ---- TQ3 (tq3_core.py) ------------------------------------------------------------------- */
/* tq3_quantize over n_vec contiguous 128-element vectors. x is fp32 (x_is_bf16 = 0) or raw bf16
 * bits (x_is_bf16 = 1). signs[128] are the +-1.0 sign flips. Outputs: packed[n_vec][48],
 * norms[n_vec], scales[n_vec]. */
void or_tq3_encode(const void *x, int x_is_bf16, int64_t n_vec, const float *signs,
                   uint8_t *packed, float *norms, float *scales);
/* Diagnostic twin of or_tq3_encode: writes the scaled coefficients xs[n_vec][128] (the values
 * bucketized) and the indices idx[n_vec][128] instead of packing. Used to count boundary ties. */
void or_tq3_encode_debug(const void *x, int x_is_bf16, int64_t n_vec, const float *signs,
                         float *xs, uint8_t *idx, float *norms, float *scales);
/* tq3_dequantize. out is fp32 (out_is_bf16 = 0) or bf16 bits rounded once from the fp32 result. */
void or_tq3_decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec,
                   const float *signs, void *out, int out_is_bf16);
/* _quantize_to_indices against TQ3_BOUNDARIES, _pack_3bit, _unpack_3bit. */
uint8_t or_tq3_bucketize(float xs);
void or_tq3_pack(const uint8_t *idx, int64_t n_vec, uint8_t *packed);
void or_tq3_unpack(const uint8_t *packed, int64_t n_vec, uint8_t *idx);
/* tq3_memory_bytes for a shape: returns compressed bytes, writes fp16 bytes. -1 on a bad shape. */
int64_t or_tq3_memory_bytes(const int64_t *shape, int ndim, int64_t *original_bytes);
/* The printed codebook and boundaries (8 and 7 floats). */
void or_tq3_tables(float *centroids, float *boundaries);

/* ---- Lloyd-Max (orbit_quant.py gaussian_lloyd_max) --------------------------------------- */
double or_erfinv(double t);
/* 2^bits centroids, ascending, double iteration then one cast to fp32. */
void or_gaussian_lloyd_max(int bits, int iters, float *out);
/* Same iteration, left in double (for the fixed-point and textbook pins). */
void or_gaussian_lloyd_max_f64(int bits, int iters, double *out);

/* ---- RPBH (orbit_quant.py) --------------------------------------------------------------- */
int64_t or_hadamard_block_size(int64_t d);     /* d & -d */
/* Scaled codebook of OrbitQuantizer.quantize_: fp32(lloyd_max(bits)) * fp32(d ** -0.5). */
void or_rpbh_codebook(int bits, int64_t d, float *out);
/* rpbh_forward on fp32 rows: y[r][j] = x[r][perm[j]] * signs[j], then _fwht per h-block. */
void or_rpbh_forward(const float *x, int64_t rows, int64_t d, const int32_t *perm,
                     const int8_t *signs, int64_t h, float *y);
/* rpbh_inverse: z = _fwht(y) * signs, out[r][i] = z[r][inv_perm[i]]. */
void or_rpbh_inverse(const float *y, int64_t rows, int64_t d, const int32_t *inv_perm,
                     const int8_t *signs, int64_t h, float *out);
/* pack_codes / unpack_codes: flat MSB-first bitstream, zero padded to a multiple of 8 codes. */
int64_t or_packed_bytes(int64_t numel, int bits);
void or_pack_codes(const uint8_t *codes, int64_t numel, int bits, uint8_t *out);
void or_unpack_codes(const uint8_t *packed, int64_t numel, int bits, uint8_t *codes);
/* _quantize_rows on W given as fp32 (w_is_bf16 = 0) or raw bf16 bits (1). Writes the packed
 * bitstream, the fp32 row norms and (if codes != NULL) the unpacked codes and (if unit != NULL)
 * the unit directions that were bucketized. */
void or_rpbh_quantize(const void *w, int w_is_bf16, int64_t rows, int64_t d,
                      const int32_t *perm, const int8_t *signs, int64_t h,
                      const float *codebook, int bits, uint8_t *packed, float *row_norms,
                      uint8_t *codes, float *unit);
/* _dequantize_rotated: W'[r][j] = codebook[code] * row_norm[r] in fp32 (out_is_bf16 = 0), or
 * bf16(bf16(codebook[code]) * bf16(row_norm[r])) (out_is_bf16 = 1). row_norms are given as the
 * stored values already in fp32. */
void or_rpbh_dequantize_rotated(const uint8_t *packed, const float *row_norms, int64_t rows,
                                int64_t d, int bits, const float *codebook, void *out,
                                int out_is_bf16);
/* dequantize: _dequantize_rotated in fp32, then rpbh_inverse. Output fp32. */
void or_rpbh_dequantize(const uint8_t *packed, const float *row_norms, int64_t rows, int64_t d,
                        int bits, const float *codebook, const int32_t *inv_perm,
                        const int8_t *signs, int64_t h, float *out);
/* Activation rotation of OrbitQuantizer.forward on bf16 rows: rpbh_forward computed in fp32 and
 * rounded once to bf16 (x_bits, out_bits are raw bf16). */
void or_rpbh_rotate_bf16(const uint16_t *x_bits, int64_t rows, int64_t d, const int32_t *perm,
                         const int8_t *signs, int64_t h, uint16_t *out_bits);

/* ---- brute-force cross-checks (tiny n only) ---------------------------------------------- */
/* Sylvester Hadamard H[i][j] = (-1)^popcount(i & j), n x n, as int8. */
void or_hadamard_dense(int64_t n, int8_t *H);
/* Index of the nearest of L ascending centroids (lower index on an exact tie). */
int or_nearest_centroid(float v, const float *c, int L);

#ifdef __cplusplus
}
#endif
#endif
