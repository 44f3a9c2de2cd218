/*
 * wq.h -- C ABI of libwq_b200.so: the TQ3 KV-cache codec and the OrbitQuant RPBH weight path
 * on NVIDIA B200 (sm_100a).
 *
 * Sources. Every entry point restates an operation of one of two pages:
 *   "tq3_core.py" (ComfyUI-TurboQuant): module docstring (format and algorithm), tq3_quantize,
 *       tq3_dequantize, _fwht_inplace, _quantize_to_indices, _pack_3bit, _unpack_3bit,
 *       tq3_memory_bytes, and the page's commit note (the attention layer that reads the cache).
 *   "orbit_quant.py" (OrbitQuant weight-only backend): gaussian_lloyd_max, hadamard_block_size,
 *       rpbh_forward, rpbh_inverse, _fwht, pack_codes, unpack_codes, _quantize_rows,
 *       OrbitQuantizer.quantize_, _dequantize_rotated, dequantize, forward.
 *
 * Conventions shared by every call:
 *   - Pointers named "device" are CUDA device memory owned by the caller. Pointers named "host"
 *     are ordinary host memory read during the call (their contents are copied into the launch,
 *     so the caller may reuse them as soon as the call returns).
 *   - The library allocates no memory and never synchronises. Device work is enqueued on
 *     `stream` (a cudaStream_t; NULL means the legacy default stream) and runs asynchronously.
 *   - Arguments are validated before anything is enqueued; a call that returns an error has
 *     enqueued nothing. Data VALUES are not validated (NaN/Inf give unspecified output).
 *   - An empty problem (n_vec == 0, rows == 0) returns WQ_OK and enqueues nothing; its pointers
 *     may then be NULL.
 *   - Element types: WQ_F32 = IEEE binary32, WQ_BF16 = bfloat16 (raw 16-bit patterns).
 *   - Unless an entry point states otherwise (tq3_encode, rpbh_linear, tq3_attention reorder the
 *     arithmetic and say how), all arithmetic is fp32 in the order the pages give, except the two
 *     L2 norms, whose squares are summed in fp64 and rounded once to fp32 after the square root.
 */
#ifndef WQ_H
#define WQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WQ_OK = 0,
    WQ_ERR_NULL = -1,             /* a required pointer is NULL                                */
    WQ_ERR_SHAPE = -2,            /* negative count, bad dimension, or d beyond the maximum     */
    WQ_ERR_DTYPE = -3,            /* dtype code not one of wq_dtype                            */
    WQ_ERR_ALIGN = -4,            /* a pointer is not aligned as its call requires             */
    WQ_ERR_BITS = -5,             /* bits not in {2, 3, 4}                                      */
    WQ_ERR_NOT_QUANTIZABLE = -6,  /* d & -d < 32: the page skips such layers                    */
    WQ_ERR_CUDA = -7              /* the CUDA runtime reported an error at launch               */
} wq_status;

typedef enum { WQ_F32 = 0, WQ_BF16 = 1 } wq_dtype;

/* Largest power-of-two block the RPBH rotation uses, and the page's floor for it
 * ("orbit_quant.py", MIN_HADAMARD_BLOCK). */
#define WQ_RPBH_MIN_BLOCK 32
/* Largest RPBH input dimension d the kernels accept (one weight row is held on chip). */
#define WQ_RPBH_MAX_D 32768

/* ============================================================================================
 * TQ3 ("tq3_core.py")
 * A TQ3 record encodes one 128-element vector as 48 bytes of 3-bit indices plus an fp32 norm
 * and an fp32 scale (56 bytes, 3.5 bits per value; module docstring). tq3_encode / tq3_decode
 * store records as three arrays: packed[n_vec][48], norms[n_vec], scales[n_vec] (the dict
 * tq3_quantize returns); the _aos, pool and attention calls use one 56-byte record per vector.
 * A [..., D] tensor with D a multiple of 128 is n_vec = numel / 128 consecutive vectors.
 * ============================================================================================ */

/* tq3_encode -- tq3_quantize. For each vector: n = max(||x||_2, 1e-8); y = (x / n) * s with s
 * the sign flips; y = FWHT_128(y) * fp32(1/sqrt(128)) (7 butterfly stages, h = 1..64);
 * scale = max(max|y|, 1e-8); idx_i = #{j : B_j < y_i / scale} against TQ3_BOUNDARIES;
 * indices packed 8 per 24-bit little-endian group (_pack_3bit).
 * Precision: the kernel takes each decision y_i / scale > B_j as |fwht(s x)_i| > B_j * T on the
 * unnormalised transform (T = max|fwht(s x)|, or the value the 1e-8 scale floor implies), which
 * is the same comparison in exact arithmetic. An index can therefore differ from the page's
 * step-by-step fp32 rounding only where y_i / scale lies within about 1e-6 of a boundary (exact
 * ties included); norms (fp32 sum of squares) and scales agree to within 1e-6 relative. Use
 * tq3_encode_exact for output that reproduces the page's rounding bit for bit.
 *   x          device, n_vec x 128 elements of x_dtype, 16-byte aligned.
 *   sign_mask  host, 4 words: bit i of the 128-bit little-endian mask is sign draw i
 *              (1 -> +1, 0 -> -1), i.e. _generate_sign_flips(128, seed).
 *   packed     device, n_vec x 48 bytes, 16-byte aligned.  norms, scales  device, n_vec fp32.
 * Errors: WQ_ERR_NULL, WQ_ERR_SHAPE (n_vec < 0), WQ_ERR_DTYPE, WQ_ERR_ALIGN, WQ_ERR_CUDA. */
wq_status tq3_encode(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                     uint8_t *packed, float *norms, float *scales, void *stream);

/* tq3_encode_exact -- tq3_quantize with the page's rounding reproduced step by step: the norm
 * rounded once from an fp64 sum of squares, x / n and y / scale as correctly rounded fp32
 * quotients, the butterflies and post-multiplier as single fp32 operations, and the
 * searchsorted tie rule (a value equal to a boundary takes the lower index). Packed bytes, norms
 * and scales equal those of that definition bit for bit. Same arguments and errors as tq3_encode;
 * slower (about twice the instructions per element). */
wq_status tq3_encode_exact(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                           uint8_t *packed, float *norms, float *scales, void *stream);

/* tq3_decode -- tq3_dequantize. For each record: y_i = TQ3_CENTROIDS[idx_i] * scale;
 * y = FWHT_128(y) * fp32(1/sqrt(128)); out_i = (y_i * s_i) * norm. With out_dtype = WQ_BF16
 * the fp32 result is rounded once to nearest-even bf16.
 *   packed device, n_vec x 48 bytes, 16-byte aligned.  norms, scales  device, n_vec fp32.
 *   sign_mask host, as for tq3_encode.  out  device, n_vec x 128 of out_dtype, 16-byte aligned.
 * Errors: as tq3_encode. */
wq_status tq3_decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec,
                     const uint32_t *sign_mask, void *out, int out_dtype, void *stream);

/* tq3_encode_aos / tq3_decode_aos -- tq3_encode and tq3_decode on 56-byte records (the "56 bytes
 * per vector" of tq3_memory_bytes as one array of structures): record v is the 48 packed bytes,
 * then the norm, then the scale (fp32, little-endian), at byte 56 v. Same arithmetic, precision and
 * errors as the three-array forms.
 *   records    device, n_vec x 56 bytes, 8-byte aligned.
 *   x, out     device, n_vec x 128 elements, 16-byte aligned. */
wq_status tq3_encode_aos(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                         uint8_t *records, void *stream);
wq_status tq3_decode_aos(const uint8_t *records, int64_t n_vec, const uint32_t *sign_mask, void *out,
                         int out_dtype, void *stream);

/* tq3_encode_slots / tq3_decode_paged -- the same codec on a KV cache kept as a pool of 56-byte
 * records (the record of tq3_encode_aos) that is written and read through indirection, as a paged
 * cache is: appended vectors are scattered to free slots, and a sequence is read back through its
 * page table. No counterpart on the page beyond the record itself; the arithmetic is that of
 * tq3_encode_aos / tq3_decode_aos, record by record.
 * tq3_encode_slots: vector v of x goes to record slots[v] of the pool.
 *   slots      device, n_vec x int64, 8-byte aligned. A negative slot skips the vector (padding);
 *              a slot >= n_pool is skipped and sets device fault bit 6. Two vectors with the same
 *              slot race (one of them is stored).
 *   pool       device, n_pool x 56 bytes, 8-byte aligned; records not named by a slot are untouched.
 * tq3_decode_paged: out[p] = decode(record page_table[p / page_size] * page_size + p % page_size)
 * for p = 0 .. n_vec-1.
 *   page_table device, n_pages x int32, 4-byte aligned; n_vec <= n_pages * page_size (else
 *              WQ_ERR_SHAPE). A negative entry, or one whose record lies at or beyond n_pool,
 *              decodes as zeros and sets device fault bit 6.
 *   page_size  a power of two, 1 .. 2^30 (else WQ_ERR_SHAPE).
 *   out        device, n_vec x 128 elements of out_dtype, 16-byte aligned. */
wq_status tq3_encode_slots(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                           const int64_t *slots, uint8_t *pool, int64_t n_pool, void *stream);
wq_status tq3_decode_paged(const uint8_t *pool, int64_t n_pool, const int32_t *page_table, int64_t n_pages,
                           int64_t page_size, int64_t n_vec, const uint32_t *sign_mask, void *out,
                           int out_dtype, void *stream);

/* tq3_attention -- scaled dot-product attention over a TQ3-compressed K/V cache (page "tq3_core.py":
 * the cache is what tq3_quantize compresses and tq3_dequantize restores; the page's commit note
 * names the attention layer that reads it). For every head h and query row r:
 *   out[h][r] = sum_j p_j v_j / sum_j p_j,  p_j = exp(softmax_scale * q[h][r] . k_j - max),
 * where k_j, v_j (j = 0 .. S-1) are tq3_dequantize of the records k_records[h][j], v_records[h][j].
 * No mask: every row attends to all S keys of its head.
 *   q          device, heads x m x 128 elements of q_dtype. The m rows of a head share its keys and
 *              values (grouped-query attention: m = query heads per KV head x query tokens).
 *   m          1 .. 2^20 (rows are served 16 at a time; each group of 16 reads the records again).
 *   k_records, v_records  device, heads x S x 56 bytes (the tq3_encode_aos record), 8-byte aligned.
 *   S          1 .. 2^31 keys per head.
 *   softmax_scale  finite; 1/sqrt(128) is the usual value. (Any finite fp32 scale keeps the
 *              kernel's coefficient scale * 2^-3.5 * log2(e) finite, as that factor is below 1.)
 *              The logits softmax_scale * q . k_j themselves must be finite in fp32: a logit that
 *              overflows makes the head's output undefined, as NaN or Inf inputs do.
 *   out        device, heads x m x 128 elements of out_dtype (bf16: rounded once, to nearest even).
 * Precision: the keys and values are never decoded; the query is rotated once into the basis the
 * indices live in and the output rotated back once, in fp32. Below 48 rows per head the products run
 * on the CUDA cores in fp32 and the result differs from attention over the decoded fp32 vectors by
 * fp32 rounding only. From 48 rows on they run on the tensor cores (tcgen05, 128 rows per CTA) on
 * bf16 operands, each fp32 operand split into hi + lo and three passes accumulated in fp32: a logit
 * is then within about 2^-14 softmax_scale |q| |k| of its fp32 value and a value sum within
 * (3 * 2^-18 + (432 + S / 128) 2^-24) max|v| per element.
 * Errors: WQ_ERR_SHAPE (heads < 0, m or S out of range, softmax_scale not finite), WQ_ERR_DTYPE,
 * WQ_ERR_NULL, WQ_ERR_ALIGN (q and out to their element size). heads == 0 enqueues nothing. */
wq_status tq3_attention(const void *q, int q_dtype, int64_t heads, int64_t m, const uint8_t *k_records,
                        const uint8_t *v_records, int64_t S, const uint32_t *sign_mask, float softmax_scale,
                        void *out, int out_dtype, void *stream);

/* tq3_attention_paged -- tq3_attention with the keys and values read from a paged cache: pools of
 * 56-byte records (as tq3_encode_slots writes them) shared by all heads, and a page table. Key j of
 * head h is record page_table[h * pages_per_head + j / page_size] * page_size + j % page_size of
 * k_pool and of v_pool (a K page and its V page share the entry).
 *   k_pool, v_pool  device, n_pool x 56 bytes each, 8-byte aligned.
 *   page_table device, heads x pages_per_head int32, 4-byte aligned; S <= pages_per_head * page_size.
 *   page_size  a power of two, 1 .. 2^30.
 * A page-table entry that is negative or names records at or beyond n_pool masks those keys out
 * (weight 0) and sets device fault bit 6; a head whose keys are all masked gives NaN rows.
 * Other arguments, precision and errors: as tq3_attention. */
wq_status tq3_attention_paged(const void *q, int q_dtype, int64_t heads, int64_t m, const uint8_t *k_pool,
                              const uint8_t *v_pool, int64_t n_pool, const int32_t *page_table,
                              int64_t pages_per_head, int64_t page_size, int64_t S, const uint32_t *sign_mask,
                              float softmax_scale, void *out, int out_dtype, void *stream);

/* tq3_compressed_bytes -- tq3_memory_bytes' compressed size for n_vec vectors: 56 * n_vec
 * (-1 if n_vec < 0 or the product overflows). */
int64_t tq3_compressed_bytes(int64_t n_vec);

/* ============================================================================================
 * RPBH ("orbit_quant.py")
 * A weight W[rows][d] (out x in, row-major) is rotated row by row with the shared randomized
 * permuted block-Hadamard R = blkdiag(H_h) D P, h = d & -d (hadamard_block_size):
 * (R w)_j = FWHT_h-block( w[perm[j]] * signs[j] ) * fp32(h ** -0.5).
 * perm is a permutation of 0..d-1 (int32, device) and signs are +-1 (int8, device), i.e.
 * rpbh_params(d). Entries of perm outside 0..d-1 are not rejected; they are clamped so that no
 * access leaves the row, and the output is then unspecified.
 * Packed codes form one flat MSB-first bitstream over the row-major [rows][d] codes, zero padded
 * to a multiple of 8 codes (pack_codes): rpbh_packed_bytes(rows, d, bits) bytes.
 * ============================================================================================ */

/* rpbh_quantize_weight -- _quantize_rows. For each row: w_rot = R w (fp32);
 * rho = ||w_rot||_2; u_j = w_rot_j / (rho + 1e-10); code_j = #{k : e_k < u_j} with
 * e_k = (c_k + c_{k+1}) / 2 over the scaled codebook; codes packed MSB-first; row_norms[r] = rho
 * stored in w_dtype (OrbitQuantizer.quantize_ keeps the norms in the weight dtype).
 *   W          device, rows x d of w_dtype, 16-byte aligned.
 *   perm, signs device, d entries each.   bits  2, 3 or 4.
 *   codebook   host, 2^bits ascending fp32 centroids, already scaled (wq_rpbh_codebook).
 *   packed     device, rpbh_packed_bytes(rows, d, bits) bytes, 4-byte aligned.
 *   row_norms  device, rows entries of w_dtype.
 * Errors: WQ_ERR_NULL, WQ_ERR_SHAPE (rows < 0, d <= 0, d > WQ_RPBH_MAX_D or the row does not
 * fit on chip), WQ_ERR_NOT_QUANTIZABLE (d & -d < 32), WQ_ERR_BITS, WQ_ERR_DTYPE, WQ_ERR_ALIGN,
 * WQ_ERR_CUDA. */
wq_status rpbh_quantize_weight(const void *W, int w_dtype, int64_t rows, int64_t d,
                               const int32_t *perm, const int8_t *signs, int bits,
                               const float *codebook, uint8_t *packed, void *row_norms,
                               void *stream);

/* rpbh_requantize_weight -- OrbitQuantizer.requantize_: the new weight, cast to fp32, is quantized
 * by _quantize_rows with the module's stored perm, signs and codebook (exactly as
 * rpbh_quantize_weight), and the row norms are stored in the module's original dtype rather than
 * the new weight's: row_norms[r] = rho in norm_dtype (WQ_BF16: rounded to nearest even).
 * rpbh_quantize_weight is this call with norm_dtype = w_dtype.
 *   row_norms  device, rows entries of norm_dtype, aligned to its size.
 * Other arguments and errors: as rpbh_quantize_weight (WQ_ERR_DTYPE also for a bad norm_dtype). */
wq_status rpbh_requantize_weight(const void *W, int w_dtype, int64_t rows, int64_t d,
                                 const int32_t *perm, const int8_t *signs, int bits,
                                 const float *codebook, uint8_t *packed, void *row_norms,
                                 int norm_dtype, void *stream);

/* rpbh_pack_codes / rpbh_unpack_codes -- pack_codes and unpack_codes for any number of codes, on
 * the device. pack: the low `bits` bits of each of the numel codes go MSB-first into a flat
 * stream, code k at stream bits bits*k .. bits*k + bits - 1 (stream bit p = bit 7 - p % 8 of byte
 * p / 8), zero padded to a multiple of 8 codes: ceil(numel / 8) * bits bytes. unpack: the first
 * numel codes of such a stream, one per byte. A code stream need not start a row on a byte
 * boundary (the page packs any tensor flat), so this is the form for arrays whose rows hold a
 * number of codes that is not a multiple of 8; rpbh_quantize_weight writes the same stream for
 * whole weights.
 *   codes      device, numel bytes (any alignment; 8-byte aligned is faster).
 *   packed     device, ceil(numel / 8) * bits bytes (any alignment).
 *   bits       1 .. 8.
 * Errors: WQ_ERR_SHAPE (numel < 0 or above 2^46), WQ_ERR_BITS, WQ_ERR_NULL, WQ_ERR_CUDA.
 * numel == 0 enqueues nothing. */
wq_status rpbh_pack_codes(const uint8_t *codes, int64_t numel, int bits, uint8_t *packed, void *stream);
wq_status rpbh_unpack_codes(const uint8_t *packed, int64_t numel, int bits, uint8_t *codes, void *stream);

/* rpbh_dequantize_weight -- _dequantize_rotated, and with unrotate = 1 dequantize.
 * Rotated (unrotate = 0): out[r][j] = codebook[code] * row_norm[r] in out_dtype; for WQ_BF16 the
 * page's bf16 product bf16(bf16(codebook[code]) * bf16(row_norm[r])).
 * Unrotated (unrotate = 1): the fp32 rotated weight is mapped back with rpbh_inverse,
 * z = FWHT_h-block(w') * fp32(h ** -0.5) * signs, out[r][perm[j]] = z[r][j]
 * (the same as out[r][i] = z[r][inv_perm[i]]); WQ_BF16 output rounds that fp32 result once.
 *   packed     device, as written by rpbh_quantize_weight, 4-byte aligned.
 *   row_norms  device, rows entries of norm_dtype.  codebook  host, 2^bits fp32.
 *   perm, signs device (read only when unrotate = 1; may be NULL otherwise).
 *   out        device, rows x d of out_dtype, 16-byte aligned.
 * Errors: as rpbh_quantize_weight. */
wq_status rpbh_dequantize_weight(const uint8_t *packed, const void *row_norms, int norm_dtype,
                                 int64_t rows, int64_t d, int bits, const float *codebook,
                                 const int32_t *perm, const int8_t *signs, int unrotate,
                                 void *out, int out_dtype, void *stream);

/* rpbh_rotate_activations -- the activation side of OrbitQuantizer.forward: x_rot = R x per row,
 * computed in fp32 and rounded once to the output dtype (the page runs the butterflies in the
 * activation dtype; one final rounding is at least as accurate).
 *   x, x_rot   device, rows x d of dtype, 16-byte aligned (x_rot may not alias x).
 *   perm, signs device, d entries each.
 * Errors: WQ_ERR_NULL, WQ_ERR_SHAPE, WQ_ERR_NOT_QUANTIZABLE, WQ_ERR_DTYPE, WQ_ERR_ALIGN,
 * WQ_ERR_CUDA. */
wq_status rpbh_rotate_activations(const void *x, int dtype, int64_t rows, int64_t d,
                                  const int32_t *perm, const int8_t *signs, void *x_rot,
                                  void *stream);

/* rpbh_linear -- the linear layer of OrbitQuantizer.forward on the rotated activations,
 * y = F.linear(x_rot, W', bias) with W' the rotated-basis dequantized weight (as
 * rpbh_dequantize_weight with unrotate = 0 and bf16 output), without writing W' out: the codes
 * are unpacked into the tensor-core operand on chip. y[i][n] = bf16(sum_k x_rot[i][k] *
 * bf16(codebook[code[n][k]]) * bf16(row_norm[n]) + bias[n]), the sum in fp32 on the tensor cores;
 * the row norm scales the sum instead of each product, so y agrees with the product of the bf16
 * W' to within 2^-8 relative per term (plus fp32 summation and the final bf16 rounding).
 *   packed     device, as written by rpbh_quantize_weight for out_features x d, 16-byte aligned.
 *   row_norms  device, out_features entries of norm_dtype.  codebook  host, 2^bits fp32.
 *   x_rot      device, m x d bf16 (rpbh_rotate_activations output), 16-byte aligned.
 *   bias       device, out_features bf16, or NULL for none.
 *   y          device, m x out_features bf16 (row-major), 2-byte aligned.
 * d must be a multiple of 64. Errors: WQ_ERR_NULL, WQ_ERR_SHAPE (negative sizes, d not a
 * multiple of 64 or above 2^20), WQ_ERR_BITS, WQ_ERR_DTYPE, WQ_ERR_ALIGN, WQ_ERR_CUDA. */
wq_status rpbh_linear(const uint8_t *packed, const void *row_norms, int norm_dtype,
                      int64_t out_features, int64_t d, int bits, const float *codebook,
                      const void *x_rot, int64_t m, const void *bias, void *y, void *stream);

/* rpbh_packed_bytes -- size of the packed bitstream: ceil(rows * d / 8) * bits (-1 on a bad
 * argument). */
int64_t rpbh_packed_bytes(int64_t rows, int64_t d, int bits);

/* ============================================================================================
 * Host helpers (run on the CPU, synchronous)
 * ============================================================================================ */

/* wq_gaussian_lloyd_max -- gaussian_lloyd_max: the 2^bits MSE-optimal levels for N(0,1),
 * ascending. Initialised at sqrt(2) * erfinv(2q - 1), q = (k + 0.5) / 2^bits, then `iters`
 * rounds of midpoint edges and conditional means (phi(lo) - phi(hi)) / (Phi(hi) - Phi(lo)),
 * in fp64; the result is rounded once to fp32. `out` is host memory for 2^bits floats.
 * Errors: WQ_ERR_NULL, WQ_ERR_BITS (bits outside 1..4), WQ_ERR_SHAPE (iters < 0). */
wq_status wq_gaussian_lloyd_max(int bits, int iters, float *out);

/* wq_rpbh_codebook -- the codebook OrbitQuantizer.quantize_ stores for input dimension d:
 * fp32(gaussian_lloyd_max(bits, 200)) * fp32(d ** -0.5). `out` host, 2^bits floats.
 * Errors: WQ_ERR_NULL, WQ_ERR_BITS, WQ_ERR_SHAPE (d <= 0). */
wq_status wq_rpbh_codebook(int bits, int64_t d, float *out);

/* wq_device_fault -- reads and clears the library's sticky device fault bits. A kernel whose
 * bounded wait runs out (which does not happen in normal operation) sets a bit and returns early,
 * leaving its outputs unspecified: bit 0 a TQ3 kernel waiting for a TMA tile, bit 1 an RPBH kernel
 * waiting for a row copy or the CUDA-core attention waiting for a tile's records, bit 3 the tensor-core TQ3 encoder waiting for a tile or its product,
 * bit 4 rpbh_linear waiting for a tile, the unpacked weights or its product, bit 5 the self-test
 * wq_selftest_wait_timeout, bit 7 the tensor-core attention waiting for its product. Bit 6 is not a wait: tq3_encode_slots, tq3_decode_paged or
 * tq3_attention_paged met a slot or page-table entry outside the pool (that record was skipped,
 * decoded as zeros, or masked out of the attention; the rest of the call is complete).
 * Synchronous (a device-to-host copy on the legacy default stream); `flags` is host memory.
 * Errors: WQ_ERR_NULL, WQ_ERR_CUDA. */
wq_status wq_device_fault(unsigned int *flags);

/* wq_selftest_wait_timeout -- exercises the fault path without a GPU fault (no counterpart in the
 * pages): one thread waits, with the library's bounded wait, on an mbarrier that nothing arrives
 * at; after the wait's 2 s limit it sets fault bit 5 and returns, so wq_device_fault then reports
 * 32 and the context stays usable. Enqueued on `stream`; takes about 2 s of GPU time.
 * Errors: WQ_ERR_CUDA. */
wq_status wq_selftest_wait_timeout(void *stream);

/* wq_status_string -- a static, NUL-terminated description of a status code. */
const char *wq_status_string(int status);

/* wq_version -- library version, (major << 16) | minor. */
int wq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* WQ_H */
