// Register-blocked RPBH kernels (see rpbh_fast.cu). Internal interface between the C ABI in
// rpbh.cu and the fast kernels; not part of the exported library surface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "wq.h"

namespace wq {
namespace rpbh_fast {

// True when the fast kernels handle this (d, dtype) pair: Hadamard block h = d & -d with an even
// log2 between 6 and 12 (h = 64, 256, 1024, 4096) and a row that fits in shared memory.
bool supported(int64_t d, int in_esz, int out_esz);

wq_status rotate(const void *x, int dtype, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                 void *out, cudaStream_t s);

// Row norms are written in norm_dtype (WQ_F32 or WQ_BF16), whatever the weight's dtype.
wq_status quantize(const void *w, int w_dtype, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                   int bits, const float *codebook, uint8_t *packed, void *row_norms, int norm_dtype, cudaStream_t s);

wq_status dequantize_unrotate(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t rows, int64_t d,
                              int bits, const float *codebook, const int32_t *perm, const int8_t *signs, void *out,
                              int out_dtype, cudaStream_t s);

// _dequantize_rotated for rows whose codes (d/8 * bits bytes) are a multiple of 16 bytes and fit
// twice in shared memory: a persistent kernel that fetches each row's codes ahead by bulk copy.
bool dequantize_rotated_fits(int64_t d, int bits);
wq_status dequantize_rotated(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t rows, int64_t d,
                             int bits, const float *codebook, void *out, int out_dtype, cudaStream_t s);

// Reads and clears the fault bits of these kernels (bit 1: a bounded wait for a row copy ran out).
unsigned int read_and_clear_fault();

}  // namespace rpbh_fast
}  // namespace wq
