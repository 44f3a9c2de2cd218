// One-thread-per-vector TQ3 kernels (see tq3_rows.cu). Internal interface between the C ABI in
// tq3.cu and these kernels; not part of the exported library surface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tq3_common.cuh"
#include "wq.h"

namespace wq {
namespace tq3_rows {

// tq3_quantize with the decisions taken on |fwht(D x)| against per-vector thresholds (see
// tq3_rows.cu for what this changes against the page's step-by-step rounding).
wq_status encode(const void *x, int x_dtype, int64_t n_vec, const tq3::SignMask &m, uint8_t *packed, float *norms,
                 float *scales, cudaStream_t s, int layout = tq3::kSoA, const tq3::PoolMap &pool = {});

// tq3_dequantize, rounding as the page does (bit-identical to the step-by-step definition).
wq_status decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec,
                 const tq3::SignMask &m, void *out, int out_dtype, cudaStream_t s, int layout = tq3::kSoA,
                 const tq3::PoolMap &pool = {});
// (layout is a tq3::Layout: for kAoS and kPool `packed` holds 56-byte records and norms and scales
// are unused; for kPool it is the whole pool, placed through `pool`)

// Reads and clears the fault bits of these kernels (bit 0: a bounded wait for a TMA tile ran out;
// bit 6: a slot or page-table entry outside the pool).
unsigned int read_and_clear_fault();

}  // namespace tq3_rows
}  // namespace wq
