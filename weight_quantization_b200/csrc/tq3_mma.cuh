// TQ3 encoder for bf16 input with the transform on the tensor cores (see tq3_mma.cu). Internal
// interface between the C ABI in tq3.cu and that kernel; not part of the exported library surface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tq3_common.cuh"
#include "wq.h"

namespace wq {
namespace tq3_mma {

// tq3_quantize of n_vec bf16 vectors (same contract and precision as the fast TQ3 encoder).
// layout is a tq3::Layout: for kAoS `packed` receives 56-byte records (packed bytes, norm, scale),
// for kPool record v goes to slot pool.index[v] of the pool at `packed`; norms and scales are then
// unused.
wq_status encode_bf16(const void *x, int64_t n_vec, const tq3::SignMask &m, uint8_t *packed, float *norms,
                      float *scales, cudaStream_t s, int layout = tq3::kSoA, const tq3::PoolMap &pool = {});

// Reads and clears the fault bits of this kernel (bit 3: a bounded wait for a TMA tile or for the
// tensor-core product ran out; bit 6: a slot outside the pool).
unsigned int read_and_clear_fault();

}  // namespace tq3_mma
}  // namespace wq
