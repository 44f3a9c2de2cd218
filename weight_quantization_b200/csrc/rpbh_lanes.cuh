// Warp-lane RPBH kernels for bf16 rows with a Hadamard block of 256 or 1024 (see rpbh_lanes.cu).
// Internal interface between the dispatchers in rpbh_fast.cu and these kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rpbh_edges.cuh"
#include "wq.h"

namespace wq {
namespace rpbh_lanes {

// True when the kernels take rows of length d (bf16): h = d & -d is 256 or 1024, d <= 16384 and
// the layout fits the device's shared memory.
bool rotate_fits(int64_t d);
bool quantize_fits(int64_t d, const rpbh_fast::Edges &E);

wq_status rotate(const uint16_t *x, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, uint16_t *out,
                 cudaStream_t s);
wq_status quantize(const uint16_t *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, int bits,
                   const rpbh_fast::Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s);

// Reads and clears the fault bits of these kernels (bit 1: a bounded wait for a row copy ran out).
unsigned int read_and_clear_fault();

}  // namespace rpbh_lanes
}  // namespace wq
