// Attention over a TQ3 K/V cache on the tensor cores, for many query rows per head (see
// tq3_attn_mma.cu). Internal interface between tq3_attn.cu and that kernel; not part of the exported
// library surface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tq3_common.cuh"
#include "wq.h"

namespace wq {

// Where the records of (head, key) live: contiguous [heads][S] records, or a pool reached through a
// page table of pages_per_head int32 entries per head (table == nullptr: contiguous).
struct AttnCache {
    const uint8_t *k, *v;
    const int32_t *table;
    int64_t pages_per_head, n_pool;
    int shift;  // log2 of the page size
};

namespace tq3_attn_mma {

using Cache = AttnCache;

// softmax(softmax_scale q k^T) v for all m query rows of every head, 128 rows per CTA; coef is
// post * softmax_scale * log2(e). Same contract as tq3_attention.
wq_status run(const void *q, int q_dtype, int64_t heads, int64_t m, const Cache &kv, int64_t S,
              const tq3::SignMask &mask, float coef, void *out, int out_dtype, cudaStream_t s);

// Reads and clears this kernel's fault bits (bit 7: a bounded wait for a tensor-core product ran
// out; bit 6: a page-table entry outside the pool).
unsigned int read_and_clear_fault();

}  // namespace tq3_attn_mma
}  // namespace wq
