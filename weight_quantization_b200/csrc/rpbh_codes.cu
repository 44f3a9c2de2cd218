// pack_codes / unpack_codes on sm_100a for any number of codes: page "orbit_quant.py" (pack_codes,
// unpack_codes).
//
// The stream is MSB-first: code k occupies stream bits bits*k .. bits*k + bits - 1, the first of
// them the code's most significant bit, and stream bit p is bit 7 - p % 8 of byte p / 8. Eight
// codes make exactly `bits` bytes, so the stream splits into independent groups of eight codes
// whatever `bits` is; a group is one thread's work: the eight codes (the tail group zero padded, as
// the page pads) are shifted into one 64-bit word, whose top 8 * bits bits are the group's bytes.
// Codes of a row whose first code does not start on a byte boundary (rows * d not a multiple of 8
// in a flattened stream) need nothing special: only the group index matters.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "wq.h"

namespace wq {
namespace rpbh_codes {

constexpr int kThreads = 256;

// codes8 = 1 when `codes` is 8-byte aligned, so a full group loads as one 8-byte access.
__global__ void __launch_bounds__(kThreads)
    pack_kernel(const uint8_t *__restrict__ codes, int64_t numel, int bits, int codes8, uint8_t *__restrict__ packed) {
    const int64_t groups = (numel + 7) >> 3;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k0 = g << 3;
        uint64_t c8 = 0;  // code k0 + i in byte i
        if (codes8 && k0 + 8 <= numel) {
            c8 = *reinterpret_cast<const uint64_t *>(codes + k0);
        } else {
            for (int i = 0; i < 8 && k0 + i < numel; ++i) c8 |= (uint64_t)codes[k0 + i] << (8 * i);
        }
        uint64_t acc = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = (acc << bits) | ((uint32_t)(c8 >> (8 * i)) & mask);
        uint8_t *dst = packed + g * bits;
        for (int b = 0; b < bits; ++b) dst[b] = (uint8_t)(acc >> (8 * (bits - 1 - b)));
    }
}

__global__ void __launch_bounds__(kThreads)
    unpack_kernel(const uint8_t *__restrict__ packed, int64_t numel, int bits, int codes8, uint8_t *__restrict__ codes) {
    const int64_t groups = (numel + 7) >> 3;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        const uint8_t *src = packed + g * bits;
        uint64_t acc = 0;
        for (int b = 0; b < bits; ++b) acc = (acc << 8) | src[b];
        uint64_t c8 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) c8 |= (uint64_t)((uint32_t)(acc >> (bits * (7 - i))) & mask) << (8 * i);
        const int64_t k0 = g << 3;
        if (codes8 && k0 + 8 <= numel) {
            *reinterpret_cast<uint64_t *>(codes + k0) = c8;
        } else {
            for (int i = 0; i < 8 && k0 + i < numel; ++i) codes[k0 + i] = (uint8_t)(c8 >> (8 * i));
        }
    }
}

unsigned grid_for(int64_t numel) {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
    }
    const int64_t blocks = (((numel + 7) >> 3) + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sms * 8;
    return (unsigned)(blocks < cap ? blocks : cap);
}

}  // namespace rpbh_codes
}  // namespace wq

using namespace wq;

namespace {
wq_status check_codes_args(const void *a, const void *b, int64_t numel, int bits) {
    if (numel < 0 || numel > ((int64_t)1 << 46)) return WQ_ERR_SHAPE;
    if (bits < 1 || bits > 8) return WQ_ERR_BITS;
    if (numel == 0) return WQ_OK;
    if (!a || !b) return WQ_ERR_NULL;
    return WQ_OK;
}
}  // namespace

extern "C" wq_status rpbh_pack_codes(const uint8_t *codes, int64_t numel, int bits, uint8_t *packed, void *stream) {
    const wq_status st = check_codes_args(codes, packed, numel, bits);
    if (st != WQ_OK || numel == 0) return st;
    rpbh_codes::pack_kernel<<<rpbh_codes::grid_for(numel), rpbh_codes::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        codes, numel, bits, (int)aligned(codes, 8), packed);
    return launch_status();
}

extern "C" wq_status rpbh_unpack_codes(const uint8_t *packed, int64_t numel, int bits, uint8_t *codes, void *stream) {
    const wq_status st = check_codes_args(packed, codes, numel, bits);
    if (st != WQ_OK || numel == 0) return st;
    rpbh_codes::unpack_kernel<<<rpbh_codes::grid_for(numel), rpbh_codes::kThreads, 0,
                                static_cast<cudaStream_t>(stream)>>>(packed, numel, bits, (int)aligned(codes, 8), codes);
    return launch_status();
}
