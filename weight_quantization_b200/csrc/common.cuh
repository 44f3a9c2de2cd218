// Shared device/host helpers of libwq_b200 (no codec arithmetic lives here).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "wq.h"

namespace wq {

// Raw bf16 <-> fp32. Widening is exact (bf16 is the top half of an fp32).
__device__ __forceinline__ float bf16_lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t pair) { return __uint_as_float(pair & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Round-to-nearest-even narrowing of two fp32 values into one bf16x2 word (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    return (uint16_t)(pack_bf16x2(f, 0.0f) & 0xffffu);
}

// Streaming 16-byte global accesses: inputs are read once, outputs written once.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream16(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline wq_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

inline bool valid_dtype(int t) { return t == WQ_F32 || t == WQ_BF16; }
inline int dtype_size(int t) { return t == WQ_F32 ? 4 : 2; }

}  // namespace wq
