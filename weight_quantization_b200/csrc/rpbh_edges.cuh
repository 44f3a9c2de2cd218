// Decisions and bit packing of the RPBH weight quantizer, shared by its kernels: page
// "orbit_quant.py" (_quantize_rows: bucketize against the codebook midpoints; pack_codes).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace wq {
namespace rpbh_fast {

struct Edges {
    float e[15];  // (c_k + c_{k+1}) / 2
    // for an antisymmetric codebook, the positive edges e[L/2 .. L-2] as exact steps (see
    // step_count): M[i] = 2^(24 - E) with E the binary exponent of the edge, K[i] = -edge * M[i];
    // steps = 1 when every positive edge is at least 2^-103 (so that M is a normal fp32 value)
    float M[7], K[7];
    int steps;
    int norm_bf16;  // row norms are stored as bf16 (RNE) when set, fp32 otherwise
};

// a * b + c on both lanes, rounded up / down.
__device__ __forceinline__ f32x2 fma_rp2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rp.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ f32x2 fma_rm2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 d;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The codes of two quotients u (both lanes) for an antisymmetric codebook with E.steps set, as
// fp32 values 2^23 + code (the code is the value's low byte). The same decisions as bucketize<.., true>:
// a' = |u| - u 2^-24 rounded up (|u| for u > 0, next(|u|) for u <= 0) is compared with the positive
// edges strictly, each compare an exact 0/1 step sat(a' M + K) (a' > e means a' >= e + ulp, and
// M = 2 / ulp(e)); with c the number of edges below a', the code is mid + 1/2 + sgn (c + 1/2),
// sgn the sign of u + (-0) rounded down, which is -0 for both zeros (the page gives zero the
// code below the middle edge).
template <int BITS>
__device__ __forceinline__ f32x2 sym_codes(f32x2 u, const Edges &E) {
    constexpr int L = 1 << BITS, kPos = L / 2 - 1;
    float u0, u1;
    upk2(u, u0, u1);
    const f32x2 ap = fma_rp2(u, pk2(-0x1p-24f, -0x1p-24f), pk2(fabsf(u0), fabsf(u1)));
    float a0, a1;
    upk2(ap, a0, a1);
    f32x2 c = pk2(0.5f, 0.5f);
#pragma unroll
    for (int i = 0; i < kPos; ++i)
        c = add2(c, pk2(__saturatef(__fmaf_rn(a0, E.M[i], E.K[i])), __saturatef(__fmaf_rn(a1, E.M[i], E.K[i]))));
    float b0, b1, c0, c1;
    upk2(fma_rm2(u, pk2(1.0f, 1.0f), pk2(-0.0f, -0.0f)), b0, b1);
    upk2(c, c0, c1);
    const f32x2 sc = pk2(__uint_as_float(__float_as_uint(c0) | (__float_as_uint(b0) & 0x80000000u)),
                         __uint_as_float(__float_as_uint(c1) | (__float_as_uint(b1) & 0x80000000u)));
    constexpr float kBase = 8388608.0f + (float)(L / 2 - 1);  // 2^23 + mid
    return add2(add2(sc, pk2(0.5f, 0.5f)), pk2(kBase, kBase));
}

// bucketize(u, edges, right=False): the number of edges strictly below u.
// kSym: the codebook is antisymmetric (c_k = -c_{L-1-k}), so the middle edge is 0 and the other
// edges come in +- pairs: count the positive edges below a' = |u| for u > 0, or below
// a' = next(|u|) for u < 0 (fma with upward rounding: |u| - u 2^-24 rounded up), which turns the
// "<=" a negative value needs into a strict compare. Otherwise every edge is compared directly.
template <int BITS, bool kSym>
__device__ __forceinline__ uint32_t bucketize(float u, const Edges &E) {
    constexpr int L = 1 << BITS;
    if (kSym) {
        constexpr int mid = L / 2 - 1;
        const float ap = __fmaf_ru(u, -0x1p-24f, fabsf(u));
        uint32_t c = 0;
#pragma unroll
        for (int k = mid + 1; k < L - 1; ++k) c += (uint32_t)(ap > E.e[k]);
        return u > 0.0f ? (uint32_t)(mid + 1) + c : (uint32_t)mid - c;
    } else {
        uint32_t c = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) c += (uint32_t)(u > E.e[k]);
        return c;
    }
}

// pack_codes for one group of 32 codes (code i in byte i of cw): BITS 32-bit words of the MSB-first
// stream, word k holding stream bits 32k .. 32k + 31 with the first at bit 31. Code i occupies
// stream bits BITS*i .. BITS*i + BITS - 1; one that crosses a word boundary is split between two.
template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&cw)[8], uint32_t (&word)[BITS]) {
#pragma unroll
    for (int k = 0; k < BITS; ++k) word[k] = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const uint32_t c = __byte_perm(cw[i >> 2], 0u, 0x4440u + (uint32_t)(i & 3));
        const int o = BITS * i, k = o >> 5, r = o & 31;
        if (r + BITS <= 32) {
            word[k] += c << (32 - r - BITS);
        } else {
            word[k] += c >> (r + BITS - 32);
            word[k + 1] += c << (64 - r - BITS);
        }
    }
}
// pack32 for BITS = 3 with the codes combined four at a time: byte-reversed word r = c0 c1 c2 c3;
// (r | r >> 5) & 0x003F003F holds c0 c1 at bits 16 .. 21 and c2 c3 at bits 0 .. 5, and one more
// shift and mask gives the 12-bit chunk c0 c1 c2 c3 (MSB first); eight chunks make the three words.
__device__ __forceinline__ void pack32_b3(const uint32_t (&cw)[8], uint32_t (&word)[3]) {
    uint32_t ch[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t r = __byte_perm(cw[j], 0u, 0x0123);
        const uint32_t t = (r | (r >> 5)) & 0x003F003Fu;
        ch[j] = (t >> 10) | (t & 0x3Fu);
    }
    word[0] = (ch[0] << 20) | (ch[1] << 8) | (ch[2] >> 4);
    word[1] = (ch[2] << 28) | (ch[3] << 16) | (ch[4] << 4) | (ch[5] >> 8);
    word[2] = (ch[5] << 24) | (ch[6] << 12) | ch[7];
}

// unpack_codes for one group: the inverse of pack32, code i into byte i of cw.
}  // namespace rpbh_fast
}  // namespace wq
