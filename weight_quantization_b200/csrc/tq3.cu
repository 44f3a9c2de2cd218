// TQ3 KV-cache codec on sm_100a: page "tq3_core.py" (tq3_quantize, tq3_dequantize).
//
// Layout: one thread owns one 128-element vector for the whole transform. The 128 values live in
// registers, so the 7 butterfly stages of the FWHT need no shuffles and no shared memory, every
// element index is a compile-time constant, and the per-vector scalars (norm, reciprocal, scale)
// are computed once per vector rather than once per lane.
//
// Rounding follows the page step by step in fp32 (the library is built with -fmad=false, so no
// multiply is fused into a following add), which makes the packed bytes reproducible bit for
// bit by any IEEE implementation of the same steps. The one reading the page leaves open is
// the L2 norm's reduction: squares are summed in fp64 and the fp64 square root is rounded once.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "wq.h"

namespace wq {
namespace tq3 {

constexpr int kD = 128;
constexpr int kThreads = 128;

// TQ3_CENTROIDS (positive half; the negative half is its exact mirror) and TQ3_BOUNDARIES as
// printed on the page, rounded to fp32 like torch.tensor(..., dtype=float32).
__device__ __forceinline__ float centroid(uint32_t idx) {
    const uint32_t m = (idx & 4u) ? (idx & 3u) : (3u - idx);
    const float mag = m == 0 ? 0.1129f : m == 1 ? 0.3479f : m == 2 ? 0.6168f : 0.9816f;
    return (idx & 4u) ? mag : -mag;
}

// searchsorted(TQ3_BOUNDARIES, v, right=False): the number of boundaries strictly below v.
__device__ __forceinline__ uint32_t bucketize(float v) {
    return (uint32_t)(v > -0.7992f) + (uint32_t)(v > -0.4824f) + (uint32_t)(v > -0.2304f) +
           (uint32_t)(v > 0.0f) + (uint32_t)(v > 0.2304f) + (uint32_t)(v > 0.4824f) +
           (uint32_t)(v > 0.7992f);
}

// fp32(1.0 / math.sqrt(128)), the post-multiplier of _fwht_inplace.
__device__ __forceinline__ float fwht_post() { return __uint_as_float(0x3DB504F3u); }

struct SignMask {
    uint32_t w[4];  // bit i = sign draw i (1 -> +1, 0 -> -1)
};

// y * s_i for s_i = +-1 is exact: flip the sign bit where the draw was 0.
__device__ __forceinline__ float apply_sign(float v, const SignMask &m, int i) {
    const uint32_t keep = (m.w[i >> 5] >> (i & 31)) & 1u;
    return __uint_as_float(__float_as_uint(v) ^ ((keep ^ 1u) << 31));
}

// _fwht_inplace without its final scaling: stages h = 1, 2, ..., 64 of (a, b) -> (a + b, a - b)
// on positions (i, i + h) inside each 2h-block.
__device__ __forceinline__ void fwht128(float (&a)[kD]) {
#pragma unroll
    for (int h = 1; h < kD; h <<= 1) {
#pragma unroll
        for (int i = 0; i < kD; ++i) {
            if ((i & h) == 0) {
                const float x = a[i], y = a[i + h];
                a[i] = __fadd_rn(x, y);
                a[i + h] = __fsub_rn(x, y);
            }
        }
    }
}

template <bool kBf16In>
__global__ void __launch_bounds__(kThreads)
    encode_kernel(const void *__restrict__ xin, int64_t n_vec, SignMask mask,
                  uint8_t *__restrict__ packed, float *__restrict__ norms,
                  float *__restrict__ scales) {
    const int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (v >= n_vec) return;

    // x.float(): bf16 widening is exact.
    float a[kD];
    if (kBf16In) {
        const uint8_t *src = static_cast<const uint8_t *>(xin) + v * (kD * 2);
#pragma unroll
        for (int q = 0; q < kD / 8; ++q) {
            const uint4 u = ld_stream16(src + 16 * q);
            a[8 * q + 0] = bf16_lo(u.x);
            a[8 * q + 1] = bf16_hi(u.x);
            a[8 * q + 2] = bf16_lo(u.y);
            a[8 * q + 3] = bf16_hi(u.y);
            a[8 * q + 4] = bf16_lo(u.z);
            a[8 * q + 5] = bf16_hi(u.z);
            a[8 * q + 6] = bf16_lo(u.w);
            a[8 * q + 7] = bf16_hi(u.w);
        }
    } else {
        const uint8_t *src = static_cast<const uint8_t *>(xin) + v * (kD * 4);
#pragma unroll
        for (int q = 0; q < kD / 4; ++q) {
            const uint4 u = ld_stream16(src + 16 * q);
            a[4 * q + 0] = __uint_as_float(u.x);
            a[4 * q + 1] = __uint_as_float(u.y);
            a[4 * q + 2] = __uint_as_float(u.z);
            a[4 * q + 3] = __uint_as_float(u.w);
        }
    }

    // Step 1: n = max(||x||, 1e-8). Squares of fp32 values are exact in fp64.
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
    for (int i = 0; i < kD; i += 4) {
        s0 = __dadd_rn(s0, __dmul_rn((double)a[i + 0], (double)a[i + 0]));
        s1 = __dadd_rn(s1, __dmul_rn((double)a[i + 1], (double)a[i + 1]));
        s2 = __dadd_rn(s2, __dmul_rn((double)a[i + 2], (double)a[i + 2]));
        s3 = __dadd_rn(s3, __dmul_rn((double)a[i + 3], (double)a[i + 3]));
    }
    float n = __double2float_rn(__dsqrt_rn(__dadd_rn(__dadd_rn(s0, s1), __dadd_rn(s2, s3))));
    n = fmaxf(n, 1e-8f);

    // xn = x / n, then the sign flips (exact), then the FWHT and its fp32 post-multiplier.
#pragma unroll
    for (int i = 0; i < kD; ++i) a[i] = apply_sign(__fdiv_rn(a[i], n), mask, i);
    fwht128(a);
    const float post = fwht_post();
#pragma unroll
    for (int i = 0; i < kD; ++i) a[i] = __fmul_rn(a[i], post);

    // Step 4: absmax scale, clamp(min=1e-8).
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kD; ++i) s = fmaxf(s, fabsf(a[i]));
    s = fmaxf(s, 1e-8f);

    // Steps 5-6: indices of xs = xh / s, packed 8 per 24-bit little-endian group.
    uint32_t grp[16];
#pragma unroll
    for (int g = 0; g < 16; ++g) {
        uint32_t bits = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) bits |= bucketize(__fdiv_rn(a[8 * g + i], s)) << (3 * i);
        grp[g] = bits;
    }
    uint8_t *dst = packed + v * 48;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        // groups 4c..4c+3 are 96 bits = three 32-bit little-endian words
        const uint32_t g0 = grp[4 * c], g1 = grp[4 * c + 1], g2 = grp[4 * c + 2], g3 = grp[4 * c + 3];
        grp[4 * c + 0] = g0 | (g1 << 24);
        grp[4 * c + 1] = (g1 >> 8) | (g2 << 16);
        grp[4 * c + 2] = (g2 >> 16) | (g3 << 8);
    }
    st_stream16(dst + 0, make_uint4(grp[0], grp[1], grp[2], grp[4]));
    st_stream16(dst + 16, make_uint4(grp[5], grp[6], grp[8], grp[9]));
    st_stream16(dst + 32, make_uint4(grp[10], grp[12], grp[13], grp[14]));
    norms[v] = n;
    scales[v] = s;
}

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads)
    decode_kernel(const uint8_t *__restrict__ packed, const float *__restrict__ norms,
                  const float *__restrict__ scales, int64_t n_vec, SignMask mask,
                  void *__restrict__ out) {
    const int64_t v = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (v >= n_vec) return;

    const uint8_t *src = packed + v * 48;
    const uint4 p0 = ld_stream16(src), p1 = ld_stream16(src + 16), p2 = ld_stream16(src + 32);
    const uint32_t w[12] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w, p2.x, p2.y, p2.z, p2.w};
    const float scale = scales[v];
    const float n = norms[v];

    // _unpack_3bit, centroids[idx] * scale
    float a[kD];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t w0 = w[3 * c], w1 = w[3 * c + 1], w2 = w[3 * c + 2];
        const uint32_t g[4] = {w0 & 0xffffffu, (w0 >> 24) | ((w1 & 0xffffu) << 8),
                               (w1 >> 16) | ((w2 & 0xffu) << 16), w2 >> 8};
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                a[32 * c + 8 * k + i] = __fmul_rn(centroid((g[k] >> (3 * i)) & 7u), scale);
    }

    // inverse FWHT (the normalised transform is its own inverse), then signs, then the norm
    fwht128(a);
    const float post = fwht_post();
#pragma unroll
    for (int i = 0; i < kD; ++i) a[i] = __fmul_rn(apply_sign(__fmul_rn(a[i], post), mask, i), n);

    if (kBf16Out) {
        uint8_t *dst = static_cast<uint8_t *>(out) + v * (kD * 2);
#pragma unroll
        for (int q = 0; q < kD / 8; ++q)
            st_stream16(dst + 16 * q,
                        make_uint4(pack_bf16x2(a[8 * q + 0], a[8 * q + 1]), pack_bf16x2(a[8 * q + 2], a[8 * q + 3]),
                                   pack_bf16x2(a[8 * q + 4], a[8 * q + 5]), pack_bf16x2(a[8 * q + 6], a[8 * q + 7])));
    } else {
        uint8_t *dst = static_cast<uint8_t *>(out) + v * (kD * 4);
#pragma unroll
        for (int q = 0; q < kD / 4; ++q)
            st_stream16(dst + 16 * q, make_uint4(__float_as_uint(a[4 * q + 0]), __float_as_uint(a[4 * q + 1]),
                                                 __float_as_uint(a[4 * q + 2]), __float_as_uint(a[4 * q + 3])));
    }
}

inline unsigned grid_for(int64_t n_vec) { return (unsigned)((n_vec + kThreads - 1) / kThreads); }

}  // namespace tq3
}  // namespace wq

using namespace wq;

extern "C" wq_status tq3_encode(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                                uint8_t *packed, float *norms, float *scales, void *stream) {
    if (n_vec < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(x_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!x || !sign_mask || !packed || !norms || !scales) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(norms, 4) || !aligned(scales, 4)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_dtype == WQ_BF16)
        tq3::encode_kernel<true><<<tq3::grid_for(n_vec), tq3::kThreads, 0, s>>>(x, n_vec, m, packed, norms, scales);
    else
        tq3::encode_kernel<false><<<tq3::grid_for(n_vec), tq3::kThreads, 0, s>>>(x, n_vec, m, packed, norms, scales);
    return launch_status();
}

extern "C" wq_status tq3_decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec,
                                const uint32_t *sign_mask, void *out, int out_dtype, void *stream) {
    if (n_vec < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!packed || !norms || !scales || !sign_mask || !out) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(packed, 16) || !aligned(out, 16) || !aligned(norms, 4) || !aligned(scales, 4)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (out_dtype == WQ_BF16)
        tq3::decode_kernel<true><<<tq3::grid_for(n_vec), tq3::kThreads, 0, s>>>(packed, norms, scales, n_vec, m, out);
    else
        tq3::decode_kernel<false><<<tq3::grid_for(n_vec), tq3::kThreads, 0, s>>>(packed, norms, scales, n_vec, m, out);
    return launch_status();
}

extern "C" int64_t tq3_compressed_bytes(int64_t n_vec) {
    if (n_vec < 0 || n_vec > INT64_MAX / 56) return -1;
    return n_vec * 56;
}
