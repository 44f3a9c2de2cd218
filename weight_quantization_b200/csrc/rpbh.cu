// OrbitQuant RPBH weight path on sm_100a: page "orbit_quant.py" (rpbh_forward, rpbh_inverse,
// _fwht, _quantize_rows, pack_codes, unpack_codes, _dequantize_rotated, dequantize, forward).
//
// One CTA owns one row. The row is staged in shared memory with coalesced 16-byte loads, the
// permutation is a gather out of shared memory (it spans the whole row, not one Hadamard block),
// and the block FWHT runs stage by stage in shared memory. Rounding follows the page in fp32
// (the library is built with -fmad=false); the row norm sums squares in fp64.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "common.cuh"
#include "rpbh_fast.cuh"
#include "wq.h"

namespace wq {
namespace rpbh {

constexpr int kThreads = 256;

struct Codebook {
    float c[16];  // 2^bits ascending centroids, already scaled by d ** -0.5
};

__device__ __forceinline__ int clamp_index(int32_t p, int d) { return (uint32_t)p < (uint32_t)d ? p : 0; }

// fp32 view of one row element held in shared memory as the input dtype.
template <bool kBf16>
__device__ __forceinline__ float row_elem(const unsigned char *raw, int j) {
    if (kBf16) return bf16_to_f32(reinterpret_cast<const uint16_t *>(raw)[j]);
    return reinterpret_cast<const float *>(raw)[j];
}

// Copy `bytes` (a multiple of 16) from global to shared memory, 16 bytes per thread per step.
__device__ __forceinline__ void stage_row(unsigned char *dst, const unsigned char *src, int bytes) {
    for (int c = threadIdx.x; c < bytes / 16; c += blockDim.x)
        reinterpret_cast<uint4 *>(dst)[c] = ld_stream16(src + 16 * (size_t)c);
}

// y_j = x[perm[j]] * signs[j] (index_select then the Rademacher signs; both exact).
template <bool kBf16>
__device__ __forceinline__ void gather_signs(float *buf, const unsigned char *raw, int d,
                                             const int32_t *__restrict__ perm,
                                             const int8_t *__restrict__ signs) {
    for (int j = threadIdx.x; j < d; j += blockDim.x)
        buf[j] = __fmul_rn(row_elem<kBf16>(raw, clamp_index(__ldg(perm + j), d)), (float)__ldg(signs + j));
}

// _fwht without the final scaling, on every contiguous h-block of buf[0..d): stages
// step = 1, 2, ..., h/2 of (a, b) -> (a + b, a - b) on positions (i, i + step).
__device__ __forceinline__ void block_fwht(float *buf, int d, int h) {
    for (int step = 1; step < h; step <<= 1) {
        const int lg = __ffs(step) - 1;
        for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
            const int i = ((p >> lg) << (lg + 1)) | (p & (step - 1));
            const float a = buf[i], b = buf[i + step];
            buf[i] = __fadd_rn(a, b);
            buf[i + step] = __fsub_rn(a, b);
        }
        __syncthreads();
    }
}

__device__ __forceinline__ double block_sum(double v, double *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = __dadd_rn(t, red[w]);
        red[32] = t;
    }
    __syncthreads();
    return red[32];
}

template <bool kBf16>
__global__ void __launch_bounds__(kThreads)
    rotate_kernel(const void *__restrict__ x, int d, int h, float post, const int32_t *__restrict__ perm,
                  const int8_t *__restrict__ signs, void *__restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem[];
    float *buf = reinterpret_cast<float *>(smem);
    unsigned char *raw = smem + (size_t)d * 4;
    const int64_t r = blockIdx.x;
    const int esz = kBf16 ? 2 : 4;
    stage_row(raw, static_cast<const unsigned char *>(x) + r * (int64_t)d * esz, d * esz);
    __syncthreads();
    gather_signs<kBf16>(buf, raw, d, perm, signs);
    __syncthreads();
    block_fwht(buf, d, h);
    if (kBf16) {
        uint32_t *o = reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(out) + r * (int64_t)d);
        for (int j = threadIdx.x; j < d / 2; j += blockDim.x)
            o[j] = pack_bf16x2(__fmul_rn(buf[2 * j], post), __fmul_rn(buf[2 * j + 1], post));
    } else {
        float *o = static_cast<float *>(out) + r * (int64_t)d;
        for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = __fmul_rn(buf[j], post);
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(kThreads)
    quantize_kernel(const void *__restrict__ w, int d, int h, float post, const int32_t *__restrict__ perm,
                    const int8_t *__restrict__ signs, int bits, Codebook cb, uint8_t *__restrict__ packed,
                    void *__restrict__ row_norms, int norm_bf16) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ double red[33];
    __shared__ float edges[16];
    float *buf = reinterpret_cast<float *>(smem);
    unsigned char *raw = smem + (size_t)d * 4;
    const int64_t r = blockIdx.x;
    const int esz = kBf16 ? 2 : 4;
    const int L = 1 << bits;
    // edges = (codebook[:-1] + codebook[1:]) / 2
    if (threadIdx.x + 1 < (unsigned)L) edges[threadIdx.x] = __fdiv_rn(__fadd_rn(cb.c[threadIdx.x], cb.c[threadIdx.x + 1]), 2.0f);
    stage_row(raw, static_cast<const unsigned char *>(w) + r * (int64_t)d * esz, d * esz);
    __syncthreads();
    gather_signs<kBf16>(buf, raw, d, perm, signs);
    __syncthreads();
    block_fwht(buf, d, h);
    // w_rot = fwht * h^-0.5; rho = ||w_rot|| (fp64 sum of exact squares, one rounding)
    double ss = 0.0;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        const float v = __fmul_rn(buf[j], post);
        buf[j] = v;
        ss = __dadd_rn(ss, __dmul_rn((double)v, (double)v));
    }
    const float rho = __double2float_rn(__dsqrt_rn(block_sum(ss, red)));
    const float den = __fadd_rn(rho, 1e-10f);
    // codes of 8 consecutive elements -> `bits` bytes of the MSB-first stream
    uint8_t *dst = packed + (r * (int64_t)d / 8) * bits;
    for (int g = threadIdx.x; g < d / 8; g += blockDim.x) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float u = __fdiv_rn(buf[8 * g + i], den);
            uint32_t code = 0;
            for (int k = 0; k + 1 < L; ++k) code += (uint32_t)(u > edges[k]);
            word = (word << bits) | code;
        }
        for (int b = 0; b < bits; ++b) dst[g * bits + b] = (uint8_t)(word >> (8 * (bits - 1 - b)));
    }
    if (threadIdx.x == 0) {
        if (norm_bf16)
            static_cast<uint16_t *>(row_norms)[r] = f32_to_bf16(rho);
        else
            static_cast<float *>(row_norms)[r] = rho;
    }
}

// _dequantize_rotated, optionally followed by rpbh_inverse.
template <bool kNormBf16, bool kOutBf16, bool kUnrotate>
__global__ void __launch_bounds__(kThreads)
    dequantize_kernel(const uint8_t *__restrict__ packed, const void *__restrict__ row_norms, int d, int h,
                      float post, int bits, Codebook cb, const int32_t *__restrict__ perm,
                      const int8_t *__restrict__ signs, void *__restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float cbs[16];
    const int64_t r = blockIdx.x;
    const int L = 1 << bits;
    const float rho = kNormBf16 ? bf16_to_f32(static_cast<const uint16_t *>(row_norms)[r])
                                : static_cast<const float *>(row_norms)[r];
    if (threadIdx.x < (unsigned)L) {
        // codebook.to(dtype): the bf16 rotated output multiplies bf16-rounded operands
        const float c = cb.c[threadIdx.x];
        cbs[threadIdx.x] = (kOutBf16 && !kUnrotate) ? bf16_to_f32(f32_to_bf16(c)) : c;
    }
    __syncthreads();
    const float rho_op = (kOutBf16 && !kUnrotate) ? bf16_to_f32(f32_to_bf16(rho)) : rho;
    const uint8_t *src = packed + (r * (int64_t)d / 8) * bits;
    float *buf = reinterpret_cast<float *>(smem);
    const uint32_t mask = (1u << bits) - 1u;
    for (int g = threadIdx.x; g < d / 8; g += blockDim.x) {
        uint32_t word = 0;
        for (int b = 0; b < bits; ++b) word = (word << 8) | src[g * bits + b];
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(cbs[(word >> (bits * (7 - i))) & mask], rho_op);
        if (kUnrotate) {
#pragma unroll
            for (int i = 0; i < 8; ++i) buf[8 * g + i] = v[i];
        } else if (kOutBf16) {
            uint4 o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                 pack_bf16x2(v[6], v[7]));
            st_stream16(static_cast<uint16_t *>(out) + r * (int64_t)d + 8 * g, o);
        } else {
            float *o = static_cast<float *>(out) + r * (int64_t)d + 8 * g;
            st_stream16(o, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                                      __float_as_uint(v[3])));
            st_stream16(o + 4, make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                                          __float_as_uint(v[7])));
        }
    }
    if (!kUnrotate) return;
    __syncthreads();
    block_fwht(buf, d, h);
    // z = fwht * h^-0.5 * signs; out[perm[j]] = z[j]  (== out[i] = z[inv_perm[i]])
    float *ob = buf + d;
    for (int j = threadIdx.x; j < d; j += blockDim.x)
        ob[clamp_index(__ldg(perm + j), d)] = __fmul_rn(__fmul_rn(buf[j], post), (float)__ldg(signs + j));
    __syncthreads();
    if (kOutBf16) {
        uint32_t *o = reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(out) + r * (int64_t)d);
        for (int j = threadIdx.x; j < d / 2; j += blockDim.x) o[j] = pack_bf16x2(ob[2 * j], ob[2 * j + 1]);
    } else {
        float *o = static_cast<float *>(out) + r * (int64_t)d;
        for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = ob[j];
    }
}

// h ** -0.5 evaluated in double (as Python does) and applied as an fp32 scalar.
inline float fwht_post(int64_t h) { return (float)std::pow((double)h, -0.5); }

inline wq_status check_dims(int64_t rows, int64_t d) {
    if (rows < 0 || d <= 0 || d > WQ_RPBH_MAX_D) return WQ_ERR_SHAPE;
    if ((d & -d) < WQ_RPBH_MIN_BLOCK) return WQ_ERR_NOT_QUANTIZABLE;
    if (rows > 0x7fffffffLL) return WQ_ERR_SHAPE;
    return WQ_OK;
}

// Opt in to more than 48 KB of dynamic shared memory when a row needs it. The attribute is set
// once per kernel (and again only if a later call needs more), so calls made while a stream is
// being captured into a CUDA graph issue no attribute changes.
inline size_t optin_limit() {
    static size_t cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) {
        int optin = 0;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
        cached[dev] = (size_t)optin;
    }
    return cached[dev];
}

template <typename K>
inline wq_status prepare(K kernel, size_t smem) {
    if (smem + 1024 > optin_limit()) return WQ_ERR_SHAPE;
    return ensure_dynamic_smem(reinterpret_cast<const void *>(kernel), smem) ? WQ_OK : WQ_ERR_CUDA;
}

}  // namespace rpbh
}  // namespace wq

using namespace wq;

extern "C" int64_t rpbh_packed_bytes(int64_t rows, int64_t d, int bits) {
    if (rows < 0 || d < 0 || bits < 1 || bits > 8) return -1;
    if (d != 0 && rows > INT64_MAX / d) return -1;
    const int64_t n = rows * d;
    return (n / 8 + (n % 8 != 0)) * bits;
}

extern "C" wq_status rpbh_rotate_activations(const void *x, int dtype, int64_t rows, int64_t d,
                                             const int32_t *perm, const int8_t *signs, void *x_rot, void *stream) {
    wq_status st = rpbh::check_dims(rows, d);
    if (st != WQ_OK) return st;
    if (!valid_dtype(dtype)) return WQ_ERR_DTYPE;
    if (rows == 0) return WQ_OK;
    if (!x || !perm || !signs || !x_rot) return WQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(x_rot, 16) || !aligned(perm, 4)) return WQ_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rpbh_fast::supported(d, dtype_size(dtype), dtype_size(dtype)) && aligned(perm, 16) && aligned(signs, 16))
        return rpbh_fast::rotate(x, dtype, rows, d, perm, signs, x_rot, s);
    const int h = (int)(d & -d);
    const size_t smem = (size_t)d * (4 + dtype_size(dtype));
    const float post = rpbh::fwht_post(h);
    if (dtype == WQ_BF16) {
        if ((st = rpbh::prepare(rpbh::rotate_kernel<true>, smem)) != WQ_OK) return st;
        rpbh::rotate_kernel<true><<<(unsigned)rows, rpbh::kThreads, smem, s>>>(x, (int)d, h, post, perm, signs, x_rot);
    } else {
        if ((st = rpbh::prepare(rpbh::rotate_kernel<false>, smem)) != WQ_OK) return st;
        rpbh::rotate_kernel<false><<<(unsigned)rows, rpbh::kThreads, smem, s>>>(x, (int)d, h, post, perm, signs, x_rot);
    }
    return launch_status();
}

extern "C" wq_status rpbh_requantize_weight(const void *W, int w_dtype, int64_t rows, int64_t d, const int32_t *perm,
                                            const int8_t *signs, int bits, const float *codebook, uint8_t *packed,
                                            void *row_norms, int norm_dtype, void *stream) {
    wq_status st = rpbh::check_dims(rows, d);
    if (st != WQ_OK) return st;
    if (bits < 2 || bits > 4) return WQ_ERR_BITS;
    if (!valid_dtype(w_dtype) || !valid_dtype(norm_dtype)) return WQ_ERR_DTYPE;
    if (rows == 0) return WQ_OK;
    if (!W || !perm || !signs || !codebook || !packed || !row_norms) return WQ_ERR_NULL;
    if (!aligned(W, 16) || !aligned(packed, 4) || !aligned(perm, 4) || !aligned(row_norms, dtype_size(norm_dtype)))
        return WQ_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (rpbh_fast::supported(d, dtype_size(w_dtype), 1) && aligned(perm, 16) && aligned(signs, 16))
        return rpbh_fast::quantize(W, w_dtype, rows, d, perm, signs, bits, codebook, packed, row_norms, norm_dtype, s);
    rpbh::Codebook cb = {};
    for (int k = 0; k < (1 << bits); ++k) cb.c[k] = codebook[k];
    const int h = (int)(d & -d);
    const size_t smem = (size_t)d * (4 + dtype_size(w_dtype));
    const float post = rpbh::fwht_post(h);
    const int nb = norm_dtype == WQ_BF16;
    if (w_dtype == WQ_BF16) {
        if ((st = rpbh::prepare(rpbh::quantize_kernel<true>, smem)) != WQ_OK) return st;
        rpbh::quantize_kernel<true><<<(unsigned)rows, rpbh::kThreads, smem, s>>>(W, (int)d, h, post, perm, signs, bits,
                                                                                 cb, packed, row_norms, nb);
    } else {
        if ((st = rpbh::prepare(rpbh::quantize_kernel<false>, smem)) != WQ_OK) return st;
        rpbh::quantize_kernel<false><<<(unsigned)rows, rpbh::kThreads, smem, s>>>(W, (int)d, h, post, perm, signs, bits,
                                                                                  cb, packed, row_norms, nb);
    }
    return launch_status();
}

extern "C" wq_status rpbh_quantize_weight(const void *W, int w_dtype, int64_t rows, int64_t d, const int32_t *perm,
                                          const int8_t *signs, int bits, const float *codebook, uint8_t *packed,
                                          void *row_norms, void *stream) {
    return rpbh_requantize_weight(W, w_dtype, rows, d, perm, signs, bits, codebook, packed, row_norms, w_dtype,
                                  stream);
}

namespace {
template <bool kNormBf16, bool kOutBf16, bool kUnrotate>
wq_status launch_dequant(const uint8_t *packed, const void *row_norms, int64_t rows, int d, int bits,
                         const rpbh::Codebook &cb, const int32_t *perm, const int8_t *signs, void *out,
                         cudaStream_t s) {
    const int h = d & -d;
    const size_t smem = kUnrotate ? (size_t)d * 8 : 0;
    auto k = rpbh::dequantize_kernel<kNormBf16, kOutBf16, kUnrotate>;
    wq_status st = rpbh::prepare(k, smem);
    if (st != WQ_OK) return st;
    k<<<(unsigned)rows, rpbh::kThreads, smem, s>>>(packed, row_norms, d, h, rpbh::fwht_post(h), bits, cb, perm, signs,
                                                   out);
    return launch_status();
}
}  // namespace

extern "C" wq_status rpbh_dequantize_weight(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t rows,
                                            int64_t d, int bits, const float *codebook, const int32_t *perm,
                                            const int8_t *signs, int unrotate, void *out, int out_dtype,
                                            void *stream) {
    wq_status st = rpbh::check_dims(rows, d);
    if (st != WQ_OK) return st;
    if (bits < 2 || bits > 4) return WQ_ERR_BITS;
    if (!valid_dtype(norm_dtype) || !valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    if (rows == 0) return WQ_OK;
    if (!packed || !row_norms || !codebook || !out) return WQ_ERR_NULL;
    if (unrotate && (!perm || !signs)) return WQ_ERR_NULL;
    if (!aligned(packed, 4) || !aligned(out, 16) || !aligned(row_norms, dtype_size(norm_dtype)) ||
        (unrotate && !aligned(perm, 4)))
        return WQ_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (unrotate && rpbh_fast::supported(d, 1, dtype_size(out_dtype)) && aligned(perm, 16) && aligned(signs, 16))
        return rpbh_fast::dequantize_unrotate(packed, row_norms, norm_dtype, rows, d, bits, codebook, perm, signs, out,
                                              out_dtype, s);
    if (!unrotate && aligned(packed, 16) && rpbh_fast::dequantize_rotated_fits(d, bits))
        return rpbh_fast::dequantize_rotated(packed, row_norms, norm_dtype, rows, d, bits, codebook, out, out_dtype, s);
    rpbh::Codebook cb = {};
    for (int k = 0; k < (1 << bits); ++k) cb.c[k] = codebook[k];
    const int di = (int)d;
    const bool nb = norm_dtype == WQ_BF16, ob = out_dtype == WQ_BF16;
#define WQ_DQ(NB, OB, UR) launch_dequant<NB, OB, UR>(packed, row_norms, rows, di, bits, cb, perm, signs, out, s)
    if (unrotate) {
        if (nb) return ob ? WQ_DQ(true, true, true) : WQ_DQ(true, false, true);
        return ob ? WQ_DQ(false, true, true) : WQ_DQ(false, false, true);
    }
    if (nb) return ob ? WQ_DQ(true, true, false) : WQ_DQ(true, false, false);
    return ob ? WQ_DQ(false, true, false) : WQ_DQ(false, false, false);
#undef WQ_DQ
}
