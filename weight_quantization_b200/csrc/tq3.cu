// TQ3 KV-cache codec on sm_100a: page "tq3_core.py" (tq3_quantize, tq3_dequantize). This file
// holds the C ABI of the TQ3 entry points and the step-by-step encoder behind tq3_encode_exact;
// the fast encoders are in tq3_mma.cu (bf16) and tq3_rows.cu (fp32), the decoder in tq3_rows.cu.
//
// Step-by-step encoder layout: two threads own one 128-element vector. Lanes 0-15 of a warp hold
// elements 0..63 of 16 vectors and lanes 16-31 hold elements 64..127 of the same vectors, so six of
// the seven FWHT stages run in registers and only the last one (h = 64) exchanges values with a
// shuffle. A CTA of 128 threads handles 64 vectors; its input tile is loaded from HBM by TMA into
// shared memory with 128-byte swizzling, so every thread reads its own 128-byte row segment
// without bank conflicts and global traffic is whole, contiguous tiles.
//
// Rounding follows the page step by step in fp32 (the library is built with -fmad=false; fused
// operations are written explicitly only where they are exact), so packed bytes, norms and scales
// are reproducible bit for bit:
//   * the L2 norm sums exact fp64 squares and rounds the fp64 square root once to fp32;
//   * x / n and xh / scale are computed with Markstein's method: with r = RN(1/d),
//     q0 = RN(x r), e = RN(x - q0 d) (one FMA), RN(q0 + e r) = RN(x / d) whenever |x| >= 2^-100
//     and the quotient is a normal value (P. Markstein, "Computation of elementary functions on the
//     IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990); below that the result can be
//     one unit in the last place off (a unit of at least 2^-149), never of the other sign. The
//     tests check the kernels bit for bit against IEEE division on vectors spanning 80 binades;
//   * the butterflies and post-multipliers are single IEEE additions and multiplications (the
//     last stage as one fused a * (+-1) + b, which rounds once like an addition);
//   * the indices come from exact 0/1 saturated steps summed on the FMA pipe (add_index).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "rpbh_fast.cuh"
#include "tq3_common.cuh"
#include "tq3_mma.cuh"
#include "rpbh_linear.cuh"
#include "tq3_rows.cuh"
#include "wq.h"

namespace wq {
namespace tq3 {

constexpr int kRows = 64;       // vectors per CTA
constexpr int kThreads = 128;   // two threads per vector
constexpr int kBoxBytes = kRows * 128;
constexpr uint32_t kMaxPolls = 1u << 24;

// Set (sticky) by a kernel whose bounded wait for its TMA tile ran out; read by wq_device_fault.
__device__ unsigned int g_fault;

// Sign-bit XOR pattern for the pair of elements (e, e + 1), e = 64 * half + 2k, laid out like a
// bf16x2 word (bit 15 = element e, bit 31 = element e + 1). H is all ones for half 1.
template <bool kDefault>
__device__ __forceinline__ uint32_t pair_flip(int k, uint32_t H, uint32_t mlo, uint32_t mhi) {
    if (kDefault) {
        const uint32_t c0 = (default_flip(2 * k) >> 16) | default_flip(2 * k + 1);
        const uint32_t c1 = (default_flip(64 + 2 * k) >> 16) | default_flip(64 + 2 * k + 1);
        return c0 ^ (H & (c0 ^ c1));
    } else {
        const uint32_t word = k < 16 ? mlo : mhi;
        const uint32_t b = (~word >> ((2 * k) & 31)) & 3u;
        return ((b & 1u) << 15) | ((b & 2u) << 30);
    }
}

// Encoder split of the flips: with the page's table the half-0 pattern C0 is applied later as
// operand negation in the first butterfly stage, so the words only take (C0 ^ C1) for half 1;
// any other table takes the whole pattern on the words.
template <bool kDefault>
__device__ __forceinline__ uint32_t word_flip(int k, uint32_t H, uint32_t mlo, uint32_t mhi) {
    if (kDefault) {
        const uint32_t c0 = (default_flip(2 * k) >> 16) | default_flip(2 * k + 1);
        const uint32_t c1 = (default_flip(64 + 2 * k) >> 16) | default_flip(64 + 2 * k + 1);
        return H & (c0 ^ c1);
    }
    return pair_flip<false>(k, H, mlo, mhi);
}
template <bool kDefault>
__host__ __device__ constexpr bool stage1_neg(int e) {
    return kDefault && default_flip(e) != 0;
}

// Stage h = 64: element i (half 0) with element i + 64 (half 1). Half 0 keeps a + o and half 1
// keeps o - a, both as one rounding of a * (+-1) + o.
__device__ __forceinline__ void stage64(float (&a)[64], int half) {
    const float sg = half ? -1.0f : 1.0f;
    const f32x2 S = pk2(sg, sg);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float o0 = __shfl_xor_sync(0xffffffffu, a[2 * k], 16);
        const float o1 = __shfl_xor_sync(0xffffffffu, a[2 * k + 1], 16);
        upk2(fma2(pk2(a[2 * k], a[2 * k + 1]), S, pk2(o0, o1)), a[2 * k], a[2 * k + 1]);
    }
}

// Correctly rounded x / d given r = RN(1/d) (Markstein), two lanes at a time.
__device__ __forceinline__ f32x2 div2(f32x2 x, f32x2 r, f32x2 neg_d) {
    const f32x2 q0 = mul2(x, r);
    const f32x2 e = fma2(q0, neg_d, x);
    return fma2(e, r, q0);
}

// Adds 8^i * idx to the fp32 group word, idx = searchsorted(TQ3_BOUNDARIES, q, right=False), the
// number of boundaries strictly below q. With a' = RU(|q| - q 2^-24) -- |q| for q > 0 (or the
// float just below it when q is a power of two, which no boundary sits next to) and next(|q|) for
// q < 0 -- the count of positive boundaries b with b < a' is c = #{b < q} for q > 0 and
// c = #{b <= |q|} for q < 0, so idx = 4 + c for q > 0 and idx = 3 - c otherwise (q = +-0 gives
// a' = 0 and idx 3). Each [b < a'] is an exact 0/1: a' and b are floats of magnitude >= 2^-3,
// so a' > b implies (a' - b) 2^26 >= 1 and the saturated value is 1; a' <= b saturates to 0.
// Every term is an integer below 2^24, so the word is exact.
__device__ __forceinline__ float add_index(float q, float w8, float word) {
    const float ap = __fmaf_ru(q, -0x1p-24f, fabsf(q));
    const float M = 67108864.0f;  // 2^26
    float c = __saturatef(__fmaf_rn(ap, M, -0.2304f * M));
    c = __fadd_rn(c, __saturatef(__fmaf_rn(ap, M, -0.4824f * M)));
    c = __fadd_rn(c, __saturatef(__fmaf_rn(ap, M, -0.7992f * M)));
    const bool pos = q > 0.0f;
    return __fmaf_rn(pos ? w8 : -w8, c, __fadd_rn(word, pos ? 4.0f * w8 : 3.0f * w8));
}

// Stages h = 2 .. 32 of the butterfly on 64 values held as 32 pairs (2k, 2k + 1).
__device__ __forceinline__ void fwht_local_2_32(float (&a)[64]) {
    f32x2 P[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) P[k] = pk2(a[2 * k], a[2 * k + 1]);
#pragma unroll
    for (int hp = 1; hp < 32; hp <<= 1)
#pragma unroll
        for (int k = 0; k < 32; ++k)
            if ((k & hp) == 0) {
                const f32x2 A = P[k], B = P[k + hp];
                P[k] = add2(A, B);
                P[k + hp] = sub2(A, B);
            }
#pragma unroll
    for (int k = 0; k < 32; ++k) upk2(P[k], a[2 * k], a[2 * k + 1]);
}

template <bool kBf16In, bool kDefault>
__global__ void __launch_bounds__(kThreads, 4)
    encode_kernel(int64_t n_vec, const __grid_constant__ CUtensorMap tmap, SignMask mask,
                  uint8_t *__restrict__ packed, float *__restrict__ norms, float *__restrict__ scales) {
    constexpr int kBoxes = kBf16In ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *tile = tile_base(smem_raw);
    uint64_t *bar = reinterpret_cast<uint64_t *>(tile + kBoxes * kBoxBytes);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane >> 4;
    const int row = warp * 16 + (lane & 15);
    const int64_t v = (int64_t)blockIdx.x * kRows + row;

    if (threadIdx.x == 0) mbar_init(bar, 1);
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_expect_tx(bar, kBoxes * kBoxBytes);
#pragma unroll
        for (int b = 0; b < kBoxes; ++b)
            tma_load_2d(tile + b * kBoxBytes, &tmap, b * (kBf16In ? 64 : 32), blockIdx.x * kRows, bar);
    }
    // the bounded wait's outcome is made CTA-uniform so that no lane is left inside a shuffle
    if (__syncthreads_or(!mbar_wait_bounded(bar, 0, kMaxPolls))) {
        if (threadIdx.x == 0) atomicOr(&g_fault, 1u);
        mbar_wait_bounded(bar, 0, kMaxPolls);  // give an in-flight copy a second chance to land
        return;
    }

    const uint32_t H = half ? 0xffffffffu : 0u;
    const uint32_t mlo = half ? mask.w[2] : mask.w[0], mhi = half ? mask.w[3] : mask.w[1];

    // x.float() with the sign flips applied (exact), as 32 pairs (2k, 2k + 1)
    float x[64];
    if (kBf16In) {
        unsigned char *box = tile + half * kBoxBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 q = *reinterpret_cast<const uint4 *>(swz(box, row, j));
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = 4 * j + u;
                const uint32_t w = w4[u] ^ word_flip<kDefault>(k, H, mlo, mhi);
                x[2 * k] = bf16_lo(w);
                x[2 * k + 1] = bf16_hi(w);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            unsigned char *box = tile + (2 * half + (j >> 3)) * kBoxBytes;
            const uint4 q = *reinterpret_cast<const uint4 *>(swz(box, row, j & 7));
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int u = 0; u < 4; u += 2) {
                const int k = 2 * j + u / 2;
                const uint32_t f = word_flip<kDefault>(k, H, mlo, mhi);
                x[2 * k] = __uint_as_float(w4[u] ^ (f << 16));
                x[2 * k + 1] = __uint_as_float(w4[u + 1] ^ (f & 0x80000000u));
            }
        }
    }

    // Step 1: n = max(||x||, 1e-8); squares of fp32 values are exact in fp64
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const double d = (double)x[i];
        acc[i & 3] = __fma_rn(d, d, acc[i & 3]);
    }
    const double mine = __dadd_rn(__dadd_rn(acc[0], acc[1]), __dadd_rn(acc[2], acc[3]));
    const double other = __shfl_xor_sync(0xffffffffu, mine, 16);
    const float n = fmaxf(__double2float_rn(__dsqrt_rn(__dadd_rn(mine, other))), 1e-8f);

    // xn = x / n (signs already applied), then stage 1 of the FWHT
    float a[64];
    {
        const float r = __frcp_rn(n);
        const f32x2 R = pk2(r, r), ND = pk2(-n, -n);
#pragma unroll
        for (int k = 0; k < 32; ++k) upk2(div2(pk2(x[2 * k], x[2 * k + 1]), R, ND), a[2 * k], a[2 * k + 1]);
    }
    // stage 1, with the rest of the default-table flips as (exact) operand negations
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float p = stage1_neg<kDefault>(2 * k) ? -a[2 * k] : a[2 * k];
        const float q = stage1_neg<kDefault>(2 * k + 1) ? -a[2 * k + 1] : a[2 * k + 1];
        a[2 * k] = __fadd_rn(p, q);
        a[2 * k + 1] = __fsub_rn(p, q);
    }
    fwht_local_2_32(a);
    stage64(a, half);

    // Step 4: scale = max(max|xh|, 1e-8) with xh = fwht * c; max|fl(y c)| = fl(max|y| c)
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 64; i += 2) m = max3(m, fabsf(a[i]), fabsf(a[i + 1]));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    const float c = fwht_post();
    const float s = fmaxf(__fmul_rn(m, c), 1e-8f);

    // Steps 5-6: idx = bucketize(RN(RN(y c) / s)), 8 indices per 24-bit little-endian group
    uint32_t grp[8];
    {
        const float rs = __frcp_rn(s);
        const f32x2 C2 = pk2(c, c), RS = pk2(rs, rs), NS = pk2(-s, -s);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float wf = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float q0, q1;
                upk2(div2(mul2(pk2(a[8 * g + i], a[8 * g + i + 1]), C2), RS, NS), q0, q1);
                wf = add_index(q0, (float)(1u << (3 * i)), wf);
                wf = add_index(q1, (float)(1u << (3 * i + 3)), wf);
            }
            grp[g] = __float2uint_rz(wf);  // exact: an integer below 2^24
        }
    }
    if (v < n_vec) {
        // this thread's 24 bytes are 48v + 24 * half ...; both halves write one 16-byte chunk at
        // 48v + 32 * half and one 8-byte chunk at 48v + 16 + 8 * half (aligned for either half,
        // with no lane-divergent branch around the accesses)
        const uint32_t w0 = grp[0] | (grp[1] << 24), w1 = (grp[1] >> 8) | (grp[2] << 16),
                       w2 = (grp[2] >> 16) | (grp[3] << 8);
        const uint32_t w3 = grp[4] | (grp[5] << 24), w4 = (grp[5] >> 8) | (grp[6] << 16),
                       w5 = (grp[6] >> 16) | (grp[7] << 8);
        uint8_t *rec = packed + v * 48;
        st_stream16(rec + 32 * half, half ? make_uint4(w2, w3, w4, w5) : make_uint4(w0, w1, w2, w3));
        st_stream8(rec + 16 + 8 * half, half ? make_uint2(w0, w1) : make_uint2(w4, w5));
        if (half == 0)
            norms[v] = n;
        else
            scales[v] = s;
    }
}

// Dynamic shared memory of the step-by-step encoder: the input tile plus alignment and barrier.
inline size_t smem_bytes(bool bf16) { return (size_t)(bf16 ? 2 : 4) * kBoxBytes + 1024 + 64; }

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
    if (x_dtype == WQ_BF16) return tq3_mma::encode_bf16(x, n_vec, m, packed, norms, scales, s);
    return tq3_rows::encode(x, x_dtype, n_vec, m, packed, norms, scales, s);
}

extern "C" wq_status tq3_encode_exact(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                                      uint8_t *packed, float *norms, float *scales, void *stream) {
    if (n_vec < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(x_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!x || !sign_mask || !packed || !norms || !scales) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(norms, 4) || !aligned(scales, 4)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    const bool def = tq3::is_default(m), bf = x_dtype == WQ_BF16;
    const int esz = bf ? 2 : 4;
    const size_t smem = tq3::smem_bytes(bf);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int64_t off = 0; off < n_vec; off += tq3::kMaxChunk) {
        const int64_t cnt = n_vec - off < tq3::kMaxChunk ? n_vec - off : tq3::kMaxChunk;
        const unsigned char *xc = static_cast<const unsigned char *>(x) + off * (tq3::kD * esz);
        CUtensorMap tm;
        if (!make_tmap_2d(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, xc, tq3::kD,
                          (uint64_t)cnt, tq3::kD * esz, bf ? 64 : 32, tq3::kRows))
            return WQ_ERR_CUDA;
        const unsigned grid = (unsigned)((cnt + tq3::kRows - 1) / tq3::kRows);
        uint8_t *pc = packed + off * 48;
        float *nc = norms + off, *sc = scales + off;
        if (bf && def)
            tq3::encode_kernel<true, true><<<grid, tq3::kThreads, smem, s>>>(cnt, tm, m, pc, nc, sc);
        else if (bf)
            tq3::encode_kernel<true, false><<<grid, tq3::kThreads, smem, s>>>(cnt, tm, m, pc, nc, sc);
        else if (def)
            tq3::encode_kernel<false, true><<<grid, tq3::kThreads, smem, s>>>(cnt, tm, m, pc, nc, sc);
        else
            tq3::encode_kernel<false, false><<<grid, tq3::kThreads, smem, s>>>(cnt, tm, m, pc, nc, sc);
        const wq_status st = launch_status();
        if (st != WQ_OK) return st;
    }
    return WQ_OK;
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
    return tq3_rows::decode(packed, norms, scales, n_vec, m, out, out_dtype, static_cast<cudaStream_t>(stream));
}

extern "C" wq_status tq3_encode_aos(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                                    uint8_t *records, void *stream) {
    if (n_vec < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(x_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!x || !sign_mask || !records) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(records, 8)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_dtype == WQ_BF16) return tq3_mma::encode_bf16(x, n_vec, m, records, nullptr, nullptr, s, tq3::kAoS);
    return tq3_rows::encode(x, x_dtype, n_vec, m, records, nullptr, nullptr, s, tq3::kAoS);
}

extern "C" wq_status tq3_decode_aos(const uint8_t *records, int64_t n_vec, const uint32_t *sign_mask, void *out,
                                    int out_dtype, void *stream) {
    if (n_vec < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!records || !sign_mask || !out) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(records, 8) || !aligned(out, 16)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    return tq3_rows::decode(records, nullptr, nullptr, n_vec, m, out, out_dtype, static_cast<cudaStream_t>(stream),
                            tq3::kAoS);
}

extern "C" wq_status tq3_encode_slots(const void *x, int x_dtype, int64_t n_vec, const uint32_t *sign_mask,
                                      const int64_t *slots, uint8_t *pool, int64_t n_pool, void *stream) {
    if (n_vec < 0 || n_pool < 0) return WQ_ERR_SHAPE;
    if (!valid_dtype(x_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!x || !sign_mask || !slots || !pool) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40) || n_pool > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(pool, 8) || !aligned(slots, 8)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    const tq3::PoolMap pm{slots, 0, n_pool, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (x_dtype == WQ_BF16) return tq3_mma::encode_bf16(x, n_vec, m, pool, nullptr, nullptr, s, tq3::kPool, pm);
    return tq3_rows::encode(x, x_dtype, n_vec, m, pool, nullptr, nullptr, s, tq3::kPool, pm);
}

extern "C" wq_status tq3_decode_paged(const uint8_t *pool, int64_t n_pool, const int32_t *page_table,
                                      int64_t n_pages, int64_t page_size, int64_t n_vec, const uint32_t *sign_mask,
                                      void *out, int out_dtype, void *stream) {
    if (n_vec < 0 || n_pool < 0 || n_pages < 0) return WQ_ERR_SHAPE;
    if (page_size < 1 || page_size > ((int64_t)1 << 30) || (page_size & (page_size - 1))) return WQ_ERR_SHAPE;
    if (!valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    if (n_vec == 0) return WQ_OK;
    if (!pool || !page_table || !sign_mask || !out) return WQ_ERR_NULL;
    if (n_vec > ((int64_t)1 << 40) || n_pool > ((int64_t)1 << 40) || n_pages > ((int64_t)1 << 40)) return WQ_ERR_SHAPE;
    if ((n_vec + page_size - 1) / page_size > n_pages) return WQ_ERR_SHAPE;  // the table must cover every vector read
    if (!aligned(pool, 8) || !aligned(page_table, 4) || !aligned(out, 16)) return WQ_ERR_ALIGN;
    tq3::SignMask m;
    for (int i = 0; i < 4; ++i) m.w[i] = sign_mask[i];
    int shift = 0;
    while ((int64_t(1) << shift) < page_size) ++shift;
    const tq3::PoolMap pm{page_table, 0, n_pool, shift};
    return tq3_rows::decode(pool, nullptr, nullptr, n_vec, m, out, out_dtype, static_cast<cudaStream_t>(stream),
                            tq3::kPool, pm);
}

extern "C" int64_t tq3_compressed_bytes(int64_t n_vec) {
    if (n_vec < 0 || n_vec > INT64_MAX / 56) return -1;
    return n_vec * 56;
}

namespace wq {
namespace tq3 {
// One thread waits, through the same bounded wait the kernels use, on an mbarrier that nothing
// arrives at; when the wait gives up (after 2 s of %globaltimer) it sets fault bit 5 and returns.
__global__ void selftest_wait_kernel() {
    __shared__ uint64_t bar;
    mbar_init(&bar, 1);
    if (!mbar_wait_bounded(&bar, 0u, 1u << 30)) atomicOr(&g_fault, 32u);
}
}  // namespace tq3
}  // namespace wq

extern "C" wq_status wq_selftest_wait_timeout(void *stream) {
    wq::tq3::selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
    return launch_status();
}

namespace wq {
unsigned int tq3_attn_read_and_clear_fault();  // tq3_attn.cu
namespace rpbh_lanes {
unsigned int read_and_clear_fault();  // rpbh_lanes.cu
}
}

extern "C" wq_status wq_device_fault(unsigned int *flags) {
    if (!flags) return WQ_ERR_NULL;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, tq3::g_fault, sizeof v) != cudaSuccess) return WQ_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(tq3::g_fault, &zero, sizeof zero) != cudaSuccess) return WQ_ERR_CUDA;
    const unsigned int r = rpbh_fast::read_and_clear_fault();
    const unsigned int q = tq3_rows::read_and_clear_fault();
    const unsigned int t = tq3_mma::read_and_clear_fault();
    const unsigned int l = rpbh_linear::read_and_clear_fault();
    const unsigned int a = tq3_attn_read_and_clear_fault();
    const unsigned int n = rpbh_lanes::read_and_clear_fault();
    if ((r | q | t | l | a | n) & 0x80000000u) return WQ_ERR_CUDA;
    *flags = v | r | q | t | l | a | n;
    return WQ_OK;
}
