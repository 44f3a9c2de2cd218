// Fused RPBH linear layer on sm_100a: page "orbit_quant.py", forward (x_rot = rpbh_forward(x),
// then F.linear(x_rot, W', bias)), with W' the rotated-basis dequantized weight
// (_dequantize_rotated: codebook[codes] * norms in the weight dtype). W' is never written out: its
// packed codes are unpacked straight into the tensor-core operand in shared memory.
//
// One CTA computes a 256 x 256 tile of D = W'_tile x_rot_tile^T (256 output features as two
// halves of 128 = the product's M and the accumulators' lanes, 256 activation rows = N and their
// columns), K = d in chunks of 64 (one 128-byte swizzle atom of bf16); the two halves share each
// x_rot tile, so x_rot is read once per 256 output features:
//   * warp 0, lane 0: TMA loads of x_rot [256 x 64] bf16 tiles (128-byte swizzle) into a ring of
//     three stages, and the products: per chunk and K = 16 step one tcgen05.mma.kind::f16
//     (M = 128, N = 256) per half, accumulating in 2 x 256 tensor-memory columns, each chunk's
//     commit releasing its stage;
//   * warps 4..11: thread p owns output feature n0 + p: it loads the chunk's 8 * bits code bytes
//     of its row, unpacks the 64 codes (MSB-first stream, pack_codes) and looks each up in the
//     codebook rounded to bf16 (a shuffle: lane l holds centroid l mod 2^bits), writing the 128-byte
//     row of the operand tile with the 128-byte swizzle; then, after the last product, the
//     epilogue: accumulator row p, column j is y[m0 + j][n0 + p] / rho, so
//     y = bf16(acc * bf16(rho_n) + bias_n), stored so that a warp writes 32 consecutive features.
// The row norm is applied to the accumulated sum instead of to every element: the standalone
// dequantizer rounds bf16(codebook) * bf16(rho) to bf16 per element, this kernel does not, so
// the two differ by at most 2^-8 relative per term (the tolerance the tests use).
// Every wait is bounded; a timeout sets the fault flag, after which no wait or issue happens
// and the kernel runs out, results void.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>
#include <cstring>

#include "common.cuh"
#include "tcgen05.cuh"
#include "rpbh_linear.cuh"
#include "wq.h"

namespace wq {
namespace rpbh_linear {

constexpr int kTM = 256;  // output features per tile (two halves of 128: the product's M)
constexpr int kTK = 64;   // K per chunk
constexpr int kStages = 3;
constexpr int kProducerWarps = kTM / 32;
constexpr int kThreads = 128 + 32 * kProducerWarps;
constexpr int kAHalf = 128 * kTK * 2;  // one half of the weight tile
constexpr int kABytes = kTM * kTK * 2;
constexpr int kOffA = 0;
constexpr int kOffB = kStages * kABytes;
constexpr uint32_t kTmemCols = 512;  // the two accumulators at columns 0 and 256
constexpr uint32_t kMaxPolls = 1u << 24;

// TN activation rows per tile (the product's N: a multiple of 16 up to 256; the host picks the
// one that fills the SMs best)
template <int TN>
struct Tile {
    static constexpr int kTN = TN;
    static constexpr int kBBytes = TN * kTK * 2;
    static constexpr int kOffBar = kOffB + kStages * kBBytes;  // full_a, full_b, empty (per stage), done, TMEM address
    static constexpr int kSmem = 1024 + kOffBar + 8 * (3 * kStages + 1) + 16;
    static_assert(TN % 16 == 0 && TN <= 256 && kBBytes % 1024 == 0, "N of one tcgen05.mma, whole swizzle atoms");
    static_assert(kSmem <= 232448, "the ring must fit the 227 KB a CTA may use");
    // fp32 accumulator, bf16 A and B, both K-major, N = TN, M = 128
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
};

__device__ unsigned int g_fault;

struct CodebookBf16 {
    uint16_t c[16];  // the codebook rounded to bf16 (codebook.to(dtype))
};

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Code i (0 .. 63) of a chunk whose 8 * BITS bytes are held as big-endian 32-bit words W
// (stream bit b is bit 31 - b % 32 of W[b / 32]), in the low BITS bits of the result; the bits
// above it are whatever follows in the word. A shuffle takes its source lane modulo 32, and lane l
// holds centroid l mod 2^BITS, so the lookup needs no mask.
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&W)[2 * BITS], int i) {
    const int o = BITS * i, q = o >> 5, r = o & 31;
    if (r + BITS <= 32) return W[q] >> (32 - r - BITS);
    return __funnelshift_l(W[q + 1], W[q], r + BITS - 32);
}

// The lookup of 2- and 3-bit codes by byte permutes, on the integer pipe: the 2^BITS bf16 entries
// split into an 8-byte table of their low bytes and one of their high bytes; a byte permute whose
// selector nibble k holds a code copies that code's byte into byte k of the result, so two permutes
// look up four codes and two more interleave the low and high bytes into bf16 pairs.
struct ByteTables {
    uint32_t lo0, lo1, hi0, hi1;  // byte k of lo0 (k < 4) / lo1 (k >= 4): low byte of entry k
};

__device__ __forceinline__ ByteTables byte_tables(const CodebookBf16 &cb, int entries) {
    ByteTables t = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t e = k < entries ? cb.c[k] : 0u;
        if (k < 4) {
            t.lo0 |= (e & 0xffu) << (8 * k);
            t.hi0 |= (e >> 8) << (8 * k);
        } else {
            t.lo1 |= (e & 0xffu) << (8 * (k - 4));
            t.hi1 |= (e >> 8) << (8 * (k - 4));
        }
    }
    return t;
}

// The four BITS-bit codes of x (4 BITS bits, first code in the top bits, nothing above) as the
// four nibbles of a byte-permute selector, the last code in nibble 0. Two steps, each an exact
// multiply-add that moves the upper half of every field group up: for 3 bits
// (x & 0x3f) | (x & 0xfc0) << 2, then (y & 0x0707) | (y & 0x3838) << 1.
template <int BITS>
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
    if constexpr (BITS == 3) {
        const uint32_t y = (x & 0xfc0u) * 3u + x;
        return (y & 0x3838u) + y;
    } else {
        const uint32_t y = (x & 0xf0u) * 15u + x;
        return (y & 0x0c0cu) * 3u + y;
    }
}

// Codes 8j .. 8j + 7 of a chunk (stream bytes BITS j .. BITS j + BITS - 1 of the little-endian
// words R) as four bf16 pairs, code 8j in the low half of w[0].
template <int BITS>
__device__ __forceinline__ void lookup8(const uint32_t (&R)[2 * BITS], int j, const ByteTables &t, uint32_t (&w)[4]) {
    uint32_t xa, xb;  // codes 8j .. 8j + 3 and 8j + 4 .. 8j + 7
    if constexpr (BITS == 3) {
        const int b0 = 3 * j, q = b0 >> 2, u = b0 & 3;
        // the group's three bytes, first in bits 16 .. 23 (byte 3 of the result is not used)
        const uint32_t g = __byte_perm(R[q], q + 1 < 2 * BITS ? R[q + 1] : 0u, (u + 2) | ((u + 1) << 4) | (u << 8));
        xa = (g >> 12) & 0xfffu;
        xb = g & 0xfffu;
    } else {
        const int b0 = 2 * j, q = b0 >> 2, u = b0 & 3;
        const uint32_t g = __byte_perm(R[q], 0u, (u + 1) | (u << 4));
        xa = (g >> 8) & 0xffu;
        xb = g & 0xffu;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = spread4<BITS>(h ? xb : xa);
        const uint32_t L = __byte_perm(t.lo0, t.lo1, sel), H = __byte_perm(t.hi0, t.hi1, sel);
        w[2 * h] = __byte_perm(L, H, 0x6273);      // first and second code of the four
        w[2 * h + 1] = __byte_perm(L, H, 0x4051);  // third and fourth
    }
}

template <int BITS, bool kNormBf16, int TN>
__global__ void __launch_bounds__(kThreads, 1)
    linear_kernel(const uint8_t *__restrict__ packed, const void *__restrict__ row_norms, int out_f, int d,
                  const __grid_constant__ CUtensorMap xmap, int m_rows, const uint16_t *__restrict__ bias,
                  CodebookBf16 cb, uint16_t *__restrict__ y) {
    using T = Tile<TN>;
    constexpr int kTN = TN, kBBytes = T::kBBytes, kOffBar = T::kOffBar;
    constexpr uint32_t kIdesc = T::kIdesc;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *const base = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTM, m0 = blockIdx.y * kTN;
    const int nchunks = d / kTK;
    uint64_t *const full_a = reinterpret_cast<uint64_t *>(base + kOffBar);  // the unpacking warps arrive
    uint64_t *const full_b = full_a + kStages;                             // the TMA of x_rot lands
    uint64_t *const empty = full_b + kStages;                              // the chunk's products are done
    uint64_t *const done = empty + kStages;                                // every product is done
    uint32_t *const tslot = reinterpret_cast<uint32_t *>(done + 1);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_a[s], kProducerWarps);
            mbar_init(&full_b[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    bool fault = false;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t issued[kStages] = {};  // x_rot copies issued per stage (fault path)
            auto load_b = [&](int c) {
                const int s = c % kStages;
                mbar_expect_tx(&full_b[s], kBBytes);
                tma_load_2d(base + kOffB + s * kBBytes, &xmap, c * kTK, m0, &full_b[s]);
                ++issued[s];
            };
            for (int c = 0; c < kStages && c < nchunks; ++c) load_b(c);
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                const uint32_t ph = (uint32_t)(c / kStages) & 1u;
                if (!mbar_wait_bounded(&full_b[s], ph, kMaxPolls) || !mbar_wait_bounded(&full_a[s], ph, kMaxPolls)) {
                    fault = true;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = sw128_desc(smem_u32(base + kOffA + s * kABytes));
                const uint64_t bd = sw128_desc(smem_u32(base + kOffB + s * kBBytes));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {  // K = 16 per instruction: 32 bytes into each 128-byte row
                    const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
                    mma_bf16(tmem, ad + (uint32_t)(ks * 2), bd + (uint32_t)(ks * 2), kIdesc, acc);
                    mma_bf16(tmem + 256u, ad + (uint32_t)((kAHalf >> 4) + ks * 2), bd + (uint32_t)(ks * 2), kIdesc,
                             acc);
                }
                mma_commit(&empty[s]);
                // the previous chunk's stage takes the chunk kStages after it once its products are done
                if (c >= 1 && c - 1 + kStages < nchunks) {
                    const int sp = (c - 1) % kStages;
                    if (!mbar_wait_bounded(&empty[sp], (uint32_t)((c - 1) / kStages) & 1u, kMaxPolls)) {
                        fault = true;
                        break;
                    }
                    load_b(c - 1 + kStages);
                }
            }
            mma_commit(done);  // arrives once every product issued above is done
            if (fault) {
                // give the copies still in flight a bounded chance to land before the memory goes away
                for (int s = 0; s < kStages; ++s)
                    if (issued[s] > 0) mbar_wait_bounded(&full_b[s], (issued[s] - 1) & 1u, kMaxPolls);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int p = threadIdx.x - 128;  // this thread's output feature within the tile (accumulator lane)
        const int n = n0 + p;
        const bool valid = n < out_f;
        const uint8_t *const src = packed + (int64_t)(valid ? n : 0) * (d / 8 * BITS);
        // 4 bits: lane l holds the bf16 centroid l mod 16, and a shuffle from the lane named by a code
        // is the lookup; 2 and 3 bits: byte permutes
        const uint32_t cbv = cb.c[lane & ((1 << BITS) - 1)];
        const ByteTables tabs = byte_tables(cb, 1 << BITS);
        unsigned char *const rowA = base + kOffA + (p >> 7) * kAHalf + (p & 127) * 128;
        const int sw = p & 7;
        // the code bytes of chunk c + 2 are loaded while chunk c is unpacked (two register sets
        // ahead, so the loads' latency is hidden behind two chunks of work)
        uint2 raw[2][BITS];
        auto fetch = [&](int c, uint2 (&r)[BITS]) {
#pragma unroll
            for (int q = 0; q < BITS; ++q)
                r[q] = c < nchunks ? __ldg(reinterpret_cast<const uint2 *>(src + c * 8 * BITS) + q) : make_uint2(0u, 0u);
        };
        fetch(0, raw[0]);
        fetch(1, raw[1]);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            if (c >= kStages && !fault) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait_bounded(&empty[s], (uint32_t)(c / kStages - 1) & 1u, kMaxPolls);
                if (!__all_sync(0xffffffffu, ok)) fault = true;
            }
            // the chunk's 8 * BITS code bytes, as little-endian words (R) and as big-endian words (W)
            uint32_t R[2 * BITS], W[2 * BITS];
#pragma unroll
            for (int q = 0; q < BITS; ++q) {
                const uint2 v = (c & 1) ? raw[1][q] : raw[0][q];
                R[2 * q] = v.x;
                R[2 * q + 1] = v.y;
                W[2 * q] = __byte_perm(v.x, 0u, 0x0123);
                W[2 * q + 1] = __byte_perm(v.y, 0u, 0x0123);
            }
            if (c & 1)
                fetch(c + 2, raw[1]);
            else
                fetch(c + 2, raw[0]);
            unsigned char *const A = rowA + s * kABytes;
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // 16-byte chunk j: k = 8j .. 8j + 7 (rows past out_features: never stored)
                uint32_t w4[4];
                if constexpr (BITS == 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t lo = __shfl_sync(0xffffffffu, cbv, (int)code_at<BITS>(W, 8 * j + 2 * u));
                        const uint32_t hi = __shfl_sync(0xffffffffu, cbv, (int)code_at<BITS>(W, 8 * j + 2 * u + 1));
                        w4[u] = __byte_perm(lo, hi, 0x5410);
                    }
                } else {
                    lookup8<BITS>(R, j, tabs, w4);
                }
                *reinterpret_cast<uint4 *>(A + ((j ^ sw) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            fence_proxy_async_smem();  // written by threads, read by the tensor core
            __syncwarp();
            if (lane == 0 && !fault) mbar_arrive(&full_a[s]);
        }
        // epilogue: y[m][n] = bf16(acc[p][m - m0] * bf16(rho_n) + bias_n)
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(done, 0u, kMaxPolls);
        if (!__all_sync(0xffffffffu, ok)) fault = true;
        tc_fence_after();
        float rho = 0.0f, b = 0.0f;
        if (valid) {
            rho = kNormBf16 ? bf16_to_f32(static_cast<const uint16_t *>(row_norms)[n])
                            : static_cast<const float *>(row_norms)[n];
            rho = bf16_to_f32(f32_to_bf16(rho));
            if (bias) b = bf16_to_f32(bias[n]);
        }
        // warps 4..7 read the first half's accumulator, warps 8..11 the second's (lanes 32 (warp % 4) ..)
        const uint32_t lanes = tmem + (uint32_t)((p >> 7) * 256) + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll 1
        for (int j = 0; j < (kTN + 31) / 32; ++j) {
            float v[32];
            tmem_ld32(lanes + 32u * j, v);  // (past column kTN the values are not this tile's: not stored)
            tmem_wait(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int m = m0 + 32 * j + i;
                if (valid && 32 * j + i < kTN && m < m_rows) y[(int64_t)m * out_f + n] = f32_to_bf16(__fmaf_rn(v[i], rho, b));
            }
        }
    }
    if (fault && (lane == 0)) atomicOr(&g_fault, 16u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
namespace {
// fp32 -> bf16, round to nearest even (the codebook's .to(dtype)); the codebook is finite
uint16_t bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

template <int BITS, bool kNB, int TN>
wq_status launch_tn(const uint8_t *packed, const void *row_norms, int64_t out_f, int64_t d, const void *x_rot,
                    int64_t m, const uint16_t *bias, const CodebookBf16 &cb, uint16_t *y, cudaStream_t s) {
    CUtensorMap xm;
    if (!make_tmap_2d(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x_rot, (uint64_t)d, (uint64_t)m, (uint64_t)d * 2, kTK, TN))
        return WQ_ERR_CUDA;
    auto k = linear_kernel<BITS, kNB, TN>;
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), Tile<TN>::kSmem)) return WQ_ERR_CUDA;
    const dim3 grid((unsigned)((out_f + kTM - 1) / kTM), (unsigned)((m + TN - 1) / TN));
    k<<<grid, kThreads, Tile<TN>::kSmem, s>>>(packed, row_norms, (int)out_f, (int)d, xm, (int)m, bias, cb, y);
    return launch_status();
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
    return cached[dev];
}

// One CTA per SM: a tile width of 240 rows instead of 256 is taken when it needs fewer rounds of
// CTAs times the width (e.g. 16 x 9 = 144 tiles in one round on 148 SMs instead of 16 x 8 = 128).
template <int BITS, bool kNB>
wq_status launch(const uint8_t *packed, const void *row_norms, int64_t out_f, int64_t d, const void *x_rot,
                 int64_t m, const uint16_t *bias, const CodebookBf16 &cb, uint16_t *y, cudaStream_t s) {
    const int64_t sms = sm_count() > 0 ? sm_count() : 1, tn = (out_f + kTM - 1) / kTM;
    auto cost = [&](int64_t w) { return ((tn * ((m + w - 1) / w) + sms - 1) / sms) * w; };
    if (cost(240) < cost(256)) return launch_tn<BITS, kNB, 240>(packed, row_norms, out_f, d, x_rot, m, bias, cb, y, s);
    return launch_tn<BITS, kNB, 256>(packed, row_norms, out_f, d, x_rot, m, bias, cb, y, s);
}

template <bool kNB>
wq_status by_bits(int bits, const uint8_t *packed, const void *row_norms, int64_t out_f, int64_t d,
                  const void *xm, int64_t m, const uint16_t *bias, const CodebookBf16 &cb, uint16_t *y,
                  cudaStream_t s) {
    switch (bits) {
        case 2: return launch<2, kNB>(packed, row_norms, out_f, d, xm, m, bias, cb, y, s);
        case 3: return launch<3, kNB>(packed, row_norms, out_f, d, xm, m, bias, cb, y, s);
        case 4: return launch<4, kNB>(packed, row_norms, out_f, d, xm, m, bias, cb, y, s);
        default: return WQ_ERR_BITS;
    }
}
}  // namespace

unsigned int read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(g_fault, &zero, sizeof zero);
    return v;
}

}  // namespace rpbh_linear
}  // namespace wq

using namespace wq;

extern "C" wq_status rpbh_linear(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t out_features,
                                 int64_t d, int bits, const float *codebook, const void *x_rot, int64_t m,
                                 const void *bias, void *y, void *stream) {
    if (out_features < 0 || d < 0 || m < 0) return WQ_ERR_SHAPE;
    if (bits < 2 || bits > 4) return WQ_ERR_BITS;
    if (norm_dtype != WQ_F32 && norm_dtype != WQ_BF16) return WQ_ERR_DTYPE;
    if (d % 64 != 0 || d > (int64_t)1 << 20 || out_features > INT32_MAX / 2 || m > INT32_MAX / 2) return WQ_ERR_SHAPE;
    if (out_features == 0 || m == 0) return WQ_OK;
    if (d == 0) return WQ_ERR_SHAPE;
    if (!packed || !row_norms || !codebook || !x_rot || !y) return WQ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(packed) & 15) || (reinterpret_cast<uintptr_t>(x_rot) & 15) ||
        (reinterpret_cast<uintptr_t>(y) & 1) || (reinterpret_cast<uintptr_t>(bias) & 1) ||
        (reinterpret_cast<uintptr_t>(row_norms) & (norm_dtype == WQ_BF16 ? 1 : 3)))
        return WQ_ERR_ALIGN;
    rpbh_linear::CodebookBf16 cb = {};
    for (int k = 0; k < (1 << bits); ++k) cb.c[k] = rpbh_linear::bf16_rne(codebook[k]);
    const void *xm = x_rot;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto *b = static_cast<const uint16_t *>(bias);
    auto *yo = static_cast<uint16_t *>(y);
    return norm_dtype == WQ_BF16
               ? rpbh_linear::by_bits<true>(bits, packed, row_norms, out_features, d, xm, m, b, cb, yo, s)
               : rpbh_linear::by_bits<false>(bits, packed, row_norms, out_features, d, xm, m, b, cb, yo, s);
}
