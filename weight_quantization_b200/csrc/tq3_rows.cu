// TQ3 with one thread per 128-element vector, on sm_100a: page "tq3_core.py" (tq3_quantize,
// tq3_dequantize, _fwht_inplace, _quantize_to_indices, _pack_3bit, _unpack_3bit).
//
// A thread keeps its whole vector in registers as 64 packed fp32 pairs: six of the seven FWHT
// stages are two-lane IEEE adds or subtracts between registers and one is a scalar butterfly
// inside each pair (the encoder pairs (k, k + 64), so its scalar stage is h = 64; the decoder
// pairs (2k, 2k + 1), so its scalar stage is h = 1). No value crosses threads. CTAs are persistent over 128-vector tiles: the encoder streams its
// input tiles through shared memory with TMA (two stages, the next tile landing while this one is
// processed); the decoder prefetches the next tile's records into registers and writes each output
// tile with TMA stores from a 128-byte-swizzled staging buffer.
//
// Decoder numerics are the page's, step by step: dequantised values RN(centroid * scale), the seven
// butterfly stages as single roundings, RN(. * fp32(1/sqrt(128))), the sign flips (exact), then
// RN(. * norm) -- bit-identical to the definition.
//
// Encoder numerics. The page normalises x, transforms, scales by the absmax and compares
// xs = RN(RN(y c) / scale) with the boundaries. In exact arithmetic xs_i = z_i / max|z| with
// z = fwht(D x) (the norm and c cancel), unless the 1e-8 floor on the scale is active. This kernel
// therefore transforms the unnormalised input, forms x_i = RN(z_i RN(1 / T)) with T = max|z|
// (T = 1e-8 * norm * sqrt(128) when the floor is active) and takes the index from the decision
// polynomial, 3 + ceil(Q(x_i)) (tq3_common.cuh). The rounding of x and the polynomial's fp32
// evaluation move each boundary by a few 1e-7 in xs, so an index can differ from the step-by-step
// result only for a coefficient within 1e-6 of a boundary (ties included). Norms come from an fp32 sum of
// squares (within 1e-6 relative), scales = max(RN(RN(max|z| / norm) * c), 1e-8). A vector whose
// fp32 sum of squares is not finite (|x| beyond about 1e19, where the unnormalised transform can
// itself overflow although the page's normalised one does not) is encoded by the page's steps
// instead, from global memory (tq3::encode_vector_exact).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "tq3_common.cuh"
#include "tq3_rows.cuh"

namespace wq {
namespace tq3_rows {

using tq3::SignMask;

constexpr int kTile = 32;                // vectors per tile = threads per CTA (one warp)
constexpr int kThreads = kTile;
constexpr int kBoxBytes = kTile * 128;   // one 128-byte-wide TMA box of a tile
constexpr int kMinBlocks = 12;           // CTAs per SM the register budget is sized for
constexpr uint32_t kMaxPolls = 1u << 24;

// Set (sticky) by a kernel whose bounded wait for its TMA tile ran out; read by wq_device_fault.
__device__ unsigned int g_fault;

// Sign carried by element e's register before the first stage: the page's draw when the kernel
// folds its table into the butterflies; -1 when the flips are applied to the data as it is loaded
// (the encoder then loads -s_e x_e, so that every table ends with the same carried sign -1 below).
template <bool kFold>
__host__ __device__ constexpr int sg(int e) {
    return kFold ? tq3::default_sign(e) : -1;
}
// Before stage h the register at index i holds s_j * (true value), j = i & ~(h - 1).
template <bool kFold>
__host__ __device__ constexpr int carried(int h, int i) {
    return sg<kFold>(i & ~(h - 1));
}
// Stage h on (i, i + h): the true pair is (c_i r_i, c_{i+h} r_{i+h}); the sum c_i (r_i + sigma
// r_{i+h}) and the difference c_i (r_i - sigma r_{i+h}) both carry c_i, sigma = c_i c_{i+h}.
template <bool kFold>
__host__ __device__ constexpr int sigma(int h, int i) {
    return carried<kFold>(h, i) * carried<kFold>(h, i + h);
}

// Stages h = 1 .. 32 on the register pairs, with the carried signs as compile-time choices
// between a + b, a - b and a + (+-1) b (one rounding each, like an addition).
template <bool kFold>
__device__ __forceinline__ void stages_1_32(f32x2 (&P)[64]) {
    const f32x2 PM = pk2(1.0f, -1.0f), MP = pk2(-1.0f, 1.0f);
#pragma unroll
    for (int h = 1; h <= 32; h <<= 1)
#pragma unroll
        for (int k = 0; k < 64; ++k)
            if ((k & h) == 0) {
                const int sx = sigma<kFold>(h, k), sy = sigma<kFold>(h, k + 64);
                const f32x2 A = P[k], B = P[k + h];
                if (sx == 1 && sy == 1) {
                    P[k] = add2(A, B);
                    P[k + h] = sub2(A, B);
                } else if (sx == -1 && sy == -1) {
                    P[k] = sub2(A, B);
                    P[k + h] = add2(A, B);
                } else if (sx == 1) {
                    P[k] = fma2(B, PM, A);
                    P[k + h] = fma2(B, MP, A);
                } else {
                    P[k] = fma2(B, MP, A);
                    P[k + h] = fma2(B, PM, A);
                }
            }
}

// ---------------------------------------------------------------------------------------------
// Encoder
// ---------------------------------------------------------------------------------------------
template <bool kBf16>
struct EncGeo {
    static constexpr int kBoxes = kBf16 ? 2 : 4;
    static constexpr int kStages = kBf16 ? 2 : 1;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;
    static constexpr int kFlipWords = kBf16 ? 64 : 128;
    static constexpr int kBarOff = kStages * kTileBytes;
    static constexpr int kFlipOff = kBarOff + 64;
    static constexpr int kSmem = 1024 + kFlipOff + 4 * kFlipWords;
};

// kLay (tq3::Layout): kSoA writes packed, norms and scales; kAoS writes 56-byte records at
// `packed`; kPool writes record v to slot pm.index[v] of the pool at `packed` (here and in
// decode_rows, norms and scales are unused for the record layouts).
template <bool kBf16, bool kFold, int kLay = tq3::kSoA>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    encode_rows(int64_t n_vec, const __grid_constant__ CUtensorMap tmap, const void *__restrict__ x, SignMask mask,
                uint8_t *__restrict__ packed, float *__restrict__ norms, float *__restrict__ scales, tq3::PoolMap pm) {
    using G = EncGeo<kBf16>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *const base = tq3::tile_base(smem_raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + G::kBarOff);
    uint32_t *flipw = reinterpret_cast<uint32_t *>(base + G::kFlipOff);
    const int tid = threadIdx.x;
    const int64_t n_tiles = (n_vec + kTile - 1) / kTile;
    const int64_t my_tiles = (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

    if (!kFold) {
        // sign-bit XOR words giving -s_e x_e: bf16 pairs (2i, 2i + 1) in bits 15 and 31, or one
        // fp32 per word
        for (int i = tid; i < G::kFlipWords; i += kThreads) {
            if (kBf16) {
                const uint32_t b = (mask.w[i >> 4] >> ((2 * i) & 31)) & 3u;
                flipw[i] = ((b & 1u) << 15) | ((b & 2u) << 30);
            } else {
                flipw[i] = ((mask.w[i >> 5] >> (i & 31)) & 1u) << 31;
            }
        }
    }
    if (tid == 0) {
        for (int s = 0; s < G::kStages; ++s) mbar_init(&full[s], 1);
    }
    __syncthreads();
    auto issue = [&](int64_t i) {  // load this CTA's i-th tile into stage i % kStages
        uint64_t *bar = &full[i % G::kStages];
        unsigned char *dst = base + (i % G::kStages) * G::kTileBytes;
        const int y = (int)((blockIdx.x + i * gridDim.x) * kTile);
        fence_proxy_async_smem();  // the stage's earlier generic-proxy reads come first
        mbar_expect_tx(bar, G::kTileBytes);
#pragma unroll
        for (int b = 0; b < G::kBoxes; ++b) tma_load_2d(dst + b * kBoxBytes, &tmap, b * (kBf16 ? 64 : 32), y, bar);
    };
    if (tid == 0)
        for (int64_t i = 0; i < G::kStages && i < my_tiles; ++i) issue(i);

    const float post = tq3::fwht_post();
    for (int64_t it = 0; it < my_tiles; ++it) {
        const int st = (int)(it % G::kStages);
        const uint32_t phase = (uint32_t)((it / G::kStages) & 1);
        if (__syncthreads_or(!mbar_wait_bounded(&full[st], phase, kMaxPolls))) {
            if (tid == 0) {
                atomicOr(&g_fault, 1u);
                // let copies already issued land before the CTA's shared memory goes away
                for (int64_t i = it + 1; i < it + G::kStages && i < my_tiles; ++i)
                    mbar_wait_bounded(&full[i % G::kStages], (uint32_t)((i / G::kStages) & 1), kMaxPolls);
            }
            return;
        }
        // x.float() (with the flips if they are not folded), as register pairs (k, k + 64)
        f32x2 P[64];
        const unsigned char *sb = base + st * G::kTileBytes;
        if (kBf16) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 q0 = *reinterpret_cast<const uint4 *>(tq3::swz(const_cast<unsigned char *>(sb), tid, j));
                const uint4 q1 =
                    *reinterpret_cast<const uint4 *>(tq3::swz(const_cast<unsigned char *>(sb) + kBoxBytes, tid, j));
                uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w}, w1[4] = {q1.x, q1.y, q1.z, q1.w};
                if (!kFold) {
                    const uint4 f0 = *reinterpret_cast<const uint4 *>(flipw + 4 * j);
                    const uint4 f1 = *reinterpret_cast<const uint4 *>(flipw + 32 + 4 * j);
                    w0[0] ^= f0.x; w0[1] ^= f0.y; w0[2] ^= f0.z; w0[3] ^= f0.w;
                    w1[0] ^= f1.x; w1[1] ^= f1.y; w1[2] ^= f1.z; w1[3] ^= f1.w;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    P[8 * j + 2 * u] = pk2(__uint_as_float(__byte_perm(w0[u], 0u, 0x1044)),
                                           __uint_as_float(__byte_perm(w1[u], 0u, 0x1044)));
                    P[8 * j + 2 * u + 1] = pk2(__uint_as_float(__byte_perm(w0[u], 0u, 0x3244)),
                                               __uint_as_float(__byte_perm(w1[u], 0u, 0x3244)));
                }
            }
        } else {
#pragma unroll
            for (int bb = 0; bb < 2; ++bb)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    unsigned char *s0 = const_cast<unsigned char *>(sb);
                    const uint4 q0 = *reinterpret_cast<const uint4 *>(tq3::swz(s0 + bb * kBoxBytes, tid, j));
                    const uint4 q1 = *reinterpret_cast<const uint4 *>(tq3::swz(s0 + (2 + bb) * kBoxBytes, tid, j));
                    uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w}, w1[4] = {q1.x, q1.y, q1.z, q1.w};
                    const int k0 = 32 * bb + 4 * j;
                    if (!kFold) {
                        const uint4 f0 = *reinterpret_cast<const uint4 *>(flipw + k0);
                        const uint4 f1 = *reinterpret_cast<const uint4 *>(flipw + 64 + k0);
                        w0[0] ^= f0.x; w0[1] ^= f0.y; w0[2] ^= f0.z; w0[3] ^= f0.w;
                        w1[0] ^= f1.x; w1[1] ^= f1.y; w1[2] ^= f1.z; w1[3] ^= f1.w;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) P[k0 + u] = pk2(__uint_as_float(w0[u]), __uint_as_float(w1[u]));
                }
        }
        __syncthreads();  // every thread has its row: the stage can take the tile after next
        if (tid == 0 && it + G::kStages < my_tiles) issue(it + G::kStages);

        // sum of squares (fp32, eight partial sums)
        f32x2 acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int k = 0; k < 64; ++k) acc[k & 3] = fma2(P[k], P[k], acc[k & 3]);
        float n2;
        {
            float a0, a1;
            upk2(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), a0, a1);
            n2 = __fadd_rn(a0, a1);
        }

        // z = -(true fwht): stages 1 .. 32, then stage 64 with the carried sign and the final
        // negation folded into its operands (an exact cancellation gives z = +0, i.e. a true -0)
        stages_1_32<kFold>(P);
        {
            constexpr int F = sg<kFold>(0), S64 = sg<kFold>(0) * sg<kFold>(64);
#pragma unroll
            for (int k = 0; k < 64; ++k) {
                float a, b;
                upk2(P[k], a, b);
                const float aa = (F == 1) ? -a : a;
                const float bb = (F * S64 == 1) ? -b : b;
                P[k] = pk2(__fadd_rn(aa, bb), __fsub_rn(aa, bb));
            }
        }
        float mm[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int k = 0; k < 64; ++k) {
            float a, b;
            upk2(P[k], a, b);
            mm[k & 3] = max3(mm[k & 3], fabsf(a), fabsf(b));
        }
        const float m = fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3]));

        // norm, scale and the |z| thresholds. A vector whose fp32 squares overflowed (|x| beyond
        // about 1e19; z itself may have overflowed) is re-encoded step by step at the store below.
        const bool big = !(n2 <= 3.0e38f);
        const float nrm = fmaxf(__fsqrt_rn(n2), 1e-8f);
        const float sraw = __fmul_rn(__fdiv_rn(m, nrm), post);
        const float scale = fmaxf(sraw, 1e-8f);
        const float T = (sraw >= 1e-8f) ? m : __fmul_rn(__fmul_rn(1e-8f, nrm), 11.3137085f);
        // the indices by the decision polynomial (tq3::q_coef): x = u / T with u = -z, the true
        // coefficient, then idx = 3 + ceil(Q(x)), accumulated as 8^j-weighted fp32 words (exact
        // integers below 2^24); the low half of W[g] is group g, the high half group g + 8
        const f32x2 NR = pk2(-__frcp_rn(T), -__frcp_rn(T));
        const f32x2 Q1 = pk2(tq3::q_coef(1), tq3::q_coef(1)), Q3 = pk2(tq3::q_coef(3), tq3::q_coef(3)),
                    Q5 = pk2(tq3::q_coef(5), tq3::q_coef(5));
        const f32x2 KK = pk2(8388612.0f, 8388612.0f), NC = pk2(-8388609.0f, -8388609.0f);
        f32x2 W[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) W[g] = 0ull;
#pragma unroll
        for (int kk = 0; kk < 64; ++kk) {
            // slot-major order: consecutive steps update different words (independent chains)
            const int j = kk >> 3, k = 8 * (kk & 7) + j;
            const float w8s = __uint_as_float((127u + 3u * j) << 23);  // 8^j
            const f32x2 x = mul2(P[k], NR);
            const f32x2 x2 = mul2(x, x);
            const f32x2 h = fma2(fma2(Q5, x2, Q3), x2, Q1);
            const f32x2 idx = add2(tq3::fma2_rp(h, x, KK), NC);  // 3 + ceil(Q(x))
            W[k >> 3] = fma2(pk2(w8s, w8s), idx, W[k >> 3]);
        }
        const int64_t v = (blockIdx.x + it * gridDim.x) * kTile + tid;
        if (v < n_vec) {
            int64_t slot = v;
            if constexpr (kLay == tq3::kPool) slot = __ldg(static_cast<const int64_t *>(pm.index) + v);
            uint32_t g[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float lo, hi;
                upk2(W[q], lo, hi);
                g[q] = __float2uint_rn(lo);
                g[q + 8] = __float2uint_rn(hi);
            }
            // _pack_3bit: group i = bytes 3i .. 3i + 2 of the record, little-endian
            uint32_t o[12];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                o[3 * q] = g[4 * q] | (g[4 * q + 1] << 24);
                o[3 * q + 1] = (g[4 * q + 1] >> 8) | (g[4 * q + 2] << 16);
                o[3 * q + 2] = (g[4 * q + 2] >> 16) | (g[4 * q + 3] << 8);
            }
            if constexpr (kLay != tq3::kSoA) {  // a 56-byte record is 8-byte aligned
                if (kLay == tq3::kPool && slot >= pm.n_pool) atomicOr(&g_fault, tq3::kFaultPoolIndex);
                if (kLay == tq3::kAoS || (slot >= 0 && slot < pm.n_pool)) {
                    uint8_t *rec = packed + slot * 56;
                    if (big) {
                        tq3::encode_vector_exact(x, kBf16, v, mask, rec, reinterpret_cast<float *>(rec + 48),
                                                 reinterpret_cast<float *>(rec + 52));
                    } else {
#pragma unroll
                        for (int q = 0; q < 6; ++q) st_stream8(rec + 8 * q, make_uint2(o[2 * q], o[2 * q + 1]));
                        st_stream8(rec + 48, make_uint2(__float_as_uint(nrm), __float_as_uint(scale)));
                    }
                }
            } else {
                uint8_t *rec = packed + v * 48;
                if (big) {
                    tq3::encode_vector_exact(x, kBf16, v, mask, rec, norms + v, scales + v);
                } else {
                    st_stream16(rec, make_uint4(o[0], o[1], o[2], o[3]));
                    st_stream16(rec + 16, make_uint4(o[4], o[5], o[6], o[7]));
                    st_stream16(rec + 32, make_uint4(o[8], o[9], o[10], o[11]));
                    norms[v] = nrm;
                    scales[v] = scale;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Decoder
// ---------------------------------------------------------------------------------------------
struct Rec {
    uint4 q[3];
    float n, s;
};

// Page-table entry of logical vector p (launch-relative, inside the launch).
__device__ __forceinline__ int32_t page_of(const tq3::PoolMap &pm, int64_t p) {
    return __ldg(static_cast<const int32_t *>(pm.index) + ((pm.v0 + p) >> pm.shift));
}

// Record of logical vector p (launch-relative) whose page-table entry is `page`, or -1 (and the
// fault bit) for an entry outside the pool.
__device__ __forceinline__ int64_t pool_record(const tq3::PoolMap &pm, int64_t p, int32_t page) {
    const int64_t lp = pm.v0 + p;
    const int64_t r = ((int64_t)page << pm.shift) | (lp & ((int64_t(1) << pm.shift) - 1));
    if (page < 0 || r >= pm.n_pool) {
        atomicOr(&g_fault, tq3::kFaultPoolIndex);
        return -1;
    }
    return r;
}

// The record of vector v (launch-relative; zeros past n_vec). In the pool layout `page` is v's
// page-table entry, read ahead by the caller.
template <int kLay>
__device__ __forceinline__ Rec load_rec(const uint8_t *__restrict__ packed, const float *__restrict__ norms,
                                        const float *__restrict__ scales, int64_t n_vec, int64_t v,
                                        const tq3::PoolMap &pm, int32_t page) {
    Rec r;
    int64_t at = v < n_vec ? v : -1;
    if constexpr (kLay == tq3::kPool)
        if (at >= 0) at = pool_record(pm, v, page);
    if (at >= 0) {
        if constexpr (kLay != tq3::kSoA) {  // a 56-byte record is 8-byte aligned
            const uint8_t *p = packed + at * 56;
            uint2 w[7];
#pragma unroll
            for (int q = 0; q < 7; ++q) w[q] = __ldg(reinterpret_cast<const uint2 *>(p) + q);
            r.q[0] = make_uint4(w[0].x, w[0].y, w[1].x, w[1].y);
            r.q[1] = make_uint4(w[2].x, w[2].y, w[3].x, w[3].y);
            r.q[2] = make_uint4(w[4].x, w[4].y, w[5].x, w[5].y);
            r.n = __uint_as_float(w[6].x);
            r.s = __uint_as_float(w[6].y);
        } else {
            const uint8_t *p = packed + v * 48;
            r.q[0] = ld_nc16(p);
            r.q[1] = ld_nc16(p + 16);
            r.q[2] = ld_nc16(p + 32);
            r.n = __ldg(norms + v);
            r.s = __ldg(scales + v);
        }
    } else {
        r.q[0] = r.q[1] = r.q[2] = make_uint4(0u, 0u, 0u, 0u);
        r.n = r.s = 0.0f;
    }
    return r;
}

template <bool kBf16>
struct DecGeo {
    static constexpr int kBoxes = kBf16 ? 2 : 4;
    static constexpr int kBufs = kBf16 ? 2 : 1;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;
    static constexpr int kSmem = 1024 + kBufs * kTileBytes;
};

template <bool kBf16Out, bool kFold, int kLay = tq3::kSoA>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    decode_rows(const uint8_t *__restrict__ packed, const float *__restrict__ norms, const float *__restrict__ scales,
                int64_t n_vec, SignMask mask, const __grid_constant__ CUtensorMap omap, tq3::PoolMap pm) {
    using G = DecGeo<kBf16Out>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *const obuf = tq3::tile_base(smem_raw);
    const int tid = threadIdx.x;
    // lane l holds TQ3_CENTROIDS[l & 7]: a shuffle whose source lane has the index in its low
    // three bits is the table lookup
    const float cb = tq3::centroid(tid & 7);
    const int64_t n_tiles = (n_vec + kTile - 1) / kTile;
    const float post = tq3::fwht_post();

    int64_t tile = blockIdx.x;
    const bool pf_ok = ((reinterpret_cast<uintptr_t>(packed) | reinterpret_cast<uintptr_t>(norms) |
                         reinterpret_cast<uintptr_t>(scales)) & 15) == 0;
    // Paged pool: the records of a tile two rounds ahead are prefetched page by page. With pages of
    // 4 to 16 records a tile covers 32 >> shift whole pages (tiles start on multiples of 32), lane l
    // taking page l; with 32 or more, one page, lane 0. A lane reads its page-table entry one round
    // before the prefetch that needs it, so no lane waits on that read.
    const int pf_lanes = kLay != tq3::kPool ? 0 : pm.shift >= 5 ? 1 : pm.shift >= 2 ? (kTile >> pm.shift) : 0;
    auto page_entry = [&](int64_t t) -> int32_t {  // this lane's page-table entry for tile t, or -1
        if constexpr (kLay == tq3::kPool) {
            const int64_t first = pm.shift >= 5 ? 0 : (int64_t)tid << pm.shift;
            if (tid < pf_lanes && t < n_tiles && t * kTile + first < n_vec)
                return __ldg(static_cast<const int32_t *>(pm.index) + ((pm.v0 + t * kTile + first) >> pm.shift));
        }
        return -1;
    };
    // pool layout: the page-table entry of this thread's vector in a tile, read one round before
    // the record load that needs it
    auto vec_page = [&](int64_t t) -> int32_t {
        if constexpr (kLay == tq3::kPool) {
            const int64_t v = t * kTile + tid;
            if (v < n_vec) return page_of(pm, v);
        }
        return -1;
    };
    pdl_wait();  // the records may come from the kernel before this one
    Rec cur = load_rec<kLay>(packed, norms, scales, n_vec, tile * kTile + tid, pm, vec_page(tile));
    int32_t pv = vec_page(tile + gridDim.x);
    int32_t pe = page_entry(tile + 2 * (int64_t)gridDim.x);
    for (int it = 0; tile < n_tiles; ++it, tile += gridDim.x) {
        // on its last tile the block lets the next kernel in the stream be scheduled: its set-up
        // overlaps this kernel's tail (it still waits for this kernel to finish before reading)
        if (tile + gridDim.x >= n_tiles) pdl_trigger();
        const Rec nxt = load_rec<kLay>(packed, norms, scales, n_vec, (tile + gridDim.x) * kTile + tid, pm, pv);
        pv = vec_page(tile + 2 * (int64_t)gridDim.x);
        // the records of the tile after that go into L2 now, so next iteration's load finds them
        // there (whole 16-byte units inside the arrays only)
        if constexpr (kLay == tq3::kPool) {
            // a page's run of records starts on a 16-byte boundary and spans a multiple of 4 records:
            // its first record is a multiple of 4 (page << shift, plus a multiple of 32 inside pages of
            // 32 or more), and 56 * 4 = 224
            const int32_t pe_next = page_entry(tile + 3 * (int64_t)gridDim.x);
            if (pf_ok && pe >= 0) {
                const int64_t v0 = (tile + 2 * gridDim.x) * kTile;
                const int64_t cnt = (n_vec - v0 < kTile ? n_vec - v0 : kTile) & ~int64_t(3);
                const int64_t first = pm.shift >= 5 ? 0 : (int64_t)tid << pm.shift;
                const int64_t per = pm.shift >= 5 ? kTile : (int64_t(1) << pm.shift);
                const int64_t c = cnt - first < per ? cnt - first : per;
                const int64_t lp = pm.v0 + v0 + first;
                const int64_t r0 = ((int64_t)pe << pm.shift) | (lp & ((int64_t(1) << pm.shift) - 1));
                if (c > 0 && r0 + c <= pm.n_pool) bulk_prefetch_l2(packed + r0 * 56, (uint32_t)(c * 56));
            }
            pe = pe_next;
        } else if (tid == 0 && pf_ok && tile + 2 * gridDim.x < n_tiles) {
            const int64_t v0 = (tile + 2 * gridDim.x) * kTile;
            const int64_t cnt = (n_vec - v0 < kTile ? n_vec - v0 : kTile) & ~int64_t(3);
            if (cnt > 0) {
                if constexpr (kLay == tq3::kAoS) {
                    bulk_prefetch_l2(packed + v0 * 56, (uint32_t)(cnt * 56));
                } else {
                    // the packed bytes only: prefetching the tile's 128-byte runs of norms and
                    // scales as well measured 2.2 us slower per launch on the KV cache
                    bulk_prefetch_l2(packed + v0 * 48, (uint32_t)(cnt * 48));
                }
            }
        }
        unsigned char *buf = obuf + (it % G::kBufs) * G::kTileBytes;
        if (tid == 0) bulk_wait_read<G::kBufs - 1>();  // the store that last read this buffer is done
        __syncthreads();
        const uint32_t W[12] = {cur.q[0].x, cur.q[0].y, cur.q[0].z, cur.q[0].w, cur.q[1].x, cur.q[1].y,
                                cur.q[1].z, cur.q[1].w, cur.q[2].x, cur.q[2].y, cur.q[2].z, cur.q[2].w};
        // _unpack_3bit + centroids[idx] * scale: element e's index is bits 3e .. 3e + 2 of the
        // little-endian record
        float v[128];
#pragma unroll
        for (int e = 0; e < 128; ++e) {
            const int o = 3 * e, q = o >> 5, sh = o & 31;
            const uint32_t sel = sh == 0 ? W[q] : sh <= 29 ? (W[q] >> sh) : __funnelshift_r(W[q], W[q + 1], sh);
            v[e] = __shfl_sync(0xffffffffu, cb, (int)sel);
        }
        // Register pairs (2k, 2k + 1) here: stage 1 is the scalar butterfly inside each pair and
        // stages 2 .. 64 are packed operations between registers. (A packed product that feeds a
        // packed addition can be contracted into one fused operation by the compiler, which would
        // skip the rounding of centroid * scale; no packed addition here reads a product.)
        f32x2 P[64];
        {
            const f32x2 S2 = pk2(cur.s, cur.s);
#pragma unroll
            for (int k = 0; k < 64; ++k) {
                float a, b;
                upk2(mul2(pk2(v[2 * k], v[2 * k + 1]), S2), a, b);
                P[k] = pk2(__fadd_rn(a, b), __fsub_rn(a, b));
            }
        }
#pragma unroll
        for (int hp = 1; hp <= 32; hp <<= 1)  // stage h = 2 hp: register k with register k + hp
#pragma unroll
            for (int k = 0; k < 64; ++k)
                if ((k & hp) == 0) {
                    const f32x2 A = P[k], B = P[k + hp];
                    P[k] = add2(A, B);
                    P[k + hp] = sub2(A, B);
                }
        // * post, then * (s_i * norm): the flip is exact, so it rides on the norm's sign
        {
            const f32x2 C2 = pk2(post, post);
            const float n = cur.n;
            f32x2 NS[4];
            if (kFold) {
                NS[0] = pk2(n, n);
                NS[1] = pk2(n, -n);
                NS[2] = pk2(-n, n);
                NS[3] = pk2(-n, -n);
            }
#pragma unroll
            for (int k = 0; k < 64; ++k) {
                f32x2 N2;
                if (kFold) {
                    N2 = NS[(tq3::default_sign(2 * k) < 0 ? 2 : 0) + (tq3::default_sign(2 * k + 1) < 0 ? 1 : 0)];
                } else {
                    const uint32_t fb = ~mask.w[k >> 4] >> ((2 * k) & 31);
                    N2 = pk2(__uint_as_float(__float_as_uint(n) ^ ((fb & 1u) << 31)),
                             __uint_as_float(__float_as_uint(n) ^ ((fb & 2u) << 30)));
                }
                P[k] = mul2(mul2(P[k], C2), N2);
            }
        }
        // stage the tile (row = vector, 128-byte swizzle) and write it with TMA stores
        if (kBf16Out) {
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t o[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {  // elements 64 b + 8 j + 2 u, + 1
                        float x0, x1;
                        upk2(P[32 * b + 4 * j + u], x0, x1);
                        o[u] = pack_bf16x2(x0, x1);
                    }
                    *reinterpret_cast<uint4 *>(tq3::swz(buf + b * kBoxBytes, tid, j)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int j = 0; j < 8; ++j) {  // elements 32 b + 4 j .. + 3
                    float o[4];
                    upk2(P[16 * b + 2 * j], o[0], o[1]);
                    upk2(P[16 * b + 2 * j + 1], o[2], o[3]);
                    *reinterpret_cast<float4 *>(tq3::swz(buf + b * kBoxBytes, tid, j)) = make_float4(o[0], o[1], o[2], o[3]);
                }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            // decoded output is written once and read by a later kernel: evict it from L2 first
            const uint64_t pol = l2_evict_first_policy();
#pragma unroll
            for (int b = 0; b < G::kBoxes; ++b)
                tma_store_2d_hint(&omap, b * (kBf16Out ? 64 : 32), (int)(tile * kTile), buf + b * kBoxBytes, pol);
            bulk_commit();
        }
        cur = nxt;
    }
    if (tid == 0) bulk_wait_all<0>();
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
    return cached[dev];
}

// Persistent grid: as many CTAs as fit on the GPU at once, never more than there are tiles.
template <typename K>
int grid_for(K k, size_t smem, int64_t tiles) {
    int per_sm = blocks_per_sm_cached(reinterpret_cast<const void *>(k), kThreads, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t g = (int64_t)per_sm * (sm_count() > 0 ? sm_count() : 1);
    return (int)(g < tiles ? g : tiles);
}

template <typename K>
wq_status launch_enc(K k, size_t smem, int64_t cnt, const CUtensorMap &tm, const void *xc, const SignMask &m,
                     uint8_t *pc, float *nc, float *sc, const tq3::PoolMap &pm, cudaStream_t s) {
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return WQ_ERR_CUDA;
    const int64_t tiles = (cnt + kTile - 1) / kTile;
    k<<<grid_for(k, smem, tiles), kThreads, smem, s>>>(cnt, tm, xc, m, pc, nc, sc, pm);
    return launch_status();
}

template <int kLay>
wq_status launch_enc_lay(bool bf, bool def, size_t smem, int64_t cnt, const CUtensorMap &tm, const void *xc,
                         const SignMask &m, uint8_t *pc, float *nc, float *sc, const tq3::PoolMap &pm,
                         cudaStream_t s) {
    if (bf)
        return def ? launch_enc(encode_rows<true, true, kLay>, smem, cnt, tm, xc, m, pc, nc, sc, pm, s)
                   : launch_enc(encode_rows<true, false, kLay>, smem, cnt, tm, xc, m, pc, nc, sc, pm, s);
    return def ? launch_enc(encode_rows<false, true, kLay>, smem, cnt, tm, xc, m, pc, nc, sc, pm, s)
               : launch_enc(encode_rows<false, false, kLay>, smem, cnt, tm, xc, m, pc, nc, sc, pm, s);
}

wq_status encode(const void *x, int x_dtype, int64_t n_vec, const SignMask &m, uint8_t *packed, float *norms,
                 float *scales, cudaStream_t s, int layout, const tq3::PoolMap &pool) {
    const bool def = tq3::is_default(m), bf = x_dtype == WQ_BF16;
    const int esz = bf ? 2 : 4;
    const size_t smem = bf ? EncGeo<true>::kSmem : EncGeo<false>::kSmem;
    for (int64_t off = 0; off < n_vec; off += tq3::kMaxChunk) {
        const int64_t cnt = n_vec - off < tq3::kMaxChunk ? n_vec - off : tq3::kMaxChunk;
        const unsigned char *xc = static_cast<const unsigned char *>(x) + off * (tq3::kD * esz);
        CUtensorMap tm;
        if (!make_tmap_2d(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, xc, tq3::kD,
                          (uint64_t)cnt, tq3::kD * esz, bf ? 64 : 32, kTile))
            return WQ_ERR_CUDA;
        wq_status st;
        if (layout == tq3::kPool) {  // the pool is not offset; the chunk's slots are
            tq3::PoolMap pm = pool;
            pm.index = static_cast<const int64_t *>(pool.index) + off;
            st = launch_enc_lay<tq3::kPool>(bf, def, smem, cnt, tm, xc, m, packed, nullptr, nullptr, pm, s);
        } else if (layout == tq3::kAoS) {
            st = launch_enc_lay<tq3::kAoS>(bf, def, smem, cnt, tm, xc, m, packed + off * 56, nullptr, nullptr, pool,
                                           s);
        } else {
            st = launch_enc_lay<tq3::kSoA>(bf, def, smem, cnt, tm, xc, m, packed + off * 48, norms + off,
                                           scales + off, pool, s);
        }
        if (st != WQ_OK) return st;
    }
    return WQ_OK;
}

template <typename K>
wq_status launch_dec(K k, size_t smem, const uint8_t *pc, const float *nc, const float *sc, int64_t cnt,
                     const SignMask &m, const CUtensorMap &tm, const tq3::PoolMap &pm, cudaStream_t s) {
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return WQ_ERR_CUDA;
    const int64_t tiles = (cnt + kTile - 1) / kTile;
    k<<<grid_for(k, smem, tiles), kThreads, smem, s>>>(pc, nc, sc, cnt, m, tm, pm);
    return launch_status();
}

template <int kLay>
wq_status launch_dec_lay(bool bf, bool def, size_t smem, const uint8_t *pc, const float *nc, const float *sc,
                         int64_t cnt, const SignMask &m, const CUtensorMap &tm, const tq3::PoolMap &pm,
                         cudaStream_t s) {
    if (bf)
        return def ? launch_dec(decode_rows<true, true, kLay>, smem, pc, nc, sc, cnt, m, tm, pm, s)
                   : launch_dec(decode_rows<true, false, kLay>, smem, pc, nc, sc, cnt, m, tm, pm, s);
    return def ? launch_dec(decode_rows<false, true, kLay>, smem, pc, nc, sc, cnt, m, tm, pm, s)
               : launch_dec(decode_rows<false, false, kLay>, smem, pc, nc, sc, cnt, m, tm, pm, s);
}

wq_status decode(const uint8_t *packed, const float *norms, const float *scales, int64_t n_vec, const SignMask &m,
                 void *out, int out_dtype, cudaStream_t s, int layout, const tq3::PoolMap &pool) {
    const bool def = tq3::is_default(m), bf = out_dtype == WQ_BF16;
    const int esz = bf ? 2 : 4;
    const size_t smem = bf ? DecGeo<true>::kSmem : DecGeo<false>::kSmem;
    for (int64_t off = 0; off < n_vec; off += tq3::kMaxChunk) {
        const int64_t cnt = n_vec - off < tq3::kMaxChunk ? n_vec - off : tq3::kMaxChunk;
        unsigned char *oc = static_cast<unsigned char *>(out) + off * (tq3::kD * esz);
        CUtensorMap tm;
        if (!make_tmap_2d(&tm, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, oc, tq3::kD,
                          (uint64_t)cnt, tq3::kD * esz, bf ? 64 : 32, kTile))
            return WQ_ERR_CUDA;
        wq_status st;
        if (layout == tq3::kPool) {  // the pool is not offset; the page-table position is
            tq3::PoolMap pm = pool;
            pm.v0 = pool.v0 + off;
            st = launch_dec_lay<tq3::kPool>(bf, def, smem, packed, nullptr, nullptr, cnt, m, tm, pm, s);
        } else if (layout == tq3::kAoS) {
            st = launch_dec_lay<tq3::kAoS>(bf, def, smem, packed + off * 56, nullptr, nullptr, cnt, m, tm, pool, s);
        } else {
            st = launch_dec_lay<tq3::kSoA>(bf, def, smem, packed + off * 48, norms + off, scales + off, cnt, m, tm,
                                           pool, s);
        }
        if (st != WQ_OK) return st;
    }
    return WQ_OK;
}

unsigned int read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(g_fault, &zero, sizeof zero);
    return v;
}

}  // namespace tq3_rows
}  // namespace wq
