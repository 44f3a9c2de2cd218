// Register-blocked RPBH kernels on sm_100a: page "orbit_quant.py" (rpbh_forward, _fwht,
// _quantize_rows, pack_codes, unpack_codes, dequantize / rpbh_inverse).
//
// For a Hadamard block h = 2^(2B) each h-block is viewed as an S x S matrix (S = 2^B, element
// k = row * S + col). Butterfly stages 1 .. S/2 act on the column index and stages S .. h/2 on
// the row index, so the block FWHT is two passes of in-register butterflies over S values:
//   pass 0: one thread takes one matrix row (S contiguous elements), gathers them through the
//           permutation from the row staged in shared memory, applies the signs and the first B
//           stages, and writes the row to a transpose buffer;
//   pass 1: one thread takes one matrix column, applies the remaining B stages and the epilogue.
// Stages stay in the page's order (h = 1, 2, 4, ...) and every butterfly is one IEEE add or
// subtract, so results match the stage-by-stage definition bit for bit. The transpose buffer
// swizzles 16-byte chunks by row (and flips the row parity of odd blocks when S < 32) so that
// pass 0's 16-byte stores and pass 1's 4-byte loads are free of shared-memory bank conflicts.
// One CTA owns one weight/activation row; the row norm of the quantizer is a CTA reduction.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "common.cuh"
#include "rpbh_edges.cuh"
#include "rpbh_fast.cuh"
#include "rpbh_lanes.cuh"

namespace wq {
namespace rpbh_fast {

constexpr int kMaxThreads = 256;

template <int B>
struct Geo {
    static constexpr int S = 1 << B;
    static constexpr int H = 1 << (2 * B);
    static constexpr int NCH = S / 4;
    static constexpr bool kParity = S < 32;
};

template <int B>
__device__ __forceinline__ int chunk_swz(int row) {
    return B == 3 ? ((row >> 2) & 1) : B == 4 ? ((row >> 1) & 3) : (row & 7);
}

// Physical float index of element (row, col) of h-block `blk` in the transpose buffer.
template <int B>
__device__ __forceinline__ int bufpos(int blk, int row, int col) {
    using G = Geo<B>;
    const int prow = G::kParity ? (row ^ (blk & 1)) : row;
    const int ch = (col >> 2) ^ (chunk_swz<B>(row) & (G::NCH - 1));
    return blk * G::H + prow * G::S + ch * 4 + (col & 3);
}

// Stages 1, 2, ..., S/2 of the butterfly on S register values; pairs are packed two at a time
// from the second stage on.
template <int S>
__device__ __forceinline__ void butterfly(float (&y)[S]) {
#pragma unroll
    for (int k = 0; k < S; k += 2) {
        const float p = y[k], q = y[k + 1];
        y[k] = __fadd_rn(p, q);
        y[k + 1] = __fsub_rn(p, q);
    }
    f32x2 P[S / 2];
#pragma unroll
    for (int k = 0; k < S / 2; ++k) P[k] = pk2(y[2 * k], y[2 * k + 1]);
#pragma unroll
    for (int hp = 1; hp < S / 2; hp <<= 1)
#pragma unroll
        for (int k = 0; k < S / 2; ++k)
            if ((k & hp) == 0) {
                const f32x2 A = P[k], Bv = P[k + hp];
                P[k] = add2(A, Bv);
                P[k + hp] = sub2(A, Bv);
            }
#pragma unroll
    for (int k = 0; k < S / 2; ++k) upk2(P[k], y[2 * k], y[2 * k + 1]);
}

__device__ __forceinline__ unsigned char *align16(unsigned char *p) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 15) & ~uintptr_t(15));
}

// Copy `bytes` (a multiple of 16) global -> shared with 16-byte accesses.
__device__ __forceinline__ void copy_in(unsigned char *dst, const unsigned char *src, int bytes) {
    for (int c = threadIdx.x; c < bytes / 16; c += blockDim.x)
        *reinterpret_cast<uint4 *>(dst + 16 * c) = ld_stream16(src + 16 * (size_t)c);
}
__device__ __forceinline__ void copy_out(unsigned char *dst, const unsigned char *src, int bytes) {
    for (int c = threadIdx.x; c < bytes / 16; c += blockDim.x)
        st_stream16(dst + 16 * (size_t)c, *reinterpret_cast<const uint4 *>(src + 16 * c));
}

__device__ __forceinline__ int clampi(int32_t p, int d) { return (uint32_t)p < (uint32_t)d ? p : 0; }

// pass 0 for one matrix row: y[t] = x[perm[j0 + t]] * signs[j0 + t], then the first B stages
template <int B, bool kBf16>
__device__ __forceinline__ void gather_row(float (&y)[1 << B], const unsigned char *raw, int j0, int d,
                                           const int32_t *__restrict__ perm, const int8_t *__restrict__ signs) {
    constexpr int S = 1 << B;
    int32_t pi[S];
#pragma unroll
    for (int q = 0; q < S / 4; ++q) {
        const int4 v = __ldg(reinterpret_cast<const int4 *>(perm + j0) + q);
        pi[4 * q] = v.x; pi[4 * q + 1] = v.y; pi[4 * q + 2] = v.z; pi[4 * q + 3] = v.w;
    }
    uint32_t sw[S / 4];
    if (S >= 16) {
#pragma unroll
        for (int q = 0; q < S / 16; ++q) {
            const int4 v = __ldg(reinterpret_cast<const int4 *>(signs + j0) + q);
            sw[4 * q] = v.x; sw[4 * q + 1] = v.y; sw[4 * q + 2] = v.z; sw[4 * q + 3] = v.w;
        }
    } else {
        const int2 v = __ldg(reinterpret_cast<const int2 *>(signs + j0));
        sw[0] = v.x; sw[1] = v.y;
    }
#pragma unroll
    for (int t = 0; t < S; ++t) {
        const int p = clampi(pi[t], d);
        const float xv = kBf16 ? bf16_to_f32(reinterpret_cast<const uint16_t *>(raw)[p])
                               : reinterpret_cast<const float *>(raw)[p];
        const float sg = (float)(int8_t)(sw[t >> 2] >> (8 * (t & 3)));
        y[t] = __fmul_rn(xv, sg);  // index_select(x, perm) * signs (exact)
    }
    butterfly<S>(y);
}

template <int B>
__device__ __forceinline__ void store_row(unsigned char *buf_raw, const float (&y)[1 << B], int blk, int r) {
    constexpr int S = 1 << B;
    float *buf = reinterpret_cast<float *>(buf_raw);
#pragma unroll
    for (int q = 0; q < S / 4; ++q)
        *reinterpret_cast<float4 *>(buf + bufpos<B>(blk, r, 4 * q)) =
            make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
}

template <int B>
__device__ __forceinline__ void load_col(float (&y)[1 << B], const unsigned char *buf_raw, int blk, int c) {
    constexpr int S = 1 << B;
    const float *buf = reinterpret_cast<const float *>(buf_raw);
#pragma unroll
    for (int t = 0; t < S; ++t) y[t] = buf[bufpos<B>(blk, t, c)];
}

// ---------------------------------------------------------------------------------------------
// rpbh_rotate_activations: x_rot = blkdiag(H_h) D P x, computed in fp32, rounded once.
// ---------------------------------------------------------------------------------------------
template <int B, bool kBf16>
__global__ void __launch_bounds__(kMaxThreads)
    rotate_kernel(const void *__restrict__ x, int d, float post, const int32_t *__restrict__ perm,
                  const int8_t *__restrict__ signs, void *__restrict__ out) {
    using G = Geo<B>;
    constexpr int esz = kBf16 ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *raw = align16(smem_raw);
    unsigned char *buf = raw + (size_t)d * esz;
    const int64_t row = blockIdx.x;
    copy_in(raw, static_cast<const unsigned char *>(x) + row * (int64_t)d * esz, d * esz);
    __syncthreads();
    const int nslots = d >> B;
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, r = s & (G::S - 1);
        float y[G::S];
        gather_row<B, kBf16>(y, raw, blk * G::H + r * G::S, d, perm, signs);
        store_row<B>(buf, y, blk, r);
    }
    __syncthreads();
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, c = s & (G::S - 1);
        float y[G::S];
        load_col<B>(y, buf, blk, c);
        butterfly<G::S>(y);
#pragma unroll
        for (int t = 0; t < G::S; ++t) {
            const int j = blk * G::H + c + (t << B);
            const float z = __fmul_rn(y[t], post);
            if (kBf16)
                reinterpret_cast<uint16_t *>(raw)[j] = f32_to_bf16(z);
            else
                reinterpret_cast<float *>(raw)[j] = z;
        }
    }
    __syncthreads();
    copy_out(static_cast<unsigned char *>(out) + row * (int64_t)d * esz, raw, d * esz);
}

// ---------------------------------------------------------------------------------------------
// rpbh_quantize_weight: _quantize_rows
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ double block_sum_f64(double v, double *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = __dadd_rn(t, red[w]);
        red[32] = t;
    }
    __syncthreads();
    return red[32];
}

template <int BITS>
__device__ __forceinline__ void unpack32(const uint32_t (&word)[BITS], uint32_t (&cw)[8]) {
    constexpr uint32_t kMask = (1u << BITS) - 1u;
#pragma unroll
    for (int q = 0; q < 8; ++q) cw[q] = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int o = BITS * i, k = o >> 5, r = o & 31;
        uint32_t c;
        if (r + BITS <= 32)
            c = (word[k] >> (32 - r - BITS)) & kMask;
        else
            c = ((word[k] << (r + BITS - 32)) | (word[k + 1] >> (64 - r - BITS))) & kMask;
        cw[i >> 2] += c << (8 * (i & 3));
    }
}

template <int B, bool kBf16, int BITS, bool kSym>
__global__ void __launch_bounds__(kMaxThreads)
    quantize_kernel(const void *__restrict__ w, int d, float post, const int32_t *__restrict__ perm,
                    const int8_t *__restrict__ signs, Edges E, uint8_t *__restrict__ packed,
                    void *__restrict__ row_norms) {
    using G = Geo<B>;
    constexpr int esz = kBf16 ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    __shared__ double red[33];
    unsigned char *raw = align16(smem_raw);
    unsigned char *buf = raw + (size_t)d * esz;
    const int64_t row = blockIdx.x;
    copy_in(raw, static_cast<const unsigned char *>(w) + row * (int64_t)d * esz, d * esz);
    __syncthreads();
    const int nslots = d >> B;
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, r = s & (G::S - 1);
        float y[G::S];
        gather_row<B, kBf16>(y, raw, blk * G::H + r * G::S, d, perm, signs);
        store_row<B>(buf, y, blk, r);
    }
    __syncthreads();
    // pass 1: w_rot = fwht * h^-0.5, written back in place; fp64 sum of exact squares
    double ss = 0.0;
    float *fb = reinterpret_cast<float *>(buf);
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, c = s & (G::S - 1);
        float y[G::S];
        load_col<B>(y, buf, blk, c);
        butterfly<G::S>(y);
#pragma unroll
        for (int t = 0; t < G::S; ++t) {
            const float z = __fmul_rn(y[t], post);
            fb[bufpos<B>(blk, t, c)] = z;
            const double dz = (double)z;
            ss = __fma_rn(dz, dz, ss);
        }
    }
    // rho = ||w_rot||; unit = w_rot / (rho + 1e-10)
    const float rho = __double2float_rn(__dsqrt_rn(block_sum_f64(ss, red)));
    const float den = __fadd_rn(rho, 1e-10f);
    const float rden = __frcp_rn(den);
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, c = s & (G::S - 1);
#pragma unroll
        for (int t = 0; t < G::S; ++t) {
            const float z = fb[bufpos<B>(blk, t, c)];
            // z / den by Markstein's correction (r = RN(1/den), q0 = RN(z r), e = RN(z - q0 den),
            // RN(q0 + e r)): correctly rounded for |z| >= 2^-100 and a normal quotient
            const float q0 = __fmul_rn(z, rden);
            const float u = __fmaf_rn(__fmaf_rn(-q0, den, z), rden, q0);
            raw[blk * G::H + c + (t << B)] = (uint8_t)bucketize<BITS, kSym>(u, E);
        }
    }
    __syncthreads();
    // pack_codes: 32 codes -> BITS big-endian 32-bit words of the MSB-first stream
    uint8_t *dst = packed + (row * (int64_t)d / 8) * BITS;
    for (int g = threadIdx.x; g < d / 32; g += blockDim.x) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(raw + 32 * g);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(raw + 32 * g + 16);
        const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        uint32_t word[BITS];
        pack32<BITS>(cw, word);
#pragma unroll
        for (int k = 0; k < BITS; ++k) reinterpret_cast<uint32_t *>(dst + 4 * BITS * g)[k] = __byte_perm(word[k], 0, 0x0123);
    }
    if (threadIdx.x == 0) {
        if (E.norm_bf16)
            static_cast<uint16_t *>(row_norms)[row] = f32_to_bf16(rho);
        else
            static_cast<float *>(row_norms)[row] = rho;
    }
}

// ---------------------------------------------------------------------------------------------
// rpbh_dequantize_weight with unrotate: _dequantize_rotated(fp32) then rpbh_inverse
// ---------------------------------------------------------------------------------------------
struct Codebook {
    float c[16];
};

template <int B, bool kNormBf16, bool kOutBf16, int BITS>
__global__ void __launch_bounds__(kMaxThreads)
    dequant_unrotate_kernel(const uint8_t *__restrict__ packed, const void *__restrict__ row_norms, int d,
                            float post, Codebook cb, const int32_t *__restrict__ perm,
                            const int8_t *__restrict__ signs, void *__restrict__ out) {
    using G = Geo<B>;
    constexpr int oesz = kOutBf16 ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    __shared__ float cbs[16];
    unsigned char *codes = align16(smem_raw);
    unsigned char *buf = codes + d;
    unsigned char *stage = buf + (size_t)d * 4;
    const int64_t row = blockIdx.x;
    if (threadIdx.x < (1u << BITS)) cbs[threadIdx.x] = cb.c[threadIdx.x];
    const float rho = kNormBf16 ? bf16_to_f32(static_cast<const uint16_t *>(row_norms)[row])
                                : static_cast<const float *>(row_norms)[row];
    // unpack_codes: BITS big-endian words -> 32 codes
    const uint8_t *src = packed + (row * (int64_t)d / 8) * BITS;
    for (int g = threadIdx.x; g < d / 32; g += blockDim.x) {
        uint32_t word[BITS];
#pragma unroll
        for (int k = 0; k < BITS; ++k)
            word[k] = __byte_perm(__ldg(reinterpret_cast<const uint32_t *>(src + 4 * BITS * g) + k), 0, 0x0123);
        uint32_t cw[8];
        unpack32<BITS>(word, cw);
        *reinterpret_cast<uint4 *>(codes + 32 * g) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4 *>(codes + 32 * g + 16) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    }
    __syncthreads();
    const int nslots = d >> B;
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, r = s & (G::S - 1);
        const int j0 = blk * G::H + r * G::S;
        float y[G::S];
#pragma unroll
        for (int t = 0; t < G::S; ++t) y[t] = __fmul_rn(cbs[codes[j0 + t]], rho);  // W' = codebook[code] * rho
        butterfly<G::S>(y);
        store_row<B>(buf, y, blk, r);
    }
    __syncthreads();
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int blk = s >> B, c = s & (G::S - 1);
        float y[G::S];
        load_col<B>(y, buf, blk, c);
        butterfly<G::S>(y);
#pragma unroll
        for (int t = 0; t < G::S; ++t) {
            const int j = blk * G::H + c + (t << B);
            // z = fwht * h^-0.5 * signs; out[perm[j]] = z
            const float z = __fmul_rn(__fmul_rn(y[t], post), (float)__ldg(signs + j));
            const int p = clampi(__ldg(perm + j), d);
            if (kOutBf16)
                reinterpret_cast<uint16_t *>(stage)[p] = f32_to_bf16(z);
            else
                reinterpret_cast<float *>(stage)[p] = z;
        }
    }
    __syncthreads();
    copy_out(static_cast<unsigned char *>(out) + row * (int64_t)d * oesz, stage, d * oesz);
}

// ---------------------------------------------------------------------------------------------
// Persistent variants: each CTA keeps the permutation (16-bit) and the sign bits in shared memory
// and walks rows blockIdx.x, blockIdx.x + gridDim.x, ...; the next row is fetched with a 1-D bulk
// copy into the other of two row buffers while the current row is processed.
// ---------------------------------------------------------------------------------------------
constexpr uint32_t kMaxPolls = 1u << 24;
__device__ unsigned int g_fault;

__host__ __device__ constexpr int a16(int x) { return (x + 15) & ~15; }

struct PLayout {
    int perm, bits, row0, row1, buf, bar, total;
    __host__ __device__ PLayout(int d, int esz) {
        perm = 0;
        bits = a16(2 * d);
        row0 = bits + a16(d / 8);
        row1 = row0 + d * esz;
        buf = row1 + d * esz;
        bar = buf + 4 * d;  // row barriers 0 and 1, table barrier 2
        total = bar + 32;
    }
};

// pass 0 from the staged row: y[t] = x[perm[j0 + t]] * signs[j0 + t] (the sign as a bit flip)
template <int B, bool kBf16>
__device__ __forceinline__ void gather_row_smem(float (&y)[1 << B], const unsigned char *raw, int j0,
                                                const uint16_t *perm16, const uint32_t *sbits) {
    constexpr int S = 1 << B;
    uint32_t pw[S / 2];
#pragma unroll
    for (int q = 0; q < S / 8; ++q) {
        const uint4 v = *reinterpret_cast<const uint4 *>(perm16 + j0 + 8 * q);
        pw[4 * q] = v.x; pw[4 * q + 1] = v.y; pw[4 * q + 2] = v.z; pw[4 * q + 3] = v.w;
    }
    uint32_t sw[(S + 31) / 32];
#pragma unroll
    for (int q = 0; q < (S + 31) / 32; ++q) sw[q] = sbits[(j0 >> 5) + q] >> (S < 32 ? (j0 & 31) : 0);
#pragma unroll
    for (int t = 0; t < S; ++t) {
        const uint32_t p = (pw[t >> 1] >> (16 * (t & 1))) & 0xffffu;
        const uint32_t flip = ((sw[t >> 5] >> (t & 31)) & 1u) << 31;
        const uint32_t xb = kBf16 ? (uint32_t)reinterpret_cast<const uint16_t *>(raw)[p] << 16
                                  : reinterpret_cast<const uint32_t *>(raw)[p];
        y[t] = __uint_as_float(xb ^ flip);
    }
    butterfly<S>(y);
}

// Waits for this row's bulk copy; if the bounded wait runs out anywhere in the CTA, every thread
// learns it (so no thread is left at a later barrier), the fault flag is set and the caller stops.
__device__ __forceinline__ bool row_ready(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(bar, parity, kMaxPolls);
    const bool any_fail = __syncthreads_or(!ok);
    if (any_fail && threadIdx.x == 0) atomicOr(&g_fault, 2u);
    return !any_fail;
}

// Prologue of the persistent kernels. The tables arrive by bulk copy into buffers the row loop
// reuses later (perm as int32 into the transpose buffer, signs into the second row buffer), and
// the CTA's first row into the first row buffer; the tables are then converted in place: perm to
// 16-bit indices clamped into the row, signs to bits (bit t of word w set when signs[32 w + t] is
// negative). Returns false, CTA-uniformly and with the fault flag set, if the tables never land.
__device__ bool persistent_prologue(const PLayout &Lo, unsigned char *base, const int32_t *__restrict__ perm,
                                    const int8_t *__restrict__ signs, int d, const unsigned char *first_row,
                                    uint32_t row_bytes) {
    uint16_t *perm16 = reinterpret_cast<uint16_t *>(base + Lo.perm);
    uint32_t *sbits = reinterpret_cast<uint32_t *>(base + Lo.bits);
    unsigned char *rb0 = base + Lo.row0, *rb1 = base + Lo.row1, *buf = base + Lo.buf;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + Lo.bar);
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_init(&bar[2], 1);
        mbar_expect_tx(&bar[2], 5u * (uint32_t)d);
        bulk_load(buf, perm, 4u * (uint32_t)d, &bar[2]);
        bulk_load(rb1, signs, (uint32_t)d, &bar[2]);
        if (first_row) {
            mbar_expect_tx(&bar[0], row_bytes);
            bulk_load(rb0, first_row, row_bytes, &bar[0]);
        }
    }
    __syncthreads();  // the barriers are initialised before anyone waits on them
    if (!row_ready(&bar[2], 0)) {
        if (threadIdx.x == 0 && first_row) mbar_wait_bounded(&bar[0], 0, kMaxPolls);
        return false;
    }
    const int32_t *p32 = reinterpret_cast<const int32_t *>(buf);
    for (int j = threadIdx.x; j < d; j += blockDim.x) perm16[j] = (uint16_t)clampi(p32[j], d);
    for (int w = threadIdx.x; w < d / 32; w += blockDim.x) {
        uint32_t bits = 0;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 v = *reinterpret_cast<const uint4 *>(rb1 + 32 * w + 16 * q);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int b = 0; b < 4; ++b) bits |= ((wv[u] >> (8 * b + 7)) & 1u) << (16 * q + 4 * u + b);
        }
        sbits[w] = bits;
    }
    fence_proxy_async_smem();  // these reads of buf and rb1 precede the bulk copies that reuse them
    __syncthreads();
    return true;
}

template <int B, bool kBf16>
__global__ void __launch_bounds__(kMaxThreads)
    rotate_persistent(const void *__restrict__ x, int rows, int d, float post, const int32_t *__restrict__ perm,
                      const int8_t *__restrict__ signs, void *__restrict__ out) {
    using G = Geo<B>;
    constexpr int esz = kBf16 ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align16(smem_raw);
    const PLayout Lo(d, esz);
    uint16_t *perm16 = reinterpret_cast<uint16_t *>(base + Lo.perm);
    uint32_t *sbits = reinterpret_cast<uint32_t *>(base + Lo.bits);
    unsigned char *const rb0 = base + Lo.row0;  // row buffers rb0 and rb0 + row_bytes
    unsigned char *buf = base + Lo.buf;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + Lo.bar);
    const uint32_t row_bytes = (uint32_t)d * esz;
    const unsigned char *xb = static_cast<const unsigned char *>(x);
    int row = blockIdx.x;
    if (!persistent_prologue(Lo, base, perm, signs, d, row < rows ? xb + (int64_t)row * row_bytes : nullptr,
                             row_bytes))
        return;
    const int nslots = d >> B;
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int cur = it & 1;
        const int nrow = row + gridDim.x;
        if (threadIdx.x == 0 && nrow < rows) {
            bulk_wait_read<0>();  // the store of the row that last used the other buffer has read it
            mbar_expect_tx(&bar[cur ^ 1], row_bytes);
            bulk_load((rb0 + (cur ^ 1) * row_bytes), xb + (int64_t)nrow * row_bytes, row_bytes, &bar[cur ^ 1]);
        }
        if (!row_ready(&bar[cur], (it >> 1) & 1)) {
            if (threadIdx.x == 0 && nrow < rows) mbar_wait_bounded(&bar[cur ^ 1], ((it + 1) >> 1) & 1, kMaxPolls);
            return;
        }
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            const int blk = s >> B, r = s & (G::S - 1);
            float y[G::S];
            gather_row_smem<B, kBf16>(y, (rb0 + cur * row_bytes), blk * G::H + r * G::S, perm16, sbits);
            store_row<B>(buf, y, blk, r);
        }
        __syncthreads();
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            const int blk = s >> B, c = s & (G::S - 1);
            float y[G::S];
            load_col<B>(y, buf, blk, c);
            butterfly<G::S>(y);
#pragma unroll
            for (int t = 0; t < G::S; ++t) {
                const int j = blk * G::H + c + (t << B);
                const float z = __fmul_rn(y[t], post);
                if (kBf16)
                    reinterpret_cast<uint16_t *>((rb0 + cur * row_bytes))[j] = f32_to_bf16(z);
                else
                    reinterpret_cast<float *>((rb0 + cur * row_bytes))[j] = z;
            }
        }
        // the rotated row goes out with one bulk copy; the buffer is refilled only once it has been read
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            bulk_store(static_cast<unsigned char *>(out) + (int64_t)row * row_bytes, rb0 + cur * row_bytes, row_bytes);
            bulk_commit();
        }
    }
    if (threadIdx.x == 0) bulk_wait_all<0>();
}

template <int B, bool kBf16, int BITS, bool kSym>
__global__ void __launch_bounds__(kMaxThreads, 2)
    quantize_persistent(const void *__restrict__ w, int rows, int d, float post, const int32_t *__restrict__ perm,
                        const int8_t *__restrict__ signs, Edges E, uint8_t *__restrict__ packed,
                        void *__restrict__ row_norms) {
    using G = Geo<B>;
    constexpr int esz = kBf16 ? 2 : 4;
    extern __shared__ unsigned char smem_raw[];
    __shared__ double red[33];
    unsigned char *base = align16(smem_raw);
    const PLayout Lo(d, esz);
    uint16_t *perm16 = reinterpret_cast<uint16_t *>(base + Lo.perm);
    uint32_t *sbits = reinterpret_cast<uint32_t *>(base + Lo.bits);
    unsigned char *const rb0 = base + Lo.row0;  // row buffers rb0 and rb0 + row_bytes
    unsigned char *buf = base + Lo.buf;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + Lo.bar);
    const uint32_t row_bytes = (uint32_t)d * esz;
    const unsigned char *wb = static_cast<const unsigned char *>(w);
    int row = blockIdx.x;
    if (!persistent_prologue(Lo, base, perm, signs, d, row < rows ? wb + (int64_t)row * row_bytes : nullptr,
                             row_bytes))
        return;
    const int nslots = d >> B;
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int cur = it & 1;
        const int nrow = row + gridDim.x;
        if (threadIdx.x == 0 && nrow < rows) {
            mbar_expect_tx(&bar[cur ^ 1], row_bytes);
            bulk_load((rb0 + (cur ^ 1) * row_bytes), wb + (int64_t)nrow * row_bytes, row_bytes, &bar[cur ^ 1]);
        }
        if (!row_ready(&bar[cur], (it >> 1) & 1)) {
            if (threadIdx.x == 0 && nrow < rows) mbar_wait_bounded(&bar[cur ^ 1], ((it + 1) >> 1) & 1, kMaxPolls);
            return;
        }
        for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
            const int blk = s >> B, r = s & (G::S - 1);
            float y[G::S];
            gather_row_smem<B, kBf16>(y, (rb0 + cur * row_bytes), blk * G::H + r * G::S, perm16, sbits);
            store_row<B>(buf, y, blk, r);
        }
        __syncthreads();
        // pass 1 keeps w_rot in registers (the host guarantees nslots <= kSlots * blockDim.x):
        // thread slots s = threadIdx.x + k blockDim.x, k < kSlots, in the order of the plain loop
        constexpr int kSlots = 64 / G::S;
        float zk[kSlots][G::S];
        double ss = 0.0;
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
            const int s = threadIdx.x + k * (int)blockDim.x;
            if (s < nslots) {
                const int blk = s >> B, c = s & (G::S - 1);
                load_col<B>(zk[k], buf, blk, c);
                butterfly<G::S>(zk[k]);
#pragma unroll
                for (int t = 0; t < G::S; ++t) {
                    zk[k][t] = __fmul_rn(zk[k][t], post);
                    const double dz = (double)zk[k][t];
                    ss = __fma_rn(dz, dz, ss);
                }
            }
        }
        const float rho = __double2float_rn(__dsqrt_rn(block_sum_f64(ss, red)));
        const float den = __fadd_rn(rho, 1e-10f);
        const float rden = __frcp_rn(den);
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
            const int s = threadIdx.x + k * (int)blockDim.x;
            if (s < nslots) {
                const int blk = s >> B, c = s & (G::S - 1);
                unsigned char *cb = (rb0 + cur * row_bytes) + blk * G::H + c;
#pragma unroll
                for (int t = 0; t < G::S; ++t) {
                    const float z = zk[k][t];
                    const float q0 = __fmul_rn(z, rden);
                    const float u = __fmaf_rn(__fmaf_rn(-q0, den, z), rden, q0);
                    cb[t << B] = (uint8_t)bucketize<BITS, kSym>(u, E);
                }
            }
        }
        __syncthreads();
        uint8_t *dst = packed + ((int64_t)row * d / 8) * BITS;
        for (int g = threadIdx.x; g < d / 32; g += blockDim.x) {
            const uint4 c0 = *reinterpret_cast<const uint4 *>((rb0 + cur * row_bytes) + 32 * g);
            const uint4 c1 = *reinterpret_cast<const uint4 *>((rb0 + cur * row_bytes) + 32 * g + 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t word[BITS];
            pack32<BITS>(cw, word);
#pragma unroll
            for (int k = 0; k < BITS; ++k)
                reinterpret_cast<uint32_t *>(dst + 4 * BITS * g)[k] = __byte_perm(word[k], 0, 0x0123);
        }
        if (threadIdx.x == 0) {
            if (E.norm_bf16)
                static_cast<uint16_t *>(row_norms)[row] = f32_to_bf16(rho);
            else
                static_cast<float *>(row_norms)[row] = rho;
        }
        fence_proxy_async_smem();
        __syncthreads();
    }
}

// Warp-local form of quantize_persistent, for h-blocks of at most 32 x 32 (S <= 32): warp w always
// owns the same h-blocks, groups g = w, w + nwarps, ... of 32 / S blocks each, in every row. Both
// butterfly passes of a block, its codes and their packing stay inside the owning warp (its part
// of the transpose buffer is private), so a row needs one CTA barrier, for the norm; the partial
// sums alternate between two sets by row, so a set is rewritten only after the barrier between.
// A timed-out wait sets the fault flag but ends no thread's loop early, so every thread meets
// every barrier.
// kSlotsT = 1: the form for rows with at most one block group per warp (h = 1024 rows of a few
// blocks): one register slot per lane, so more CTAs fit an SM.
template <int B, bool kBf16, int BITS, bool kSym, int kSlotsT = 0>
__global__ void __launch_bounds__(kSlotsT == 1 ? 128 : kMaxThreads, kSlotsT == 1 ? 5 : 2)
    quantize_warp(const void *__restrict__ w, int rows, int d, float post, const int32_t *__restrict__ perm,
                  const int8_t *__restrict__ signs, Edges E, uint8_t *__restrict__ packed,
                  void *__restrict__ row_norms) {
    using G = Geo<B>;
    constexpr int S = G::S, H = G::H;
    constexpr int kBpw = 32 / S;  // blocks a warp works on at once: lane = sub-block * S + row / column
    // register slots per lane (the host checks the warp's share fits)
    constexpr int kSlots = kSlotsT ? kSlotsT : 64 / S;
    constexpr int esz = kBf16 ? 2 : 4;
    static_assert(S <= 32, "a block's rows must fit one warp");
    extern __shared__ unsigned char smem_raw[];
    __shared__ double red[2][kMaxThreads / 32];
    unsigned char *base = align16(smem_raw);
    const PLayout Lo(d, esz);
    const uint16_t *perm16 = reinterpret_cast<const uint16_t *>(base + Lo.perm);
    const uint32_t *sbits = reinterpret_cast<const uint32_t *>(base + Lo.bits);
    unsigned char *const rb0 = base + Lo.row0;  // row buffers rb0 and rb0 + row_bytes
    unsigned char *buf = base + Lo.buf;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + Lo.bar);
    const uint32_t row_bytes = (uint32_t)d * esz;
    const unsigned char *wb = static_cast<const unsigned char *>(w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = (int)(blockDim.x >> 5);
    const int sub = lane / S, rc = lane % S;
    const int nb = d / H, ngroups = (nb + kBpw - 1) / kBpw;
    int row = blockIdx.x;
    if (!persistent_prologue(Lo, base, perm, signs, d, row < rows ? wb + (int64_t)row * row_bytes : nullptr,
                             row_bytes))
        return;
    bool fault = false;
    int last_buf = -1;  // thread 0: the buffer and phase of the last row copy it issued
    uint32_t last_par = 0;
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int cur = it & 1;
        const int nrow = row + gridDim.x;
        // every thread passed the previous row's barrier after its last read of the other buffer
        if (threadIdx.x == 0 && nrow < rows && !fault) {
            mbar_expect_tx(&bar[cur ^ 1], row_bytes);
            bulk_load((rb0 + (cur ^ 1) * row_bytes), wb + (int64_t)nrow * row_bytes, row_bytes, &bar[cur ^ 1]);
            last_buf = cur ^ 1;
            last_par = (uint32_t)(((it + 1) >> 1) & 1);
        }
        if (!fault && !mbar_wait_bounded(&bar[cur], (it >> 1) & 1, kMaxPolls)) {
            fault = true;
            atomicOr(&g_fault, 2u);
        }
        const unsigned char *rbc = rb0 + cur * row_bytes;
        // pass 0 and pass 1 of the warp's blocks; w_rot stays in registers
        float zk[kSlots][S];
        double ss = 0.0;
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
            const int g = warp + k * nwarps;
            const int blk = g * kBpw + sub;
            if (g < ngroups) {  // warp-uniform
                if (blk < nb) {
                    float y[S];
                    gather_row_smem<B, kBf16>(y, rbc, blk * H + rc * S, perm16, sbits);
                    store_row<B>(buf, y, blk, rc);
                }
                __syncwarp();
                if (blk < nb) {
                    load_col<B>(zk[k], buf, blk, rc);
                    butterfly<S>(zk[k]);
#pragma unroll
                    for (int t = 0; t < S; ++t) {
                        zk[k][t] = __fmul_rn(zk[k][t], post);
                        const double dz = (double)zk[k][t];
                        ss = __fma_rn(dz, dz, ss);
                    }
                }
            }
        }
        // rho = ||w_rot||: every lane of a warp gets the same warp sum, every thread the same total
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        if (lane == 0) red[cur][warp] = ss;
        fence_proxy_async_smem();  // this thread's reads of the row buffer precede the copy that refills it
        __syncthreads();
        double tot = 0.0;
        for (int v = 0; v < nwarps; ++v) tot = __dadd_rn(tot, red[cur][v]);
        const float rho = __double2float_rn(__dsqrt_rn(tot));
        const float den = __fadd_rn(rho, 1e-10f);
        const float rden = __frcp_rn(den);
        // codes, one byte each in element order, into the block's own part of the transpose buffer
        // (its columns are in registers by now); u = z / den by Markstein's correction
        // (q0 = RN(z r), r = RN(1 / den), rem = RN(z - q0 den), u = RN(q0 + rem r)), correctly
        // rounded for |z| >= 2^-100 and a normal quotient, two elements at a time
        const f32x2 RDEN = pk2(rden, rden), NDEN = pk2(-den, -den);
#pragma unroll
        for (int k = 0; k < kSlots; ++k) {
            const int g = warp + k * nwarps;
            const int blk = g * kBpw + sub;
            if (g < ngroups && blk < nb) {
                unsigned char *cb = buf + 4 * blk * H + rc;
#pragma unroll
                for (int t = 0; t < S; t += 2) {
                    const f32x2 z = pk2(zk[k][t], zk[k][t + 1]);
                    const f32x2 q0 = mul2(z, RDEN);
                    const f32x2 u = fma2(fma2(q0, NDEN, z), RDEN, q0);
                    if constexpr (kSym) {
                        float v0, v1;
                        upk2(sym_codes<BITS>(u, E), v0, v1);
                        cb[t * S] = (uint8_t)__float_as_uint(v0);
                        cb[(t + 1) * S] = (uint8_t)__float_as_uint(v1);
                    } else {
                        float u0, u1;
                        upk2(u, u0, u1);
                        cb[t * S] = (uint8_t)bucketize<BITS, false>(u0, E);
                        cb[(t + 1) * S] = (uint8_t)bucketize<BITS, false>(u1, E);
                    }
                }
            }
        }
        __syncwarp();
        // pack_codes: the warp's groups of 32 codes (S per block group, over all its block groups)
        // spread over the 32 lanes
        uint8_t *dst = packed + ((int64_t)row * d / 8) * BITS;
#pragma unroll
        for (int j0 = 0; j0 < kSlots * S; j0 += 32) {
            const int unit = j0 + lane, k = unit / S;
            const int g = warp + k * nwarps;
            const int blk = g * kBpw + (unit % S) / (H / 32), q = (unit % S) % (H / 32);
            if (k < kSlots && g < ngroups && blk < nb) {
                const unsigned char *src = buf + 4 * blk * H + 32 * q;
                const uint4 c0 = *reinterpret_cast<const uint4 *>(src);
                const uint4 c1 = *reinterpret_cast<const uint4 *>(src + 16);
                const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t word[BITS];
                if constexpr (BITS == 3)
                    pack32_b3(cw, word);
                else
                    pack32<BITS>(cw, word);
                uint32_t *out = reinterpret_cast<uint32_t *>(dst + (blk * H + 32 * q) / 8 * BITS);
#pragma unroll
                for (int j = 0; j < BITS; ++j) out[j] = __byte_perm(word[j], 0, 0x0123);
            }
        }
        __syncwarp();  // the codes are read before the next row's pass 0 rewrites this part of the buffer
        if (threadIdx.x == 0) {
            if (E.norm_bf16)
                static_cast<uint16_t *>(row_norms)[row] = f32_to_bf16(rho);
            else
                static_cast<float *>(row_norms)[row] = rho;
        }
    }
    // a fault may leave thread 0's last row copy in flight: give it a bounded chance to land
    if (fault && threadIdx.x == 0 && last_buf >= 0) mbar_wait_bounded(&bar[last_buf], last_par, kMaxPolls);
}

// Warp-local form of the activation rotation (S <= 32): warp w always owns the same h-blocks,
// groups g = w, w + nwarps, ... of 32 / S blocks, and runs both butterfly passes of a group
// through its own 128 S-byte transpose scratch; the outputs go from registers straight to global
// memory (for each t, the S lanes of a block store S consecutive elements). Rows are
// double-buffered by 1-D bulk copies; one CTA barrier per row tells thread 0 that every warp
// has finished gathering from a row buffer, which then takes the row after next.
struct RLayout {
    int perm, bits, row0, row1, scr, bar, total;
    __host__ __device__ RLayout(int d, int esz, int nwarps, int S) {
        perm = 0;
        bits = a16(2 * d);
        row0 = bits + a16(d / 8);
        row1 = row0 + d * esz;
        scr = row1 + d * esz;
        bar = scr + nwarps * 128 * S;
        total = bar + 32;
    }
};

constexpr int kRotWarps = 12;  // warps per CTA of rotate_warp (two CTAs per SM fit the register file)

template <int B, bool kBf16>
__global__ void __launch_bounds__(32 * kRotWarps, 2)
    rotate_warp(const void *__restrict__ x, int rows, int d, float post, const int32_t *__restrict__ perm,
                const int8_t *__restrict__ signs, void *__restrict__ out) {
    using G = Geo<B>;
    constexpr int S = G::S, H = G::H, kBpw = 32 / S;
    constexpr int esz = kBf16 ? 2 : 4;
    static_assert(S <= 32, "a block's rows must fit one warp");
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = align16(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = (int)(blockDim.x >> 5);
    const RLayout Lo(d, esz, nwarps, S);
    uint16_t *perm16 = reinterpret_cast<uint16_t *>(base + Lo.perm);
    uint32_t *sbits = reinterpret_cast<uint32_t *>(base + Lo.bits);
    unsigned char *const rb0 = base + Lo.row0;  // row buffers rb0 and rb0 + row_bytes
    unsigned char *const scr = base + Lo.scr + warp * 128 * S;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + Lo.bar);
    const uint32_t row_bytes = (uint32_t)d * esz;
    const unsigned char *xb = static_cast<const unsigned char *>(x);
    const int sub = lane / S, rc = lane % S;
    const int nb = d / H, ngroups = (nb + kBpw - 1) / kBpw;

    // tables: perm (int32) lands in the row buffers, the signs in the scratch; both are converted
    // in place before the first row is fetched
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_init(&bar[2], 1);
        mbar_expect_tx(&bar[2], 5u * (uint32_t)d);
        bulk_load(rb0, perm, 4u * (uint32_t)d, &bar[2]);
        bulk_load(base + Lo.scr, signs, (uint32_t)d, &bar[2]);
    }
    __syncthreads();
    if (!row_ready(&bar[2], 0)) return;
    {
        const int32_t *p32 = reinterpret_cast<const int32_t *>(rb0);
        for (int j = threadIdx.x; j < d; j += blockDim.x) perm16[j] = (uint16_t)clampi(p32[j], d);
        const unsigned char *sg = base + Lo.scr;
        for (int w = threadIdx.x; w < d / 32; w += blockDim.x) {
            uint32_t bits = 0;
            for (int t = 0; t < 32; ++t) bits |= (uint32_t)(((uint8_t)sg[32 * w + t]) >> 7) << t;
            sbits[w] = bits;
        }
    }
    fence_proxy_async_smem();  // these reads of the row buffers precede the copies that refill them
    __syncthreads();
    int row = blockIdx.x;
    uint32_t n_iss0 = 0u, n_iss1 = 0u;  // thread 0: row copies issued into each buffer
    if (threadIdx.x == 0)
        for (int b = 0; b < 2; ++b) {
            const int r = row + b * (int)gridDim.x;
            if (r < rows) {
                mbar_expect_tx(&bar[b], row_bytes);
                bulk_load(rb0 + b * row_bytes, xb + (int64_t)r * row_bytes, row_bytes, &bar[b]);
                if (b == 0) ++n_iss0; else ++n_iss1;
            }
        }
    bool fault = false;
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int cur = it & 1;
        if (!fault && !mbar_wait_bounded(&bar[cur], (it >> 1) & 1, kMaxPolls)) {
            fault = true;
            atomicOr(&g_fault, 2u);
        }
        const unsigned char *rbc = rb0 + cur * row_bytes;
        unsigned char *orow = static_cast<unsigned char *>(out) + (int64_t)row * row_bytes;
        for (int g = warp; g < ngroups; g += nwarps) {
            const int blk = g * kBpw + sub;
            if (blk < nb) {
                float y[S];
                gather_row_smem<B, kBf16>(y, rbc, blk * H + rc * S, perm16, sbits);
                store_row<B>(scr, y, sub, rc);
            }
            __syncwarp();
            if (blk < nb) {
                float y[S];
                load_col<B>(y, scr, sub, rc);
                butterfly<S>(y);
#pragma unroll
                for (int t = 0; t < S; ++t) {
                    const int j = blk * H + rc + t * S;
                    const float z = __fmul_rn(y[t], post);
                    if (kBf16)
                        reinterpret_cast<uint16_t *>(orow)[j] = f32_to_bf16(z);
                    else
                        reinterpret_cast<float *>(orow)[j] = z;
                }
            }
            __syncwarp();  // the columns are read before the warp's next group rewrites the scratch
        }
        // every warp has gathered from this buffer: it takes the row after next
        fence_proxy_async_smem();
        __syncthreads();
        const int r2 = row + 2 * (int)gridDim.x;
        if (threadIdx.x == 0 && r2 < rows && !fault) {
            mbar_expect_tx(&bar[cur], row_bytes);
            bulk_load(rb0 + cur * row_bytes, xb + (int64_t)r2 * row_bytes, row_bytes, &bar[cur]);
            if (cur == 0) ++n_iss0; else ++n_iss1;
        }
    }
    // a fault may leave row copies in flight: give the last one into each buffer a bounded chance
    if (fault && threadIdx.x == 0) {
        if (n_iss0 > 0) mbar_wait_bounded(&bar[0], (n_iss0 - 1) & 1u, kMaxPolls);
        if (n_iss1 > 0) mbar_wait_bounded(&bar[1], (n_iss1 - 1) & 1u, kMaxPolls);
    }
}

// ---------------------------------------------------------------------------------------------
// rpbh_dequantize_weight without unrotate (_dequantize_rotated), persistent: each CTA walks rows
// blockIdx.x, blockIdx.x + gridDim.x, ...; a row's codes (d/8 * bits bytes, a multiple of 16) come
// in by 1-D bulk copy two rows ahead into one of two buffers, and its norm one row ahead into a
// register, so no thread waits for memory in the middle of a row. Group g of 8 codes (bits
// bytes, MSB first) gives 8 outputs, stored 16 bytes at a time.
// ---------------------------------------------------------------------------------------------
template <bool kNormBf16, bool kOutBf16, int BITS>
__global__ void __launch_bounds__(256)
    deq_rot_persistent(const uint8_t *__restrict__ packed, const void *__restrict__ row_norms, int rows, int d,
                       Codebook cb, void *__restrict__ out) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ float cbs[16];
    unsigned char *base = align16(smem_raw);
    const uint32_t nbytes = (uint32_t)(d / 8 * BITS);
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + 2 * nbytes);
    constexpr int L = 1 << BITS;
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    if (threadIdx.x < L) {
        // codebook.to(dtype): the bf16 rotated output multiplies bf16-rounded operands
        const float c = cb.c[threadIdx.x];
        cbs[threadIdx.x] = kOutBf16 ? bf16_to_f32(f32_to_bf16(c)) : c;
    }
    auto norm_of = [&](int r) {
        return kNormBf16 ? bf16_to_f32(static_cast<const uint16_t *>(row_norms)[r])
                         : static_cast<const float *>(row_norms)[r];
    };
    int row = blockIdx.x;
    uint32_t n_iss0 = 0u, n_iss1 = 0u;  // thread 0: row copies issued into each buffer
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        for (int b = 0; b < 2; ++b) {
            const int r = row + b * (int)gridDim.x;
            if (r < rows) {
                mbar_expect_tx(&bar[b], nbytes);
                bulk_load(base + b * nbytes, packed + (int64_t)r * nbytes, nbytes, &bar[b]);
                if (b == 0) ++n_iss0; else ++n_iss1;
            }
        }
    }
    __syncthreads();
    float rho_next = row < rows ? norm_of(row) : 0.0f;
    bool fault = false;
    for (int it = 0; row < rows; ++it, row += gridDim.x) {
        const int cur = it & 1;
        const float rho = rho_next;
        if (row + (int)gridDim.x < rows) rho_next = norm_of(row + gridDim.x);
        const float rho_op = kOutBf16 ? bf16_to_f32(f32_to_bf16(rho)) : rho;
        if (!fault && !mbar_wait_bounded(&bar[cur], (it >> 1) & 1, kMaxPolls)) {
            fault = true;
            atomicOr(&g_fault, 2u);
        }
        const unsigned char *src = base + cur * nbytes;
        for (int g = threadIdx.x; g < d / 8; g += blockDim.x) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < BITS; ++b) word = (word << 8) | src[g * BITS + b];
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(cbs[(word >> (BITS * (7 - i))) & kMask], rho_op);
            if (kOutBf16) {
                st_stream16(static_cast<uint16_t *>(out) + (int64_t)row * d + 8 * g,
                            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                       pack_bf16x2(v[6], v[7])));
            } else {
                float *o = static_cast<float *>(out) + (int64_t)row * d + 8 * g;
                st_stream16(o, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                                          __float_as_uint(v[3])));
                st_stream16(o + 4, make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                                              __float_as_uint(v[7])));
            }
        }
        // every thread has read this buffer: it takes the row after next
        fence_proxy_async_smem();
        __syncthreads();
        const int r2 = row + 2 * (int)gridDim.x;
        if (threadIdx.x == 0 && r2 < rows && !fault) {
            mbar_expect_tx(&bar[cur], nbytes);
            bulk_load(base + cur * nbytes, packed + (int64_t)r2 * nbytes, nbytes, &bar[cur]);
            if (cur == 0) ++n_iss0; else ++n_iss1;
        }
    }
    // a fault may leave row copies in flight: give the last one into each buffer a bounded chance
    if (fault && threadIdx.x == 0) {
        if (n_iss0 > 0) mbar_wait_bounded(&bar[0], (n_iss0 - 1) & 1u, kMaxPolls);
        if (n_iss1 > 0) mbar_wait_bounded(&bar[1], (n_iss1 - 1) & 1u, kMaxPolls);
    }
}

// ---------------------------------------------------------------------------------------------
// host dispatch
// ---------------------------------------------------------------------------------------------
int log2_block(int64_t d) {
    const int64_t h = d & -d;
    int l = 0;
    while ((int64_t(1) << l) < h) ++l;
    return l;
}

size_t smem_limit() {
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

size_t rot_smem(int64_t d, int esz) { return (size_t)d * (esz + 4) + 16; }
size_t deq_smem(int64_t d, int oesz) { return (size_t)d * (1 + 4 + oesz) + 16; }

bool supported(int64_t d, int in_esz, int out_esz) {
    const int l = log2_block(d);
    if (l < 6 || l > 12 || (l & 1)) return false;
    if (d > 65536) return false;
    const size_t a = rot_smem(d, in_esz > out_esz ? in_esz : out_esz), b = deq_smem(d, out_esz);
    return (a > b ? a : b) + 2048 <= smem_limit();
}

int threads_for(int64_t d, int B) {
    const int64_t slots = d >> B;
    int64_t t = ((slots + 31) / 32) * 32;
    if (t > kMaxThreads) t = kMaxThreads;
    if (t < 128) t = 128;
    return (int)t;
}

// Raise a kernel's dynamic shared-memory limit once (and again only when a call needs more).
template <typename K>
wq_status prep(K k, size_t smem) {
    return ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem) ? WQ_OK : WQ_ERR_CUDA;
}

float fwht_post(int64_t h) { return (float)std::pow((double)h, -0.5); }

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
    return cached[dev];
}

size_t pers_smem(int64_t d, int esz) { return (size_t)PLayout((int)d, esz).total + 16; }

bool persistent_fits(int64_t d, int esz) { return d <= 32768 && pers_smem(d, esz) + 1024 <= smem_limit(); }

int blocks_per_sm(const void *k, int threads, size_t smem) { return blocks_per_sm_cached(k, threads, smem); }

// The persistent form (tables resident, rows double-buffered by bulk copies) is taken whenever it
// fits on an SM: measured faster than one row per CTA for the LLM and DiT shapes even where its
// larger shared-memory footprint leaves fewer CTAs per SM.
template <typename KP, typename KR>
bool prefer_persistent(KP kp, size_t pers, KR kr, size_t plain, int threads) {
    (void)kr;
    (void)plain;
    return blocks_per_sm(reinterpret_cast<const void *>(kp), threads, pers) >= 1;
}

// Grid for a persistent kernel: every SM gets as many CTAs as fit, but never more CTAs than rows.
template <typename K>
int persistent_grid(K k, int threads, size_t smem, int64_t rows) {
    int per_sm = blocks_per_sm_cached(reinterpret_cast<const void *>(k), threads, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t g = (int64_t)per_sm * sm_count();
    return (int)(g < rows ? g : rows);
}

template <int B, bool kBf16>
wq_status rotate_b(const void *x, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, void *out,
                   cudaStream_t s) {
    const int threads = threads_for(d, B);
    const size_t smem = rot_smem(d, kBf16 ? 2 : 4);
    auto k = rotate_kernel<B, kBf16>;
    wq_status st = prep(k, smem);
    if (st != WQ_OK) return st;
    // the warp-local form: kRotWarps warps, each with a 128 S-byte transpose scratch (which also
    // stages the signs at set-up, so it must hold d bytes)
    if constexpr (B <= 5) {
        constexpr int S = 1 << B, kW = kRotWarps;
        const size_t wsmem = (size_t)RLayout((int)d, kBf16 ? 2 : 4, kW, S).total + 16;
        // (only when every warp has a block group of each row: with fewer, most warps would idle)
        const int64_t groups = ((d >> (2 * B)) + 32 / S - 1) / (32 / S);
        if (groups >= kW && d <= 32768 && (int64_t)kW * 128 * S >= d && wsmem + 1024 <= smem_limit()) {
            auto kw = rotate_warp<B, kBf16>;
            st = prep(kw, wsmem);
            if (st != WQ_OK) return st;
            if (blocks_per_sm(reinterpret_cast<const void *>(kw), 32 * kW, wsmem) >= 1) {
                kw<<<persistent_grid(kw, 32 * kW, wsmem, rows), 32 * kW, wsmem, s>>>(
                    x, (int)rows, (int)d, fwht_post(d & -d), perm, signs, out);
                return launch_status();
            }
        }
    }
    if (persistent_fits(d, kBf16 ? 2 : 4)) {
        const size_t psmem = pers_smem(d, kBf16 ? 2 : 4);
        auto kp = rotate_persistent<B, kBf16>;
        st = prep(kp, psmem);
        if (st != WQ_OK) return st;
        if (prefer_persistent(kp, psmem, k, smem, threads)) {
            kp<<<persistent_grid(kp, threads, psmem, rows), threads, psmem, s>>>(x, (int)rows, (int)d,
                                                                                 fwht_post(d & -d), perm, signs, out);
            return launch_status();
        }
    }
    k<<<(unsigned)rows, threads, smem, s>>>(x, (int)d, fwht_post(d & -d), perm, signs, out);
    return launch_status();
}

wq_status rotate(const void *x, int dtype, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                 void *out, cudaStream_t s) {
    const bool bf = dtype == WQ_BF16;
    if (bf && rpbh_lanes::rotate_fits(d))
        return rpbh_lanes::rotate(static_cast<const uint16_t *>(x), rows, d, perm, signs, static_cast<uint16_t *>(out), s);
    switch (log2_block(d) / 2) {
        case 3: return bf ? rotate_b<3, true>(x, rows, d, perm, signs, out, s) : rotate_b<3, false>(x, rows, d, perm, signs, out, s);
        case 4: return bf ? rotate_b<4, true>(x, rows, d, perm, signs, out, s) : rotate_b<4, false>(x, rows, d, perm, signs, out, s);
        case 5: return bf ? rotate_b<5, true>(x, rows, d, perm, signs, out, s) : rotate_b<5, false>(x, rows, d, perm, signs, out, s);
        case 6: return bf ? rotate_b<6, true>(x, rows, d, perm, signs, out, s) : rotate_b<6, false>(x, rows, d, perm, signs, out, s);
        default: return WQ_ERR_SHAPE;
    }
}

template <int B, bool kBf16, int BITS, bool kSym>
wq_status quantize_b(const void *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                     const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    const int threads = threads_for(d, B);
    const size_t smem = rot_smem(d, kBf16 ? 2 : 4);
    auto k = quantize_kernel<B, kBf16, BITS, kSym>;
    wq_status st = prep(k, smem);
    if (st != WQ_OK) return st;
    // the warp-local form (where its register-resident slots compile without spilling): each warp's
    // share of block groups must fit its 64 / S register slots
    if constexpr (B == 5 || (B == 4 && kBf16)) {
        constexpr int64_t S = int64_t(1) << B;
        const int64_t groups = ((d >> (2 * B)) + 32 / S - 1) / (32 / S);
        // at most one block group per warp: the one-slot form
        if constexpr (B == 5) {
            if ((!kSym || E.steps) && persistent_fits(d, kBf16 ? 2 : 4) && groups <= threads / 32 &&
                threads <= 128) {
                const size_t psmem = pers_smem(d, kBf16 ? 2 : 4);
                auto kw = quantize_warp<B, kBf16, BITS, kSym, 1>;
                st = prep(kw, psmem);
                if (st != WQ_OK) return st;
                if (blocks_per_sm(reinterpret_cast<const void *>(kw), threads, psmem) >= 1) {
                    kw<<<persistent_grid(kw, threads, psmem, rows), threads, psmem, s>>>(
                        w, (int)rows, (int)d, fwht_post(d & -d), perm, signs, E, packed, row_norms);
                    return launch_status();
                }
            }
        }
        if ((!kSym || E.steps) && persistent_fits(d, kBf16 ? 2 : 4) &&
            (groups + threads / 32 - 1) / (threads / 32) <= 64 / S) {
            const size_t psmem = pers_smem(d, kBf16 ? 2 : 4);
            auto kw = quantize_warp<B, kBf16, BITS, kSym>;
            st = prep(kw, psmem);
            if (st != WQ_OK) return st;
            if (blocks_per_sm(reinterpret_cast<const void *>(kw), threads, psmem) >= 1) {
                kw<<<persistent_grid(kw, threads, psmem, rows), threads, psmem, s>>>(
                    w, (int)rows, (int)d, fwht_post(d & -d), perm, signs, E, packed, row_norms);
                return launch_status();
            }
        }
    }
    // the persistent form keeps each thread's slots of the row in registers: at most 64 / S of them
    if (persistent_fits(d, kBf16 ? 2 : 4) && (d >> B) <= (int64_t)(64 >> B) * threads) {
        const size_t psmem = pers_smem(d, kBf16 ? 2 : 4);
        auto kp = quantize_persistent<B, kBf16, BITS, kSym>;
        st = prep(kp, psmem);
        if (st != WQ_OK) return st;
        if (prefer_persistent(kp, psmem, k, smem, threads)) {
            kp<<<persistent_grid(kp, threads, psmem, rows), threads, psmem, s>>>(
                w, (int)rows, (int)d, fwht_post(d & -d), perm, signs, E, packed, row_norms);
            return launch_status();
        }
    }
    k<<<(unsigned)rows, threads, smem, s>>>(w, (int)d, fwht_post(d & -d), perm, signs, E, packed, row_norms);
    return launch_status();
}

template <int B, bool kBf16, bool kSym>
wq_status quantize_bits(int bits, const void *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                        const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    switch (bits) {
        case 2: return quantize_b<B, kBf16, 2, kSym>(w, rows, d, perm, signs, E, packed, row_norms, s);
        case 3: return quantize_b<B, kBf16, 3, kSym>(w, rows, d, perm, signs, E, packed, row_norms, s);
        case 4: return quantize_b<B, kBf16, 4, kSym>(w, rows, d, perm, signs, E, packed, row_norms, s);
        default: return WQ_ERR_BITS;
    }
}

template <int B>
wq_status quantize_sym(bool bf, bool sym, int bits, const void *w, int64_t rows, int64_t d, const int32_t *perm,
                       const int8_t *signs, const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    if (bf)
        return sym ? quantize_bits<B, true, true>(bits, w, rows, d, perm, signs, E, packed, row_norms, s)
                   : quantize_bits<B, true, false>(bits, w, rows, d, perm, signs, E, packed, row_norms, s);
    return sym ? quantize_bits<B, false, true>(bits, w, rows, d, perm, signs, E, packed, row_norms, s)
               : quantize_bits<B, false, false>(bits, w, rows, d, perm, signs, E, packed, row_norms, s);
}

wq_status quantize(const void *w, int w_dtype, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                   int bits, const float *codebook, uint8_t *packed, void *row_norms, int norm_dtype, cudaStream_t s) {
    const int L = 1 << bits;
    Edges E = {};
    E.norm_bf16 = norm_dtype == WQ_BF16;
    // edges = (codebook[:-1] + codebook[1:]) / 2, in fp32 as the page computes them
    for (int k = 0; k + 1 < L; ++k) {
        volatile float sum = codebook[k] + codebook[k + 1];
        E.e[k] = sum / 2.0f;
    }
    bool sym = true;
    for (int k = 0; k < L; ++k)
        if (!(codebook[k] == -codebook[L - 1 - k])) sym = false;
    if (sym && !(E.e[L / 2 - 1] == 0.0f)) sym = false;
    if (sym) {
        E.steps = 1;
        for (int i = 0; i < L / 2 - 1; ++i) {
            const float e = E.e[L / 2 + i];
            int ex = 0;
            std::frexp(e, &ex);  // e = f 2^ex, f in [0.5, 1): binary exponent ex - 1
            if (!(e >= 0x1p-103f) || !std::isfinite(e)) {
                E.steps = 0;
                break;
            }
            E.M[i] = std::ldexp(1.0f, 25 - ex);
            E.K[i] = -e * E.M[i];  // exact: e scaled by a power of two into [2^24, 2^25)
        }
    }
    const bool bf = w_dtype == WQ_BF16;
    if (bf && sym && rpbh_lanes::quantize_fits(d, E))
        return rpbh_lanes::quantize(static_cast<const uint16_t *>(w), rows, d, perm, signs, bits, E, packed, row_norms,
                                    s);
    switch (log2_block(d) / 2) {
        case 3: return quantize_sym<3>(bf, sym, bits, w, rows, d, perm, signs, E, packed, row_norms, s);
        case 4: return quantize_sym<4>(bf, sym, bits, w, rows, d, perm, signs, E, packed, row_norms, s);
        case 5: return quantize_sym<5>(bf, sym, bits, w, rows, d, perm, signs, E, packed, row_norms, s);
        case 6: return quantize_sym<6>(bf, sym, bits, w, rows, d, perm, signs, E, packed, row_norms, s);
        default: return WQ_ERR_SHAPE;
    }
}

template <int B, bool kNB, bool kOB, int BITS>
wq_status deq_b(const uint8_t *packed, const void *norms, int64_t rows, int64_t d, const Codebook &cb,
                const int32_t *perm, const int8_t *signs, void *out, cudaStream_t s) {
    const size_t smem = deq_smem(d, kOB ? 2 : 4);
    auto k = dequant_unrotate_kernel<B, kNB, kOB, BITS>;
    wq_status st = prep(k, smem);
    if (st != WQ_OK) return st;
    k<<<(unsigned)rows, threads_for(d, B), smem, s>>>(packed, norms, (int)d, fwht_post(d & -d), cb, perm, signs, out);
    return launch_status();
}

template <int B, bool kNB, bool kOB>
wq_status deq_bits(int bits, const uint8_t *packed, const void *norms, int64_t rows, int64_t d, const Codebook &cb,
                   const int32_t *perm, const int8_t *signs, void *out, cudaStream_t s) {
    switch (bits) {
        case 2: return deq_b<B, kNB, kOB, 2>(packed, norms, rows, d, cb, perm, signs, out, s);
        case 3: return deq_b<B, kNB, kOB, 3>(packed, norms, rows, d, cb, perm, signs, out, s);
        case 4: return deq_b<B, kNB, kOB, 4>(packed, norms, rows, d, cb, perm, signs, out, s);
        default: return WQ_ERR_BITS;
    }
}

template <int B>
wq_status deq_dt(bool nb, bool ob, int bits, const uint8_t *packed, const void *norms, int64_t rows, int64_t d,
                 const Codebook &cb, const int32_t *perm, const int8_t *signs, void *out, cudaStream_t s) {
    if (nb)
        return ob ? deq_bits<B, true, true>(bits, packed, norms, rows, d, cb, perm, signs, out, s)
                  : deq_bits<B, true, false>(bits, packed, norms, rows, d, cb, perm, signs, out, s);
    return ob ? deq_bits<B, false, true>(bits, packed, norms, rows, d, cb, perm, signs, out, s)
              : deq_bits<B, false, false>(bits, packed, norms, rows, d, cb, perm, signs, out, s);
}

wq_status dequantize_unrotate(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t rows, int64_t d,
                              int bits, const float *codebook, const int32_t *perm, const int8_t *signs, void *out,
                              int out_dtype, cudaStream_t s) {
    Codebook cb = {};
    for (int k = 0; k < (1 << bits); ++k) cb.c[k] = codebook[k];
    const bool nb = norm_dtype == WQ_BF16, ob = out_dtype == WQ_BF16;
    switch (log2_block(d) / 2) {
        case 3: return deq_dt<3>(nb, ob, bits, packed, row_norms, rows, d, cb, perm, signs, out, s);
        case 4: return deq_dt<4>(nb, ob, bits, packed, row_norms, rows, d, cb, perm, signs, out, s);
        case 5: return deq_dt<5>(nb, ob, bits, packed, row_norms, rows, d, cb, perm, signs, out, s);
        case 6: return deq_dt<6>(nb, ob, bits, packed, row_norms, rows, d, cb, perm, signs, out, s);
        default: return WQ_ERR_SHAPE;
    }
}

bool dequantize_rotated_fits(int64_t d, int bits) {
    const int64_t nbytes = d / 8 * bits;
    return d % 8 == 0 && nbytes % 16 == 0 && 2 * nbytes + 64 + 1024 <= (int64_t)smem_limit();
}

template <bool kNB, bool kOB, int BITS>
wq_status deq_rot_launch(const uint8_t *packed, const void *row_norms, int64_t rows, int64_t d, const Codebook &cb,
                         void *out, cudaStream_t s) {
    auto k = deq_rot_persistent<kNB, kOB, BITS>;
    const size_t smem = (size_t)(d / 8 * BITS) * 2 + 16 + 16;
    const wq_status st = prep(k, smem);
    if (st != WQ_OK) return st;
    // 128 or 256 threads, whichever leaves fewer idle group slots in a row's last pass
    const int64_t groups = d / 8;
    const int64_t idle128 = (groups + 127) / 128 * 128 - groups, idle256 = (groups + 255) / 256 * 256 - groups;
    const int threads = idle128 < idle256 ? 128 : 256;
    k<<<persistent_grid(k, threads, smem, rows), threads, smem, s>>>(packed, row_norms, (int)rows, (int)d, cb, out);
    return launch_status();
}

template <bool kNB, bool kOB>
wq_status deq_rot_bits(int bits, const uint8_t *packed, const void *row_norms, int64_t rows, int64_t d,
                       const Codebook &cb, void *out, cudaStream_t s) {
    switch (bits) {
        case 2: return deq_rot_launch<kNB, kOB, 2>(packed, row_norms, rows, d, cb, out, s);
        case 3: return deq_rot_launch<kNB, kOB, 3>(packed, row_norms, rows, d, cb, out, s);
        case 4: return deq_rot_launch<kNB, kOB, 4>(packed, row_norms, rows, d, cb, out, s);
        default: return WQ_ERR_BITS;
    }
}

wq_status dequantize_rotated(const uint8_t *packed, const void *row_norms, int norm_dtype, int64_t rows, int64_t d,
                             int bits, const float *codebook, void *out, int out_dtype, cudaStream_t s) {
    Codebook cb = {};
    for (int k = 0; k < (1 << bits); ++k) cb.c[k] = codebook[k];
    const bool nb = norm_dtype == WQ_BF16, ob = out_dtype == WQ_BF16;
    if (nb) return ob ? deq_rot_bits<true, true>(bits, packed, row_norms, rows, d, cb, out, s)
                      : deq_rot_bits<true, false>(bits, packed, row_norms, rows, d, cb, out, s);
    return ob ? deq_rot_bits<false, true>(bits, packed, row_norms, rows, d, cb, out, s)
              : deq_rot_bits<false, false>(bits, packed, row_norms, rows, d, cb, out, s);
}

unsigned int read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(g_fault, &zero, sizeof zero);
    return v;
}

}  // namespace rpbh_fast
}  // namespace wq
