// Warp-lane RPBH kernels on sm_100a for bf16 rows whose Hadamard block is h = 256 or 1024: page
// "orbit_quant.py" (rpbh_forward, _fwht, _quantize_rows, pack_codes).
//
// The arithmetic is rpbh_fast.cu's (an h-block viewed as S x S, S = 16 or 32; pass 0 takes one
// matrix row per lane and the stages 1 .. S/2, pass 1 one matrix column per lane and the stages
// S .. h/2; every butterfly one IEEE add or subtract in the page's stage order; the scale
// 1/sqrt(h) one rounded product), arranged so that few instructions are spent per element:
//  - permutation and signs are one shared table of 16-bit entries, entry j = 2 perm[j] with bit 15
//    set when signs[j] < 0: the byte offset of the source element in the staged row and its sign.
//    One 32-bit table word drives the gather of an adjacent pair, its sign flips and its stage 1.
//    The table is stored in the order the lanes read it (16-byte chunks of consecutive lanes
//    adjacent), so the 16-byte table loads are free of bank conflicts.
//  - rows are double-buffered at two fixed shared-memory offsets (0 and kStride) and the gather is
//    compiled once per buffer (a row takes the instance of its buffer; the rotation's loop is
//    unrolled by two), so every gather address is a table offset plus a constant.
//  - warp w always owns the same h-blocks (block groups g = w, w + nwarps, ...; a group is the
//    32 / S blocks that fill the warp's lanes) and transposes them through its own scratch, whose
//    per-lane addresses are computed once per launch; pass 0's 16-byte stores are chunk-swizzled
//    by row and the blocks of a group are 16 banks apart, so the transpose is conflict free.
//  - the stages after the first of each pass, the scale and, in the quantizer, the division and
//    the decisions run on packed fp32 pairs.
// Quantizer: the row norm is an fp64 sum of the squares (each warp's part reduced in the warp);
// the last warp to deliver its part adds the parts in warp order, takes the root and publishes
// rho, rho + 1e-10 and its reciprocal; one CTA barrier per row makes them visible. Codes go
// through the warp's scratch as bytes and are packed 32 to a lane.
// Activation rotation: a producer warp streams rows into the two buffers (a buffer is refilled
// once every compute warp has released it), and outputs go from registers to global memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "rpbh_lanes.cuh"

namespace wq {
namespace rpbh_lanes {

using rpbh_fast::Edges;

constexpr uint32_t kMaxPolls = 1u << 24;
__device__ unsigned int g_fault;

template <int B>
struct Geo {
    static constexpr int S = 1 << B, H = S * S, KB = 32 / S;
    static constexpr int KS = B == 4 ? 2 : 1;           // block groups a warp holds at once (quantizer)
    static constexpr int BS = B == 4 ? 4 * H + 64 : 0;  // transpose bytes between the blocks of a group
    static constexpr int CS = H + 16;                   // code bytes between blocks
    static constexpr int SCR = B == 4 ? 2 * BS : 4 * H; // scratch bytes per warp
    static_assert(KS * KB * H / 32 == 32, "a warp's codes are one 32-code unit per lane");
    static_assert(KS * KB * CS <= SCR, "codes fit the transpose scratch");
};

// chunk swizzle of the transpose: row r's 16-byte chunk q lives at chunk q ^ swz(r)
template <int B>
__host__ __device__ constexpr int swz(int r) {
    return B == 4 ? ((r >> 1) & 3) : (r & 7);
}

__host__ __device__ constexpr int a128(int x) { return (x + 127) & ~127; }

// Shared-memory layout. Row buffers at 0 and stride; the table right after the second buffer's
// row; warp scratch in the gap after the first buffer's row while it fits, the rest after the
// table; then the reduction slots and the barriers.
struct Lay {
    int rowb, stride, tab, tabb, scr, nw, per_gap, hi, misc, total;
    __host__ __device__ Lay(int d, int stride_, int nw_, int S, int KS, int scr_) {
        rowb = 2 * d;
        stride = stride_;
        nw = nw_;
        scr = scr_;
        tabb = nw * KS * S * 64;
        tab = stride + a128(rowb);
        per_gap = (stride - a128(rowb)) / scr;
        if (per_gap > nw) per_gap = nw;
        if (per_gap < 0) per_gap = 0;
        hi = tab + a128(tabb);
        misc = hi + (nw - per_gap) * scr;
        total = misc + 512;
    }
    __host__ __device__ int scratch(int w) const { return w < per_gap ? a128(rowb) + w * scr : hi + (w - per_gap) * scr; }
};

// misc region: barriers (4 x 8 bytes: rows, buffers released), per-warp fp64 partial sums
// [2][16], published row parameters [2][4] (rho, den, 1 / den), arrival counters [2]
constexpr int kBarOff = 0, kRedOff = 64, kPrmOff = kRedOff + 2 * 16 * 8, kCntOff = kPrmOff + 2 * 4 * 4;

// Builds the gather table: chunk ch = ((w KS + k) S/8 + q) 32 + lane holds the entries of positions
// j0 .. j0 + 7, j0 = blk h + rc S + 8 q, of the lane's row in slot k (zero where the lane has no
// block). One step per chunk: perm[j0 .. j0 + 7] and signs[j0 .. j0 + 7] by vector loads (perm
// 16-byte and signs 8-byte aligned, as j0 is a multiple of 8), one 16-byte store. Runs while the
// first rows are in flight.
template <int B>
__device__ void build_table(unsigned char *sm, const Lay &L, int d, int KS, const int32_t *__restrict__ perm,
                            const int8_t *__restrict__ signs, int tid, int nthreads) {
    using G = Geo<B>;
    constexpr int S = G::S, H = G::H, KB = G::KB;
    const int nb = d / H, ngroups = (nb + KB - 1) / KB;
    uint4 *tab = reinterpret_cast<uint4 *>(sm + L.tab);
    const int nch = L.nw * KS * (S / 8) * 32;
    for (int ch = tid; ch < nch; ch += nthreads) {
        const int lane = ch & 31, rest = ch >> 5;
        const int q = rest % (S / 8), wk = rest / (S / 8);
        const int k = wk % KS, w = wk / KS;
        const int g = w + k * L.nw, blk = g * KB + lane / S, rc = lane % S;
        uint32_t e[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (g < ngroups && blk < nb) {
            const int j0 = blk * H + rc * S + 8 * q;
            const int4 p0 = __ldg(reinterpret_cast<const int4 *>(perm + j0));
            const int4 p1 = __ldg(reinterpret_cast<const int4 *>(perm + j0 + 4));
            const uint2 sv = __ldg(reinterpret_cast<const uint2 *>(signs + j0));
            const int32_t pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t pc = (uint32_t)pv[i] < (uint32_t)d ? (uint32_t)pv[i] : 0u;
                const uint32_t sb = ((i < 4 ? sv.x : sv.y) >> (8 * (i & 3) + 7)) & 1u;
                e[i] = (pc << 1) | (sb << 15);
            }
        }
        tab[ch] = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
    }
}

// Thread 0, before the kernel waits for the one it depends on: L2 prefetches of the CTA's first
// two rows (bulk prefetches: 16-byte aligned, 2 d bytes a multiple of 16). The tables are left
// out: every CTA reads the same ones, which stay in L2 from launch to launch, and prefetching
// them from every CTA measured slower on rows of 3072.
__device__ __forceinline__ void prefetch_start(const uint16_t *x, int rows, int d) {
    for (int b = 0; b < 2; ++b) {
        const int r = (int)blockIdx.x + b * (int)gridDim.x;
        if (r < rows) bulk_prefetch_l2(x + (int64_t)r * d, 2u * (uint32_t)d);
    }
}

// Pass 0 of one matrix row: the S positions a lane owns, through the table chunks tw[0], tw[32],
// ... Each 32-bit table word gathers a pair from the row buffer at byte kOff: the entry's low
// 15 bits are the byte offset, bit 15 flips the element's sign; the pair's stage-1 butterfly
// follows, then stages 2 .. S/2 on packed pairs.
template <int S, int kOff>
__device__ __forceinline__ void gather_pass0(float (&y)[S], const unsigned char *sm, const uint4 *tw) {
    uint32_t W[S / 2];
#pragma unroll
    for (int q = 0; q < S / 8; ++q) {
        const uint4 v = tw[32 * q];
        W[4 * q] = v.x;
        W[4 * q + 1] = v.y;
        W[4 * q + 2] = v.z;
        W[4 * q + 3] = v.w;
    }
#pragma unroll
    for (int k = 0; k < S / 2; ++k) {
        const uint32_t v0 = *reinterpret_cast<const uint16_t *>(sm + kOff + (W[k] & 0x7ffeu));
        const uint32_t v1 = *reinterpret_cast<const uint16_t *>(sm + kOff + ((W[k] >> 16) & 0x7ffeu));
        const float x0 = __uint_as_float((v0 ^ (W[k] & 0x8000u)) << 16);
        const float x1 = __uint_as_float((v1 << 16) ^ (W[k] & 0x80000000u));
        y[2 * k] = __fadd_rn(x0, x1);
        y[2 * k + 1] = __fsub_rn(x0, x1);
    }
    f32x2 P[S / 2];
#pragma unroll
    for (int k = 0; k < S / 2; ++k) P[k] = pk2(y[2 * k], y[2 * k + 1]);
#pragma unroll
    for (int hp = 1; hp < S / 2; hp <<= 1)
#pragma unroll
        for (int k = 0; k < S / 2; ++k)
            if ((k & hp) == 0) {
                const f32x2 a = P[k], b = P[k + hp];
                P[k] = add2(a, b);
                P[k + hp] = sub2(a, b);
            }
#pragma unroll
    for (int k = 0; k < S / 2; ++k) upk2(P[k], y[2 * k], y[2 * k + 1]);
}

// Pass 1 of one matrix column: stages S .. h/2 (stage 1 of the column scalar, the rest on packed
// pairs (y[2i], y[2i + 1])), then the scale; the result stays packed.
template <int S>
__device__ __forceinline__ void column_pass(float (&y)[S], f32x2 (&P)[S / 2], f32x2 post2) {
#pragma unroll
    for (int k = 0; k < S; k += 2) {
        const float a = y[k], b = y[k + 1];
        y[k] = __fadd_rn(a, b);
        y[k + 1] = __fsub_rn(a, b);
    }
#pragma unroll
    for (int k = 0; k < S / 2; ++k) P[k] = pk2(y[2 * k], y[2 * k + 1]);
#pragma unroll
    for (int hp = 1; hp < S / 2; hp <<= 1)
#pragma unroll
        for (int k = 0; k < S / 2; ++k)
            if ((k & hp) == 0) {
                const f32x2 a = P[k], b = P[k + hp];
                P[k] = add2(a, b);
                P[k + hp] = sub2(a, b);
            }
#pragma unroll
    for (int k = 0; k < S / 2; ++k) P[k] = mul2(P[k], post2);
}

// Per-lane transpose addresses (byte offsets into shared memory), fixed for the launch.
template <int B>
struct Xpose {
    static constexpr int S = 1 << B, NSW = B == 4 ? 4 : 8;
    int st[S / 4];  // pass 0: chunk q of the lane's row
    int ld[NSW];    // pass 1: element (t, c) at ld[swz(t)] + 4 S t
    __device__ void init(int scr, int sub, int r) {
        using G = Geo<B>;
        const int base = scr + sub * G::BS;
#pragma unroll
        for (int q = 0; q < S / 4; ++q) st[q] = base + 4 * S * r + 16 * (q ^ swz<B>(r));
#pragma unroll
        for (int s = 0; s < NSW; ++s) ld[s] = base + 16 * ((r >> 2) ^ s) + 4 * (r & 3);
    }
    __device__ __forceinline__ void store(unsigned char *sm, const float (&y)[S]) const {
#pragma unroll
        for (int q = 0; q < S / 4; ++q)
            *reinterpret_cast<float4 *>(sm + st[q]) = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
    }
    __device__ __forceinline__ void load(const unsigned char *sm, float (&y)[S]) const {
#pragma unroll
        for (int t = 0; t < S; ++t) y[t] = *reinterpret_cast<const float *>(sm + ld[swz<B>(t)] + 4 * S * t);
    }
};

// 3-bit decisions as rpbh_fast::sym_codes, with the sign applied by one packed fma:
// 2^22 + mid + 1/2 + sgn (c + 1/2), exact, whose low byte is twice the code.
__device__ __forceinline__ f32x2 sym_codes3x2(f32x2 u, const Edges &E) {
    float u0, u1;
    upk2(u, u0, u1);
    const f32x2 ap = rpbh_fast::fma_rp2(u, pk2(-0x1p-24f, -0x1p-24f), pk2(fabsf(u0), fabsf(u1)));
    float a0, a1;
    upk2(ap, a0, a1);
    f32x2 c = pk2(0.5f, 0.5f);
#pragma unroll
    for (int i = 0; i < 3; ++i)
        c = add2(c, pk2(__saturatef(__fmaf_rn(a0, E.M[i], E.K[i])), __saturatef(__fmaf_rn(a1, E.M[i], E.K[i]))));
    float b0, b1;
    upk2(rpbh_fast::fma_rm2(u, pk2(1.0f, 1.0f), pk2(-0.0f, -0.0f)), b0, b1);
    const f32x2 sg = pk2(__uint_as_float((__float_as_uint(b0) & 0x80000000u) | 0x3f800000u),
                         __uint_as_float((__float_as_uint(b1) & 0x80000000u) | 0x3f800000u));
    constexpr float kB = 4194304.0f + 3.5f;  // 2^22 + mid + 1/2
    return fma2(sg, c, pk2(kB, kB));
}

// 32 codes to BITS words of the MSB-first stream: code i in byte i of cw (3 bits: twice the code,
// as sym_codes3x2 leaves it).
template <int BITS>
__device__ __forceinline__ void pack_unit(const uint32_t (&cw)[8], uint32_t (&word)[BITS]) {
    if constexpr (BITS == 3) {
        // each word of four bytes (twice the codes c0 .. c3) gives twice the 12-bit chunk
        // c0 c1 c2 c3 (MSB first) by two 16x8-bit dot products (weights 512, 64 on bytes 0, 1, then
        // 8, 1 on bytes 2, 3); the shifts below halve it while placing the eight chunks
        uint32_t ch[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t r;
            asm("dp2a.lo.u32.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(0x00400200u), "r"(cw[j]), "r"(0u));
            asm("dp2a.hi.u32.u32 %0, %1, %2, %3;" : "=r"(ch[j]) : "r"(0x00010008u), "r"(cw[j]), "r"(r));
        }
        word[0] = (ch[0] << 19) | (ch[1] << 7) | (ch[2] >> 5);
        word[1] = (ch[2] << 27) | (ch[3] << 15) | (ch[4] << 3) | (ch[5] >> 9);
        word[2] = (ch[5] << 23) | (ch[6] << 11) | (ch[7] >> 1);
    } else {
        rpbh_fast::pack32<BITS>(cw, word);
    }
}

// ---------------------------------------------------------------------------------------------
// _quantize_rows
// ---------------------------------------------------------------------------------------------
template <int B, int BITS, int kStride>
__global__ void __maxnreg__(B == 4 ? 80 : 96)
    quantize_lanes(const uint16_t *__restrict__ w, int rows, int d, float post, const int32_t *__restrict__ perm,
                   const int8_t *__restrict__ signs, Edges E, uint8_t *__restrict__ packed,
                   void *__restrict__ row_norms) {
    using G = Geo<B>;
    constexpr int S = G::S, H = G::H, KB = G::KB, KS = G::KS;
    extern __shared__ __align__(128) unsigned char sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (int)(blockDim.x >> 5);
    const int sub = lane / S, rc = lane % S;
    const int nb = d / H, ngroups = (nb + KB - 1) / KB;
    const Lay L(d, kStride, nw, S, KS, G::SCR);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L.misc + kBarOff);
    double *red = reinterpret_cast<double *>(sm + L.misc + kRedOff);
    float *prm = reinterpret_cast<float *>(sm + L.misc + kPrmOff);
    int *cnt = reinterpret_cast<int *>(sm + L.misc + kCntOff);
    const uint32_t rowb = (uint32_t)L.rowb;
    int row = blockIdx.x;

    bool fault = false;
    // While the kernel before this one finishes, its tail overlaps the fetch of this CTA's first
    // rows into L2 (a prefetch only warms the cache: the rows are read after the wait below, and
    // L2 keeps them coherent with that kernel's writes).
    if (threadIdx.x == 0) prefetch_start(w, rows, d);
    pdl_wait();  // the rows, tables and outputs may belong to the kernel before this one
    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        cnt[0] = 0;
        cnt[1] = 0;
        // the CTA's first two rows, one into each buffer
        for (int b = 0; b < 2; ++b) {
            const int r = row + b * (int)gridDim.x;
            if (r < rows) {
                mbar_expect_tx(&bar[b], rowb);
                bulk_load(sm + b * kStride, w + (int64_t)r * d, rowb, &bar[b]);
            }
        }
    }
    build_table<B>(sm, L, d, KS, perm, signs, threadIdx.x, blockDim.x);
    __syncthreads();  // table, barriers and counters are ready
    const int scr = L.scratch(warp);
    Xpose<B> X;
    X.init(scr, sub, rc);
    const int cbase = scr + sub * G::CS + rc;  // this lane's codes: + slot block offset + t S
    const uint4 *tw = reinterpret_cast<const uint4 *>(sm + L.tab) + warp * KS * (S / 8) * 32 + lane;
    // pack: lane -> (block of the warp's KS x KB, 32-code unit)
    const int pbw = lane / (H / 32), pq = lane % (H / 32);
    const int pk = pbw / KB, pg = warp + pk * nw, pblk = pg * KB + pbw % KB;
    const bool pvalid = pg < ngroups && pblk < nb;
    const int psrc = scr + pbw * G::CS + 32 * pq;
    const int64_t prow_bytes = (int64_t)d / 8 * BITS;
    const int pdst = (pblk * H + 32 * pq) / 8 * BITS;
    const f32x2 post2 = pk2(post, post);

    // thread 0: the buffer and phase of the last row copy it issued (the set-up copies first)
    int last_buf = row + (int)gridDim.x < rows ? 1 : (row < rows ? 0 : -1);
    uint32_t last_par = 0;
    int it = 0;
    for (; row < rows; row += (int)gridDim.x, ++it) {
        const int kBuf = it & 1;
        if (row + (int)gridDim.x >= rows) pdl_trigger();  // the CTA's last row: the next kernel may be scheduled
        if (!fault && !mbar_wait_bounded(&bar[kBuf], (uint32_t)((it >> 1) & 1), kMaxPolls)) {
            fault = true;
            atomicOr(&g_fault, 2u);
        }
        f32x2 zk[KS][S / 2];
        double ss = 0.0;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int g = warp + k * nw, blk = g * KB + sub;
            if (g < ngroups) {  // warp-uniform
                if (blk < nb) {
                    float y[S];
                    if (kBuf)
                        gather_pass0<S, kStride>(y, sm, tw + k * (S / 8) * 32);
                    else
                        gather_pass0<S, 0>(y, sm, tw + k * (S / 8) * 32);
                    X.store(sm, y);
                }
                __syncwarp();
                if (blk < nb) {
                    float y[S];
                    X.load(sm, y);
                    column_pass<S>(y, zk[k], post2);
#pragma unroll
                    for (int i = 0; i < S / 2; ++i) {
                        float a, b;
                        upk2(zk[k][i], a, b);
                        ss = __fma_rn((double)a, (double)a, ss);
                        ss = __fma_rn((double)b, (double)b, ss);
                    }
                }
                __syncwarp();  // the columns are read before the next slot's rows overwrite the scratch
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
        fence_proxy_async_smem();  // this thread's reads of the row buffer precede the copy that refills it
        const int set = it & 1;
        if (lane == 0) {
            red[set * 16 + warp] = ss;
            __threadfence_block();
            if (atomicAdd(&cnt[set], 1) == nw - 1) {
                __threadfence_block();
                const volatile double *rv = red + set * 16;
                double tot = 0.0;
                for (int v = 0; v < nw; ++v) tot = __dadd_rn(tot, rv[v]);
                const float rho = __double2float_rn(__dsqrt_rn(tot));
                const float den = __fadd_rn(rho, 1e-10f);
                prm[set * 4 + 0] = rho;
                prm[set * 4 + 1] = den;
                prm[set * 4 + 2] = __frcp_rn(den);
                cnt[set] = 0;
                if (E.norm_bf16)
                    static_cast<uint16_t *>(row_norms)[row] = f32_to_bf16(rho);
                else
                    static_cast<float *>(row_norms)[row] = rho;
            }
        }
        __syncthreads();
        // every thread has gathered from this buffer: it takes the row after next
        const int r2 = row + 2 * (int)gridDim.x;
        if (threadIdx.x == 0 && r2 < rows && !fault) {
            mbar_expect_tx(&bar[kBuf], rowb);
            bulk_load(sm + kBuf * kStride, w + (int64_t)r2 * d, rowb, &bar[kBuf]);
            last_buf = kBuf;
            last_par = (uint32_t)(((it + 2) >> 1) & 1);
        }
        const float den = prm[set * 4 + 1], rden = prm[set * 4 + 2];
        // u = z / den by Markstein's correction (q0 = RN(z r), rem = RN(z - q0 den) by one fma,
        // u = RN(q0 + rem r)): the correctly rounded quotient whenever |z| >= 2^-100 and z / den is
        // a normal value, at most one unit in the last place off below that; then the codes, one
        // byte each in element order
        const f32x2 RDEN = pk2(rden, rden), NDEN = pk2(-den, -den);
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int g = warp + k * nw, blk = g * KB + sub;
            if (g < ngroups && blk < nb) {
                unsigned char *cb = sm + cbase + k * KB * G::CS;
#pragma unroll
                for (int i = 0; i < S / 2; ++i) {
                    const f32x2 z = zk[k][i];
                    const f32x2 q0 = mul2(z, RDEN);
                    const f32x2 u = fma2(fma2(q0, NDEN, z), RDEN, q0);
                    float v0, v1;
                    if constexpr (BITS == 3)
                        upk2(sym_codes3x2(u, E), v0, v1);
                    else
                        upk2(rpbh_fast::sym_codes<BITS>(u, E), v0, v1);
                    cb[(2 * i) * S] = (uint8_t)__float_as_uint(v0);
                    cb[(2 * i + 1) * S] = (uint8_t)__float_as_uint(v1);
                }
            }
        }
        __syncwarp();
        if (pvalid) {
            const uint4 c0 = *reinterpret_cast<const uint4 *>(sm + psrc);
            const uint4 c1 = *reinterpret_cast<const uint4 *>(sm + psrc + 16);
            const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t word[BITS];
            pack_unit<BITS>(cw, word);
            uint32_t *out = reinterpret_cast<uint32_t *>(packed + (int64_t)row * prow_bytes + pdst);
#pragma unroll
            for (int j = 0; j < BITS; ++j) out[j] = __byte_perm(word[j], 0, 0x0123);
        }
        __syncwarp();  // the codes are read before the next row's transposes rewrite the scratch
    }
    // a fault may leave thread 0's last row copy in flight: give it a bounded chance to land
    if (fault && threadIdx.x == 0 && last_buf >= 0) mbar_wait_bounded(&bar[last_buf], last_par, kMaxPolls);
}

// ---------------------------------------------------------------------------------------------
// rpbh_forward on activation rows (bf16 in, bf16 out)
// ---------------------------------------------------------------------------------------------
template <int B, int kStride>
__global__ void __maxnreg__(80)
    rotate_lanes(const uint16_t *__restrict__ x, int rows, int d, float post, const int32_t *__restrict__ perm,
                 const int8_t *__restrict__ signs, uint16_t *__restrict__ out) {
    using G = Geo<B>;
    constexpr int S = G::S, H = G::H, KB = G::KB, KS = G::KS;
    extern __shared__ __align__(128) unsigned char sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (int)(blockDim.x >> 5) - 1;
    const int sub = lane / S, rc = lane % S;
    const int nb = d / H, ngroups = (nb + KB - 1) / KB;
    const Lay L(d, kStride, nw, S, KS, G::SCR);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L.misc + kBarOff);
    uint64_t *empty = full + 2;
    const uint32_t rowb = (uint32_t)L.rowb;

    bool fault = false;
    if (threadIdx.x == 0) prefetch_start(x, rows, d);  // as in quantize_lanes
    pdl_wait();  // the rows, tables and outputs may belong to the kernel before this one
    if (threadIdx.x == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], (uint32_t)nw);
        mbar_init(&empty[1], (uint32_t)nw);
    }
    __syncthreads();  // the barriers are initialised before the producer's first copies land on them

    if (warp == nw) {  // producer: one lane streams the CTA's rows into the two buffers
        if (lane == 0) {
            int n = 0;
            uint32_t issued[2] = {0u, 0u};
            bool ok = true;
            for (int row = blockIdx.x; row < rows; row += (int)gridDim.x, ++n) {
                const int b = n & 1;
                if (n >= 2 && !mbar_wait_bounded(&empty[b], (uint32_t)(((n >> 1) - 1) & 1), kMaxPolls)) {
                    atomicOr(&g_fault, 2u);
                    ok = false;
                    break;
                }
                mbar_expect_tx(&full[b], rowb);
                bulk_load(sm + b * kStride, x + (int64_t)row * d, rowb, &full[b]);
                ++issued[b];
            }
            // after a fault, give the copies in flight a bounded chance to land before the CTA exits
            if (!ok)
                for (int b = 0; b < 2; ++b)
                    if (issued[b]) mbar_wait_bounded(&full[b], (issued[b] - 1) & 1u, kMaxPolls);
        }
        return;
    }
    // the compute warps build the table while the first rows are in flight
    build_table<B>(sm, L, d, KS, perm, signs, threadIdx.x, 32 * nw);
    asm volatile("bar.sync 1, %0;" ::"r"(32 * nw) : "memory");

    const int scr = L.scratch(warp);
    Xpose<B> X;
    X.init(scr, sub, rc);
    const uint4 *tw = reinterpret_cast<const uint4 *>(sm + L.tab) + warp * KS * (S / 8) * 32 + lane;
    const f32x2 post2 = pk2(post, post);
    int it = 0;
    int row = blockIdx.x;
    auto body = [&](auto kb) {
        constexpr int kBuf = decltype(kb)::value;
        if (row + (int)gridDim.x >= rows) pdl_trigger();  // the CTA's last row: the next kernel may be scheduled
        if (!fault && !mbar_wait_bounded(&full[kBuf], (uint32_t)((it >> 1) & 1), kMaxPolls)) {
            fault = true;
            atomicOr(&g_fault, 2u);
        }
        uint16_t *orow = out + (int64_t)row * d;
        for (int g = warp; g < ngroups; g += nw) {
            const int blk = g * KB + sub;
            const int k = (g - warp) / nw;  // slot: which of the warp's table runs
            if (blk < nb) {
                float y[S];
                gather_pass0<S, kBuf * kStride>(y, sm, tw + k * (S / 8) * 32);
                X.store(sm, y);
            }
            __syncwarp();
            if (blk < nb) {
                float y[S];
                f32x2 P[S / 2];
                X.load(sm, y);
                column_pass<S>(y, P, post2);
                uint16_t *o = orow + blk * H + rc;
#pragma unroll
                for (int i = 0; i < S / 2; ++i) {
                    float a, b;
                    upk2(P[i], a, b);
                    o[(2 * i) * S] = f32_to_bf16(a);
                    o[(2 * i + 1) * S] = f32_to_bf16(b);
                }
            }
            __syncwarp();  // the columns are read before the warp's next group rewrites the scratch
        }
        fence_proxy_async_smem();  // this lane's reads of the row buffer precede the copy that refills it
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[kBuf]);
    };
    while (row < rows) {
        body(std::integral_constant<int, 0>{});
        row += (int)gridDim.x;
        ++it;
        if (row >= rows) break;
        body(std::integral_constant<int, 1>{});
        row += (int)gridDim.x;
        ++it;
    }
}

// ---------------------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------------------
namespace {

int block_log2(int64_t d) {
    const int64_t h = d & -d;
    int l = 0;
    while ((int64_t(1) << l) < h) ++l;
    return l;
}

int stride_for(int64_t d) { return d <= 4096 ? 8192 : d <= 12288 ? 24576 : 32768; }

size_t smem_optin() {
    static size_t cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
        cached[dev] = (size_t)v;
    }
    return cached[dev];
}

int sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
    return cached[dev];
}

// warps holding block groups: every group in KS slots per warp (quantizer) or one slot per warp
// pass (rotation, with the same warp count so that the table layouts agree)
int compute_warps(int64_t d, int B) {
    const int S = 1 << B, H = S * S, KB = 32 / S, KS = B == 4 ? 2 : 1;
    const int nb = (int)(d / H), ngroups = (nb + KB - 1) / KB;
    return (ngroups + KS - 1) / KS;
}

bool shape_ok(int64_t d) {
    if (d <= 0 || d > 16384) return false;
    const int l = block_log2(d);
    return l == 8 || l == 10;
}

size_t lay_total(int64_t d, int B) {
    const int S = 1 << B, KS = B == 4 ? 2 : 1, scr = B == 4 ? 2 * (4 * S * S + 64) : 4 * S * S;
    const Lay L((int)d, stride_for(d), compute_warps(d, B), S, KS, scr);
    return (size_t)L.total;
}

template <typename K>
int grid_for(K k, int threads, size_t smem, int64_t rows) {
    int per = blocks_per_sm_cached(reinterpret_cast<const void *>(k), threads, smem);
    if (per < 1) per = 1;
    const int64_t g = (int64_t)per * sms();
    return (int)(g < rows ? g : rows);
}

template <int B, int kStride>
wq_status rotate_launch(const uint16_t *x, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                        uint16_t *out, cudaStream_t s) {
    auto k = rotate_lanes<B, kStride>;
    const size_t smem = lay_total(d, B);
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return WQ_ERR_CUDA;
    const int threads = 32 * (compute_warps(d, B) + 1);
    const float post = (float)std::pow((double)(d & -d), -0.5);
    if (launch_pdl(k, (unsigned)grid_for(k, threads, smem, rows), (unsigned)threads, smem, s, x, (int)rows, (int)d, post,
                   perm, signs, out) != cudaSuccess)
        return WQ_ERR_CUDA;
    return launch_status();
}

template <int B, int BITS, int kStride>
wq_status quantize_launch(const uint16_t *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                          const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    auto k = quantize_lanes<B, BITS, kStride>;
    const size_t smem = lay_total(d, B);
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), smem)) return WQ_ERR_CUDA;
    const int threads = 32 * compute_warps(d, B);
    const float post = (float)std::pow((double)(d & -d), -0.5);
    if (launch_pdl(k, (unsigned)grid_for(k, threads, smem, rows), (unsigned)threads, smem, s, w, (int)rows, (int)d, post,
                   perm, signs, E, packed, row_norms) != cudaSuccess)
        return WQ_ERR_CUDA;
    return launch_status();
}

template <int B>
wq_status rotate_b(const uint16_t *x, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, uint16_t *out,
                   cudaStream_t s) {
    switch (stride_for(d)) {
        case 8192: return rotate_launch<B, 8192>(x, rows, d, perm, signs, out, s);
        case 24576: return rotate_launch<B, 24576>(x, rows, d, perm, signs, out, s);
        default: return rotate_launch<B, 32768>(x, rows, d, perm, signs, out, s);
    }
}

template <int B, int BITS>
wq_status quantize_bs(const uint16_t *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                      const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    switch (stride_for(d)) {
        case 8192: return quantize_launch<B, BITS, 8192>(w, rows, d, perm, signs, E, packed, row_norms, s);
        case 24576: return quantize_launch<B, BITS, 24576>(w, rows, d, perm, signs, E, packed, row_norms, s);
        default: return quantize_launch<B, BITS, 32768>(w, rows, d, perm, signs, E, packed, row_norms, s);
    }
}

template <int B>
wq_status quantize_b(int bits, const uint16_t *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs,
                     const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    switch (bits) {
        case 2: return quantize_bs<B, 2>(w, rows, d, perm, signs, E, packed, row_norms, s);
        case 3: return quantize_bs<B, 3>(w, rows, d, perm, signs, E, packed, row_norms, s);
        case 4: return quantize_bs<B, 4>(w, rows, d, perm, signs, E, packed, row_norms, s);
        default: return WQ_ERR_BITS;
    }
}

}  // namespace

bool rotate_fits(int64_t d) {
    if (!shape_ok(d)) return false;
    const int B = block_log2(d) / 2;
    return compute_warps(d, B) + 1 <= 32 && lay_total(d, B) + 1024 <= smem_optin();
}

bool quantize_fits(int64_t d, const Edges &E) {
    if (!shape_ok(d) || !E.steps) return false;
    const int B = block_log2(d) / 2;
    return compute_warps(d, B) <= 16 && lay_total(d, B) + 1024 <= smem_optin();
}

wq_status rotate(const uint16_t *x, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, uint16_t *out,
                 cudaStream_t s) {
    if (rows <= 0) return WQ_OK;
    return block_log2(d) == 8 ? rotate_b<4>(x, rows, d, perm, signs, out, s)
                              : rotate_b<5>(x, rows, d, perm, signs, out, s);
}

wq_status quantize(const uint16_t *w, int64_t rows, int64_t d, const int32_t *perm, const int8_t *signs, int bits,
                   const Edges &E, uint8_t *packed, void *row_norms, cudaStream_t s) {
    if (rows <= 0) return WQ_OK;
    return block_log2(d) == 8 ? quantize_b<4>(bits, w, rows, d, perm, signs, E, packed, row_norms, s)
                              : quantize_b<5>(bits, w, rows, d, perm, signs, E, packed, row_norms, s);
}

unsigned int read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(g_fault, &zero, sizeof zero);
    return v;
}

}  // namespace rpbh_lanes
}  // namespace wq
