// Attention over a TQ3-compressed K/V cache on the tensor cores (tcgen05), for many query rows per
// head (prefill): the same operation and the same rotated-basis identities as tq3_attn.cu (page
// "tq3_core.py": tq3_dequantize gives the vectors the attention reads),
//     logit_j = coef * norm_j * scale_j * (q~ . c[idx_j]),       q~ = H (s . q),
//     out     = s . H( sum_j p_j norm_j scale_j c[idx'_j] / sum_j p_j ) * post,
// computed for 128 query rows at a time as two products per tile of 128 keys:
//     S = Q~ C_K^T            (M = 128 rows, N = 128 keys, K = 128 rotated coordinates)
//     O += P C_V              (M = 128 rows, N = 128 coordinates, K = 128 keys)
// with the key factor coef * norm_j * scale_j folded into C_K's row j and norm_j * scale_j into
// C_V's row j. The operands are bf16 on the tensor core, so every fp32 operand x is split into
// x = hi + lo (hi = bf16(x), lo = bf16(x - hi), |x - hi - lo| <= 2^-18 |x|) and each product takes
// three passes, hi hi + hi lo + lo hi (the dropped lo lo is below 2^-18 of a term), all accumulating
// in fp32 in tensor memory.
//
// One CTA of 256 threads serves one (head, 128-row chunk); all of the head's keys, tile by tile:
//   1. the tile's key and value records arrive by 8-byte cp.async;
//   2. all threads expand the key centroids, times the key factor, into C_K (hi and lo, bf16,
//      128-byte-swizzled K-major operand tiles); thread 0 issues S = Q~ C_K^T (3 x 8 mma);
//   3. warps 0-3 (thread r = query row r = tensor-memory lane r) read their row of S, update the
//      running max (raised only when it grows by more than 8 in log2 units, so the output
//      accumulator is rescaled rarely), form p = 2^(s - max), add it to the row sum and write P
//      (hi and lo) as their row of the next A operand; warps 4-7 meanwhile expand the value
//      centroids, times norm * scale, into C_V^T (coordinate-major, so that K = keys);
//   4. thread 0 issues O += P C_V (3 x 8 mma).
// At the end thread r reads its row of O, divides by its row sum, applies the inverse transform
// (seven butterfly stages in registers), post and the signs, and stores the row. Every wait on the
// tensor core is bounded: on a timeout the fault flag is set and the CTA gives in-flight products a
// bounded chance to finish, frees its tensor memory and returns.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "tcgen05.cuh"
#include "tq3_attn_mma.cuh"
#include "tq3_common.cuh"

namespace cg = cooperative_groups;

namespace wq {
namespace tq3_attn_mma {

using tq3::SignMask;

constexpr int kRows = 128;     // query rows per CTA (M)
constexpr int kKeys = 128;     // keys per tile
constexpr int kThreads = 256;
constexpr int kWords = 14;
constexpr int kBox = 128 * 128;   // one 64-column half of a 128 x 128 bf16 operand, in bytes
constexpr int kOp = 2 * kBox;     // one operand tile
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kMaxPolls = 1u << 24;
constexpr float kLazy = 8.0f;     // the running max is raised only past this margin (log2 units)

// shared memory (offsets from a 1024-byte aligned base)
constexpr int kOffQh = 0, kOffQl = kOp, kOffBh = 2 * kOp, kOffBl = 3 * kOp, kOffPh = 4 * kOp, kOffPl = 5 * kOp;
constexpr int kRecBytes = kKeys * kWords * 4;   // one tensor's records of one tile
constexpr int kOffRec = 6 * kOp;                  // [buffer][K, V] records, double-buffered by tile
constexpr int kOffFac = kOffRec + 4 * kRecBytes;  // per key: coef norm scale (K), norm scale (V)
constexpr int kOffValid = kOffFac + 2 * kKeys * 4;  // [buffer][key]
constexpr int kOffMerge = kOffValid + 2 * kKeys * 4;  // per row: running max and sum (cluster merge)
constexpr int kOffBar = kOffMerge + 2 * kRows * 4;
constexpr int kSmem = 1024 + kOffBar + 32;
constexpr int kMaxSplit = 8;  // CTAs of a cluster sharing one (head, row chunk)
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

__device__ unsigned int g_fault;

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// 16-byte chunk `chunk` (elements 8 chunk .. 8 chunk + 7 of K) of operand row `row`.
__device__ __forceinline__ uint4 *op_chunk(unsigned char *op, int row, int chunk) {
    return reinterpret_cast<uint4 *>(op + (chunk >> 3) * kBox + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// x = hi + lo for a pair of fp32 values, as two bf16x2 words (element a in the low half).
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16x2(a, b);
    const float ha = __uint_as_float(hi << 16), hb = __uint_as_float(hi & 0xffff0000u);
    lo = pack_bf16x2(__fsub_rn(a, ha), __fsub_rn(b, hb));
}

// Eight fp32 values as one chunk of the hi operand and one of the lo operand.
__device__ __forceinline__ void put8(unsigned char *oph, unsigned char *opl, int row, int chunk, const float (&v)[8]) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split2(v[2 * i], v[2 * i + 1], h[i], l[i]);
    *op_chunk(oph, row, chunk) = make_uint4(h[0], h[1], h[2], h[3]);
    *op_chunk(opl, row, chunk) = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Record index of key j of head h (contiguous or through the page table), or -1 outside the pool.
__device__ __forceinline__ int64_t record_of(const Cache &kv, int64_t head, int64_t S, int64_t j) {
    if (kv.table == nullptr) return head * S + j;
    const int32_t page = __ldg(kv.table + head * kv.pages_per_head + (j >> kv.shift));
    const int64_t r = ((int64_t)page << kv.shift) | (j & ((int64_t(1) << kv.shift) - 1));
    return (page >= 0 && r < kv.n_pool) ? r : -1;
}

__device__ __forceinline__ float sign_of(const SignMask &m, int e) { return ((m.w[e >> 5] >> (e & 31)) & 1u) ? 1.0f : -1.0f; }

// Unnormalised 128-point FWHT of 128 register values, stages h = 1 .. 64.
__device__ __forceinline__ void fwht128(float (&v)[128]) {
#pragma unroll
    for (int h = 1; h < 128; h <<= 1)
#pragma unroll
        for (int i = 0; i < 128; ++i)
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = __fadd_rn(a, b);
                v[i + h] = __fsub_rn(a, b);
            }
}

// D (+)= A B^T over K = 128 in three passes hi hi + hi lo + lo hi.
__device__ __forceinline__ void mma3(uint32_t d, unsigned char *ah, unsigned char *al, unsigned char *bh,
                                     unsigned char *bl, uint32_t acc0) {
    const uint64_t dah = sw128_desc(smem_u32(ah)), dal = sw128_desc(smem_u32(al));
    const uint64_t dbh = sw128_desc(smem_u32(bh)), dbl = sw128_desc(smem_u32(bl));
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        const uint64_t a = pass == 2 ? dal : dah, b = pass == 1 ? dbl : dbh;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * kBox + (ks & 3) * 32) >> 4;
            mma_bf16(d, a + off, b + off, kIdesc, (pass > 0 || ks > 0) ? 1u : acc0);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_mma_kernel(const void *__restrict__ q, int q_bf16, int m, Cache kv, int64_t S, SignMask mask, float coef,
                    void *__restrict__ out, int out_bf16, int64_t head0) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *const base = tq3::tile_base(smem_raw);
    unsigned char *const Qh = base + kOffQh, *const Ql = base + kOffQl;
    unsigned char *const Bh = base + kOffBh, *const Bl = base + kOffBl;
    unsigned char *const Ph = base + kOffPh, *const Pl = base + kOffPl;
    float *const facK = reinterpret_cast<float *>(base + kOffFac);
    float *const facV = facK + kKeys;
    float *const mrow = reinterpret_cast<float *>(base + kOffMerge);
    float *const lrow = mrow + kRows;
    uint64_t *const bar = reinterpret_cast<uint64_t *>(base + kOffBar);  // [0] S done, [1] O done
    uint32_t *const tslot = reinterpret_cast<uint32_t *>(base + kOffBar + 16);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    cg::cluster_group cluster = cg::this_cluster();
    const int split = (int)cluster.block_rank(), n_split = (int)cluster.num_blocks();
    const int64_t head = head0 + blockIdx.y;
    const int r0 = (int)(blockIdx.x / n_split) * kRows;
    const float cb = tq3::centroid((uint32_t)(lane & 7));  // lane l holds centroid l mod 8
    const float post = tq3::fwht_post();

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
    }
    if (warp == 0) tmem_alloc(tslot, kTmemCols);
    // Q~ = H (s . q) for this CTA's rows (thread r < 128 owns row r; rows past m are zeros), split
    // into the two A operands of S
    if (tid < kRows) {
        float v[128];
        const int r = r0 + tid;
#pragma unroll
        for (int e = 0; e < 128; ++e) {
            float x = 0.0f;
            if (r < m) {
                const int64_t at = (head * m + r) * 128 + e;
                x = q_bf16 ? __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t *>(q) + at) << 16)
                           : __ldg(static_cast<const float *>(q) + at);
            }
            v[e] = __fmul_rn(x, sign_of(mask, e));
        }
        fwht128(v);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float w8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w8[i] = v[8 * c + i];
            put8(Qh, Ql, tid, c, w8);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tS = tmem, tO = tmem + 128;
    const uint32_t my_lanes = ((uint32_t)((warp & 3) * 32) << 16);

    float run_max = -INFINITY, run_sum = 0.0f;
    bool fault = false;
    uint32_t n_s = 0, n_o = 0;  // products committed (for the phases and the fault path)
    // this CTA's share of the head's key tiles
    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const int64_t t_begin = n_tiles * split / n_split, t_end = n_tiles * (split + 1) / n_split;
    // the records of a tile into buffer b (thread t < 128: key t's key record; t >= 128: key
    // t - 128's value record), with the key's validity
    auto fetch = [&](int64_t tile, int b) {
        const int key = tid & 127;
        const int64_t j = tile * kKeys + key;
        const int64_t rec = j < S ? record_of(kv, head, S, j) : -1;
        if (tid < 128) {
            if (j < S && rec < 0) atomicOr(&g_fault, tq3::kFaultPoolIndex);
            reinterpret_cast<int *>(base + kOffValid)[b * kKeys + key] = rec >= 0;
        }
        if (rec >= 0) {
            const uint8_t *src = (tid < 128 ? kv.k : kv.v) + rec * 56;
            uint32_t *dst = reinterpret_cast<uint32_t *>(base + kOffRec + (2 * b + (tid >= 128)) * kRecBytes) + key * kWords;
#pragma unroll
            for (int w = 0; w < kWords / 2; ++w) cp_async8(dst + 2 * w, src + 8 * w);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (t_begin < t_end) fetch(t_begin, 0);
    for (int64_t tile = t_begin; tile < t_end && !fault; ++tile) {
        // 1. this tile's records have landed; the next tile's are requested into the other buffer
        //    (its previous contents, tile - 1's, were last read before the last barrier)
        const int b = (int)((tile - t_begin) & 1);
        if (tile + 1 < t_end) {
            fetch(tile + 1, b ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        uint32_t(*const recK)[kWords] = reinterpret_cast<uint32_t(*)[kWords]>(base + kOffRec + 2 * b * kRecBytes);
        uint32_t(*const recV)[kWords] = reinterpret_cast<uint32_t(*)[kWords]>(base + kOffRec + (2 * b + 1) * kRecBytes);
        const int *const valid = reinterpret_cast<const int *>(base + kOffValid) + b * kKeys;
        // the previous tile's O product has read C_V and P before they are rewritten below
        if (n_o > 0) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(&bar[1], (n_o - 1) & 1u, kMaxPolls);
            if (__syncthreads_or(!ok)) {
                fault = true;
                break;
            }
            tc_fence_after();
        }
        // 2. C_K: thread t expands half t >> 7 (64 coordinates) of key t & 127, times the key factor
        {
            const int key = tid & 127, half = tid >> 7;
            const bool ok = valid[key] != 0;
            const float f = ok ? __fmul_rn(__fmul_rn(__uint_as_float(recK[key][12]), __uint_as_float(recK[key][13])), coef)
                               : 0.0f;
            if (half == 0) {
                facK[key] = f;
                facV[key] = valid[key] ? __fmul_rn(__uint_as_float(recV[key][12]), __uint_as_float(recV[key][13])) : 0.0f;
            }
            uint32_t W[7];
#pragma unroll
            for (int w = 0; w < 7; ++w) W[w] = ok ? recK[key][6 * half + w] : 0u;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                float v8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int o = 3 * (8 * g + i), wq = o >> 5, sh = o & 31;
                    const uint32_t idx = wq < 6 ? __funnelshift_r(W[wq], W[wq + 1], sh) : (W[wq] >> sh);
                    v8[i] = __fmul_rn(__shfl_sync(0xffffffffu, cb, (int)idx), f);
                }
                put8(Bh, Bl, key, 8 * half + g, v8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            mma3(tS, Qh, Ql, Bh, Bl, 0u);
            mma_commit(&bar[0]);
        }
        ++n_s;
        {
            bool ok = true;
            if (lane == 0) ok = mbar_wait_bounded(&bar[0], (n_s - 1) & 1u, kMaxPolls);
            if (__syncthreads_or(!ok)) {
                fault = true;
                break;
            }
        }
        tc_fence_after();
        if (warp < 4) {
            // 3a. softmax of row tid against the tile's keys
            float s[128];
            tmem_ld32(tS + my_lanes + 0, *reinterpret_cast<float(*)[32]>(&s[0]));
            tmem_ld32(tS + my_lanes + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
            tmem_ld32(tS + my_lanes + 64, *reinterpret_cast<float(*)[32]>(&s[64]));
            tmem_ld32(tS + my_lanes + 96, *reinterpret_cast<float(*)[32]>(&s[96]));
            tmem_wait(*reinterpret_cast<float(*)[32]>(&s[0]));
            tmem_wait(*reinterpret_cast<float(*)[32]>(&s[32]));
            tmem_wait(*reinterpret_cast<float(*)[32]>(&s[64]));
            tmem_wait(*reinterpret_cast<float(*)[32]>(&s[96]));
            if (tile * kKeys + kKeys > S || kv.table != nullptr) {
#pragma unroll
                for (int j = 0; j < 128; ++j)
                    if (!valid[j]) s[j] = -INFINITY;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 128; j += 2) mx = max3(mx, s[j], s[j + 1]);
            // raise the running max when it grows past the margin; the accumulated row and sum then
            // scale by 2^(old - new). The accumulator is read and written by whole warps (the
            // tensor-memory accesses are warp-collective): a row that keeps its max scales by 1.
            const bool raise = mx > run_max + kLazy || run_max == -INFINITY;
            float alpha = 1.0f;
            if (raise) {
                alpha = run_max == -INFINITY ? 0.0f : exp2f(__fsub_rn(run_max, mx));
                run_max = mx;
                run_sum = __fmul_rn(run_sum, alpha);
            }
            if (n_o > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32(tO + my_lanes + 32 * c, o);
                    tmem_wait(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __fmul_rn(o[i], alpha);
                    tmem_st32(tO + my_lanes + 32 * c, o);
                }
                tmem_st_wait();
            }
            float psum = 0.0f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float p8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    p8[i] = run_max == -INFINITY ? 0.0f : exp2f(__fsub_rn(s[8 * c + i], run_max));
                    psum = __fadd_rn(psum, p8[i]);
                }
                put8(Ph, Pl, tid, c, p8);
            }
            run_sum = __fadd_rn(run_sum, psum);
        } else {
            // 3b. C_V^T: thread t owns coordinate c = t - 128, key rows 0 .. 127 (16 chunks of 8 keys)
            const int c = tid - 128;
            const int o = 3 * c, wq = o >> 5, sh = o & 31;
#pragma unroll 2
            for (int g = 0; g < 16; ++g) {
                float v8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int key = 8 * g + i;
                    const uint32_t idx = wq < 11 ? __funnelshift_r(recV[key][wq], recV[key][wq + 1], sh)
                                                 : (recV[key][wq] >> sh);
                    v8[i] = __fmul_rn(__shfl_sync(0xffffffffu, cb, (int)idx), facV[key]);
                }
                put8(Bh, Bl, c, g, v8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            mma3(tO, Ph, Pl, Bh, Bl, n_o > 0 ? 1u : 0u);
            mma_commit(&bar[1]);
        }
        ++n_o;
    }
    // the last O product
    if (!fault && n_o > 0) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&bar[1], (n_o - 1) & 1u, kMaxPolls);
        if (__syncthreads_or(!ok)) fault = true;
        tc_fence_after();
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // each CTA leaves its rows' running max, sum and accumulator (staged from tensor memory into
    // the B operand buffers, free now) in shared memory; cluster rank 0 merges them
    float *const Ostage = reinterpret_cast<float *>(Bh);  // [kRows][128] fp32 = Bh and Bl
    if (!fault && warp < 4) {
        float v[128];
        if (n_o > 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tO + my_lanes + 32 * c, *reinterpret_cast<float(*)[32]>(&v[32 * c]));
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_wait(*reinterpret_cast<float(*)[32]>(&v[32 * c]));
        } else {
#pragma unroll
            for (int e = 0; e < 128; ++e) v[e] = 0.0f;
        }
#pragma unroll
        for (int e4 = 0; e4 < 32; ++e4) {  // row tid, 16-byte chunks rotated by the row (bank spread)
            const int c4 = (e4 + tid) & 31;
            *reinterpret_cast<float4 *>(Ostage + tid * 128 + 4 * c4) =
                make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
        }
        mrow[tid] = n_o > 0 ? run_max : -INFINITY;
        lrow[tid] = n_o > 0 ? run_sum : 0.0f;
    }
    // every CTA of the cluster takes part (a fault still leaves this CTA at the barriers)
    cluster.sync();
    if (!fault && split == 0 && warp < 4) {
        // out = s . H(sum_c O_c 2^(m_c - M) / sum_c l_c 2^(m_c - M)) * post for row tid
        float M = -INFINITY;
        for (int c = 0; c < n_split; ++c) M = fmaxf(M, *cluster.map_shared_rank(&mrow[tid], c));
        float L = 0.0f, fac[kMaxSplit];
        for (int c = 0; c < n_split; ++c) {
            const float mc = *cluster.map_shared_rank(&mrow[tid], c);
            fac[c] = mc == -INFINITY ? 0.0f : exp2f(__fsub_rn(mc, M));
            L = __fadd_rn(L, __fmul_rn(*cluster.map_shared_rank(&lrow[tid], c), fac[c]));
        }
        float v[128];
#pragma unroll
        for (int e4 = 0; e4 < 32; ++e4) {
            float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            const int c4 = (e4 + tid) & 31;
            for (int c = 0; c < n_split; ++c) {
                const float4 x = *cluster.map_shared_rank(reinterpret_cast<float4 *>(Ostage + tid * 128 + 4 * c4), c);
                a.x = __fadd_rn(a.x, __fmul_rn(x.x, fac[c]));
                a.y = __fadd_rn(a.y, __fmul_rn(x.y, fac[c]));
                a.z = __fadd_rn(a.z, __fmul_rn(x.z, fac[c]));
                a.w = __fadd_rn(a.w, __fmul_rn(x.w, fac[c]));
            }
            v[4 * e4] = a.x;
            v[4 * e4 + 1] = a.y;
            v[4 * e4 + 2] = a.z;
            v[4 * e4 + 3] = a.w;
        }
#pragma unroll
        for (int e = 0; e < 128; ++e) v[e] = __fdiv_rn(v[e], L);
        fwht128(v);
        const int r = r0 + tid;
        if (r < m) {
#pragma unroll
            for (int e = 0; e < 128; ++e) {
                const float x = __fmul_rn(__fmul_rn(v[e], post), sign_of(mask, e));
                const int64_t at = (head * m + r) * 128 + e;
                if (out_bf16)
                    static_cast<uint16_t *>(out)[at] = f32_to_bf16(x);
                else
                    static_cast<float *>(out)[at] = x;
            }
        }
    }
    cluster.sync();  // peers keep their shared memory until rank 0 has read it
    if (fault && lane == 0) atomicOr(&g_fault, 128u);
    tc_fence_before();
    __syncthreads();
    if (fault && tid == 0) {
        // give products still in flight a bounded chance to finish before the memory goes away
        if (n_s > 0) mbar_wait_bounded(&bar[0], (n_s - 1) & 1u, kMaxPolls);
        if (n_o > 0) mbar_wait_bounded(&bar[1], (n_o - 1) & 1u, kMaxPolls);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(*tslot, kTmemCols);
    }
}

}  // namespace tq3_attn_mma

wq_status tq3_attn_mma::run(const void *q, int q_dtype, int64_t heads, int64_t m, const Cache &kv, int64_t S,
                            const SignMask &mask, float coef, void *out, int out_dtype, cudaStream_t s) {
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(attn_mma_kernel), kSmem)) return WQ_ERR_CUDA;
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
    }
    const int64_t chunks = (m + kRows - 1) / kRows, n_tiles = (S + kKeys - 1) / kKeys;
    // one CTA per SM: split each (head, chunk) over as many CTAs as keep the grid within one wave
    int64_t split = sms / (heads * chunks < 1 ? 1 : heads * chunks);
    split = split < 1 ? 1 : split > kMaxSplit ? kMaxSplit : split;
    split = split > n_tiles ? n_tiles : split;
    for (int64_t h0 = 0; h0 < heads; h0 += 65535) {
        const unsigned hy = (unsigned)(heads - h0 < 65535 ? heads - h0 : 65535);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(chunks * split), hy, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, attn_mma_kernel, q, (int)(q_dtype == WQ_BF16), (int)m, kv, S, mask, coef, out,
                               (int)(out_dtype == WQ_BF16), h0) != cudaSuccess) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
    }
    return launch_status();
}

unsigned int tq3_attn_mma::read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(g_fault, &zero, sizeof zero);
    return v;
}

}  // namespace wq
