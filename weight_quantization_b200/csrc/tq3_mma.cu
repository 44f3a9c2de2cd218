// TQ3 encoder for bf16 input on sm_100a with the sign flips and the Walsh-Hadamard transform as
// one tensor-core product: page "tq3_core.py" (tq3_quantize, _fwht_inplace, _quantize_to_indices,
// _pack_3bit).
//
// For a tile of 128 vectors X[128 x 128] (bf16, loaded by TMA with 128-byte swizzling) the kernel
// computes Z = X B^T with B[j][i] = -H[j][i] s_i, H the 128-point Hadamard matrix ((-1)^popc(i&j))
// and s the sign flips: z_j = -fwht(s x)_j. Every product is exact (a bf16 value times +-1) and
// the sums accumulate in fp32 in tensor memory; one tcgen05.mma per 16 columns of K, issued by a
// single thread, eight per tile. Thread t of the CTA then owns vector t: it reads row t of the
// accumulator (tcgen05.ld, its warp's 32-lane quarter) in 32-column pieces, twice: the norm
// (||z||^2 / 128) and absmax T, then the indices, each from the scaled coefficient x = -z / T as
// 3 + ceil(Q(x)) with Q an odd quintic through the boundaries (bucket_piece), packed through
// 8^j-weighted fp32 words. An exact zero coefficient gets index 3, as the page's searchsorted gives.
//
// Numerics: the fp32 accumulation order of the tensor core is not the butterfly's, so z agrees
// with the step-by-step transform to a few units in the last place relative to max|z|, and the
// decision polynomial places each boundary within about 1.3e-7 of its exact position; an index can
// therefore differ from the page's rounding only for a coefficient within about 1e-6 of a
// boundary. Norms and scales agree to within 1e-6 relative. A vector whose
// fp32 sum of squares is not finite (|x| beyond about 1e19, where the unnormalised product can
// itself overflow although the page's normalised transform does not) is re-encoded by the page's
// steps from global memory (tq3::encode_vector_exact).
//
// Pipeline per CTA (persistent over tiles): TMA load of the next tile is issued as soon as the
// tensor core has consumed the current one, so it lands while the 128 threads run the epilogue;
// the accumulator is read out before the next product overwrites it. Every wait is bounded: on a
// timeout the fault flag is set, the CTA gives in-flight copies and products a bounded chance to
// land, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "tcgen05.cuh"
#include "tq3_common.cuh"
#include "tq3_mma.cuh"

namespace wq {
namespace tq3_mma {

using tq3::SignMask;

// A CTA holding tensor memory runs alone on its SM, so one CTA carries four independent groups of
// 128 threads; each group streams its own tiles through its own operand buffer and accumulator
// (128 columns each of the 512 allocated), coordinated by mbarriers only. The epilogue
// reads the accumulator in 32-column pieces (twice: norm and absmax, then the indices), so a
// thread holds 32 values rather than 128 and four groups fit the register file.
constexpr int kTile = 128;  // vectors per tile = threads per group = rows of the product
constexpr int kGroups = 4;
constexpr int kThreads = kGroups * kTile;
constexpr int kBox = kTile * 128;  // one 64-column half of a 128 x 128 bf16 operand (128 B per row)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMaxPolls = 1u << 24;
// shared-memory layout (offsets from a 1024-byte aligned base): B, then one A per group, then per
// group its full (TMA) and done (tensor core) barriers, then the TMEM address
constexpr int kStageBytes = 2 * kBox;
constexpr int kOffB = 0;
constexpr int kOffA = 2 * kBox;
constexpr int kOffBar = kOffA + kGroups * kStageBytes;
constexpr int kSmem = 1024 + kOffBar + 32 * kGroups + 16;  // ... TMEM address, then the B barrier


__device__ unsigned int g_fault;

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// Sum of squares (two lanes at a time) and absmax of a 32-column piece.
__device__ __forceinline__ void acc_piece(const float (&z)[32], f32x2 (&acc)[4], float (&mm)[4]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const f32x2 p = pk2(z[2 * i], z[2 * i + 1]);
        acc[i & 3] = fma2(p, p, acc[i & 3]);
        mm[i & 3] = max3(mm[i & 3], fabsf(z[2 * i]), fabsf(z[2 * i + 1]));
    }
}

// atomicAdd on shared memory with acquire-release ordering (CTA scope); returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}

// Chunks c0 .. c0 + 3 of row n of B = -H diag(s), K-major with the 128-byte swizzle (two 64-column
// halves): entry (n, k) is -(-1)^popc(n & k) s_k, exactly +-1 in bf16.
template <bool kFold>
__device__ __forceinline__ void build_b(unsigned char *B, const SignMask &mask, int n, int c0) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {  // 16-byte chunk c holds k = 8c .. 8c + 7
        const int c = c0 + cc;
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t pair = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int k = 8 * c + 2 * u + h;
                const uint32_t sneg = kFold ? ((~tq3::default_mask_word(k >> 5) >> (k & 31)) & 1u)
                                            : ((~mask.w[k >> 5] >> (k & 31)) & 1u);
                const uint32_t neg = ((uint32_t)__popc(n & k) & 1u) ^ sneg ^ 1u;
                pair |= (neg ? 0xBF80u : 0x3F80u) << (16 * h);
            }
            w[u] = pair;
        }
        unsigned char *half = B + (c >> 3) * kBox;
        *reinterpret_cast<uint4 *>(half + n * 128 + (((c & 7) ^ (n & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Indices of one 32-column piece (elements 32c .. 32c + 31, groups 4c .. 4c + 3) packed as the
// record's bytes 12c .. 12c + 11, three little-endian words (_pack_3bit: group i is bytes
// 3i .. 3i + 2). nr = -1 / T turns the accumulator's z = -fwht into x = z * nr. Group q is
// accumulated as two fp32 words, even slots and odd slots, each a sum of index * 8^j: integers
// below 2^24, so the words are exact.
__device__ __forceinline__ void bucket_piece(const float (&z)[32], float nr, uint32_t &o0, uint32_t &o1, uint32_t &o2) {
    const f32x2 NR = pk2(nr, nr);
    const f32x2 Q1 = pk2(tq3::q_coef(1), tq3::q_coef(1)), Q3 = pk2(tq3::q_coef(3), tq3::q_coef(3)),
               Q5 = pk2(tq3::q_coef(5), tq3::q_coef(5));
    const f32x2 KK = pk2(8388612.0f, 8388612.0f), NC = pk2(-8388609.0f, -8388609.0f);
    f32x2 W[4];
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) W[gg] = 0ull;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
            const int i = 4 * gg + p;  // local elements 2i (slot 2p) and 2i + 1 (slot 2p + 1)
            const f32x2 w8 = pk2(__uint_as_float((127u + 6u * p) << 23), __uint_as_float((127u + 6u * p + 3u) << 23));
            const f32x2 x = mul2(pk2(z[2 * i], z[2 * i + 1]), NR);
            const f32x2 x2 = mul2(x, x);
            const f32x2 h = fma2(fma2(Q5, x2, Q3), x2, Q1);
            const f32x2 idx = add2(tq3::fma2_rp(h, x, KK), NC);  // 3 + ceil(Q(x))
            W[gg] = fma2(w8, idx, W[gg]);
        }
    uint32_t g4[4];
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
        float lo, hi;
        upk2(W[gg], lo, hi);
        g4[gg] = __float2uint_rn(__fadd_rn(lo, hi));
    }
    o0 = g4[0] | (g4[1] << 24);
    o1 = (g4[1] >> 8) | (g4[2] << 16);
    o2 = (g4[2] >> 16) | (g4[3] << 8);
}

// B for the page's sign table, built at compile time in the shared-memory layout above (8192
// words), so that a CTA fetches it with one bulk copy instead of computing it.
struct BTable {
    uint32_t w[2 * kBox / 4];
};
constexpr int popc_parity(int v) {
    int p = 0;
    for (; v; v &= v - 1) p ^= 1;
    return p;
}
constexpr BTable make_default_b() {
    BTable t{};
    for (int n = 0; n < kTile; ++n)
        for (int c = 0; c < 16; ++c)
            for (int u = 0; u < 4; ++u) {
                uint32_t pair = 0;
                for (int h = 0; h < 2; ++h) {
                    const int k = 8 * c + 2 * u + h;
                    const uint32_t sneg = (~tq3::default_mask_word(k >> 5) >> (k & 31)) & 1u;
                    const uint32_t neg = (uint32_t)popc_parity(n & k) ^ sneg ^ 1u;
                    pair |= (neg ? 0xBF80u : 0x3F80u) << (16 * h);
                }
                const int byte = (c >> 3) * kBox + n * 128 + (((c & 7) ^ (n & 7)) << 4) + 4 * u;
                t.w[byte / 4] = pair;
            }
    return t;
}
__device__ __align__(128) const BTable kDefaultB = make_default_b();

// kLay (tq3::Layout): kSoA writes packed, norms and scales; kAoS writes 56-byte records (the 48
// packed bytes, the norm, the scale) at `packed`; kPool writes record v to slot pm.index[v] of the
// pool at `packed` (a negative slot: not stored). Norms and scales are unused for the record layouts.
template <bool kFold, int kLay = tq3::kSoA>
__global__ void __launch_bounds__(kThreads, 1)
    encode_mma(int64_t n_vec, const __grid_constant__ CUtensorMap tmap, const void *__restrict__ x, SignMask mask,
               uint8_t *__restrict__ packed, float *__restrict__ norms, float *__restrict__ scales, tq3::PoolMap pm) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *const base = tq3::tile_base(smem_raw);
    const int grp = threadIdx.x >> 7, tid = threadIdx.x & 127, warp = tid >> 5;
    unsigned char *const B = base + kOffB;
    unsigned char *const A = base + kOffA + grp * kStageBytes;
    uint64_t *const full = reinterpret_cast<uint64_t *>(base + kOffBar) + 4 * grp;
    uint64_t *const done = full + 1;
    // per-group counters: warps that have finished reading the accumulator (modulo 4), products issued
    uint32_t *const readers = reinterpret_cast<uint32_t *>(full + 2);
    uint32_t *const issued = readers + 1;
    uint32_t *const tslot = reinterpret_cast<uint32_t *>(base + kOffBar + 32 * kGroups);
    uint64_t *const bready = reinterpret_cast<uint64_t *>(base + kOffBar + 32 * kGroups + 8);
    const int64_t n_tiles = (n_vec + kTile - 1) / kTile;
    // streams interleave across CTAs (stream = grp * gridDim.x + blockIdx.x), so the tiles left
    // over after whole rounds spread one per SM rather than piling onto the first CTAs
    const int64_t stream = (int64_t)grp * gridDim.x + blockIdx.x, n_streams = (int64_t)gridDim.x * kGroups;
    const int64_t my_tiles = stream < n_tiles ? (n_tiles - stream + n_streams - 1) / n_streams : 0;

    if (!kFold) {
        build_b<kFold>(B, mask, threadIdx.x >> 2, 4 * (threadIdx.x & 3));
        fence_proxy_async_smem();  // B is written by threads and read by the tensor core
    }
    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        *readers = 0;
        *issued = 0;
    }
    if (threadIdx.x == 0) {
        mbar_init(bready, 1);
        if (kFold) {
            mbar_expect_tx(bready, 2 * kBox);
            bulk_load(B, &kDefaultB, 2 * kBox, bready);
        } else {
            mbar_expect_tx(bready, 0);  // completes the phase at once: B was written above
        }
    }
    if (threadIdx.x < 32) tmem_alloc(tslot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything above touched only this CTA's resources and the constant table: from here on the
    // kernel reads the input and writes the outputs, so the previous kernel must be complete
    pdl_wait();
    const uint32_t tmem = *tslot + (uint32_t)(grp * kTile);  // this group's 128 columns
    const uint32_t my_lanes = tmem + ((uint32_t)(warp * 32) << 16);

    // Thread 0 of the group issues the loads: tile i + 1 once the product of tile i has consumed the
    // operand buffer (it lands during tile i's epilogue). The product of tile i + 1 is issued by
    // whichever warp is the last to finish reading tile i's accumulator, so no warp waits for the
    // others.
    int64_t n_loaded = 0;  // thread 0's count of loads issued (for the fault path)
    auto issue_load = [&](int64_t i) {
        const int y = (int)((stream + i * n_streams) * kTile);
        mbar_expect_tx(full, kStageBytes);
        tma_load_2d(A, &tmap, 0, y, full);
        tma_load_2d(A + kBox, &tmap, 64, y, full);
        n_loaded = i + 1;
    };
    const uint64_t adesc = sw128_desc(smem_u32(A)), bdesc = sw128_desc(smem_u32(B));
    auto issue_mma = [&](int64_t i) {
        if (i == 0 && !mbar_wait_bounded(bready, 0u, kMaxPolls)) return;
        if (!mbar_wait_bounded(full, (uint32_t)(i & 1), kMaxPolls)) return;  // the product's waiters time out
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // K = 16 per instruction: 32 bytes into a 128-byte row
            const uint32_t off = (uint32_t)((ks >> 2) * kBox + (ks & 3) * 32) >> 4;
            mma_bf16(tmem, adesc + off, bdesc + off, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(done);
        *issued = (uint32_t)(i + 1);
    };
    if (tid == 0 && my_tiles > 0) {
        issue_load(0);
        issue_mma(0);
    }

    const float post = tq3::fwht_post();
    bool fault = false;
    // No warp waits for another in this loop: each waits on the product's barrier itself, and the
    // last warp to finish reading the accumulator issues the next product. A timeout ends the
    // warp's loop (the decision is warp-uniform, as the accumulator reads are warp-collective).
    for (int64_t it = 0; it < my_tiles; ++it) {
        // one lane per warp polls the product's barrier; the warp synchronises on its answer
        bool ok = true;
        if ((tid & 31) == 0) ok = mbar_wait_bounded(done, (uint32_t)(it & 1), kMaxPolls);
        if (!__all_sync(0xffffffffu, ok)) {
            fault = true;
            break;
        }
        // the product has consumed the operand buffer: the next tile lands during this epilogue
        if (tid == 0 && it + 1 < my_tiles) issue_load(it + 1);
        // on a group's last tile the block lets the next kernel in the stream be scheduled: its
        // set-up overlaps this kernel's tail (it still waits for this kernel to finish before reading)
        if (it + 1 == my_tiles) pdl_trigger();
        tc_fence_after();

        // pass 1: ||x||^2 = ||z||^2 / 128 (Parseval) and max|z|. The pieces alternate between two
        // register sets, so each piece's read from tensor memory overlaps the previous piece's work;
        // the first piece of pass 2 is read while the per-vector scalars are formed.
        f32x2 acc[4] = {0ull, 0ull, 0ull, 0ull};
        float mm[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        float za[32], zb[32];
        tmem_ld32(my_lanes + 0, za);
        tmem_wait(za);
        tmem_ld32(my_lanes + 32, zb);
        acc_piece(za, acc, mm);
        tmem_wait(zb);
        tmem_ld32(my_lanes + 64, za);
        acc_piece(zb, acc, mm);
        tmem_wait(za);
        tmem_ld32(my_lanes + 96, zb);
        acc_piece(za, acc, mm);
        tmem_wait(zb);
        tmem_ld32(my_lanes + 0, za);
        acc_piece(zb, acc, mm);
        float n2;
        {
            float a0, a1;
            upk2(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), a0, a1);
            n2 = __fadd_rn(a0, a1);
        }
        const float m = fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3]));
        // A vector whose fp32 squares overflowed (|x| beyond about 1e19; z itself may have
        // overflowed) still takes part in the warp-collective accumulator reads below, and is then
        // re-encoded step by step at the store.
        const bool big = !(n2 <= 3.0e38f);
        const float nrm = fmaxf(__fsqrt_rn(__fmul_rn(n2, 0.0078125f)), 1e-8f);
        const float sraw = __fmul_rn(__fdiv_rn(m, nrm), post);
        const float scale = fmaxf(sraw, 1e-8f);
        const float T = (sraw >= 1e-8f) ? m : __fmul_rn(__fmul_rn(1e-8f, nrm), 11.3137085f);
        const float nr = -__frcp_rn(T);

        // pass 2: the indices, 32 columns at a time. Pieces 2 and 3 are both read before the next
        // product is released, so that product runs during two pieces' work.
        const int64_t v = (stream + it * n_streams) * kTile + tid;
        int64_t slot = v;  // the slot's load is issued here, ahead of its use at the store
        if constexpr (kLay == tq3::kPool) slot = v < n_vec ? __ldg(static_cast<const int64_t *>(pm.index) + v) : -1;
        uint32_t o[12];
        tmem_wait(za);
        tmem_ld32(my_lanes + 32, zb);
        bucket_piece(za, nr, o[0], o[1], o[2]);
        tmem_wait(zb);
        tmem_ld32(my_lanes + 64, za);
        bucket_piece(zb, nr, o[3], o[4], o[5]);
        tmem_wait(za);
        tmem_ld32(my_lanes + 96, zb);
        tmem_wait(zb);
        // the accumulator has been read: the next product runs during the last two pieces' work
        tc_fence_before();
        __syncwarp();
        if ((tid & 31) == 0 && it + 1 < my_tiles && (atom_add_acq_rel(readers, 1u) & 3u) == 3u)
            issue_mma(it + 1);
        bucket_piece(za, nr, o[6], o[7], o[8]);
        bucket_piece(zb, nr, o[9], o[10], o[11]);
        if (v < n_vec) {
            if constexpr (kLay != tq3::kSoA) {  // a 56-byte record is 8-byte aligned
                if (kLay == tq3::kPool && slot >= pm.n_pool) atomicOr(&g_fault, tq3::kFaultPoolIndex);
                if (kLay == tq3::kAoS || (slot >= 0 && slot < pm.n_pool)) {
                    uint8_t *const rec = packed + slot * 56;  // formed only for a slot inside the pool
                    if (big) {
                        tq3::encode_vector_exact(x, true, v, mask, rec, reinterpret_cast<float *>(rec + 48),
                                                 reinterpret_cast<float *>(rec + 52));
                    } else {
#pragma unroll
                        for (int q = 0; q < 6; ++q) st_stream8(rec + 8 * q, make_uint2(o[2 * q], o[2 * q + 1]));
                        st_stream8(rec + 48, make_uint2(__float_as_uint(nrm), __float_as_uint(scale)));
                    }
                }
            } else {
                uint8_t *const rec = packed + v * 48;
                if (big) {
                    tq3::encode_vector_exact(x, true, v, mask, rec, norms + v, scales + v);
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
    if (fault && (tid & 31) == 0) atomicOr(&g_fault, 8u);
    tc_fence_before();
    __syncthreads();
    if (__syncthreads_or(fault) && tid == 0) {
        // give what may still be in flight a bounded chance to land before the memory goes away
        if (n_loaded > 0) mbar_wait_bounded(full, (uint32_t)((n_loaded - 1) & 1), kMaxPolls);
        const uint32_t n_mma = *issued;
        if (n_mma > 0) mbar_wait_bounded(done, (n_mma - 1) & 1u, kMaxPolls);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(*tslot, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
namespace {
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev);
    return cached[dev];
}

template <typename K>
wq_status launch(K k, int64_t cnt, const CUtensorMap &tm, const void *xc, const SignMask &m, uint8_t *pc, float *nc,
                 float *sc, const tq3::PoolMap &pm, cudaStream_t s) {
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(k), kSmem)) return WQ_ERR_CUDA;
    // one CTA per SM (it holds all 512 tensor-memory columns), never more CTAs than tile triples
    const int64_t tiles = (cnt + kTile - 1) / kTile;
    const int64_t triples = (tiles + kGroups - 1) / kGroups;
    const int64_t g_ = sm_count() > 0 ? sm_count() : 1;
    const int64_t g = g_ < triples ? g_ : triples;
    if (launch_pdl(k, (unsigned)g, kThreads, kSmem, s, cnt, tm, xc, m, pc, nc, sc, pm) != cudaSuccess) {
        cudaGetLastError();
        return WQ_ERR_CUDA;
    }
    return launch_status();
}
}  // namespace

wq_status encode_bf16(const void *x, int64_t n_vec, const SignMask &m, uint8_t *packed, float *norms, float *scales,
                      cudaStream_t s, int layout, const tq3::PoolMap &pool) {
    const bool def = tq3::is_default(m);
    for (int64_t off = 0; off < n_vec; off += tq3::kMaxChunk) {
        const int64_t cnt = n_vec - off < tq3::kMaxChunk ? n_vec - off : tq3::kMaxChunk;
        const unsigned char *xc = static_cast<const unsigned char *>(x) + off * (tq3::kD * 2);
        CUtensorMap tm;
        if (!make_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xc, tq3::kD, (uint64_t)cnt, tq3::kD * 2, 64, kTile))
            return WQ_ERR_CUDA;
        wq_status st;
        if (layout == tq3::kPool) {  // the pool is not offset; the chunk's slots are
            tq3::PoolMap pm = pool;
            pm.index = static_cast<const int64_t *>(pool.index) + off;
            st = def ? launch(encode_mma<true, tq3::kPool>, cnt, tm, xc, m, packed, nullptr, nullptr, pm, s)
                     : launch(encode_mma<false, tq3::kPool>, cnt, tm, xc, m, packed, nullptr, nullptr, pm, s);
        } else if (layout == tq3::kAoS) {
            uint8_t *const pc = packed + off * 56;
            st = def ? launch(encode_mma<true, tq3::kAoS>, cnt, tm, xc, m, pc, nullptr, nullptr, pool, s)
                     : launch(encode_mma<false, tq3::kAoS>, cnt, tm, xc, m, pc, nullptr, nullptr, pool, s);
        } else {
            uint8_t *const pc = packed + off * 48;
            st = def ? launch(encode_mma<true>, cnt, tm, xc, m, pc, norms + off, scales + off, pool, s)
                     : launch(encode_mma<false>, cnt, tm, xc, m, pc, norms + off, scales + off, pool, s);
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

}  // namespace tq3_mma
}  // namespace wq
