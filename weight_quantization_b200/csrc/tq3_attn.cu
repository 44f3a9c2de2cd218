// Attention over a TQ3-compressed K/V cache, on sm_100a: softmax(q k^T * softmax_scale) v with every
// key and value a 56-byte TQ3 record (page "tq3_core.py": tq3_dequantize gives the vectors the
// attention reads; the page's commit note names the KV cache of an attention layer as the consumer).
//
// No key or value is decoded to 128 floats. tq3_dequantize gives, for a record (idx, norm, scale),
//     k = s . (H (c[idx] * scale)) * post * norm,        post = fp32(1 / sqrt(128)),
// with H the unnormalised Sylvester Hadamard matrix (symmetric), s the sign draws, c the centroids.
// So for a query q
//     q . k = norm * scale * post * sum_i (H (s . q))_i c[idx_i],
// and for weights p_j
//     sum_j p_j v_j = s . H( sum_j p_j norm_j scale_j c[idx_j] ) * post.
// The query is rotated once (q~ = H (s . q)), each logit is a 128-term dot product of q~ with the
// centroids named by the key's indices, the value side accumulates centroids weighted by
// p_j * norm_j * scale_j in the rotated basis, and one inverse transform per output row finishes.
// The result equals attention over the decoded vectors up to fp32 rounding (the page's decode
// rounds after each of its steps; this order rounds differently).
//
// Work split. A cluster of up to 8 CTAs serves one (head, chunk of up to 16 query rows): CTA x of
// the cluster takes a contiguous share of the key tiles, keeps a running max, sum and 128
// accumulators per query row (online softmax), and the cluster combines its CTAs' partial results
// through distributed shared memory, so nothing is written to global memory but the output. More
// than 16 query rows per head are served 16 at a time, each chunk re-reading the records. Within a
// CTA of 128 threads, a tile holds 128 * kKPT keys: thread t scores keys t + 128 k (k < kKPT), the
// indices of each unpacked once for every query row, two coordinates per packed multiply-add, so
// that one shared-memory read of the rotated query serves kKPT keys; for the values, each lane owns
// four rotated coordinates and each warp a quarter of the tile's keys, two query rows per packed
// multiply-add, the warps' sums being added once at the end. The records of the next tile are
// copied into shared memory asynchronously while the current one is processed: a whole tile of a
// contiguous cache by one bulk copy per tensor, other tiles by 8-byte cp.async.
//
// Records are addressed either contiguously ([heads][S] records) or through a page table over a
// pool of records (the layout tq3_encode_slots writes): key j of head h is record
// table[h][j / page_size] * page_size + j % page_size. An entry outside the pool masks its key
// out (weight 0) and sets fault bit 6.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "tq3_attn_mma.cuh"
#include "tq3_common.cuh"
#include "wq.h"

namespace cg = cooperative_groups;

namespace wq {
namespace tq3_attn {

using tq3::SignMask;

constexpr int kWords = 14;     // 32-bit words per 56-byte record
constexpr int kMaxSplit = 8;   // CTAs per cluster (portable cluster size)
constexpr int kMaxRows = 16;   // query rows per launch (chunk)
constexpr int64_t kMaxRowsTotal = 1 << 20;  // query rows per head in one call
constexpr int kThreads = 128;
constexpr uint32_t kMaxPolls = 1u << 24;

__device__ unsigned int g_fault;

using KV = AttnCache;

// From this many query rows per head on, the tensor-core kernel (tq3_attn_mma.cu) serves the call.
constexpr int64_t kMmaMinRows = 48;

// Record index of key j of head h, or -1 for a page-table entry outside the pool.
__device__ __forceinline__ int64_t record_of(const KV &kv, int64_t head, int64_t S, int64_t j) {
    if (kv.table == nullptr) return head * S + j;
    const int32_t page = __ldg(kv.table + head * kv.pages_per_head + (j >> kv.shift));
    const int64_t r = ((int64_t)page << kv.shift) | (j & ((int64_t(1) << kv.shift) - 1));
    return (page >= 0 && r < kv.n_pool) ? r : -1;
}

// 8-byte asynchronous global -> shared copy (cp.async, L1-bypassing), committed and waited in groups.
__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int kRows>
constexpr int keys_per_thread() { return kRows <= 8 ? 2 : 1; }

template <int kRows>
struct Smem {
    static constexpr int kKPT = keys_per_thread<kRows>();
    static constexpr int kKeys = kThreads * kKPT;
    static constexpr int kWarps = kThreads / 32;
    float q[kRows][128];           // q~ = H (s . q), unnormalised; at the end, the output rows
    float w[kKeys][kRows];         // p_j * norm_j * scale_j of the tile's keys, a key's rows together
    union {
        struct {
            uint32_t k[kKeys][kWords];
            uint32_t v[kKeys][kWords];
        } rec;                     // the tile's records; the next tile's keys are copied in once the
                                   // logits are done, its values once the value sums are done
        float acc[kRows][128];     // after the tiles: this CTA's accumulators, read by cluster rank 0
    } u;
    float red[kWarps][kRows];      // per-warp partial maxima and sums
    float mrow[kRows], lrow[kRows];
    int valid[2][kKeys];           // per tile parity: 1 when the key exists and its records were found
    uint64_t bar[2];               // bulk copies of a whole tile's key (0) and value (1) records
};

// Sign draw of element e: +1.0 or -1.0.
__device__ __forceinline__ float sign_of(const SignMask &m, int e) { return ((m.w[e >> 5] >> (e & 31)) & 1u) ? 1.0f : -1.0f; }

// In-place unnormalised FWHT of kRows rows of 128 floats in shared memory; all threads take part.
template <int kRows>
__device__ __forceinline__ void fwht_rows(float (*x)[128]) {
#pragma unroll
    for (int h = 1; h < 128; h <<= 1) {
        for (int p = threadIdx.x; p < kRows * 64; p += kThreads) {
            const int r = p >> 6, t = p & 63;
            const int i = (t / h) * 2 * h + (t % h);
            const float a = x[r][i], b = x[r][i + h];
            x[r][i] = __fadd_rn(a, b);
            x[r][i + h] = __fsub_rn(a, b);
        }
        __syncthreads();
    }
}

// q: [heads][m_total][128] (bf16 or fp32), of which this launch takes rows r0 .. r0 + m - 1 of
// every head; out likewise. coef = post * softmax_scale * log2(e): logits are kept in log2 units
// so that exp2 applies.
template <int kRows>
__global__ void __launch_bounds__(kThreads, 4)
    attn_kernel(const void *__restrict__ q, int q_bf16, int m, int m_total, int r0, KV kv, int64_t S, SignMask mask,
                float coef, void *__restrict__ out, int out_bf16, int64_t head0) {
    using SM = Smem<kRows>;
    constexpr int kKPT = SM::kKPT, kKeys = SM::kKeys, kWarps = SM::kWarps;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SM &sm = *reinterpret_cast<SM *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = (int)cluster.block_rank(), n_split = (int)cluster.num_blocks();
    const int64_t head = head0 + blockIdx.y;
    const float cb = tq3::centroid((uint32_t)(lane & 7));  // lane l holds centroid l mod 8
    const float post = tq3::fwht_post();

    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const int64_t t_begin = n_tiles * split / n_split, t_end = n_tiles * (split + 1) / n_split;
    // A whole tile of a contiguous cache is one run of kKeys records in global memory, laid out as
    // the shared-memory buffer is: thread 0 copies it with one bulk copy per tensor (on the copy
    // engine, not the load/store pipe), when the run starts on a 16-byte boundary (records are 56
    // bytes, so head * S must be even). Other tiles take the per-thread copies below.
    // (The 16-row form, already at its register limit, keeps the per-thread copies.)
    constexpr bool kBulk = kRows <= 8;
    const bool bulk_ok = kBulk && kv.table == nullptr &&
                         ((reinterpret_cast<uintptr_t>(kv.k) | reinterpret_cast<uintptr_t>(kv.v)) & 15) == 0 &&
                         ((head * S) & 1) == 0;
    // Only a partial last tile is not bulk, so the bulk tiles are the CTA's tiles in order: tile t
    // completes phase (t - t_begin) & 1 of each barrier.
    auto is_bulk = [&](int64_t tile) { return bulk_ok && (tile + 1) * kKeys <= S; };
    if constexpr (kBulk) {
        if (tid == 0) {
            mbar_init(&sm.bar[0], 1);
            mbar_init(&sm.bar[1], 1);
        }
        __syncthreads();  // the barriers are initialised before the first copy is issued on them
    }
    // the key (or value) records of keys tid + 128 k of a tile, by 8-byte asynchronous copies (or
    // one bulk copy); the key pass also records which keys exist (parity b of the tile index)
    auto fetch = [&](int64_t tile, bool values, int b) {
        if (is_bulk(tile)) {
            if (!values) {
#pragma unroll
                for (int k = 0; k < kKPT; ++k) sm.valid[b][tid + kThreads * k] = 1;
            }
            if (tid == 0) {
                uint64_t *bar = &sm.bar[values ? 1 : 0];
                mbar_expect_tx(bar, (uint32_t)(kKeys * 56));
                bulk_load(values ? &sm.u.rec.v[0][0] : &sm.u.rec.k[0][0],
                          (values ? kv.v : kv.k) + (head * S + tile * kKeys) * 56, (uint32_t)(kKeys * 56), bar);
            }
            return;
        }
#pragma unroll
        for (int k = 0; k < kKPT; ++k) {
            const int key = tid + kThreads * k;
            const int64_t j = tile * kKeys + key;
            const int64_t rec = j < S ? record_of(kv, head, S, j) : -1;
            if (!values) {
                if (j < S && rec < 0) atomicOr(&g_fault, tq3::kFaultPoolIndex);
                sm.valid[b][key] = rec >= 0;  // read after the barrier that follows this tile's wait
            }
            if (rec >= 0) {
                const uint8_t *src = (values ? kv.v : kv.k) + rec * 56;
                uint32_t *dst = values ? sm.u.rec.v[key] : sm.u.rec.k[key];
#pragma unroll
                for (int w = 0; w < kWords / 2; ++w) cp_async8(dst + 2 * w, src + 8 * w);
            }
        }
        cp_async_commit();
    };
    if (t_begin < t_end) {
        fetch(t_begin, false, 0);
        fetch(t_begin, true, 0);
    }

    // q~ = H (s . q) for every row (rows m .. kRows-1 are zeros and never written out)
    for (int i = tid; i < kRows * 128; i += kThreads) {
        const int r = i >> 7, e = i & 127;
        float v = 0.0f;
        if (r < m) {
            const int64_t at = (head * m_total + r0 + r) * 128 + e;
            v = q_bf16 ? __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t *>(q) + at) << 16)
                       : __ldg(static_cast<const float *>(q) + at);
        }
        sm.q[r][e] = __fmul_rn(v, sign_of(mask, e));
    }
    __syncthreads();
    fwht_rows<kRows>(sm.q);

    // per lane: rotated coordinates 4 lane .. 4 lane + 3 of every row, as pairs of rows
    constexpr int kRP = (kRows + 1) / 2;
    f32x2 acc[4][kRP];
    float lsum[kRows], mrun[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        lsum[r] = 0.0f;
        mrun[r] = -INFINITY;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int rp = 0; rp < kRP; ++rp) acc[c][rp] = 0ull;

    for (int64_t tile = t_begin; tile < t_end; ++tile) {
        const int b = (int)((tile - t_begin) & 1);
        if (is_bulk(tile)) {
            const bool ok = mbar_wait_bounded(&sm.bar[0], (uint32_t)b, kMaxPolls) &&
                            mbar_wait_bounded(&sm.bar[1], (uint32_t)b, kMaxPolls);
            if (__syncthreads_or(!ok)) {
                // a copy that did not complete in time: results void. Give it another bounded
                // chance to land before the buffers are reused, then leave the tiles.
                if (tid == 0) {
                    atomicOr(&g_fault, 2u);
                    mbar_wait_bounded(&sm.bar[0], (uint32_t)b, kMaxPolls);
                    mbar_wait_bounded(&sm.bar[1], (uint32_t)b, kMaxPolls);
                }
                __syncthreads();
                break;
            }
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // this tile's records (and valid flags) are visible to every thread
        const uint32_t(*kr)[kWords] = sm.u.rec.k;
        const uint32_t(*vr)[kWords] = sm.u.rec.v;

        // logits: thread tid scores keys tid + 128 k, four coordinates at a time, two per packed fma
        float dot[kKPT][kRows];
        {
            uint32_t W[kKPT][kWords];
#pragma unroll
            for (int k = 0; k < kKPT; ++k)
#pragma unroll
                for (int w = 0; w < kWords / 2; ++w) {
                    const uint2 x = *reinterpret_cast<const uint2 *>(&kr[tid + kThreads * k][2 * w]);
                    W[k][2 * w] = x.x;
                    W[k][2 * w + 1] = x.y;
                }
            f32x2 d2[kKPT][kRows];
#pragma unroll
            for (int k = 0; k < kKPT; ++k)
#pragma unroll
                for (int r = 0; r < kRows; ++r) d2[k][r] = 0ull;
#pragma unroll
            for (int ch = 0; ch < 32; ++ch) {
                f32x2 c01[kKPT], c23[kKPT];
#pragma unroll
                for (int k = 0; k < kKPT; ++k) {
                    float c[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {  // the index of coordinate 4 ch + e is at bit 3 (4 ch + e)
                        const int o = 12 * ch + 3 * e, wq = o >> 5, sh = o & 31;
                        c[e] = __shfl_sync(0xffffffffu, cb, (int)__funnelshift_r(W[k][wq], W[k][wq + 1], sh));
                    }
                    c01[k] = pk2(c[0], c[1]);
                    c23[k] = pk2(c[2], c[3]);
                }
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    const float4 qq = *reinterpret_cast<const float4 *>(&sm.q[r][4 * ch]);
                    const f32x2 q01 = pk2(qq.x, qq.y), q23 = pk2(qq.z, qq.w);
#pragma unroll
                    for (int k = 0; k < kKPT; ++k) {
                        d2[k][r] = fma2(q01, c01[k], d2[k][r]);
                        d2[k][r] = fma2(q23, c23[k], d2[k][r]);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kKPT; ++k) {
                const int key = tid + kThreads * k;
                const float kscale = __fmul_rn(__fmul_rn(__uint_as_float(W[k][12]), __uint_as_float(W[k][13])), coef);
                const bool ok = sm.valid[b][key] != 0;
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    float a, bb;
                    upk2(d2[k][r], a, bb);
                    dot[k][r] = ok ? __fmul_rn(__fadd_rn(a, bb), kscale) : -INFINITY;
                }
            }
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                float mx = dot[0][r];
#pragma unroll
                for (int k = 1; k < kKPT; ++k) mx = fmaxf(mx, dot[k][r]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) sm.red[warp][r] = mx;
            }
        }
        if (bulk_ok) fence_proxy_async_smem();  // these reads precede a bulk copy into the buffer
        __syncthreads();  // every thread is past its reads of the key records
        if (tile + 1 < t_end) fetch(tile + 1, false, b ^ 1);

        // new row maxima (the same in every thread), rescale factors, the weights of this thread's keys
        float alpha[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float mx = mrun[r];
#pragma unroll
            for (int g = 0; g < kWarps; ++g) mx = fmaxf(mx, sm.red[g][r]);
            // a row whose keys so far are all masked keeps max -inf; its factor is then 1 (no sum yet)
            alpha[r] = mrun[r] == -INFINITY ? 0.0f : exp2f(__fsub_rn(mrun[r], mx));
            mrun[r] = mx;
            lsum[r] = __fmul_rn(lsum[r], alpha[r]);
        }
#pragma unroll
        for (int k = 0; k < kKPT; ++k) {
            const int key = tid + kThreads * k;
            // a key without records (past S, or masked by the page table) has uninitialised record
            // words: its weight is exactly 0, whatever its value record holds
            const bool live = sm.valid[b][key] != 0;
            const float nvsv = __fmul_rn(__uint_as_float(vr[key][12]), __uint_as_float(vr[key][13]));
            float wt[kRows];
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                const float p = (!live || mrun[r] == -INFINITY) ? 0.0f : exp2f(__fsub_rn(dot[k][r], mrun[r]));
                lsum[r] = __fadd_rn(lsum[r], p);
                wt[r] = live ? __fmul_rn(p, nvsv) : 0.0f;
            }
            if constexpr (kRows % 4 == 0) {
#pragma unroll
                for (int r4 = 0; r4 < kRows; r4 += 4)
                    *reinterpret_cast<float4 *>(&sm.w[key][r4]) = make_float4(wt[r4], wt[r4 + 1], wt[r4 + 2], wt[r4 + 3]);
            } else {
#pragma unroll
                for (int r = 0; r < kRows; ++r) sm.w[key][r] = wt[r];
            }
        }
        __syncthreads();

        // values: warp g takes keys kKeys/4 g .. kKeys/4 (g + 1) - 1, lane l the rotated coordinates
        // 4l .. 4l + 3, two rows per packed fma
        {
            const int o = 12 * lane, wq = o >> 5, sh = o & 31;
#pragma unroll
            for (int rp = 0; rp < kRP; ++rp) {
                const f32x2 a2 = pk2(alpha[2 * rp], 2 * rp + 1 < kRows ? alpha[2 * rp + 1] : 0.0f);
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[c][rp] = mul2(acc[c][rp], a2);
            }
            constexpr int kPerWarp = kKeys / kWarps;
#pragma unroll 2
            for (int jj = 0; jj < kPerWarp; ++jj) {
                const int j = kPerWarp * warp + jj;
                const uint32_t bits = __funnelshift_r(vr[j][wq], vr[j][wq + 1], sh);
                f32x2 cv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float x = __shfl_sync(0xffffffffu, cb, (int)(bits >> (3 * c)));
                    cv[c] = pk2(x, x);
                }
                f32x2 wj[kRP];
                if constexpr (kRows % 4 == 0) {
#pragma unroll
                    for (int r4 = 0; r4 < kRows; r4 += 4) {
                        const float4 x = *reinterpret_cast<const float4 *>(&sm.w[j][r4]);
                        wj[r4 / 2] = pk2(x.x, x.y);
                        wj[r4 / 2 + 1] = pk2(x.z, x.w);
                    }
                } else if constexpr (kRows == 2) {
                    const float2 x = *reinterpret_cast<const float2 *>(&sm.w[j][0]);
                    wj[0] = pk2(x.x, x.y);
                } else {
                    wj[0] = pk2(sm.w[j][0], 0.0f);
                }
#pragma unroll
                for (int rp = 0; rp < kRP; ++rp)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[c][rp] = fma2(cv[c], wj[rp], acc[c][rp]);
            }
        }
        if (bulk_ok) fence_proxy_async_smem();  // these reads precede a bulk copy into the buffer
        __syncthreads();  // every thread is past its reads of the value records
        if (tile + 1 < t_end) fetch(tile + 1, true, b ^ 1);
    }
    cp_async_wait<0>();
    __syncthreads();  // the record buffers become the accumulators

    // this CTA's row sums and accumulators, in a fixed order: warp sums, then warps one by one
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        float v = lsum[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) sm.red[warp][r] = v;
    }
    __syncthreads();
    for (int g = 0; g < kWarps; ++g) {
        if (warp == g) {
#pragma unroll
            for (int rp = 0; rp < kRP; ++rp)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float a0, a1;
                    upk2(acc[c][rp], a0, a1);
                    float *d0 = &sm.u.acc[2 * rp][4 * lane + c];
                    *d0 = g == 0 ? a0 : __fadd_rn(*d0, a0);
                    if (2 * rp + 1 < kRows) {
                        float *d1 = &sm.u.acc[2 * rp + 1][4 * lane + c];
                        *d1 = g == 0 ? a1 : __fadd_rn(*d1, a1);
                    }
                }
        }
        __syncthreads();
    }
    if (tid < kRows) {
        float l = 0.0f;
        for (int g = 0; g < kWarps; ++g) l = __fadd_rn(l, sm.red[g][tid]);
        sm.lrow[tid] = l;
    }
    if (tid == 0) {  // the running maxima are the same in every thread
#pragma unroll
        for (int r = 0; r < kRows; ++r) sm.mrow[r] = mrun[r];
    }

    // combine the cluster's partial results on rank 0: shared max, rescaled sums and accumulators
    cluster.sync();
    float res[kRows];
    if (split == 0) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float M = -INFINITY;
            for (int c = 0; c < n_split; ++c) M = fmaxf(M, *cluster.map_shared_rank(&sm.mrow[r], c));
            float L = 0.0f, A = 0.0f;
            for (int c = 0; c < n_split; ++c) {
                const float mc = *cluster.map_shared_rank(&sm.mrow[r], c);
                const float f = mc == -INFINITY ? 0.0f : exp2f(__fsub_rn(mc, M));
                L = __fadd_rn(L, __fmul_rn(*cluster.map_shared_rank(&sm.lrow[r], c), f));
                A = __fadd_rn(A, __fmul_rn(*cluster.map_shared_rank(&sm.u.acc[r][tid], c), f));
            }
            res[r] = __fdiv_rn(A, L);
        }
    }
    cluster.sync();  // peers keep their shared memory until rank 0 has read it
    if (split != 0) return;
    // o = s . H(acc / L) * post
#pragma unroll
    for (int r = 0; r < kRows; ++r) sm.q[r][tid] = res[r];
    __syncthreads();
    fwht_rows<kRows>(sm.q);
    for (int i = tid; i < m * 128; i += kThreads) {
        const int r = i >> 7, e = i & 127;
        const float v = __fmul_rn(__fmul_rn(sm.q[r][e], post), sign_of(mask, e));
        const int64_t at = (head * m_total + r0 + r) * 128 + e;
        if (out_bf16)
            static_cast<uint16_t *>(out)[at] = f32_to_bf16(v);
        else
            static_cast<float *>(out)[at] = v;
    }
}

template <int kRows>
wq_status launch(const void *q, int q_dtype, int64_t heads, int m, int m_total, int r0, const KV &kv, int64_t S,
                 const SignMask &mask, float coef, void *out, int out_dtype, cudaStream_t s) {
    constexpr int kKeys = Smem<kRows>::kKeys;
    if (!ensure_dynamic_smem(reinterpret_cast<const void *>(attn_kernel<kRows>), sizeof(Smem<kRows>)))
        return WQ_ERR_CUDA;
    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const unsigned split = (unsigned)(n_tiles < kMaxSplit ? n_tiles : kMaxSplit);
    for (int64_t h0 = 0; h0 < heads; h0 += 65535) {
        const unsigned hy = (unsigned)(heads - h0 < 65535 ? heads - h0 : 65535);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(split, hy, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = sizeof(Smem<kRows>);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, attn_kernel<kRows>, q, (int)(q_dtype == WQ_BF16), m, m_total, r0, kv, S, mask,
                               coef, out, (int)(out_dtype == WQ_BF16), h0) != cudaSuccess) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
    }
    return launch_status();
}

// Every chunk of up to kMaxRows query rows of every head, one launch per chunk.
wq_status run(const void *q, int q_dtype, int64_t heads, int64_t m, const KV &kv, int64_t S, const SignMask &mask,
              float coef, void *out, int out_dtype, cudaStream_t s) {
    if (m >= kMmaMinRows) return tq3_attn_mma::run(q, q_dtype, heads, m, kv, S, mask, coef, out, out_dtype, s);
    for (int64_t r0 = 0; r0 < m; r0 += kMaxRows) {
        const int mc = (int)(m - r0 < kMaxRows ? m - r0 : kMaxRows);
        wq_status st;
        if (mc <= 1)
            st = launch<1>(q, q_dtype, heads, mc, (int)m, (int)r0, kv, S, mask, coef, out, out_dtype, s);
        else if (mc <= 2)
            st = launch<2>(q, q_dtype, heads, mc, (int)m, (int)r0, kv, S, mask, coef, out, out_dtype, s);
        else if (mc <= 4)
            st = launch<4>(q, q_dtype, heads, mc, (int)m, (int)r0, kv, S, mask, coef, out, out_dtype, s);
        else if (mc <= 8)
            st = launch<8>(q, q_dtype, heads, mc, (int)m, (int)r0, kv, S, mask, coef, out, out_dtype, s);
        else
            st = launch<16>(q, q_dtype, heads, mc, (int)m, (int)r0, kv, S, mask, coef, out, out_dtype, s);
        if (st != WQ_OK) return st;
    }
    return WQ_OK;
}

// post * softmax_scale * log2(e), in double and rounded once; false if that is not finite
bool coefficient(float softmax_scale, float *coef) {
    const uint32_t post_bits = 0x3DB504F3u;  // fp32(1 / sqrt(128))
    float post;
    memcpy(&post, &post_bits, sizeof post);
    *coef = (float)((double)post * (double)softmax_scale * 1.4426950408889634);
    return isfinite(*coef);
}

}  // namespace tq3_attn

unsigned int tq3_attn_read_and_clear_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, tq3_attn::g_fault, sizeof v) != cudaSuccess) return 0x80000000u;
    if (v) cudaMemcpyToSymbol(tq3_attn::g_fault, &zero, sizeof zero);
    return v | tq3_attn_mma::read_and_clear_fault();
}

}  // namespace wq

using namespace wq;

extern "C" wq_status tq3_attention(const void *q, int q_dtype, int64_t heads, int64_t m, const uint8_t *k_records,
                                   const uint8_t *v_records, int64_t S, const uint32_t *sign_mask, float softmax_scale,
                                   void *out, int out_dtype, void *stream) {
    if (heads < 0 || m < 1 || m > tq3_attn::kMaxRowsTotal || S < 1 || S > ((int64_t)1 << 31)) return WQ_ERR_SHAPE;
    if (heads > ((int64_t)1 << 24)) return WQ_ERR_SHAPE;
    if (!valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    float coef;
    if (!isfinite(softmax_scale) || !tq3_attn::coefficient(softmax_scale, &coef)) return WQ_ERR_SHAPE;
    if (heads == 0) return WQ_OK;
    if (!q || !k_records || !v_records || !sign_mask || !out) return WQ_ERR_NULL;
    if (!aligned(q, dtype_size(q_dtype)) || !aligned(out, dtype_size(out_dtype)) || !aligned(k_records, 8) ||
        !aligned(v_records, 8))
        return WQ_ERR_ALIGN;
    tq3::SignMask mask;
    for (int i = 0; i < 4; ++i) mask.w[i] = sign_mask[i];
    tq3_attn::KV kv = {k_records, v_records, nullptr, 0, 0, 0};
    return tq3_attn::run(q, q_dtype, heads, m, kv, S, mask, coef, out, out_dtype, static_cast<cudaStream_t>(stream));
}

extern "C" wq_status tq3_attention_paged(const void *q, int q_dtype, int64_t heads, int64_t m, const uint8_t *k_pool,
                                         const uint8_t *v_pool, int64_t n_pool, const int32_t *page_table,
                                         int64_t pages_per_head, int64_t page_size, int64_t S,
                                         const uint32_t *sign_mask, float softmax_scale, void *out, int out_dtype,
                                         void *stream) {
    if (heads < 0 || m < 1 || m > tq3_attn::kMaxRowsTotal || S < 1 || S > ((int64_t)1 << 31)) return WQ_ERR_SHAPE;
    if (heads > ((int64_t)1 << 24) || n_pool < 0 || pages_per_head < 0) return WQ_ERR_SHAPE;
    if (page_size < 1 || page_size > ((int64_t)1 << 30) || (page_size & (page_size - 1))) return WQ_ERR_SHAPE;
    if (pages_per_head > (((int64_t)1 << 40) / page_size) || S > pages_per_head * page_size) return WQ_ERR_SHAPE;
    if (!valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    float coef;
    if (!isfinite(softmax_scale) || !tq3_attn::coefficient(softmax_scale, &coef)) return WQ_ERR_SHAPE;
    if (heads == 0) return WQ_OK;
    if (!q || !k_pool || !v_pool || !page_table || !sign_mask || !out) return WQ_ERR_NULL;
    if (!aligned(q, dtype_size(q_dtype)) || !aligned(out, dtype_size(out_dtype)) || !aligned(k_pool, 8) ||
        !aligned(v_pool, 8) || !aligned(page_table, 4))
        return WQ_ERR_ALIGN;
    tq3::SignMask mask;
    for (int i = 0; i < 4; ++i) mask.w[i] = sign_mask[i];
    int shift = 0;
    while (((int64_t)1 << shift) < page_size) ++shift;
    tq3_attn::KV kv = {k_pool, v_pool, page_table, pages_per_head, n_pool, shift};
    return tq3_attn::run(q, q_dtype, heads, m, kv, S, mask, coef, out, out_dtype, static_cast<cudaStream_t>(stream));
}
