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
// Work split. A cluster of up to 8 CTAs serves one (head, query-row group): CTA x of the cluster
// takes a contiguous share of the key tiles (128 keys each), keeps a running max, sum and 128
// accumulators per query row (online softmax), and the cluster combines its CTAs' partial results
// through distributed shared memory, so nothing is written to global memory but the output. Within
// a CTA, thread t scores key t of the tile (its indices are unpacked once and serve every query
// row); for the values, each lane owns four rotated coordinates and each warp a quarter of the
// tile's keys, the warps' sums being added once at the end.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "tq3_common.cuh"
#include "wq.h"

namespace cg = cooperative_groups;

namespace wq {
namespace tq3_attn {

using tq3::SignMask;

constexpr int kWords = 14;     // 32-bit words per 56-byte record
constexpr int kMaxSplit = 8;   // CTAs per cluster (portable cluster size)
constexpr int kMaxRows = 16;   // query rows per head

// Keys per tile = threads per CTA. 128 keys keep four CTAs (up to 128 registers a thread) on an SM,
// two with 16 rows.
template <int kRows>
constexpr int keys_per_tile() { return 128; }

template <int kRows>
struct Smem {
    static constexpr int kKeys = keys_per_tile<kRows>();
    static constexpr int kWarps = kKeys / 32;
    float q[kRows][128];           // q~ = H (s . q), unnormalised; at the end, the output rows
    float w[kKeys][kRows];         // p_j * norm_j * scale_j of the tile's keys, a key's rows together
    float acc[kRows][128];         // this CTA's accumulators, read by the cluster's rank 0
    uint32_t krec[kKeys][kWords];  // the tile's key records
    uint32_t vrec[kKeys][kWords];  // the tile's value records
    float red[kWarps][kRows];      // per-warp partial maxima and sums
    float mrow[kRows], lrow[kRows];
};

// Sign draw of element e: +1.0 or -1.0.
__device__ __forceinline__ float sign_of(const SignMask &m, int e) { return ((m.w[e >> 5] >> (e & 31)) & 1u) ? 1.0f : -1.0f; }

// In-place unnormalised FWHT of kRows rows of 128 floats in shared memory; all threads take part.
template <int kRows, int kThreads>
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

// q: [heads][m][128] (bf16 or fp32); k_rec, v_rec: [heads][S] 56-byte records; out: [heads][m][128].
// coef = post * softmax_scale * log2(e): logits are kept in log2 units so that exp2 applies.
//
// Per tile of kKeys keys (one per thread): the records are stored to shared memory from registers
// (loaded during the previous tile), the next tile's loads are issued, thread t scores key t
// against every row, the CTA agrees on the new row maxima, thread t turns its logits into weights
// p_t * norm_t * scale_t of its value record, and warp g accumulates keys 32g .. 32g + 31 with lane
// l owning rotated coordinates 4l .. 4l + 3 (one funnel shift brings the four indices in).
template <int kRows>
__global__ void __launch_bounds__(keys_per_tile<kRows>(), kRows > 8 ? 2 : 4)
    attn_kernel(const void *__restrict__ q, int q_bf16, int m, const uint8_t *__restrict__ k_rec,
                const uint8_t *__restrict__ v_rec, int64_t S, SignMask mask, float coef, void *__restrict__ out,
                int out_bf16, int64_t head0) {
    using SM = Smem<kRows>;
    constexpr int kKeys = SM::kKeys, kThreads = kKeys, kWarps = SM::kWarps;
    constexpr int kLoads = kKeys * (kWords / 2) / kThreads;  // 8-byte record words per thread and tensor
    __shared__ __align__(16) SM sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = (int)cluster.block_rank(), n_split = (int)cluster.num_blocks();
    const int64_t head = head0 + blockIdx.y;
    const float cb = tq3::centroid((uint32_t)(lane & 7));  // lane l holds centroid l mod 8
    const float post = tq3::fwht_post();

    // q~ = H (s . q) for every row (rows m .. kRows-1 are zeros and never written out)
    for (int i = tid; i < kRows * 128; i += kThreads) {
        const int r = i >> 7, e = i & 127;
        float v = 0.0f;
        if (r < m) {
            const int64_t at = (head * m + r) * 128 + e;
            v = q_bf16 ? __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t *>(q) + at) << 16)
                       : __ldg(static_cast<const float *>(q) + at);
        }
        sm.q[r][e] = __fmul_rn(v, sign_of(mask, e));
    }
    __syncthreads();
    fwht_rows<kRows, kThreads>(sm.q);

    float acc[4][kRows], lsum[kRows], mrun[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        lsum[r] = 0.0f;
        mrun[r] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[c][r] = 0.0f;
    }

    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const int64_t t_begin = n_tiles * split / n_split, t_end = n_tiles * (split + 1) / n_split;
    const uint2 *kh = reinterpret_cast<const uint2 *>(k_rec + head * S * 56);
    const uint2 *vh = reinterpret_cast<const uint2 *>(v_rec + head * S * 56);
    // the tile's records, one 8-byte word per load: word i of the tile is record i / 7, part i % 7
    uint2 kbuf[kLoads], vbuf[kLoads];
    auto fetch = [&](int64_t tile) {
        const int64_t j0 = tile * kKeys;
        const int64_t n_words = (S - j0 < kKeys ? S - j0 : kKeys) * (kWords / 2);
#pragma unroll
        for (int u = 0; u < kLoads; ++u) {
            const int i = tid + u * kThreads;
            const bool ok = tile < t_end && i < n_words;
            kbuf[u] = ok ? __ldg(kh + j0 * (kWords / 2) + i) : make_uint2(0u, 0u);
            vbuf[u] = ok ? __ldg(vh + j0 * (kWords / 2) + i) : make_uint2(0u, 0u);
        }
    };
    fetch(t_begin);
    for (int64_t tile = t_begin; tile < t_end; ++tile) {
        const int n_valid = (int)(S - tile * kKeys < kKeys ? S - tile * kKeys : kKeys);
#pragma unroll
        for (int u = 0; u < kLoads; ++u) {
            reinterpret_cast<uint2 *>(&sm.krec[0][0])[tid + u * kThreads] = kbuf[u];
            reinterpret_cast<uint2 *>(&sm.vrec[0][0])[tid + u * kThreads] = vbuf[u];
        }
        __syncthreads();
        fetch(tile + 1);  // in flight during this tile's work

        // logits: thread t scores key t against every row, kChunk coordinates at a time
        constexpr int kChunk = kRows > 4 ? 16 : 32;
        float dot[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) dot[r] = 0.0f;
        {
            uint32_t W[13];
#pragma unroll
            for (int i = 0; i < 13; ++i) W[i] = sm.krec[tid][i];
#pragma unroll
            for (int ch = 0; ch < 128 / kChunk; ++ch) {
                float c[kChunk];
#pragma unroll
                for (int e = 0; e < kChunk; ++e) {  // the index of coordinate kChunk ch + e is at bit 3 (kChunk ch + e)
                    const int o = 3 * (kChunk * ch + e), wq = o >> 5, sh = o & 31;
                    c[e] = __shfl_sync(0xffffffffu, cb, (int)__funnelshift_r(W[wq], W[wq + 1], sh));
                }
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    const float4 *qr = reinterpret_cast<const float4 *>(&sm.q[r][kChunk * ch]);
#pragma unroll
                    for (int e4 = 0; e4 < kChunk / 4; ++e4) {
                        const float4 qq = qr[e4];
                        dot[r] = __fmaf_rn(qq.x, c[4 * e4], dot[r]);
                        dot[r] = __fmaf_rn(qq.y, c[4 * e4 + 1], dot[r]);
                        dot[r] = __fmaf_rn(qq.z, c[4 * e4 + 2], dot[r]);
                        dot[r] = __fmaf_rn(qq.w, c[4 * e4 + 3], dot[r]);
                    }
                }
            }
            const float kscale = __fmul_rn(__fmul_rn(__uint_as_float(W[12]), __uint_as_float(sm.krec[tid][13])), coef);
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                dot[r] = tid < n_valid ? __fmul_rn(dot[r], kscale) : -INFINITY;
                float mx = dot[r];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) sm.red[warp][r] = mx;
            }
        }
        __syncthreads();

        // new row maxima (the same in every thread), rescale factors, the weights of key t
        float alpha[kRows];
        {
            const float nv = __uint_as_float(sm.vrec[tid][12]), sv = __uint_as_float(sm.vrec[tid][13]);
            const float nvsv = __fmul_rn(nv, sv);
            float wt[kRows];
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                float mx = mrun[r];
#pragma unroll
                for (int g = 0; g < kWarps; ++g) mx = fmaxf(mx, sm.red[g][r]);
                alpha[r] = mrun[r] == -INFINITY ? 0.0f : exp2f(__fsub_rn(mrun[r], mx));
                mrun[r] = mx;
                const float p = exp2f(__fsub_rn(dot[r], mx));  // 0 for the keys past S
                lsum[r] = __fadd_rn(__fmul_rn(lsum[r], alpha[r]), p);
                wt[r] = __fmul_rn(p, nvsv);
            }
#pragma unroll
            for (int r4 = 0; r4 < kRows; r4 += 4) {
                if constexpr (kRows >= 4) {
                    *reinterpret_cast<float4 *>(&sm.w[tid][r4]) = make_float4(wt[r4], wt[r4 + 1], wt[r4 + 2], wt[r4 + 3]);
                } else {
#pragma unroll
                    for (int r = 0; r < kRows; ++r) sm.w[tid][r] = wt[r];
                }
            }
        }
        __syncthreads();

        // values: warp g takes keys 32 g .. 32 g + 31, lane l the rotated coordinates 4l .. 4l + 3
        {
            const int o = 12 * lane, wq = o >> 5, sh = o & 31;
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[c][r] = __fmul_rn(acc[c][r], alpha[r]);
#pragma unroll 2
            for (int jj = 0; jj < 32; ++jj) {
                const int j = 32 * warp + jj;
                const uint32_t bits = __funnelshift_r(sm.vrec[j][wq], sm.vrec[j][wq + 1], sh);
                float cv[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) cv[c] = __shfl_sync(0xffffffffu, cb, (int)(bits >> (3 * c)));
                float wj[kRows];
                if constexpr (kRows >= 4) {
#pragma unroll
                    for (int r4 = 0; r4 < kRows; r4 += 4) {
                        const float4 x = *reinterpret_cast<const float4 *>(&sm.w[j][r4]);
                        wj[r4] = x.x; wj[r4 + 1] = x.y; wj[r4 + 2] = x.z; wj[r4 + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int r = 0; r < kRows; ++r) wj[r] = sm.w[j][r];
                }
#pragma unroll
                for (int r = 0; r < kRows; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[c][r] = __fmaf_rn(wj[r], cv[c], acc[c][r]);
            }
        }
        __syncthreads();  // the tile's buffers are refilled next
    }

    // this CTA's row sums and accumulators, in a fixed order: warp sums, then warps one by one
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
        float v = lsum[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) sm.red[warp][r] = v;
    }
    for (int g = 0; g < kWarps; ++g) {
        if (warp == g) {
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    sm.acc[r][4 * lane + c] = g == 0 ? acc[c][r] : __fadd_rn(sm.acc[r][4 * lane + c], acc[c][r]);
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
    if (split == 0 && tid < 128) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float M = -INFINITY;
            for (int c = 0; c < n_split; ++c) M = fmaxf(M, *cluster.map_shared_rank(&sm.mrow[r], c));
            float L = 0.0f, A = 0.0f;
            for (int c = 0; c < n_split; ++c) {
                const float f = exp2f(__fsub_rn(*cluster.map_shared_rank(&sm.mrow[r], c), M));
                L = __fadd_rn(L, __fmul_rn(*cluster.map_shared_rank(&sm.lrow[r], c), f));
                A = __fadd_rn(A, __fmul_rn(*cluster.map_shared_rank(&sm.acc[r][tid], c), f));
            }
            res[r] = __fdiv_rn(A, L);
        }
    }
    cluster.sync();  // peers keep their shared memory until rank 0 has read it
    if (split != 0) return;
    // o = s . H(acc / L) * post
    if (tid < 128) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) sm.q[r][tid] = res[r];
    }
    __syncthreads();
    fwht_rows<kRows, kThreads>(sm.q);
    for (int i = tid; i < m * 128; i += kThreads) {
        const int r = i >> 7, e = i & 127;
        const float v = __fmul_rn(__fmul_rn(sm.q[r][e], post), sign_of(mask, e));
        const int64_t at = (head * m + r) * 128 + e;
        if (out_bf16)
            static_cast<uint16_t *>(out)[at] = f32_to_bf16(v);
        else
            static_cast<float *>(out)[at] = v;
    }
}

template <int kRows>
wq_status launch(const void *q, int q_dtype, int64_t heads, int m, const uint8_t *k, const uint8_t *v, int64_t S,
                 const SignMask &mask, float coef, void *out, int out_dtype, cudaStream_t s) {
    constexpr int kKeys = keys_per_tile<kRows>();
    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const unsigned split = (unsigned)(n_tiles < kMaxSplit ? n_tiles : kMaxSplit);
    for (int64_t h0 = 0; h0 < heads; h0 += 65535) {
        const unsigned hy = (unsigned)(heads - h0 < 65535 ? heads - h0 : 65535);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(split, hy, 1);
        cfg.blockDim = dim3(kKeys, 1, 1);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = split;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, attn_kernel<kRows>, q, (int)(q_dtype == WQ_BF16), m, k, v, S, mask, coef, out,
                               (int)(out_dtype == WQ_BF16), h0) != cudaSuccess) {
            cudaGetLastError();
            return WQ_ERR_CUDA;
        }
    }
    return launch_status();
}

}  // namespace tq3_attn
}  // namespace wq

using namespace wq;

extern "C" wq_status tq3_attention(const void *q, int q_dtype, int64_t heads, int64_t m, const uint8_t *k_records,
                                   const uint8_t *v_records, int64_t S, const uint32_t *sign_mask, float softmax_scale,
                                   void *out, int out_dtype, void *stream) {
    if (heads < 0 || m < 1 || m > tq3_attn::kMaxRows || S < 1 || S > ((int64_t)1 << 31)) return WQ_ERR_SHAPE;
    if (heads > ((int64_t)1 << 24)) return WQ_ERR_SHAPE;
    if (!valid_dtype(q_dtype) || !valid_dtype(out_dtype)) return WQ_ERR_DTYPE;
    if (!isfinite(softmax_scale)) return WQ_ERR_SHAPE;
    if (heads == 0) return WQ_OK;
    if (!q || !k_records || !v_records || !sign_mask || !out) return WQ_ERR_NULL;
    if (!aligned(q, dtype_size(q_dtype)) || !aligned(out, dtype_size(out_dtype)) || !aligned(k_records, 8) ||
        !aligned(v_records, 8))
        return WQ_ERR_ALIGN;
    tq3::SignMask mask;
    for (int i = 0; i < 4; ++i) mask.w[i] = sign_mask[i];
    // post * softmax_scale * log2(e), in double and rounded once
    const uint32_t post_bits = 0x3DB504F3u;  // fp32(1 / sqrt(128))
    float post;
    memcpy(&post, &post_bits, sizeof post);
    const float coef = (float)((double)post * (double)softmax_scale * 1.4426950408889634);
    if (!isfinite(coef)) return WQ_ERR_SHAPE;  // the scale times post * log2(e) must stay finite in fp32
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int mi = (int)m;
    if (mi <= 1) return tq3_attn::launch<1>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 2) return tq3_attn::launch<2>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 4) return tq3_attn::launch<4>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 8) return tq3_attn::launch<8>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    return tq3_attn::launch<16>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
}
