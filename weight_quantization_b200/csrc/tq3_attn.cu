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
// row), then thread t accumulates coordinate t over the tile's 128 values.
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

constexpr int kKeys = 128;     // keys per tile = threads per CTA
constexpr int kThreads = 128;
constexpr int kWords = 14;     // 32-bit words per 56-byte record
constexpr int kMaxSplit = 8;   // CTAs per cluster (portable cluster size)
constexpr int kMaxRows = 16;   // query rows per head

template <int kRows>
struct Smem {
    float q[kRows][128];           // q~ = H (s . q), unnormalised
    float w[kRows][kKeys];         // logits (log2 units), then p_j * norm_j * scale_j
    float acc[kRows][128];         // this CTA's accumulators, read by the cluster's rank 0
    uint32_t krec[kKeys][kWords];  // the tile's key records
    uint32_t vrec[kKeys][kWords];  // the tile's value records
    float mrow[kRows], lrow[kRows], alpha[kRows];
};

// Sign draw of element e: +1.0 or -1.0.
__device__ __forceinline__ float sign_of(const SignMask &m, int e) { return ((m.w[e >> 5] >> (e & 31)) & 1u) ? 1.0f : -1.0f; }

// In-place unnormalised FWHT of `rows` rows of 128 floats in shared memory; all threads take part.
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

// Copy n_valid records (n_valid <= kKeys) to shared memory as 8-byte words; the rest are zeros.
__device__ __forceinline__ void load_records(uint32_t (*dst)[kWords], const uint8_t *__restrict__ src, int n_valid) {
    const uint2 *s = reinterpret_cast<const uint2 *>(src);
    uint2 *d = reinterpret_cast<uint2 *>(&dst[0][0]);
    for (int i = threadIdx.x; i < kKeys * (kWords / 2); i += kThreads)
        d[i] = i < n_valid * (kWords / 2) ? __ldg(s + i) : make_uint2(0u, 0u);
}

// q: [heads][m][128] (bf16 or fp32); k_rec, v_rec: [heads][S] 56-byte records; out: [heads][m][128].
// coef = post * softmax_scale * log2(e): logits are kept in log2 units so that exp2 applies.
template <int kRows>
__global__ void __launch_bounds__(kThreads)
    attn_kernel(const void *__restrict__ q, int q_bf16, int m, const uint8_t *__restrict__ k_rec,
                const uint8_t *__restrict__ v_rec, int64_t S, SignMask mask, float coef, void *__restrict__ out,
                int out_bf16, int64_t head0) {
    __shared__ __align__(16) Smem<kRows> sm;
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
    if (tid < kRows) {
        sm.mrow[tid] = -INFINITY;
        sm.lrow[tid] = 0.0f;
    }
    __syncthreads();
    fwht_rows<kRows>(sm.q);

    float acc[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r] = 0.0f;

    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const int64_t t_begin = n_tiles * split / n_split, t_end = n_tiles * (split + 1) / n_split;
    const uint8_t *kh = k_rec + head * S * 56, *vh = v_rec + head * S * 56;
    for (int64_t tile = t_begin; tile < t_end; ++tile) {
        const int64_t j0 = tile * kKeys;
        const int n_valid = (int)(S - j0 < kKeys ? S - j0 : kKeys);
        load_records(sm.krec, kh + j0 * 56, n_valid);
        load_records(sm.vrec, vh + j0 * 56, n_valid);
        __syncthreads();

        // logits: thread t scores key t against every row, 32 coordinates at a time
        {
            uint32_t W[13];
#pragma unroll
            for (int i = 0; i < 13; ++i) W[i] = sm.krec[tid][i];
            float dot[kRows];
#pragma unroll
            for (int r = 0; r < kRows; ++r) dot[r] = 0.0f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float c[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {  // index of coordinate 32 ch + e: bits 3e' .. of the record
                    const int o = 3 * (32 * ch + e), wq = o >> 5, sh = o & 31;
                    c[e] = __shfl_sync(0xffffffffu, cb, (int)__funnelshift_r(W[wq], W[wq + 1], sh));
                }
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    const float4 *qr = reinterpret_cast<const float4 *>(&sm.q[r][32 * ch]);
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
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
            for (int r = 0; r < kRows; ++r) sm.w[r][tid] = tid < n_valid ? __fmul_rn(dot[r], kscale) : -INFINITY;
        }
        __syncthreads();

        // online softmax, one warp per row: new max, rescale factor, p_j * norm_j * scale_j
        for (int r = warp; r < kRows; r += kThreads / 32) {
            float x[4], mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                x[u] = sm.w[r][lane + 32 * u];
                mx = fmaxf(mx, x[u]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = sm.mrow[r], m_new = fmaxf(m_old, mx);
            const float a = m_old == -INFINITY ? 0.0f : exp2f(__fsub_rn(m_old, m_new));
            float sum = 0.0f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = lane + 32 * u;
                const float p = exp2f(__fsub_rn(x[u], m_new));  // 0 for the keys past S
                sum = __fadd_rn(sum, p);
                sm.w[r][j] = __fmul_rn(p, __fmul_rn(__uint_as_float(sm.vrec[j][12]), __uint_as_float(sm.vrec[j][13])));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
            if (lane == 0) {
                sm.mrow[r] = m_new;
                sm.lrow[r] = __fadd_rn(__fmul_rn(sm.lrow[r], a), sum);
                sm.alpha[r] = a;
            }
        }
        __syncthreads();

        // values: thread t accumulates rotated coordinate t over the tile's keys
        {
            const int o = 3 * tid, wq = o >> 5, sh = o & 31;
#pragma unroll
            for (int r = 0; r < kRows; ++r) acc[r] = __fmul_rn(acc[r], sm.alpha[r]);
#pragma unroll 4
            for (int j = 0; j < kKeys; ++j) {
                const float c = __shfl_sync(0xffffffffu, cb, (int)__funnelshift_r(sm.vrec[j][wq], sm.vrec[j][wq + 1], sh));
#pragma unroll
                for (int r = 0; r < kRows; ++r) acc[r] = __fmaf_rn(sm.w[r][j], c, acc[r]);
            }
        }
        __syncthreads();  // the tile's buffers are refilled next
    }

    // combine the cluster's partial results on rank 0: shared max, rescaled sums and accumulators
#pragma unroll
    for (int r = 0; r < kRows; ++r) sm.acc[r][tid] = acc[r];
    cluster.sync();
    if (split == 0) {
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
            acc[r] = __fdiv_rn(A, L);
        }
    }
    cluster.sync();  // peers keep their shared memory until rank 0 has read it
    if (split != 0) return;
    // o = s . H(acc / L) * post
#pragma unroll
    for (int r = 0; r < kRows; ++r) sm.q[r][tid] = acc[r];
    __syncthreads();
    fwht_rows<kRows>(sm.q);
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
    const int64_t n_tiles = (S + kKeys - 1) / kKeys;
    const unsigned split = (unsigned)(n_tiles < kMaxSplit ? n_tiles : kMaxSplit);
    for (int64_t h0 = 0; h0 < heads; h0 += 65535) {
        const unsigned hy = (unsigned)(heads - h0 < 65535 ? heads - h0 : 65535);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(split, hy, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int mi = (int)m;
    if (mi <= 1) return tq3_attn::launch<1>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 2) return tq3_attn::launch<2>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 4) return tq3_attn::launch<4>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    if (mi <= 8) return tq3_attn::launch<8>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
    return tq3_attn::launch<16>(q, q_dtype, heads, mi, k_records, v_records, S, mask, coef, out, out_dtype, s);
}
