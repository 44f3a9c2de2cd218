// Host-side tensor-map encoding for the TMA kernels (driver entry point fetched through the
// runtime, so the library does not link libcuda directly).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

namespace wq {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}
}  // namespace

bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    memset(map, 0, sizeof(*map));
    const cuuint64_t gdim[2] = {inner, rows};
    const cuuint64_t gstride[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A launch may use 48 KiB of shared memory in total (static + dynamic) without opting in. The
// kernel's static shared memory is read from its attributes, so a dynamic size just under 48 KiB
// on a kernel that also declares __shared__ arrays still gets the opt-in it needs. The attribute
// is raised once per (kernel, device) to the largest dynamic size asked for so far.
bool ensure_dynamic_smem(const void *kernel, size_t smem) {
    if (smem == 0) return true;
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, std::pair<size_t, size_t>> state;  // (static bytes, set to)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kernel, dev);
    auto it = state.find(key);
    if (it == state.end()) {
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return false;
        it = state.emplace(key, std::make_pair((size_t)attr.sharedSizeBytes, (size_t)0)).first;
    }
    const size_t static_bytes = it->second.first;
    size_t &cur = it->second.second;
    if (smem <= cur || static_bytes + smem <= 48 * 1024) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return false;
    cur = smem;
    return true;
}

int blocks_per_sm_cached(const void *kernel, int threads, size_t smem) {
    static std::mutex mu;
    static std::map<std::pair<std::pair<const void *, int>, std::pair<int, size_t>>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const auto key = std::make_pair(std::make_pair(kernel, dev), std::make_pair(threads, smem));
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess) return 0;
    cache[key] = n;
    return n;
}

}  // namespace wq
