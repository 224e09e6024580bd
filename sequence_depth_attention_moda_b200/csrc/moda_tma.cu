// moda_tma.cu -- host-side launch set-up shared by the kernels: TMA tensor
// maps (memoised) and the per-device dynamic shared-memory attribute.  The
// driver entry point cuTensorMapEncodeTiled is fetched through the runtime,
// so the library does not link libcuda directly.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <tuple>
#include <unordered_map>
#include <vector>

#include "moda_internal.h"

namespace moda {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

static_assert(sizeof(TmaMap) == sizeof(CUtensorMap), "TmaMap must hold a CUtensorMap");

namespace {

// Encoding a tensor map is a pure function of its arguments, so results are
// memoised: repeated calls on the same buffers (every training step, every
// decoding token) skip the driver call.  The table is cleared when it fills.
struct MapKey {
    uint64_t base, d, rows, outer;
    uint32_t box_rows, box_outer;
    bool operator==(const MapKey& o) const {
        return base == o.base && d == o.d && rows == o.rows && outer == o.outer &&
               box_rows == o.box_rows && box_outer == o.box_outer;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
        for (uint64_t v : {k.d, k.rows, k.outer, uint64_t(k.box_rows) << 32 | k.box_outer})
            h = (h ^ v) * 0x100000001B3ull;
        return static_cast<size_t>(h ^ (h >> 29));
    }
};
constexpr size_t kMapCacheEntries = 1024;
std::mutex g_map_mutex;
std::unordered_map<MapKey, TmaMap, MapKeyHash> g_map_cache;

cudaError_t encode_3d_bf16(TmaMap* out, const void* base, uint64_t d, uint64_t rows, uint64_t outer,
                           uint32_t box_rows, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t dims[3] = {d, rows, outer};
    const cuuint64_t strides[2] = {d * 2, rows * d * 2};
    const cuuint32_t box[3] = {64, box_rows, box_outer};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    std::memcpy(out->bytes, &map, sizeof(map));
    return cudaSuccess;
}

// The same for the 4-D maps (token-major views of Q and dO, the layer-major
// depth caches): keyed by base, extents, strides and box.
struct Map4Key {
    uint64_t base, dims[4], strides[3];
    uint32_t box[4];
    bool operator==(const Map4Key& o) const {
        return std::memcmp(this, &o, sizeof(Map4Key)) == 0;
    }
};
struct Map4KeyHash {
    size_t operator()(const Map4Key& k) const {
        uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
        for (int i = 0; i < 4; ++i) h = (h ^ k.dims[i]) * 0x100000001B3ull;
        for (int i = 0; i < 3; ++i) h = (h ^ k.strides[i]) * 0x100000001B3ull;
        for (int i = 0; i < 4; ++i) h = (h ^ k.box[i]) * 0x100000001B3ull;
        return static_cast<size_t>(h ^ (h >> 29));
    }
};
std::unordered_map<Map4Key, TmaMap, Map4KeyHash> g_map4_cache;

std::mutex g_attr_mutex;
std::vector<std::tuple<int, const void*, int>> g_attr_done;

}  // namespace

cudaError_t make_tma_3d_bf16(TmaMap* out, const void* base, uint64_t d, uint64_t rows,
                             uint64_t outer, uint32_t box_rows, uint32_t box_outer) {
    const MapKey key{reinterpret_cast<uint64_t>(base), d, rows, outer, box_rows, box_outer};
    {
        std::lock_guard<std::mutex> lk(g_map_mutex);
        auto it = g_map_cache.find(key);
        if (it != g_map_cache.end()) {
            *out = it->second;
            return cudaSuccess;
        }
    }
    cudaError_t e = encode_3d_bf16(out, base, d, rows, outer, box_rows, box_outer);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_map_mutex);
    if (g_map_cache.size() >= kMapCacheEntries) g_map_cache.clear();
    g_map_cache.emplace(key, *out);
    return cudaSuccess;
}

cudaError_t make_tma_4d_bf16(TmaMap* out, const void* base, const uint64_t dims[4],
                             const uint64_t strides_bytes[3], const uint32_t box[4]) {
    Map4Key key;
    std::memset(&key, 0, sizeof(key));
    key.base = reinterpret_cast<uint64_t>(base);
    for (int i = 0; i < 4; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
    for (int i = 0; i < 3; ++i) key.strides[i] = strides_bytes[i];
    {
        std::lock_guard<std::mutex> lk(g_map_mutex);
        auto it = g_map4_cache.find(key);
        if (it != g_map4_cache.end()) {
            *out = it->second;
            return cudaSuccess;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap map;
    std::memset(&map, 0, sizeof(map));
    const cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
    const cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
    const cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
    const cuuint32_t estride[4] = {1, 1, 1, 1};
    CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gd, gs, bx,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    std::memcpy(out->bytes, &map, sizeof(map));
    std::lock_guard<std::mutex> lk(g_map_mutex);
    if (g_map4_cache.size() >= kMapCacheEntries) g_map4_cache.clear();
    g_map4_cache.emplace(key, *out);
    return cudaSuccess;
}

cudaError_t set_max_dynamic_smem(const void* func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_attr_mutex);
    for (const auto& t : g_attr_done)
        if (std::get<0>(t) == dev && std::get<1>(t) == func && std::get<2>(t) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) g_attr_done.emplace_back(dev, func, bytes);
    return e;
}

}  // namespace moda
