// tma_host.h -- host-side creation of TMA tensor maps for [BH, rows, cols]
// bf16 tensors, without linking libcuda: the driver entry point is fetched
// through the runtime once per process.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <cstring>
#include <mutex>

namespace fa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Encoded maps, cached.  A tensor map is a pure function of the arguments of
// its encoder (element kind, base address, the three extents and the box
// height), so a map taken from this table is bit-for-bit the map a fresh
// encode would return; caching only removes the host cost of the encode from
// repeated calls on the same buffers.  The table is direct-mapped (a new key
// overwrites its slot) and guarded by a mutex; it is the library's only host
// state besides the per-device attributes.
enum MapKind : uint32_t { MAP_BF16 = 1, MAP_U8 = 2, MAP_F32_SW128 = 3 };

struct MapKey {
    uint32_t kind, box_rows;
    const void* base;
    uint64_t depth, rows, cols;
    bool operator==(const MapKey& o) const {
        return kind == o.kind && box_rows == o.box_rows && base == o.base && depth == o.depth &&
               rows == o.rows && cols == o.cols;
    }
};

struct MapCache {
    static constexpr int kSlots = 256;
    struct Slot {
        bool used = false;
        MapKey key{};
        CUtensorMap map;
    };
    std::mutex mu;
    Slot slot[kSlots];

    static uint32_t hash(const MapKey& k) {
        uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
        h ^= (k.depth * 31 + k.rows) * 0xC2B2AE3D27D4EB4Full;
        h ^= (k.cols * 131 + k.kind * 7 + k.box_rows) * 0x165667B19E3779F9ull;
        return static_cast<uint32_t>(h >> 40) % kSlots;
    }
    bool find(const MapKey& k, CUtensorMap* out) {
        std::lock_guard<std::mutex> lock(mu);
        const Slot& s = slot[hash(k)];
        if (!s.used || !(s.key == k)) return false;
        std::memcpy(out, &s.map, sizeof(CUtensorMap));
        return true;
    }
    void put(const MapKey& k, const CUtensorMap* m) {
        std::lock_guard<std::mutex> lock(mu);
        Slot& s = slot[hash(k)];
        s.used = true;
        s.key = k;
        std::memcpy(&s.map, m, sizeof(CUtensorMap));
    }
};

inline MapCache& map_cache() {
    static MapCache c;
    return c;
}

// A 3-D map over a contiguous [depth, rows, cols] bf16 tensor (cols fastest),
// read in boxes of [1, box_rows, 64] with the 128-byte swizzle, zero fill out
// of bounds.  Requirements checked by the driver: base 16-byte aligned,
// cols * 2 and rows * cols * 2 multiples of 16.
inline bool make_map_bf16_3d_encode(CUtensorMap* map, const void* base, uint64_t depth, uint64_t rows,
                             uint64_t cols, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, depth};
    cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Same for 8-bit elements (E4M3 stored as bytes): boxes of [1, box_rows, 128].
inline bool make_map_u8_3d_encode(CUtensorMap* map, const void* base, uint64_t depth, uint64_t rows,
                           uint64_t cols, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, depth};
    cuuint64_t strides[2] = {cols, rows * cols};
    cuuint32_t box[3] = {128, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A 3-D map over a contiguous [depth, rows, cols] fp32 tensor (cols fastest),
// boxes of [1, 128, 32] (32 floats = 128 B) with the 128-byte swizzle; used as
// the destination of shared -> global add-reductions.
inline bool make_map_f32_3d_sw128_encode(CUtensorMap* map, const void* base, uint64_t depth,
                                  uint64_t rows, uint64_t cols) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, depth};
    cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool cached_map(uint32_t kind, CUtensorMap* map, const void* base, uint64_t depth,
                       uint64_t rows, uint64_t cols, uint32_t box_rows) {
    const MapKey key{kind, box_rows, base, depth, rows, cols};
    if (map_cache().find(key, map)) return true;
    bool ok = false;
    if (kind == MAP_BF16) ok = make_map_bf16_3d_encode(map, base, depth, rows, cols, box_rows);
    else if (kind == MAP_U8) ok = make_map_u8_3d_encode(map, base, depth, rows, cols, box_rows);
    else ok = make_map_f32_3d_sw128_encode(map, base, depth, rows, cols);
    if (ok) map_cache().put(key, map);
    return ok;
}

inline bool make_map_bf16_3d(CUtensorMap* map, const void* base, uint64_t depth, uint64_t rows,
                             uint64_t cols, uint32_t box_rows) {
    return cached_map(MAP_BF16, map, base, depth, rows, cols, box_rows);
}

inline bool make_map_u8_3d(CUtensorMap* map, const void* base, uint64_t depth, uint64_t rows,
                           uint64_t cols, uint32_t box_rows) {
    return cached_map(MAP_U8, map, base, depth, rows, cols, box_rows);
}

inline bool make_map_f32_3d_sw128(CUtensorMap* map, const void* base, uint64_t depth,
                                  uint64_t rows, uint64_t cols) {
    return cached_map(MAP_F32_SW128, map, base, depth, rows, cols, 128);
}

}  // namespace fa
