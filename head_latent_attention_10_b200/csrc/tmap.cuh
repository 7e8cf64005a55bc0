// tmap.cuh -- host-side TMA tensor-map encoding (cuTensorMapEncodeTiled,
// fetched through the runtime so the library does not link libcuda) with a
// small cache keyed by every encoding parameter.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

namespace mla {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
{
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

struct TmapKey {
    const void *ptr;
    uint32_t rank, dtype;
    uint64_t dims[4], strides[3];
    uint32_t box[4];
    int swizzle;
    bool operator==(const TmapKey &o) const { return memcmp(this, &o, sizeof *this) == 0; }
};

inline CUtensorMapSwizzle swizzle_for(uint32_t inner_bytes)
{
    return inner_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                              : (inner_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// Tensor of rank 1-4 (bf16 unless `dtype` says otherwise): dims innermost
// first (elements), strides of dims 1.. in bytes, box in elements.
// Out-of-range elements read as zero and are not written by stores.
inline bool make_tmap_nd(CUtensorMap *out, const void *ptr, uint32_t rank, const uint64_t *dims,
                         const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw,
                         CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
{
    static std::mutex mu;
    static TmapKey keys[64];
    static CUtensorMap maps[64];
    static int used = 0, next = 0;
    if (rank < 1 || rank > 4) return false;
    TmapKey k;
    memset(&k, 0, sizeof k);
    k.ptr = ptr;
    k.rank = rank;
    k.dtype = (uint32_t)dtype;
    for (uint32_t i = 0; i < rank; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        if (i + 1 < rank) k.strides[i] = strides[i];
    }
    k.swizzle = (int)sw;
    {
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < used; ++i)
            if (keys[i] == k) {
                *out = maps[i];
                return true;
            }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[4], gstr[3];
    cuuint32_t cbox[4], estr[4] = {1, 1, 1, 1};
    for (uint32_t i = 0; i < rank; ++i) {
        gdim[i] = k.dims[i];
        cbox[i] = k.box[i];
        if (i + 1 < rank) gstr[i] = k.strides[i];
    }
    CUtensorMap m;
    if (fn(&m, dtype, rank, const_cast<void *>(ptr), gdim, gstr, cbox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> g(mu);
    keys[next] = k;
    maps[next] = m;
    next = (next + 1) % 64;
    if (used < 64) ++used;
    *out = m;
    return true;
}

inline bool make_tmap_3d(CUtensorMap *out, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw)
{
    const uint64_t dims[3] = {d0, d1, d2}, strides[2] = {s1, s2};
    const uint32_t box[3] = {b0, b1, b2};
    return make_tmap_nd(out, ptr, 3, dims, strides, box, sw);
}

// uint8 tensor of rank 3 (the FP8 cache), as make_tmap_3d.
inline bool make_tmap_3d_u8(CUtensorMap *out, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                            uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw)
{
    const uint64_t dims[3] = {d0, d1, d2}, strides[2] = {s1, s2};
    const uint32_t box[3] = {b0, b1, b2};
    return make_tmap_nd(out, ptr, 3, dims, strides, box, sw, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

inline bool make_tmap_4d(CUtensorMap *out, const void *ptr, const uint64_t (&dims)[4], const uint64_t (&strides)[3],
                         const uint32_t (&box)[4], CUtensorMapSwizzle sw)
{
    return make_tmap_nd(out, ptr, 4, dims, strides, box, sw);
}

}  // namespace mla
