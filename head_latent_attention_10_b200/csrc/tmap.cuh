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
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    int swizzle;
    bool operator==(const TmapKey &o) const { return memcmp(this, &o, sizeof *this) == 0; }
};

inline CUtensorMapSwizzle swizzle_for(uint32_t inner_bytes)
{
    return inner_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                              : (inner_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// bf16 tensor of rank 3: dims innermost first (elements), strides of dims 1
// and 2 in bytes, box in elements.  Out-of-range elements read as zero.
inline bool make_tmap_3d(CUtensorMap *out, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw)
{
    static std::mutex mu;
    static TmapKey keys[64];
    static CUtensorMap maps[64];
    static int used = 0, next = 0;
    TmapKey k;
    memset(&k, 0, sizeof k);
    k.ptr = ptr;
    k.dims[0] = d0; k.dims[1] = d1; k.dims[2] = d2;
    k.strides[0] = s1; k.strides[1] = s2;
    k.box[0] = b0; k.box[1] = b1; k.box[2] = b2;
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
    cuuint64_t gdim[3] = {d0, d1, d2};
    cuuint64_t gstr[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap m;
    if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), gdim, gstr, box, estr,
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

}  // namespace mla
