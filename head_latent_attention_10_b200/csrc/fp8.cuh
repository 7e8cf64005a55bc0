// fp8.cuh -- the FP8 (E4M3) latent cache: the cache writer and the
// conversions the FP8 decode uses.
//
// Layout (DeepSeek-V2 paper review, sections 4 and 9: the deployed cache keeps
// about 6 bits per element; DeepSeek-V3 report summary, the FP8 framework:
// E4M3 values with fine-grained scaling factors): a token's row
// [c^KV (512) | k^R (64), rotated] is stored as 576 E4M3 codes, and the two
// parts carry one fp32 scale each, scale = amax / 448 (an all-zero part gets
// scale 1), code = E4M3(x / scale) rounded to nearest-even and saturated at
// 448.  The value of a code is code * scale.
//   codes  [num_blocks][64][576] uint8    (576 B per row, 36,864 B per page)
//   scales [num_blocks][64][2]   fp32     (c^KV part, k^R part; 512 B per page)
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dec_common.cuh"
#include "k_simple.cuh"

namespace mla {

// E4M3 codes of x0 / scale and x1 / scale (fp32 quotients, nearest-even,
// saturated), x0 in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float x0, float x1, float scale)
{
    const float2 q = make_float2(__fdiv_rn(x0, scale), __fdiv_rn(x1, scale));
    return (uint16_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
}

// Two E4M3 codes (low byte first) -> their values as f16x2 (exact: every
// E4M3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)codes, __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// One warp per token: the token's bf16 row exactly as the bf16 cache writer
// forms it (copy or RMSNorm of the latent, RoPE of the key), then quantized
// per part.  Tokens whose slot is invalid are skipped with an error bit.
__global__ void __launch_bounds__(256)
append_latent_fp8_kernel(const bf16 *__restrict__ c_kv, const bf16 *__restrict__ k_rope, int T,
                         const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
                         const int32_t *__restrict__ block_table, int num_seqs, int max_blocks,
                         uint8_t *__restrict__ codes, float *__restrict__ scales, int num_blocks,
                         const RopeTable rope, const bf16 *__restrict__ norm_w, float eps, uint32_t *err)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int p = pos[warp];
    const long long slot = cache_slot(block_table, num_seqs, max_blocks, num_blocks, seq_idx[warp], p,
                                      lane == 0 ? err : nullptr);
    if (slot < 0) return;
    uint4 v0, v1;
    __nv_bfloat162 kr;
    latent_row_lanes(c_kv, k_rope, warp, p, lane, rope, norm_w, eps, v0, v1, kr);
    float x[16];
    const __nv_bfloat162 *h0 = reinterpret_cast<const __nv_bfloat162 *>(&v0);
    const __nv_bfloat162 *h1 = reinterpret_cast<const __nv_bfloat162 *>(&v1);
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(h0[i]), b = __bfloat1622float2(h1[i]);
        x[2 * i] = a.x; x[2 * i + 1] = a.y; x[8 + 2 * i] = b.x; x[8 + 2 * i + 1] = b.y;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(x[i]));
    const float2 r = __bfloat1622float2(kr);
    const float amc = warp_max(am), amr = warp_max(fmaxf(fabsf(r.x), fabsf(r.y)));
    const float sc = amc > 0.f ? __fdiv_rn(amc, 448.f) : 1.f;
    const float sr = amr > 0.f ? __fdiv_rn(amr, 448.f) : 1.f;
    uint8_t *row = codes + slot * kRow;
    uint16_t c[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = e4m3x2(x[2 * i], x[2 * i + 1], sc);
#pragma unroll
    for (int i = 0; i < 4; ++i) c[4 + i] = e4m3x2(x[8 + 2 * i], x[8 + 2 * i + 1], sc);
    reinterpret_cast<uint2 *>(row)[lane] = make_uint2(c[0] | ((uint32_t)c[1] << 16), c[2] | ((uint32_t)c[3] << 16));
    reinterpret_cast<uint2 *>(row + 256)[lane] =
        make_uint2(c[4] | ((uint32_t)c[5] << 16), c[6] | ((uint32_t)c[7] << 16));
    reinterpret_cast<uint16_t *>(row + kDc)[lane] = e4m3x2(r.x, r.y, sr);
    if (lane == 0) reinterpret_cast<float2 *>(scales)[slot] = make_float2(sc, sr);
}

}  // namespace mla
