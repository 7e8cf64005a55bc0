// common.cuh -- shared device helpers of the MLA decode library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

// Kernels launched by the library in this process (see mla_kernel_launches).
extern unsigned long long g_launches;
inline void count_launch(unsigned n = 1) { __atomic_fetch_add(&g_launches, n, __ATOMIC_RELAXED); }

typedef __nv_bfloat16 bf16;

constexpr int kDc = 512;      // latent width d_c
constexpr int kDr = 64;       // RoPE width d_r
constexpr int kDh = 128;      // per-head content width d_h
constexpr int kRow = kDc + kDr;  // 576 values per cached token
constexpr int kBlock = 64;    // tokens per cache block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bits)
{
    if (err) atomicOr(err, bits);
}

__device__ __forceinline__ float bf2f(bf16 v) { return __bfloat162float(v); }

// The frequency of each RoPE pair k = (x[2k], x[2k+1]), k < d_r / 2: base^(-2k/d_r)
// for plain RoPE, or its YaRN interpolation (computed on the host per call).
struct RopeTable {
    double theta[kDr / 2];
};

// RoPE of one pair (x0, x1) at position pos: turn by pos * theta.  The angle is
// formed in double precision: at positions up to 2^17 an fp32 angle would be
// off by ~1e-2 rad.
__device__ __forceinline__ void rope_turn(float x0, float x1, int pos, double theta, float *y0, float *y1)
{
    const double ang = (double)pos * theta;
    double sn, cs;
    sincos(ang, &sn, &cs);
    *y0 = (float)((double)x0 * cs - (double)x1 * sn);
    *y1 = (float)((double)x0 * sn + (double)x1 * cs);
}

// RoPE pair k of every head of token tok: one angle per (token, pair), taken
// and turned in double precision (the rotate of rope_turn), applied to the H
// heads' rows q_rope[tok][h] (64 bf16 each) and written to dst at row
// (tok * H + h) * dst_stride + dst_off; copied unturned when q_pos is null.
// A warp of consecutive k covers one token's 32 pairs: coalesced per head.
__device__ __forceinline__ void rope_heads(const bf16 *__restrict__ q_rope, const int32_t *__restrict__ q_pos,
                                           long long tok, int k, int H, const RopeTable &rope, bf16 *__restrict__ dst,
                                           int dst_stride, int dst_off)
{
    double sn = 0.0, cs = 1.0;
    if (q_pos) sincos((double)q_pos[tok] * rope.theta[k], &sn, &cs);
    for (int h = 0; h < H; ++h) {
        const long long row = tok * H + h;
        const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162 *>(q_rope + row * kDr)[k];
        __nv_bfloat162 y = x;
        if (q_pos) {
            const double x0 = __low2float(x), x1 = __high2float(x);
            y = __floats2bfloat162_rn((float)(x0 * cs - x1 * sn), (float)(x0 * sn + x1 * cs));
        }
        reinterpret_cast<__nv_bfloat162 *>(dst + row * dst_stride + dst_off)[k] = y;
    }
}

// Root mean square normalisation factor of a latent row, from the sum of its
// squares: 1 / sqrt(ss / d_c + eps).
__device__ __forceinline__ float rms_inv(float ss, float eps)
{
    return 1.0f / sqrtf(ss / (float)kDc + eps);
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 16-byte vector of 8 bf16
struct __align__(16) bf16x8 {
    __nv_bfloat162 v[4];
};

}  // namespace mla
