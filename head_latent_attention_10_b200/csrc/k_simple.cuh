// k_simple.cuh -- CUDA-core kernels: the cache writer from latents and a
// straightforward split-KV decode with its log-sum-exp combine
// (MLA_FORCE_SIMPLE), a cross-check for the tensor-core decode.
#pragma once

#include "common.cuh"

namespace mla {

// ---------------------------------------------------------------- cache slot
// Physical row of logical position `pos` in sequence `seq`, or -1 (with an
// error bit) if the sequence index, position or block-table entry is invalid.
__device__ __forceinline__ long long cache_slot(const int32_t *block_table, int num_seqs,
                                                int max_blocks, int num_blocks, int seq, int pos,
                                                uint32_t *err)
{
    if (seq < 0 || seq >= num_seqs || pos < 0 || pos >= max_blocks * kBlock) {
        set_error(err, MLA_DEVERR_SEQ_LEN);
        return -1;
    }
    const int blk = block_table[(long long)seq * max_blocks + pos / kBlock];
    if (blk < 0 || blk >= num_blocks) {
        set_error(err, MLA_DEVERR_BLOCK_ID);
        return -1;
    }
    return (long long)blk * kBlock + (pos % kBlock);
}

// RMSNorm of a latent row held by the 32 lanes of a warp (lane l: values
// [8l, 8l+8) in v0 and [256+8l, 256+8l+8) in v1), in place: sum of squares in
// fp32, x * inv * w rounded to bf16.
__device__ __forceinline__ void rmsnorm_lanes(uint4 &v0, uint4 &v1, const bf16 *__restrict__ norm_w, float eps,
                                              int lane)
{
    float x[16];
    const __nv_bfloat162 *h0 = reinterpret_cast<const __nv_bfloat162 *>(&v0);
    const __nv_bfloat162 *h1 = reinterpret_cast<const __nv_bfloat162 *>(&v1);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(h0[i]), b = __bfloat1622float2(h1[i]);
        x[2 * i] = a.x; x[2 * i + 1] = a.y; x[8 + 2 * i] = b.x; x[8 + 2 * i + 1] = b.y;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) ss += x[i] * x[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rms_inv(ss, eps);
    const uint4 w0 = reinterpret_cast<const uint4 *>(norm_w)[lane];
    const uint4 w1 = reinterpret_cast<const uint4 *>(norm_w)[lane + 32];
    const __nv_bfloat162 *g0 = reinterpret_cast<const __nv_bfloat162 *>(&w0);
    const __nv_bfloat162 *g1 = reinterpret_cast<const __nv_bfloat162 *>(&w1);
    __nv_bfloat162 *o0 = reinterpret_cast<__nv_bfloat162 *>(&v0);
    __nv_bfloat162 *o1 = reinterpret_cast<__nv_bfloat162 *>(&v1);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(g0[i]), b = __bfloat1622float2(g1[i]);
        o0[i] = __floats2bfloat162_rn(x[2 * i] * inv * a.x, x[2 * i + 1] * inv * a.y);
        o1[i] = __floats2bfloat162_rn(x[8 + 2 * i] * inv * b.x, x[8 + 2 * i + 1] * inv * b.y);
    }
}

// The cache row of token t as the lanes of a warp hold it: lane l has latent
// values [8l, 8l+8) (v0) and [256+8l, 256+8l+8) (v1), RMS-normalised if
// norm_w is given, and RoPE pair l of the key turned to position p (kr).
__device__ __forceinline__ void latent_row_lanes(const bf16 *__restrict__ c_kv, const bf16 *__restrict__ k_rope,
                                                 int t, int p, int lane, const RopeTable &rope,
                                                 const bf16 *__restrict__ norm_w, float eps, uint4 &v0, uint4 &v1,
                                                 __nv_bfloat162 &kr)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(c_kv + (long long)t * kDc);
    v0 = src[lane];
    v1 = src[lane + 32];
    if (norm_w) rmsnorm_lanes(v0, v1, norm_w, eps, lane);
    const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162 *>(k_rope + (long long)t * kDr)[lane];
    float y0, y1;
    rope_turn(__low2float(x), __high2float(x), p, rope.theta[lane], &y0, &y1);
    kr = __floats2bfloat162_rn(y0, y1);
}

// ------------------------------------------------------- append from latents
// One warp per token: lanes copy the 1 KB latent (2 x 16 B each), optionally
// RMS-normalised with weight norm_w, and turn RoPE pair `lane` of the key.
__global__ void __launch_bounds__(256)
append_latent_kernel(const bf16 *__restrict__ c_kv, const bf16 *__restrict__ k_rope, int T,
                     const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
                     const int32_t *__restrict__ block_table, int num_seqs, int max_blocks,
                     bf16 *__restrict__ cache, int num_blocks, const RopeTable rope,
                     const bf16 *__restrict__ norm_w, float eps, uint32_t *err)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int p = pos[warp];
    const long long slot = cache_slot(block_table, num_seqs, max_blocks, num_blocks,
                                      seq_idx[warp], p, lane == 0 ? err : nullptr);
    if (slot < 0) return;
    uint4 v0, v1;
    __nv_bfloat162 kr;
    latent_row_lanes(c_kv, k_rope, warp, p, lane, rope, norm_w, eps, v0, v1, kr);
    bf16 *dst = cache + slot * kRow;
    reinterpret_cast<uint4 *>(dst)[lane] = v0;
    reinterpret_cast<uint4 *>(dst)[lane + 32] = v1;
    reinterpret_cast<__nv_bfloat162 *>(dst + kDc)[lane] = kr;
}

// RoPE of the query's RoPE part for every head, into rows of stride
// dst_stride at offset dst_off (the folded absorption writes q_abs[.][512:576]).
__global__ void __launch_bounds__(256)
rope_q_kernel(const bf16 *__restrict__ q_rope, const int32_t *__restrict__ q_pos, int T, int H, bf16 *__restrict__ dst,
              int dst_stride, int dst_off, const RopeTable rope)
{
    const long long units = (long long)T * (kDr / 2);
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < units; w += (long long)gridDim.x * blockDim.x)
        rope_heads(q_rope, q_pos, w / (kDr / 2), (int)(w % (kDr / 2)), H, rope, dst, dst_stride, dst_off);
}

// RMS normalisation, in place, of the latent part of the cache rows of T
// tokens (the projection path writes the rows first): one warp per token.
__global__ void __launch_bounds__(256)
latent_rmsnorm_kernel(int T, const int32_t *__restrict__ seq_idx, const int32_t *__restrict__ pos,
                      const int32_t *__restrict__ block_table, int num_seqs, int max_blocks,
                      bf16 *__restrict__ cache, int num_blocks, const bf16 *__restrict__ norm_w, float eps)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const long long slot = cache_slot(block_table, num_seqs, max_blocks, num_blocks, seq_idx[warp], pos[warp],
                                      nullptr);
    if (slot < 0) return;
    uint4 *row = reinterpret_cast<uint4 *>(cache + slot * kRow);
    uint4 v0 = row[lane], v1 = row[lane + 32];
    rmsnorm_lanes(v0, v1, norm_w, eps, lane);
    row[lane] = v0;
    row[lane + 32] = v1;
}

// ------------------------------------------------------------- simple decode
// One CTA per (query row, group of 8 heads, KV split of kSimpleSplit tokens).
// 32-token tiles are staged in shared memory; warp w scores head w against
// the tile (one token per lane) and keeps its online-softmax state; every
// thread then accumulates two latent columns of all 8 heads.  Each split
// writes a normalized partial latent and its log2-sum-exp.
constexpr int kSimpleHeads = 8;
constexpr int kSimpleTile = 32;
constexpr int kSimpleSplit = 1024;
constexpr int kSimpleRowPad = kRow + 8;  // 1168-byte stride: 16-B reads hit distinct banks
constexpr int kSimpleSmem = kSimpleHeads * kRow * sizeof(float) + kSimpleTile * kSimpleRowPad * sizeof(bf16);

__global__ void __launch_bounds__(256)
decode_simple_kernel(const bf16 *__restrict__ q_abs, const bf16 *__restrict__ cache,
                     int num_blocks, const int32_t *__restrict__ block_table, int max_blocks,
                     const int32_t *__restrict__ seq_lens, int s, int H, float scale_log2,
                     float *__restrict__ part_o, float *__restrict__ part_lse2, int nsplit_max,
                     uint32_t *err)
{
    extern __shared__ __align__(16) unsigned char simple_smem[];
    float(*qs)[kRow] = reinterpret_cast<float(*)[kRow]>(simple_smem);
    bf16(*tile)[kSimpleRowPad] =
        reinterpret_cast<bf16(*)[kSimpleRowPad]>(simple_smem + kSimpleHeads * kRow * sizeof(float));
    __shared__ float prob[kSimpleHeads][kSimpleTile];
    __shared__ float m_run[kSimpleHeads], l_run[kSimpleHeads], corr[kSimpleHeads];
    __shared__ int tok_ok[kSimpleTile];

    const int row = blockIdx.x, hg = blockIdx.y, split = blockIdx.z;
    const int b = row / s, t = row % s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int L = seq_lens[b];
    if (L > max_blocks * kBlock || L < 0) {
        if (tid == 0 && hg == 0 && split == 0) set_error(err, MLA_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : max_blocks * kBlock;
    }
    const int nvis = L - s + t + 1;
    const int j0 = split * kSimpleSplit;
    const int j1 = min(nvis, j0 + kSimpleSplit);
    if (j0 >= j1) return;  // the combine ignores splits past the end

    for (int e = tid; e < kSimpleHeads * kRow; e += 256) {
        const int h = e / kRow, c = e % kRow;
        qs[h][c] = bf2f(q_abs[((long long)row * H + hg * kSimpleHeads + h) * kRow + c]);
    }
    if (tid < kSimpleHeads) { m_run[tid] = -INFINITY; l_run[tid] = 0.f; }
    float acc[kSimpleHeads][2] = {};
    const int c0 = tid * 2;

    for (int jt = j0; jt < j1; jt += kSimpleTile) {
        __syncthreads();
        for (int e = tid; e < kSimpleTile * (kRow / 8); e += 256) {
            const int r = e / (kRow / 8), ch = e % (kRow / 8);
            const int j = jt + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            int ok = 0;
            if (j < j1) {
                const int blk = block_table[(long long)b * max_blocks + j / kBlock];
                if (blk >= 0 && blk < num_blocks) {
                    v = reinterpret_cast<const uint4 *>(cache + ((long long)blk * kBlock + j % kBlock) * kRow)[ch];
                    ok = 1;
                } else if (ch == 0) {
                    set_error(err, MLA_DEVERR_BLOCK_ID);
                }
            }
            reinterpret_cast<uint4 *>(&tile[r][0])[ch] = v;
            if (ch == 0) tok_ok[r] = ok;
        }
        __syncthreads();
        {   // scores and online softmax: warp = head, lane = token
            const int h = warp, r = lane;
            float sc = -INFINITY;
            if (tok_ok[r]) {
                float dot = 0.f;
                const uint4 *tr = reinterpret_cast<const uint4 *>(&tile[r][0]);
                const float4 *qh = reinterpret_cast<const float4 *>(&qs[h][0]);
#pragma unroll 4
                for (int ch = 0; ch < kRow / 8; ++ch) {
                    const uint4 u = tr[ch];
                    const __nv_bfloat162 *pv = reinterpret_cast<const __nv_bfloat162 *>(&u);
                    const float4 qa = qh[2 * ch], qb = qh[2 * ch + 1];
                    dot = fmaf(qa.x, __low2float(pv[0]), dot);
                    dot = fmaf(qa.y, __high2float(pv[0]), dot);
                    dot = fmaf(qa.z, __low2float(pv[1]), dot);
                    dot = fmaf(qa.w, __high2float(pv[1]), dot);
                    dot = fmaf(qb.x, __low2float(pv[2]), dot);
                    dot = fmaf(qb.y, __high2float(pv[2]), dot);
                    dot = fmaf(qb.z, __low2float(pv[3]), dot);
                    dot = fmaf(qb.w, __high2float(pv[3]), dot);
                }
                sc = dot * scale_log2;
            }
            float mx = sc;
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = m_run[h];
            const float m_new = fmaxf(m_old, mx);
            const float pj = (sc == -INFINITY) ? 0.f : exp2f(sc - m_new);
            float sum = pj;
#pragma unroll
            for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            prob[h][r] = pj;
            __syncwarp();
            if (lane == 0) {
                const float cf = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
                corr[h] = cf;
                l_run[h] = l_run[h] * cf + sum;
                m_run[h] = m_new;
            }
        }
        __syncthreads();
        if (c0 < kDc) {
#pragma unroll
            for (int h = 0; h < kSimpleHeads; ++h) { acc[h][0] *= corr[h]; acc[h][1] *= corr[h]; }
            const int nt = min(kSimpleTile, j1 - jt);
            for (int r = 0; r < nt; ++r) {
                const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&tile[r][c0]);
                const float v0 = __low2float(v), v1 = __high2float(v);
#pragma unroll
                for (int h = 0; h < kSimpleHeads; ++h) {
                    const float p = prob[h][r];
                    acc[h][0] = fmaf(p, v0, acc[h][0]);
                    acc[h][1] = fmaf(p, v1, acc[h][1]);
                }
            }
        }
    }
    __syncthreads();
    for (int h = 0; h < kSimpleHeads; ++h) {
        const long long pi = ((long long)row * nsplit_max + split) * H + hg * kSimpleHeads + h;
        const float l = l_run[h];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (c0 < kDc) {
            float2 o = make_float2(acc[h][0] * inv, acc[h][1] * inv);
            reinterpret_cast<float2 *>(part_o + pi * kDc)[tid] = o;
        }
        if (tid == 0) part_lse2[pi] = l > 0.f ? m_run[h] + log2f(l) : -INFINITY;
    }
}

// Log-sum-exp merge of the splits of one (row, head): weights 2^(lse2_s - LSE).
__global__ void __launch_bounds__(128)
combine_simple_kernel(const float *__restrict__ part_o, const float *__restrict__ part_lse2,
                      int nsplit_max, int split_tokens, const int32_t *__restrict__ seq_lens,
                      int max_blocks, int s, int H, bf16 *__restrict__ out, float *__restrict__ out_lse,
                      uint32_t *err)
{
    const int row = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int b = row / s, t = row % s;
    int L = seq_lens[b];
    L = L < 0 ? 0 : min(L, max_blocks * kBlock);
    const int nvis = L - s + t + 1;
    const long long orow = (long long)row * H + h;
    if (nvis <= 0) {
        if (tid == 0) {
            set_error(err, MLA_DEVERR_SEQ_LEN);
            if (out_lse) out_lse[orow] = -INFINITY;
        }
        reinterpret_cast<uint2 *>(out + orow * kDc)[tid] = make_uint2(0, 0);
        return;
    }
    const int ns = (nvis + split_tokens - 1) / split_tokens;
    float M = -INFINITY;
    for (int sp = 0; sp < ns; ++sp)
        M = fmaxf(M, part_lse2[((long long)row * nsplit_max + sp) * H + h]);
    float den = 0.f;
    float4 acc = make_float4(0, 0, 0, 0);
    for (int sp = 0; sp < ns; ++sp) {
        const long long pi = ((long long)row * nsplit_max + sp) * H + h;
        const float l2 = part_lse2[pi];
        const float w = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
        den += w;
        const float4 v = reinterpret_cast<const float4 *>(part_o + pi * kDc)[tid];
        acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t *>(&lo);
    pk.y = *reinterpret_cast<uint32_t *>(&hi);
    reinterpret_cast<uint2 *>(out + orow * kDc)[tid] = pk;
    if (tid == 0 && out_lse) out_lse[orow] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
}

}  // namespace mla
