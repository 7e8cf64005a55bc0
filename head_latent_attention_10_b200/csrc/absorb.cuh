// absorb.cuh -- query absorption in one launch (sm_100a):
//   q_abs[t][i][0:512]   = (U^K_i)^T q^C_{t,i}          (fp32 accumulation -> bf16)
//   q_abs[t][i][512:576] = RoPE(q^R_{t,i}, q_pos[t])   (copied if q_pos is null)
// (DeepSeek-V2 paper review, section 2: (q^C)^T U^K c = ((U^K)^T q^C)^T c;
// section 3: a per-head RoPE query of 64 dims).
//
// CTA (i, m, p): head i, tokens [128m, 128m+128), latent columns [256p,
// 256p+256) and RoPE pairs [16p, 16p+16).  Per head the product is
// [T x 128] . [128 x 512]; two CTAs share it, so that each loads 96 KB and
// two fit on an SM: one CTA's loads then overlap another's epilogue, and the
// 256 CTAs of a 128-head batch run in one wave.  Warp 0 loads the token tile
// of q^C (two 64-column chunks) and the part's columns of U^K_i (MN-major:
// for each of the two 64-row K chunks, four 64-column N chunks) with TMA in
// one go; warp 1 issues 8 tcgen05 MMAs (M=128, N=256, K=16) into one
// accumulator; warps 2-9 read it back, two warps per TMEM lane quarter
// (thread = token row, half of the 256 columns each, and half of the part's
// RoPE pairs) into a swizzled staging tile, which one thread stores with TMA;
// the RoPE pairs leave with plain 16-byte stores (32 bytes per row and
// thread).  No TMA load uses cluster multicast.
#pragma once

#include "dec_common.cuh"

namespace mla {

constexpr int kAbThreads = 320;
constexpr int kAbParts = 2;                       // CTAs per (head, token tile)
constexpr int kAbA = 128 * 64 * 2;                // one q^C chunk: 128 tokens x 64 (16 KB)
constexpr int kAbBChunk = 64 * 64 * 2;            // one U^K box: 64 K rows x 64 N (8 KB)
constexpr int kAbB = 4 * kAbBChunk;               // one K chunk of the part's U^K_i columns: 64 x 256 (32 KB)
constexpr int kAbOffB = 2 * kAbA;                 // 32 KB
constexpr int kAbOffBar = kAbOffB + 2 * kAbB;     // 98,304
constexpr int kAbStageChunk = 128 * 128;          // one 64-column chunk of the output tile (16 KB)
constexpr int kAbSmem = kAbOffBar + 512 + 1024;   // barriers, the RoPE table (256 B), alignment slack

__global__ void __launch_bounds__(kAbThreads, 2)
absorb_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_uk,
              const __grid_constant__ CUtensorMap map_out,
              const bf16 *__restrict__ q_rope, const int32_t *__restrict__ q_pos, int T, int H,
              bf16 *__restrict__ q_abs, const RopeTable rope, uint32_t *err, unsigned long long limit_ns)
{
    extern __shared__ uint8_t ab_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(ab_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kAbOffBar);
    uint64_t *done = full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    double *theta = reinterpret_cast<double *>(smem + kAbOffBar + 64);   // [32] RoPE frequencies

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int head = blockIdx.x, m0 = blockIdx.y * 128, part = blockIdx.z;

    if (threadIdx.x == 0) {
        sm100::mbar_init(full, 1);
        sm100::mbar_init(done, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&map_q);
        sm100::prefetch_tensormap(&map_uk);
    }
    if (warp == 9)  // the frequency of RoPE pair k = lane
        theta[lane] = rope.theta[lane];
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 256);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (sm100::elect_one()) {
            sm100::mbar_arrive_expect_tx(full, 2 * kAbA + 2 * kAbB);
            for (int kc = 0; kc < 2; ++kc) {
                sm100::tma_load_3d(&map_q, full, smem + kc * kAbA, 64 * kc, m0, head);
                for (int j = 0; j < 4; ++j)
                    sm100::tma_load_3d(&map_uk, full, smem + kAbOffB + kc * kAbB + j * kAbBChunk, 256 * part + 64 * j,
                                       64 * kc, head);
            }
        }
    } else if (warp == 1) {
        if (sm100::elect_one()) {
            if (sm100::mbar_wait(full, 0, abort_flag, err, limit_ns)) {
                sm100::tc_fence_after();
                const uint32_t idesc = sm100::idesc_bf16(128, 256, 0, 1);
#pragma unroll
                for (int kc = 0; kc < 2; ++kc) {
                    const uint64_t ad = sm100::desc_kmajor(sm100::smem_u32(smem + kc * kAbA), 128, sm100::kSw128);
                    const uint64_t bd = sm100::desc_mnmajor_sw128(sm100::smem_u32(smem + kAbOffB + kc * kAbB), kAbBChunk);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        sm100::umma_ss(tmem, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 16 * 128) >> 4), idesc,
                                       (kc | kk) != 0);
                }
            }
            sm100::umma_commit(done);
        }
    } else {
        // epilogue: warp w (2..9) reads TMEM lane quarter w % 4 (thread = token
        // row r), columns [128 h, 128 h + 128) with h = (w - 2) / 4, and writes
        // its bf16 values into a staging copy of the part's output tile in the
        // (now free) input buffers: four 64-column chunks of [128 rows][128 B]
        // with 128-byte swizzle (16-byte unit u of row r at u ^ (r & 7)).  One
        // thread then stores the chunks with TMA (rows past T are not
        // written), so the global writes are whole lines instead of one
        // 16-byte piece of 32 different rows per warp instruction.
        const int qd = warp & 3, h = (warp - 2) >> 2;
        const int r = 32 * qd + lane, t = m0 + r;
        const bool ok = sm100::warp_wait(done, 0, abort_flag, err, limit_ns);
        sm100::tc_fence_after();
        auto stage_unit = [&](int chunk, int u, uint4 v) {
            *reinterpret_cast<uint4 *>(smem + chunk * kAbStageChunk + r * 128 + ((u ^ (r & 7)) << 4)) = v;
        };
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            uint32_t v[64];
            if (ok) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    sm100::tmem_ld16(sm100::tmem_addr(tmem + 128 * h, 32 * qd, 64 * c + 16 * q), v + 16 * q);
                sm100::tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] = 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                stage_unit(2 * h + c, u,
                           make_uint4(pack_bf162(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                                      pack_bf162(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                                      pack_bf162(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                                      pack_bf162(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]))));
        }
        // RoPE pairs [16 part + 8 h, 16 part + 8 h + 8) of the row's query: the
        // angle p*theta_k is formed and reduced to [-pi, pi] in double
        // precision (at positions up to 2^17 an fp32 product would be off by
        // ~1e-2 rad), then its sine and cosine are taken in fp32
        if (ok && t < T) {
            uint32_t o[8];
            const int k0 = 16 * part + 8 * h;
            const __nv_bfloat162 *src = reinterpret_cast<const __nv_bfloat162 *>(q_rope + ((long long)t * H + head) * kDr);
            const double p = q_pos ? (double)q_pos[t] : 0.0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k = k0 + e;
                const float2 x = __bfloat1622float2(src[k]);
                if (q_pos) {
                    const double ang = p * theta[k];
                    const double red = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
                    float sn, cs;
                    sincosf((float)red, &sn, &cs);
                    o[e] = pack_bf162(x.x * cs - x.y * sn, x.x * sn + x.y * cs);
                } else {
                    o[e] = pack_bf162(x.x, x.y);
                }
            }
            uint4 *dst = reinterpret_cast<uint4 *>(q_abs + ((long long)t * H + head) * kRow + kDc + 2 * k0);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 256;" ::: "memory");   // the 8 epilogue warps
        if (warp == 2 && lane == 0) {
            for (int j = 0; j < 4; ++j)
                sm100::tma_store_3d(&map_out, smem + j * kAbStageChunk, 256 * part + 64 * j, head, m0);
            sm100::tma_store_commit();
            sm100::tma_store_wait_read();
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {
            volatile int no_abort = 0;
            sm100::mbar_wait(done, 0, &no_abort, err, limit_ns);
        }
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 256);
    }
}

}  // namespace mla
