// append_proj.cuh -- the append projection of new tokens into the paged
// latent cache in one launch (sm_100a):
//   c^KV_t = W^DKV h_t,  k^R_t = RoPE(W^KR h_t, pos_t),  row [c^KV | k^R] -> slot
// (DeepSeek-V2 paper review, section 2: c^KV = W^DKV h; DeepSeek-V3 report
// summary, Method 1: k^R = RoPE(W^KR h), only c^KV and k^R are cached).
//
// Shape of the work: few tokens (M = T, one per sequence and query), a long
// K (d_model = 2048..5120) and N = 576 output columns.  Reading the 5.9 MB of
// weights fast needs many SMs, so K is split: CTA (n, m, z) computes output
// columns [64n, 64n+64) (n = 8: the 64 RoPE columns, from W^KR) of tokens
// [128m, 128m+128) over the K slice [z Ks, (z+1) Ks), Ks = d_model / 8.  The
// 8 K slices of a tile form a cluster.  Each CTA streams its slice of h and W
// through a 6-stage TMA ring into an M=128, N=64 tcgen05 accumulator, then
// sends row r of its fp32 partial to CTA r / 16 of the cluster (distributed
// shared memory), which sums the 8 partials of its 16 rows in slice order
// (the result does not depend on timing), turns the RoPE pairs and writes
// the bf16 row to the token's page slot.  No scratch outside shared memory;
// no TMA load uses cluster multicast.
#pragma once

#include "k_simple.cuh"
#include "sm100.cuh"

namespace mla {

constexpr int kApSlices = 8;                      // K slices = cluster size
constexpr int kApStages = 6;
constexpr int kApThreads = 192;
constexpr int kApA = 128 * 64 * 2;                // h chunk: 128 tokens x 64 (16 KB)
constexpr int kApB = 64 * 64 * 2;                 // W chunk: 64 outputs x 64 (8 KB)
constexpr int kApStage = kApA + kApB;
constexpr int kApOffRed = kApStages * kApStage;                  // 147,456
constexpr int kApRed = kApSlices * 16 * 64 * 4;                  // 32 KB: [slice][16 rows][64] fp32
constexpr int kApOffBar = kApOffRed + kApRed;
constexpr int kApSmem = kApOffBar + 256 + 1024;

struct AppendArgs {
    bf16 *cache;
    const int32_t *seq_idx, *pos, *block_table;
    int T, K, num_seqs, max_blocks, num_blocks;
    RopeTable rope;
    uint32_t *err;
    unsigned long long limit_ns;
};

namespace ap {

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

}  // namespace ap

__global__ void __cluster_dims__(1, 1, kApSlices) __launch_bounds__(kApThreads, 1)
append_proj_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_dkv,
                   const __grid_constant__ CUtensorMap map_kr, const AppendArgs a)
{
    extern __shared__ uint8_t ap_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(ap_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kApOffBar);
    uint64_t *empty = full + kApStages;
    uint64_t *done = empty + kApStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *red = reinterpret_cast<float *>(smem + kApOffRed);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x, m0 = blockIdx.y * 128;
    const int z = (int)ap::cluster_rank();
    const int nk = a.K / kApSlices / 64;            // 64-wide chunks of this CTA's K slice
    const int k0 = z * nk * 64;
    const CUtensorMap *mapB = n < 8 ? &map_dkv : &map_kr;
    const int nrow0 = n < 8 ? 64 * n : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kApStages; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        sm100::mbar_init(done, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&map_h);
        sm100::prefetch_tensormap(mapB);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 64);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    // every CTA of the cluster is running before any partial row is sent to it
    ap::cluster_sync();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long drain = a.limit_ns > 200000000ull ? a.limit_ns : 200000000ull;

    if (warp == 0) {
        if (sm100::elect_one()) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kApStages;
                if (kb >= kApStages &&
                    !sm100::mbar_wait(&empty[s], ((kb / kApStages) - 1) & 1, abort_flag, a.err, a.limit_ns))
                    break;
                issued = kb + 1;
                uint8_t *dst = smem + s * kApStage;
                sm100::mbar_arrive_expect_tx(&full[s], kApStage);
                sm100::tma_load_3d(&map_h, &full[s], dst, k0 + 64 * kb, m0, 0);
                sm100::tma_load_3d(mapB, &full[s], dst + kApA, k0 + 64 * kb, nrow0, 0);
            }
            if (*abort_flag) {
                volatile int no_abort = 0;
                for (int kb = issued - kApStages < 0 ? 0 : issued - kApStages; kb < issued; ++kb)
                    sm100::mbar_wait(&full[kb % kApStages], (kb / kApStages) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 1) {
        if (sm100::elect_one()) {
            const uint32_t idesc = sm100::idesc_bf16(128, 64, 0, 0);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % kApStages;
                ok = sm100::mbar_wait(&full[s], (kb / kApStages) & 1, abort_flag, a.err, a.limit_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                const uint32_t sa = sm100::smem_u32(smem + s * kApStage);
                const uint64_t ad = sm100::desc_kmajor(sa, 128, sm100::kSw128);
                const uint64_t bd = sm100::desc_kmajor(sa + kApA, 128, sm100::kSw128);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    sm100::umma_ss(tmem, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 32) >> 4), idesc,
                                   (kb | kk) != 0);
                sm100::umma_commit(&empty[s]);
            }
            sm100::umma_commit(done);
        }
    } else {
        // epilogue, part 1: warps 2..5 own TMEM lane quarters 2,3,0,1 (thread =
        // accumulator row r); row r goes to slot z of CTA r / 16's buffer
        const int q = warp & 3, r = 32 * q + lane;
        const bool ok = sm100::warp_wait(done, 0, abort_flag, a.err, a.limit_ns);
        sm100::tc_fence_after();
        uint32_t v[64];
        if (ok) {
#pragma unroll
            for (int c = 0; c < 64; c += 16) sm100::tmem_ld16(sm100::tmem_addr(tmem, 32 * q, c), v + c);
            sm100::tmem_wait_ld();
        } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) v[c] = 0u;
        }
        const uint32_t dst = ap::peer_addr(sm100::smem_u32(red + (z * 16 + (r & 15)) * 64), r >> 4);
#pragma unroll
        for (int c = 0; c < 64; c += 4)
            asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 4 * c), "r"(v[c]),
                         "r"(v[c + 1]), "r"(v[c + 2]), "r"(v[c + 3])
                         : "memory");
    }
    sm100::tc_fence_before();
    // every partial row has landed in its owner's buffer
    ap::cluster_sync();
    if (warp >= 2) {
        // epilogue, part 2: this CTA's 16 rows (tokens m0 + 16z + i), 8 columns
        // per thread, the 8 slices summed in slice order
        const int t = threadIdx.x - 64;               // 0..127
        const int i = t >> 3, c8 = (t & 7) * 8;
        const int m = m0 + 16 * z + i;
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.f;
        for (int sl = 0; sl < kApSlices; ++sl) {
            const float4 *p = reinterpret_cast<const float4 *>(red + (sl * 16 + i) * 64 + c8);
            const float4 x0 = p[0], x1 = p[1];
            o[0] += x0.x; o[1] += x0.y; o[2] += x0.z; o[3] += x0.w;
            o[4] += x1.x; o[5] += x1.y; o[6] += x1.z; o[7] += x1.w;
        }
        if (m < a.T && !*abort_flag) {
            const int p = a.pos[m];
            const long long slot = cache_slot(a.block_table, a.num_seqs, a.max_blocks, a.num_blocks, a.seq_idx[m],
                                              p, (n == 0 && c8 == 0) ? a.err : nullptr);
            if (slot >= 0) {
                if (n == 8) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float y0, y1;
                        rope_turn(o[2 * e], o[2 * e + 1], p, a.rope.theta[c8 / 2 + e], &y0, &y1);
                        o[2 * e] = y0;
                        o[2 * e + 1] = y1;
                    }
                }
                bf16x8 w;
#pragma unroll
                for (int e = 0; e < 4; ++e) w.v[e] = __floats2bfloat162_rn(o[2 * e], o[2 * e + 1]);
                *reinterpret_cast<bf16x8 *>(a.cache + slot * kRow + 64 * n + c8) = w;
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {  // every issued MMA has retired before TMEM is freed
            volatile int no_abort = 0;
            sm100::mbar_wait(done, 0, &no_abort, a.err, drain);
        }
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 64);
    }
}

}  // namespace mla
