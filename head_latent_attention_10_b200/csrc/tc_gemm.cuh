// tc_gemm.cuh -- tensor-core GEMM for the projections around the decode
// (query absorption, U^V / O up-projection, the append projection):
//   C[z][m][n] = sum_k A[z][m][k] * B[z][k][n],  bf16 in, fp32 accumulate.
//
// One CTA computes a 128 x BN tile.  Warp 0 streams 64-wide K slices of A
// and B into a 4-stage shared-memory ring with TMA (128-byte swizzle), warp 1
// issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator and frees
// each stage with tcgen05.commit, and warps 2-5 read the accumulator back
// with tcgen05.ld (one TMEM lane = one output row per thread) and hand 16
// columns at a time to the epilogue functor.
//
// A is K-major (rows of K contiguous) or, with kAmn, MN-major (A stored
// [K][M]); B is either K-major (B^T stored row-major, e.g. a weight [N][K])
// or MN-major (B stored [K][N]).
// Tensor maps are 3-D: A K-major {K, M, Z}, A MN-major {M, K, Z}, B K-major
// {K, N, Z}, B MN-major {N, K, Z}.
#pragma once

#include "sm100.cuh"

namespace mla {

constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;

template <int BN>
struct GemmSmem {
    static constexpr int A = 128 * 64 * 2;
    static constexpr int B = BN * 64 * 2;
    static constexpr int STAGE = A + B;
    static constexpr int BAR = kGemmStages * STAGE;
    static constexpr int BYTES = BAR + 256 + 1024;  // + barriers + alignment slack
    static constexpr int TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
};

template <int BN, bool kBmn, class Epi, bool kAmn = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const __grid_constant__ CUtensorMap mapC, int M, int N, int K, Epi epi, uint32_t *err,
               unsigned long long limit_ns)
{
    using S = GemmSmem<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S::BAR);
    uint64_t *empty = full + kGemmStages;
    uint64_t *done = empty + kGemmStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * 128, z = blockIdx.z;
    const int nk = K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            sm100::mbar_init(&full[s], 1);
            sm100::mbar_init(&empty[s], 1);
        }
        sm100::mbar_init(done, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&mapA);
        sm100::prefetch_tensormap(&mapB);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, S::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // launched with programmatic serialization: the set-up above overlaps the
    // end of the kernel before, whose outputs are read only from here on
    sm100::pdl_wait();

    const unsigned long long drain_ns = limit_ns > 200000000ull ? limit_ns : 200000000ull;
    if (warp == 0) {
        if (sm100::elect_one()) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kGemmStages;
                const uint32_t use = kb / kGemmStages;
                if (use > 0 && !sm100::mbar_wait(&empty[s], (use - 1) & 1, abort_flag, err, limit_ns)) break;
                issued = kb + 1;
                uint8_t *a = smem + s * S::STAGE;
                uint8_t *b = a + S::A;
                sm100::mbar_arrive_expect_tx(&full[s], S::STAGE);
                const int kx = kb * 64;
                if (kAmn) {
                    sm100::tma_load_3d(&mapA, &full[s], a, m0, kx, z);
                    sm100::tma_load_3d(&mapA, &full[s], a + 8192, m0 + 64, kx, z);
                } else {
                    sm100::tma_load_3d(&mapA, &full[s], a, kx, m0, z);
                }
                if (kBmn) {
#pragma unroll
                    for (int j = 0; j < BN / 64; ++j)
                        sm100::tma_load_3d(&mapB, &full[s], b + j * 8192, n0 + 64 * j, kx, z);
                } else {
                    sm100::tma_load_3d(&mapB, &full[s], b, kx, n0, z);
                }
            }
            if (*abort_flag) {
                // never leave a copy in flight into shared memory: wait for the
                // last load issued on every stage
                volatile int no_abort = 0;
                for (int kb = issued - kGemmStages < 0 ? 0 : issued - kGemmStages; kb < issued; ++kb)
                    sm100::mbar_wait(&full[kb % kGemmStages], (kb / kGemmStages) & 1, &no_abort, err, drain_ns);
            }
        }
    } else if (warp == 1) {
        if (sm100::elect_one()) {
            const uint32_t idesc = sm100::idesc_bf16(128, BN, kAmn ? 1 : 0, kBmn ? 1 : 0);
            bool ok = true;
            for (int kb = 0; kb < nk && ok; ++kb) {
                const int s = kb % kGemmStages;
                ok = sm100::mbar_wait(&full[s], (kb / kGemmStages) & 1, abort_flag, err, limit_ns);
                if (!ok) break;
                sm100::tc_fence_after();
                const uint32_t a = sm100::smem_u32(smem + s * S::STAGE);
                const uint32_t b = a + S::A;
                const uint64_t ad = kAmn ? sm100::desc_mnmajor_sw128(a, 8192) : sm100::desc_kmajor(a, 128, sm100::kSw128);
                const uint64_t bd = kBmn ? sm100::desc_mnmajor_sw128(b, 8192) : sm100::desc_kmajor(b, 128, sm100::kSw128);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    sm100::umma_ss(tmem, ad + (uint64_t)(((kAmn ? kk * 16 * 128 : kk * 32)) >> 4),
                                   bd + (uint64_t)(((kBmn ? kk * 16 * 128 : kk * 32)) >> 4), idesc, (kb | kk) != 0);
                sm100::umma_commit(&empty[s]);
            }
            sm100::umma_commit(done);
        }
    } else {
        // epilogue: warps 2..5 cover TMEM lane quarters 2,3,0,1
        const int q = warp & 3;
        const bool ok = sm100::warp_wait(done, 0, abort_flag, err, limit_ns);
        sm100::tc_fence_after();
        const int m = m0 + q * 32 + lane;
        if constexpr (Epi::kStaged) {
            // bf16 tile staged in the drained ring as 64-column chunks of
            // [128 rows][128 B] (128-byte swizzle), stored with TMA by one
            // thread: whole lines rather than 32 rows' pieces per instruction
            const int r = q * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                if (ok) {
                    sm100::tmem_ld16(sm100::tmem_addr(tmem, q * 32, c), v);
                    sm100::tmem_ld16(sm100::tmem_addr(tmem, q * 32, c + 16), v + 16);
                    sm100::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                }
                uint8_t *chunk = smem + (c / 64) * 16384;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int uu = ((c % 64) / 8) + u;
                    *reinterpret_cast<uint4 *>(chunk + r * 128 + ((uu ^ (r & 7)) << 4)) =
                        make_uint4(pack_bf162(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                                   pack_bf162(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                                   pack_bf162(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                                   pack_bf162(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, 128;" ::: "memory");   // the 4 epilogue warps
            if (warp == 2 && lane == 0) {
                for (int c = 0; c < BN; c += 64) {
                    // with split_n the flat column n is (n % split_n) of batch entry n / split_n
                    const int n = n0 + c;
                    if (epi.split_n > 0)
                        sm100::tma_store_3d(&mapC, smem + (c / 64) * 16384, n % epi.split_n, n / epi.split_n, m0);
                    else
                        sm100::tma_store_3d(&mapC, smem + (c / 64) * 16384, n, z, m0);
                }
                sm100::tma_store_commit();
                sm100::tma_store_wait_read();
            }
        } else if (ok) {
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                uint32_t r[16];
                sm100::tmem_ld16(sm100::tmem_addr(tmem, q * 32, c), r);
                sm100::tmem_wait_ld();
                if (m < M && n0 + c < N) epi(z, m, n0 + c, reinterpret_cast<const float *>(r));
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        if (*abort_flag) {  // every issued MMA has retired before TMEM is freed
            volatile int no_abort = 0;
            sm100::mbar_wait(done, 0, &no_abort, err, drain_ns);
        }
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, S::TMEM_COLS);
    }
}

// ------------------------------------------------------------- epilogues
// bf16 output stored with TMA from a staged tile through the kernel's output
// tensor map, which covers the output as {N, Z, M} (columns, batch entry,
// rows) with box {64, 1, 128}.  With split_n > 0 (Z = 1) the flat column n
// goes to column n % split_n of entry n / split_n: one GEMM over all heads
// writing a per-head output whose rows are interleaved with other data.
struct TcEpiTmaStore {
    static constexpr bool kStaged = true;
    int split_n = 0;
    __device__ void operator()(int, int, int, const float *) const {}
};

// 16 consecutive outputs -> bf16 at base + z*bs + m*rs + n (32-byte aligned).
struct TcEpiStore {
    static constexpr bool kStaged = false;
    bf16 *base;
    long long bs, rs;
    __device__ void operator()(int z, int m, int n, const float *v) const
    {
        uint4 pk[2];
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(pk);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        uint4 *p = reinterpret_cast<uint4 *>(base + z * bs + m * rs + n);
        p[0] = pk[0];
        p[1] = pk[1];
    }
};

// Append: token m's projected columns go to its cache slot; with `rope` the
// 16 columns are RoPE dims n..n+15 (8 pairs) and are turned first.
struct TcEpiAppend {
    static constexpr bool kStaged = false;
    bf16 *cache;
    const int32_t *seq_idx, *pos, *block_table;
    int num_seqs, max_blocks, num_blocks, col0;
    int rope;
    RopeTable tab;
    uint32_t *err;
    __device__ void operator()(int, int m, int n, const float *v) const
    {
        const int p = pos[m];
        const long long slot = cache_slot(block_table, num_seqs, max_blocks, num_blocks, seq_idx[m], p,
                                          n == 0 ? err : nullptr);
        if (slot < 0) return;
        float o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = v[i];
        if (rope) {
#pragma unroll
            for (int i = 0; i < 8; ++i) rope_turn(v[2 * i], v[2 * i + 1], p, tab.theta[n / 2 + i], &o[2 * i], &o[2 * i + 1]);
        }
        uint4 pk[2];
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(pk);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
        uint4 *dst = reinterpret_cast<uint4 *>(cache + slot * kRow + col0 + n);
        dst[0] = pk[0];
        dst[1] = pk[1];
    }
};

}  // namespace mla
