// tc_decode.cuh -- absorbed-MLA decode on tcgen05 tensor cores (sm_100a).
//
// What it computes (DeepSeek-V2 paper review, sections 2-3): for every query
// row and head i, softmax_j(scale * q_abs_i . row_j) weighted sum of the
// latents c^KV_j, where row_j = [c^KV_j | k^R_j] is the 576-value cache row
// and q_abs_i = [(U^K_i)^T q^C_i | q^R_i].  U^V is applied later.
//
// Heads are the MMA M dimension (128 rows; fewer heads leave rows zero), so
// one 64-token cache tile staged in shared memory feeds every head.  The fp32
// accumulator O = sum_j p_ij c_j for 128 heads x 512 latent columns would fill
// all 512 TMEM columns of an SM, so a 2-CTA cluster shares each tile:
//   CTA r owns latent columns [256r, 256r+256) and RoPE columns
//   [512+32r, 512+32r+32): it loads that 288-column slice of every tile,
//   computes the partial logits over it (S_r = Q_r C_r^T, M=128 N=64 K=288),
//   and keeps O_r (M=128 N=256) in its own TMEM.
//   The two CTAs swap their partial logits through distributed shared memory
//   (scaled, fp16, 16 KB per tile each way), so both hold the full logits and
//   take identical softmax decisions; no MMA work is repeated.
// P (bf16) is written from registers into TMEM and the P.C MMA reads it as
// the A operand; C is the same shared-memory tile, read MN-major.
//
// Roles (192 threads per CTA): warp 0 issues TMA loads (Q slice once per
// row, cache slices into a 3-stage ring), warp 1 issues the MMAs and zeroes
// the unused rows of a ragged last tile, warps 2-5 (one thread per head row =
// TMEM lane) run the exchange, the online softmax (log2 domain, lazy
// rescale: O and l are rescaled only when the running max grows by more than
// 8, i.e. a factor 256) and the epilogue.
//
// Work split: the (row, tile) list of the whole batch is cut into equal
// contiguous ranges, one per cluster (persistent).  A row that a range covers
// completely is normalized and written straight to the output; the pieces of
// a row cut by range ends are written as normalized fp32 partials with their
// log2-sum-exp and merged by dec_combine_kernel.
//
// Every wait is bounded (see sm100::mbar_wait); a wait that gives up sets
// MLA_DEVERR_TIMEOUT, the CTA unwinds, waits for its own copies in flight,
// meets its peer at the final cluster barrier and frees its TMEM.
#pragma once

#include "sm100.cuh"

namespace mla {

constexpr int kDecStages = 3;
constexpr int kDecThreads = 192;
constexpr int kQBytes = 4 * 16384 + 8192;    // Q slice: 4 x [128][64] SW128 + [128][32] SW64
constexpr int kStageBytes = 4 * 8192 + 4096; // cache slice: 4 x [64][64] SW128 + [64][32] SW64
constexpr int kRecvBytes = 128 * 64 * 2;     // peer partial logits, fp16 [128 rows][64 tokens]
constexpr int kOffStage = kQBytes;
constexpr int kOffRecv = kOffStage + kDecStages * kStageBytes;
constexpr int kOffBar = kOffRecv + 2 * kRecvBytes;
constexpr int kDecSmem = kOffBar + 512 + 1024;
constexpr uint32_t kTmO = 0, kTmS = 256, kTmP = 384;
constexpr int kMaxClusters = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct DecArgs {
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int32_t *plan;  // [0]=tiles per cluster, [1]=total tiles, [4..4+T] row tile starts
    bf16 *out;
    float *out_lse;
    float *part_o;        // [2*clusters][H][512] fp32
    float *part_lse2;     // [2*clusters][H]
    uint32_t *err;
    unsigned long long limit_ns;
    float scale_log2;
    int max_blocks, num_blocks, s, H, T;
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ int seq_len_clamped(const int32_t *seq_lens, int b, int max_blocks)
{
    int L = seq_lens[b];
    return L < 0 ? 0 : min(L, max_blocks * kBlock);
}

// Visible keys of query row r (query t of sequence b sees j <= L - s + t).
__device__ __forceinline__ int row_nvis(const DecArgs &a, int r)
{
    const int b = r / a.s, t = r % a.s;
    return seq_len_clamped(a.seq_lens, b, a.max_blocks) - a.s + t + 1;
}

// Largest r in [0, T] with row_start[r] <= x.
__device__ __forceinline__ int find_row(const int32_t *row_start, int T, int x)
{
    int lo = 0, hi = T;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (row_start[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Walks the segments (maximal runs of one row) of a cluster's tile range.
struct SegIter {
    const int32_t *rs;
    int T, pos, hi, r;
    int row, t0, t1, seg;  // current segment: tiles [t0, t1) of row `row`
    bool complete;
    __device__ void init(const int32_t *row_start, int T_, int lo, int hi_)
    {
        rs = row_start; T = T_; pos = lo; hi = hi_; seg = -1;
        r = find_row(rs, T, lo);
    }
    __device__ bool next()
    {
        while (pos < hi && r < T && rs[r + 1] <= pos) ++r;
        if (pos >= hi || r >= T) return false;
        const int a = rs[r], e = rs[r + 1];
        const int end = min(hi, e);
        row = r; t0 = pos - a; t1 = end - a;
        complete = (pos == a) && (end == e);
        pos = end; ++r; ++seg;
        return true;
    }
};

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v)
{
    __half2 h = *reinterpret_cast<__half2 *>(&v);
    return __half22float2(h);
}

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kDecThreads, 1)
tc_decode_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                 const __grid_constant__ CUtensorMap map_kv, const __grid_constant__ CUtensorMap map_kvr,
                 const DecArgs a)
{
    extern __shared__ uint8_t dec_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *kv_full = bars;               // [3]
    uint64_t *kv_empty = bars + 3;          // [3]
    uint64_t *q_full = bars + 6;
    uint64_t *q_empty = bars + 7;
    uint64_t *s_full = bars + 8;            // [2]
    uint64_t *s_free = bars + 10;           // [2]
    uint64_t *p_full = bars + 12;           // [2]
    uint64_t *o_done = bars + 14;           // [2]
    uint64_t *o_free = bars + 16;
    uint64_t *recv_full = bars + 17;        // [2]
    uint64_t *send_ok = bars + 19;          // [2]
    uint64_t *mma_done = bars + 21;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 22);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 23);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cr = sm100::cluster_ctarank();
    const uint32_t peer = cr ^ 1u;
    const int cl = blockIdx.x >> 1;
    const int32_t *row_start = a.plan + 4;
    const int q_per = a.plan[0], total = a.plan[1];
    const int lo = cl * q_per, hi = min(lo + q_per, total);
    if (lo >= hi) return;  // same decision in both CTAs of the cluster

    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) { sm100::mbar_init(&kv_full[i], 1); sm100::mbar_init(&kv_empty[i], 1); }
        sm100::mbar_init(q_full, 1);
        sm100::mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&s_full[i], 1);
            sm100::mbar_init(&s_free[i], 4);
            sm100::mbar_init(&p_full[i], 4);
            sm100::mbar_init(&o_done[i], 1);
            sm100::mbar_init(&recv_full[i], 1);
            sm100::mbar_init(&send_ok[i], 4);
        }
        sm100::mbar_init(o_free, 4);
        sm100::mbar_init(mma_done, 1);
        *abort_flag = 0;
        // the first two exchanges are expected before the peer may send
        sm100::mbar_arrive_expect_tx(&recv_full[0], kRecvBytes);
        sm100::mbar_arrive_expect_tx(&recv_full[1], kRecvBytes);
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&map_q);
        sm100::prefetch_tensormap(&map_qr);
        sm100::prefetch_tensormap(&map_kv);
        sm100::prefetch_tensormap(&map_kvr);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::cluster_sync();  // both CTAs' barriers exist before any remote access
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = a.limit_ns;
    const unsigned long long drain = lim > 200000000ull ? lim : 200000000ull;
    uint8_t *qs = smem;
    uint8_t *stages = smem + kOffStage;
    uint8_t *recv = smem + kOffRecv;

    SegIter it;
    it.init(row_start, a.T, lo, hi);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            int k = 0, issued_k = 0, q_issued = -1;
            bool ok = true;
            while (ok && it.next()) {
                if (it.seg > 0) ok = sm100::mbar_wait(q_empty, (it.seg - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                q_issued = it.seg;
                sm100::mbar_arrive_expect_tx(q_full, kQBytes);
                for (int j = 0; j < 4; ++j)
                    sm100::tma_load_3d(&map_q, q_full, qs + j * 16384, 256 * cr + 64 * j, 0, it.row);
                sm100::tma_load_3d(&map_qr, q_full, qs + 65536, 512 + 32 * cr, 0, it.row);
                const int b = it.row / a.s;
                for (int tt = it.t0; tt < it.t1 && ok; ++tt, ++k) {
                    const int st = k % kDecStages;
                    if (k >= kDecStages) ok = sm100::mbar_wait(&kv_empty[st], ((k / kDecStages) - 1) & 1, abort_flag, a.err, lim);
                    if (!ok) break;
                    int blk = a.block_table[(long long)b * a.max_blocks + tt];
                    if (blk < 0 || blk >= a.num_blocks) {
                        set_error(a.err, MLA_DEVERR_BLOCK_ID);
                        blk = 0;  // any valid block keeps the ring going; its tokens are masked
                    }
                    uint8_t *dst = stages + st * kStageBytes;
                    sm100::mbar_arrive_expect_tx(&kv_full[st], kStageBytes);
                    for (int j = 0; j < 4; ++j)
                        sm100::tma_load_3d(&map_kv, &kv_full[st], dst + j * 8192, 256 * cr + 64 * j, blk * kBlock, 0);
                    sm100::tma_load_3d(&map_kvr, &kv_full[st], dst + 32768, 512 + 32 * cr, blk * kBlock, 0);
                    issued_k = k + 1;
                }
            }
            if (*abort_flag) {  // wait for the copies still in flight
                volatile int no_abort = 0;
                for (int kk = issued_k - kDecStages < 0 ? 0 : issued_k - kDecStages; kk < issued_k; ++kk)
                    sm100::mbar_wait(&kv_full[kk % kDecStages], (kk / kDecStages) & 1, &no_abort, a.err, drain);
                if (q_issued >= 0) sm100::mbar_wait(q_full, q_issued & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        const uint32_t idesc_s = sm100::idesc_bf16(128, 64, 0, 0);
        const uint32_t idesc_o = sm100::idesc_bf16(128, 256, 0, 1);
        const uint32_t q_addr = sm100::smem_u32(qs);
        int k = 0;
        bool ok = true;
        auto issue_s = [&](int kk) -> bool {
            const int st = kk % kDecStages, sb = kk & 1;
            if (!sm100::mbar_wait(&kv_full[st], (kk / kDecStages) & 1, abort_flag, a.err, lim)) return false;
            if (kk >= 2 && !sm100::mbar_wait(&s_free[sb], ((kk >> 1) - 1) & 1, abort_flag, a.err, lim)) return false;
            sm100::tc_fence_after();
            if (lane == 0) {
                const uint32_t kv = sm100::smem_u32(stages + st * kStageBytes);
                const uint32_t d = tmem + kTmS + sb * 64;
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        sm100::umma_ss(d, sm100::desc_kmajor(q_addr + j * 16384 + kq * 32, 128, sm100::kSw128),
                                       sm100::desc_kmajor(kv + j * 8192 + kq * 32, 128, sm100::kSw128), idesc_s,
                                       (j | kq) != 0);
#pragma unroll
                for (int kq = 0; kq < 2; ++kq)
                    sm100::umma_ss(d, sm100::desc_kmajor(q_addr + 65536 + kq * 32, 64, sm100::kSw64),
                                   sm100::desc_kmajor(kv + 32768 + kq * 32, 64, sm100::kSw64), idesc_s, 1);
                sm100::umma_commit(&s_full[sb]);
            }
            __syncwarp();
            return true;
        };
        while (ok && it.next()) {
            ok = sm100::mbar_wait(q_full, it.seg & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            const int n = it.t1 - it.t0;
            const int nvis = row_nvis(a, it.row);
            const int b = it.row / a.s;
            ok = issue_s(k);
            for (int i = 0; i < n && ok; ++i) {
                const int kk = k + i;
                if (i + 1 < n) {
                    ok = issue_s(kk + 1);
                    if (!ok) break;
                } else {
                    if (lane == 0) sm100::umma_commit(q_empty);  // Q slice free once these S MMAs finish
                    __syncwarp();
                }
                ok = sm100::mbar_wait(&p_full[kk & 1], (kk >> 1) & 1, abort_flag, a.err, lim);
                if (ok && i == 0 && it.seg > 0) ok = sm100::mbar_wait(o_free, (it.seg - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                // a ragged or unreadable tile: zero the rows past the valid ones so 0 * garbage stays 0
                const int tt = it.t0 + i;
                int valid = min(kBlock, nvis - tt * kBlock);
                const int blk = a.block_table[(long long)b * a.max_blocks + tt];
                if (blk < 0 || blk >= a.num_blocks) valid = 0;
                uint8_t *kvp = stages + (kk % kDecStages) * kStageBytes;
                if (valid < kBlock) {
                    for (int e = lane; e < (kBlock - valid) * 4 * 8; e += 32) {
                        const int rr = valid + e / 32, j = (e >> 3) & 3, c16 = e & 7;
                        reinterpret_cast<uint4 *>(kvp + j * 8192 + rr * 128)[c16] = make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                sm100::tc_fence_after();
                if (lane == 0) {
                    const uint32_t kv = sm100::smem_u32(kvp);
                    const uint32_t pa = tmem + kTmP + (kk & 1) * 32;
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        sm100::umma_ts(tmem + kTmO, pa + kq * 8, sm100::desc_mnmajor_sw128(kv + kq * 2048, 8192),
                                       idesc_o, (i | kq) != 0);
                    sm100::umma_commit(&kv_empty[kk % kDecStages]);
                    sm100::umma_commit(&o_done[kk & 1]);
                }
                __syncwarp();
            }
            k += n;
        }
    } else {
        // -------------------------------------------------------- softmax
        const int qd = warp & 3;                 // TMEM lane quarter of this warp
        const int row_i = qd * 32 + lane;        // head row owned by this thread
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        const uint32_t peer_recv = sm100::mapa(sm100::smem_u32(recv), peer);
        const uint32_t peer_recv_full[2] = {sm100::mapa(sm100::smem_u32(&recv_full[0]), peer),
                                            sm100::mapa(sm100::smem_u32(&recv_full[1]), peer)};
        const uint32_t peer_send_ok[2] = {sm100::mapa(sm100::smem_u32(&send_ok[0]), peer),
                                          sm100::mapa(sm100::smem_u32(&send_ok[1]), peer)};
        const bool head_ok = row_i < a.H;
        int k = 0;
        bool ok = true;
        while (ok && it.next()) {
            const int n = it.t1 - it.t0;
            const int nvis = row_nvis(a, it.row);
            const int b = it.row / a.s;
            float m_run = -INFINITY, l_run = 0.f;
            for (int i = 0; i < n && ok; ++i) {
                const int kk = k + i, sb = kk & 1;
                const int tt = it.t0 + i;
                int valid = min(kBlock, nvis - tt * kBlock);
                const int blk = a.block_table[(long long)b * a.max_blocks + tt];
                if (blk < 0 || blk >= a.num_blocks) valid = 0;
                // own partial logits
                ok = sm100::mbar_wait(&s_full[sb], (kk >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                uint32_t sr[64];
#pragma unroll
                for (int c = 0; c < 4; ++c) sm100::tmem_ld16(lane_base + kTmS + sb * 64 + c * 16, sr + c * 16);
                sm100::tmem_wait_ld();
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&s_free[sb]);
                uint32_t hp[32];
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    hp[c] = pack_half2(__uint_as_float(sr[2 * c]) * a.scale_log2,
                                       __uint_as_float(sr[2 * c + 1]) * a.scale_log2);
                // send them to the peer once it has read the previous use of this buffer
                if (kk >= 2) ok = sm100::mbar_wait<true>(&send_ok[sb], ((kk >> 1) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                {
                    const uint32_t base = peer_recv + sb * kRecvBytes + row_i * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        sm100::st_async_v4(base + ((c ^ (row_i & 7)) << 4),
                                           make_uint4(hp[4 * c], hp[4 * c + 1], hp[4 * c + 2], hp[4 * c + 3]),
                                           peer_recv_full[sb]);
                }
                // and take the peer's
                ok = sm100::mbar_wait<true>(&recv_full[sb], (kk >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                float x[64];
                {
                    const uint8_t *src = recv + sb * kRecvBytes + row_i * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(src + ((c ^ (row_i & 7)) << 4));
                        const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 mine = unpack_half2(hp[4 * c + e]);
                            const float2 other = unpack_half2(pv[e]);
                            x[8 * c + 2 * e] = mine.x + other.x;
                            x[8 * c + 2 * e + 1] = mine.y + other.y;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive_remote(peer_send_ok[sb]);
                if (threadIdx.x == 64) sm100::mbar_arrive_expect_tx(&recv_full[sb], kRecvBytes);
                // online softmax over this tile (log2 domain)
                float mt = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    if (c >= valid) x[c] = -INFINITY;
                    mt = fmaxf(mt, x[c]);
                }
                const bool grow = (mt != -INFINITY) && (m_run == -INFINITY || mt > m_run + kRescaleThreshold);
                const float m_new = grow ? mt : m_run;
                const float corr = grow ? (m_run == -INFINITY ? 0.f : ex2(m_run - m_new)) : 1.f;
                const bool need_rescale = grow && m_run != -INFINITY;
                if (__any_sync(0xffffffffu, need_rescale) && i > 0) {
                    // O holds tiles up to kk-1: wait for them, then scale this row
                    const int kp = kk - 1;
                    ok = sm100::mbar_wait(&o_done[kp & 1], (kp >> 1) & 1, abort_flag, a.err, lim);
                    if (!ok) break;
                    sm100::tc_fence_after();
                    const float f = need_rescale ? corr : 1.f;
                    for (int c = 0; c < 256; c += 16) {
                        uint32_t ov[16];
                        sm100::tmem_ld16(lane_base + kTmO + c, ov);
                        sm100::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                        sm100::tmem_st16(lane_base + kTmO + c, ov);
                    }
                    sm100::tmem_wait_st();
                }
                l_run *= corr;
                m_run = m_new;
                uint32_t pw[32];
                float lsum = 0.f;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float p0 = (x[2 * c] == -INFINITY) ? 0.f : ex2(x[2 * c] - m_run);
                    const float p1 = (x[2 * c + 1] == -INFINITY) ? 0.f : ex2(x[2 * c + 1] - m_run);
                    pw[c] = pack_bf162(p0, p1);
                    const float2 back = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&pw[c]));
                    lsum += back.x + back.y;
                }
                l_run += lsum;
                // P buffer kk&1 was last read by the O MMA of tile kk-2
                if (kk >= 2) ok = sm100::mbar_wait(&o_done[kk & 1], ((kk >> 1) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                sm100::tmem_st16(lane_base + kTmP + (kk & 1) * 32, pw);
                sm100::tmem_st16(lane_base + kTmP + (kk & 1) * 32 + 16, pw + 16);
                sm100::tmem_wait_st();
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&p_full[kk & 1]);
            }
            if (!ok) break;
            // epilogue of the segment
            const int kl = k + n - 1;
            ok = sm100::mbar_wait(&o_done[kl & 1], (kl >> 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
            if (it.complete) {
                bf16 *dst = a.out + ((long long)it.row * a.H + row_i) * kDc + 256 * cr;
                for (int c = 0; c < 256; c += 16) {
                    uint32_t ov[16];
                    sm100::tmem_ld16(lane_base + kTmO + c, ov);
                    sm100::tmem_wait_ld();
                    if (head_ok) {
                        uint4 pk[2];
                        uint32_t *pp = reinterpret_cast<uint32_t *>(pk);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            pp[e] = pack_bf162(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
                        reinterpret_cast<uint4 *>(dst + c)[0] = pk[0];
                        reinterpret_cast<uint4 *>(dst + c)[1] = pk[1];
                    }
                }
                if (cr == 0 && head_ok && a.out_lse) a.out_lse[(long long)it.row * a.H + row_i] = lse2 * kLn2;
            } else {
                const long long slot = 2LL * cl + (it.seg == 0 ? 0 : 1);
                float *dst = a.part_o + (slot * a.H + row_i) * kDc + 256 * cr;
                for (int c = 0; c < 256; c += 16) {
                    uint32_t ov[16];
                    sm100::tmem_ld16(lane_base + kTmO + c, ov);
                    sm100::tmem_wait_ld();
                    if (head_ok) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d4[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                                __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
                    }
                }
                if (cr == 0 && head_ok) a.part_lse2[slot * a.H + row_i] = lse2;
            }
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(o_free);
            k += n;
        }
    }

    // ------------------------------------------------------------ teardown
    __syncwarp();
    if (*abort_flag) {
        // let DSMEM stores the peer already issued land before the cluster barrier
        const uint64_t t0 = sm100::globaltimer_ns();
        while (sm100::globaltimer_ns() - t0 < 20000ull) {}
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // every MMA this CTA issued retires before its TMEM is released
        if (lane == 0) sm100::umma_commit(mma_done);
        __syncwarp();
        volatile int no_abort = 0;
        sm100::mbar_wait(mma_done, 0, &no_abort, a.err, drain);
    }
    sm100::cluster_sync();
    if (warp == 1) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------- plan
// One CTA: tiles of every query row, their prefix sums, and the per-cluster
// quota.  plan[0] = tiles per cluster, plan[1] = total tiles,
// plan[4 + r] = first tile of row r (r = 0..T).
__global__ void __launch_bounds__(1024)
dec_plan_kernel(const int32_t *__restrict__ seq_lens, int B, int s, int max_blocks, int num_clusters,
                int32_t *__restrict__ plan, uint32_t *err)
{
    __shared__ int part[1024];
    const int T = B * s;
    const int per = (T + 1023) / 1024;
    const int r0 = threadIdx.x * per, r1 = min(T, r0 + per);
    int sum = 0;
    for (int r = r0; r < r1; ++r) {
        const int b = r / s, t = r % s;
        int L = seq_lens[b];
        if (L < 0 || L > max_blocks * kBlock) {
            if (t == 0) set_error(err, MLA_DEVERR_SEQ_LEN);
            L = L < 0 ? 0 : max_blocks * kBlock;
        }
        const int nvis = L - s + t + 1;
        if (nvis <= 0) set_error(err, MLA_DEVERR_SEQ_LEN);
        sum += nvis > 0 ? (nvis + kBlock - 1) / kBlock : 0;
    }
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = part[threadIdx.x] - sum;  // exclusive prefix
    for (int r = r0; r < r1; ++r) {
        plan[4 + r] = run;
        const int b = r / s, t = r % s;
        int L = seq_lens[b];
        L = L < 0 ? 0 : min(L, max_blocks * kBlock);
        const int nvis = L - s + t + 1;
        run += nvis > 0 ? (nvis + kBlock - 1) / kBlock : 0;
    }
    if (threadIdx.x == 1023) {
        const int total = part[1023];
        plan[4 + T] = total;
        plan[1] = total;
        plan[0] = total > 0 ? (total + num_clusters - 1) / num_clusters : 1;
    }
}

// ------------------------------------------------------------------ combine
// Rows cut by cluster ranges: merge their partials by log-sum-exp.  Rows a
// single cluster finished are already in place; rows with no visible key get
// a zero latent and lse = -inf.
__global__ void __launch_bounds__(128)
dec_combine_kernel(const int32_t *__restrict__ plan, const float *__restrict__ part_o,
                   const float *__restrict__ part_lse2, int H, bf16 *__restrict__ out,
                   float *__restrict__ out_lse)
{
    const int r = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int q = plan[0];
    const int a0 = plan[4 + r], a1 = plan[4 + r + 1];
    const long long orow = (long long)r * H + h;
    if (a1 <= a0) {
        reinterpret_cast<uint2 *>(out + orow * kDc)[tid] = make_uint2(0, 0);
        if (tid == 0 && out_lse) out_lse[orow] = -INFINITY;
        return;
    }
    const int c0 = a0 / q, c1 = (a1 - 1) / q;
    if (c0 == c1) return;
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c) {
        const int slot = 2 * c + ((c == c0 && a0 != c * q) ? 1 : 0);
        M = fmaxf(M, part_lse2[(long long)slot * H + h]);
    }
    float den = 0.f;
    float4 acc = make_float4(0, 0, 0, 0);
    for (int c = c0; c <= c1; ++c) {
        const int slot = 2 * c + ((c == c0 && a0 != c * q) ? 1 : 0);
        const float l2 = part_lse2[(long long)slot * H + h];
        const float w = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
        den += w;
        const float4 v = reinterpret_cast<const float4 *>(part_o + ((long long)slot * H + h) * kDc)[tid];
        acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 pk;
    pk.x = pack_bf162(acc.x * inv, acc.y * inv);
    pk.y = pack_bf162(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2 *>(out + orow * kDc)[tid] = pk;
    if (tid == 0 && out_lse) out_lse[orow] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
}

}  // namespace mla
