// tc_decode.cuh -- absorbed-MLA decode on tcgen05 tensor cores (sm_100a).
//
// What it computes (DeepSeek-V2 paper review, sections 2-3): for every query
// row (query token t of sequence b, head i), softmax_j(scale * q_abs . row_j)
// weighted sum of the latents c^KV_j, where row_j = [c^KV_j | k^R_j] is the
// 576-value cache row and q_abs = [(U^K_i)^T q^C | q^R].  U^V is applied later.
//
// Work unit: 64 "rows" of one sequence (its s*H (query, head) pairs, cut in
// groups of 64) against a 32-token tile of that sequence's cache.  The 64 rows
// are the MMA M dimension.  A 64-row accumulator occupies the first 16 lanes
// of each 32-lane TMEM quarter (row m at lane 32*(m/16) + m%16) across all N
// columns, so two of them interleave: O in lanes 0-15 of every quarter and S
// in lanes 16-31 (address lane offset 16):
//   S = Q C^T  : M=64, N=32 tokens, K=576   (2 buffers x 32 columns, upper lanes)
//   O += P C   : M=64, N=512 latent (2 x 256), K=32 tokens   (512 columns, lower lanes)
// and a whole group fits one CTA: no cross-CTA traffic.  The CTAs working on
// the other groups of the same sequence run at the same time on other SMs, so
// HBM delivers each cache tile once and L2 serves the repeats.
//
// Pipeline per CTA (192 threads): warp 0 streams the Q slice (per sequence)
// and 32-token cache tiles (4-stage ring) with TMA; warp 1 issues S(k+1)
// before O(k) and zeroes the unused rows of a ragged last tile; warps 2-5 (one
// warp owns 16 rows: lanes 16-31 hold a row's 32 logits each, lanes 0-15 the
// same rows' O) run the online softmax in the log2 domain with lazy
// rescaling (O and l are rescaled only when the running max grows by more
// than 8, a factor 256), write P (bf16) to shared memory for the P.C MMA, and
// write the output.
//
// Work split: the (sequence, tile) list of the batch is cut into equal
// contiguous ranges per group.  A sequence a range covers completely is
// normalized and written straight to the output; pieces of a sequence cut by
// range ends are written as normalized fp32 partials with their log2-sum-exp
// and merged by dec_combine_kernel.
//
// Every wait is bounded (see sm100::mbar_wait); a wait that gives up sets
// MLA_DEVERR_TIMEOUT, the CTA unwinds, waits for its own copies in flight and
// frees its TMEM.
#pragma once

#include "sm100.cuh"

namespace mla {

constexpr int kTN = 32;                       // tokens per tile
constexpr int kDecStages = 4;
constexpr int kDecThreads = 192;
constexpr int kGroupRows = 64;                // MMA M
constexpr int kChunkQ = kGroupRows * 128;     // one 64-column chunk of Q: 64 rows x 128 B (SW128)
constexpr int kChunkKV = kTN * 128;           // one 64-column chunk of a tile: 32 rows x 128 B
constexpr int kQBytes = 9 * kChunkQ;          // 73728
constexpr int kStageBytes = 9 * kChunkKV;     // 36864
constexpr int kPBytes = kGroupRows * kTN * 2; // 4096: P [64][32] bf16, K-major, 64-byte rows (SW64)
constexpr int kOffStage = kQBytes;
constexpr int kOffP = kOffStage + kDecStages * kStageBytes;
constexpr int kOffBar = kOffP + 2 * kPBytes;
constexpr int kOffRed = kOffBar + 512;
constexpr int kDecSmem = kOffRed + 1024;
constexpr uint32_t kTmO = 0;                   // O: lanes 0-15 of each quarter, columns [0, 512)
constexpr uint32_t kTmS = 16u << 16;           // S: lanes 16-31 of each quarter, 2 buffers x 32 columns
constexpr int kMaxRanges = 148;                // ranges per group (= CTAs / groups)
constexpr float kRescaleThreshold = 8.0f;     // log2 units

struct DecArgs {
    const bf16 *q_abs;    // [B*s][H][576]
    const int32_t *block_table;
    const int32_t *seq_lens;
    const int32_t *plan;  // [0]=tiles per range, [1]=total tiles, [2]=ranges, [4..4+B] sequence tile starts
    bf16 *out;
    float *out_lse;
    float *part_o;        // [2*ranges][s*H][512] fp32
    float *part_lse2;     // [2*ranges][s*H]
    uint32_t *err;
    unsigned long long limit_ns;
    float scale_log2;
    int max_blocks, num_blocks, s, H, B, groups;
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

// Largest r in [0, n] with start[r] <= x.
__device__ __forceinline__ int find_seq(const int32_t *start, int n, int x)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Walks a range of the (sequence, tile) list one tile at a time.
struct TileIter {
    const int32_t *rs;
    int n, pos, hi, r;
    int seq, t0, t1, seg, tt, k;
    bool complete, ok;
    __device__ bool next_seg()
    {
        while (pos < hi && r < n && rs[r + 1] <= pos) ++r;
        if (pos >= hi || r >= n) return false;
        const int a = rs[r], e = rs[r + 1];
        const int end = min(hi, e);
        seq = r; t0 = pos - a; t1 = end - a;
        complete = (pos == a) && (end == e);
        pos = end; ++r; ++seg;
        return true;
    }
    __device__ void init(const int32_t *start, int n_, int lo, int hi_)
    {
        rs = start; n = n_; pos = lo; hi = hi_; seg = -1; k = 0;
        r = find_seq(rs, n, lo);
        ok = next_seg();
        tt = t0;
    }
    __device__ bool first() const { return tt == t0; }
    __device__ bool last() const { return tt + 1 == t1; }
    __device__ void advance()
    {
        ++k;
        if (++tt >= t1) {
            ok = next_seg();
            tt = t0;
        }
    }
};

__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__global__ void __launch_bounds__(kDecThreads, 1)
tc_decode_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv,
                 const DecArgs a)
{
    extern __shared__ uint8_t dec_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint64_t *kv_full = bars;                   // [4] TMA -> MMA
    uint64_t *kv_empty = bars + 4;              // [4] MMA -> TMA
    uint64_t *q_full = bars + 8;                // TMA -> MMA
    uint64_t *q_empty = bars + 9;               // MMA -> TMA
    uint64_t *s_full = bars + 10;               // [2] MMA -> softmax
    uint64_t *s_free = bars + 12;               // [2] softmax -> MMA
    uint64_t *p_full = bars + 14;               // [2] softmax -> MMA
    uint64_t *o_done = bars + 16;               // [2] MMA -> softmax (O of tile k done, parity k&1)
    uint64_t *o_free = bars + 18;               // softmax -> MMA (epilogue read O)
    uint64_t *mma_done = bars + 19;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 26);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 27);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = blockIdx.x % a.groups, rng = blockIdx.x / a.groups;
    const int32_t *seq_start = a.plan + 4;
    const int q_per = a.plan[0], total = a.plan[1];
    const int lo = rng * q_per, hi = min(lo + q_per, total);
    if (lo >= hi) return;
    const int rows_per_seq = a.s * a.H;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecStages; ++i) { sm100::mbar_init(&kv_full[i], 1); sm100::mbar_init(&kv_empty[i], 1); }
        sm100::mbar_init(q_full, 1);
        sm100::mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&s_full[i], 1);
            sm100::mbar_init(&s_free[i], 4);
            sm100::mbar_init(&p_full[i], 4);
            sm100::mbar_init(&o_done[i], 1);
        }
        sm100::mbar_init(o_free, 4);
        sm100::mbar_init(mma_done, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&map_q);
        sm100::prefetch_tensormap(&map_kv);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = a.limit_ns;
    const unsigned long long drain = lim > 200000000ull ? lim : 200000000ull;
    uint8_t *qs = smem;
    uint8_t *stages = smem + kOffStage;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            TileIter it;
            it.init(seq_start, a.B, lo, hi);
            int issued_k = 0, q_issued = -1;
            bool ok = true;
            while (ok && it.ok) {
                const int k = it.k, st = k % kDecStages;
                if (k >= kDecStages) ok = sm100::mbar_wait(&kv_empty[st], ((k / kDecStages) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                const int pos0 = it.tt * kTN;
                int blk = a.block_table[(long long)it.seq * a.max_blocks + pos0 / kBlock];
                if (blk < 0 || blk >= a.num_blocks) {
                    // never read outside the cache: load block 0 instead; the
                    // sequence's output is then unspecified and the error bit says so
                    set_error(a.err, MLA_DEVERR_BLOCK_ID);
                    blk = 0;
                }
                uint8_t *dst = stages + st * kStageBytes;
                sm100::mbar_arrive_expect_tx(&kv_full[st], kStageBytes);
                for (int j = 0; j < 9; ++j)
                    sm100::tma_load_3d(&map_kv, &kv_full[st], dst + j * kChunkKV, 64 * j, blk * kBlock + pos0 % kBlock, 0);
                issued_k = k + 1;
                if (it.first()) {
                    // this sequence's Q slice replaces the previous one once its S MMAs retire
                    const int g = it.seg;
                    if (g > 0) ok = sm100::mbar_wait(q_empty, (g - 1) & 1, abort_flag, a.err, lim);
                    if (!ok) break;
                    q_issued = g;
                    sm100::mbar_arrive_expect_tx(q_full, kQBytes);
                    const int row0 = it.seq * rows_per_seq + group * kGroupRows;
                    for (int j = 0; j < 9; ++j) sm100::tma_load_3d(&map_q, q_full, qs + j * kChunkQ, 64 * j, row0, 0);
                }
                it.advance();
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
        const uint32_t idesc_s = sm100::idesc_bf16(kGroupRows, kTN, 0, 0);
        const uint32_t idesc_o = sm100::idesc_bf16(kGroupRows, 256, 0, 1);
        const uint32_t q_addr = sm100::smem_u32(qs);
        const uint32_t p_addr = sm100::smem_u32(smem + kOffP);
        auto issue_s = [&](int kk) -> bool {
            const int st = kk % kDecStages, sb = kk & 1;
            if (!sm100::warp_wait(&kv_full[st], (kk / kDecStages) & 1, abort_flag, a.err, lim)) return false;
            if (kk >= 2 && !sm100::warp_wait(&s_free[sb], ((kk >> 1) - 1) & 1, abort_flag, a.err, lim)) return false;
            sm100::tc_fence_after();
            if (lane == 0) {
                // base descriptors once; each K step only moves the start address
                // (the descriptor's low 14 bits hold address >> 4)
                const uint64_t qd = sm100::desc_kmajor(q_addr, 128, sm100::kSw128);
                const uint64_t kd = sm100::desc_kmajor(sm100::smem_u32(stages + st * kStageBytes), 128, sm100::kSw128);
                const uint32_t d = tmem + kTmS + sb * kTN;
                sm100::umma_ss(d, qd, kd, idesc_s, 0u);
#pragma unroll
                for (int kq = 1; kq < 4; ++kq)
                    sm100::umma_ss(d, qd + (uint64_t)((kq * 32) >> 4), kd + (uint64_t)((kq * 32) >> 4), idesc_s, 1u);
#pragma unroll
                for (int j = 1; j < 9; ++j)
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        sm100::umma_ss(d, qd + (uint64_t)((j * kChunkQ + kq * 32) >> 4),
                                       kd + (uint64_t)((j * kChunkKV + kq * 32) >> 4), idesc_s, 1u);
                sm100::umma_commit(&s_full[sb]);
            }
            __syncwarp();
            return true;
        };
        TileIter is, io;
        is.init(seq_start, a.B, lo, hi);
        io.init(seq_start, a.B, lo, hi);
        bool ok = sm100::warp_wait(q_full, 0, abort_flag, a.err, lim);
        if (ok) {
            ok = issue_s(0);
            is.advance();
        }
        int nseq = 0;
        while (ok && io.ok) {
            const int k = io.k;
            if (is.ok) {
                if (is.first()) {
                    // tile k+1 opens another sequence: swap the Q slice once this one's S MMAs retire
                    if (lane == 0) sm100::umma_commit(q_empty);
                    __syncwarp();
                    ok = sm100::warp_wait(q_full, is.seg & 1, abort_flag, a.err, lim);
                    if (!ok) break;
                    sm100::tc_fence_after();
                }
                ok = issue_s(is.k);
                if (!ok) break;
                is.advance();
            }
            ok = sm100::warp_wait(&p_full[k & 1], (k >> 1) & 1, abort_flag, a.err, lim);
            if (ok && io.first() && io.seg > 0) ok = sm100::warp_wait(o_free, (io.seg - 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            if (io.first()) nseq = seq_len_clamped(a.seq_lens, io.seq, a.max_blocks);
            // a ragged last tile: zero the rows past the sequence end so 0 * garbage stays 0
            const int valid = min(kTN, nseq - io.tt * kTN);
            uint8_t *kvp = stages + (k % kDecStages) * kStageBytes;
            if (valid < kTN) {
                for (int e = lane; e < (kTN - valid) * 8 * 8; e += 32) {
                    const int rr = valid + e / 64, j = (e >> 3) & 7, c16 = e & 7;
                    reinterpret_cast<uint4 *>(kvp + j * kChunkKV + rr * 128)[c16] = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            sm100::tc_fence_after();
            if (lane == 0) {
                const uint64_t pd = sm100::desc_kmajor(p_addr + (k & 1) * kPBytes, 64, sm100::kSw64);
                const uint64_t vd = sm100::desc_mnmajor_sw128(sm100::smem_u32(kvp), kChunkKV);
                const uint32_t acc0 = io.first() ? 0u : 1u;
#pragma unroll
                for (int kq = 0; kq < kTN / 16; ++kq)
#pragma unroll
                    for (int jh = 0; jh < 2; ++jh)
                        sm100::umma_ss(tmem + kTmO + 256 * jh, pd + (uint64_t)((kq * 32) >> 4),
                                       vd + (uint64_t)((4 * jh * kChunkKV + kq * 2048) >> 4), idesc_o,
                                       kq > 0 ? 1u : acc0);
                sm100::umma_commit(&kv_empty[k % kDecStages]);
                sm100::umma_commit(&o_done[k & 1]);
            }
            __syncwarp();
            io.advance();
        }
    } else {
        // -------------------------------------------------------- softmax
        // warp q (0..3) owns group rows [16q, 16q+16): lane 16+i holds row
        // 16q+i's logits (TMEM lane 32q+16+i), lane i its O row (lane 32q+i)
        const int qd = warp & 3;
        const bool srow = lane >= 16;
        const int r = 16 * qd + (lane & 15);
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        const uint32_t p_addr = sm100::smem_u32(smem + kOffP);
        const int grow_row = group * kGroupRows + r;  // index among the sequence's s*H rows
        const bool row_ok = grow_row < rows_per_seq;
        const int tq = row_ok ? grow_row / a.H : 0;   // query token of this row
        const int head = row_ok ? grow_row % a.H : 0;
        TileIter it;
        it.init(seq_start, a.B, lo, hi);
        float m_run = -INFINITY, l_run = 0.f;
        int nvis = 0;
        bool ok = true;
        while (ok && it.ok) {
            const int k = it.k, sb = k & 1;
            if (it.first()) {
                m_run = -INFINITY;
                l_run = 0.f;
                // query tq of a sequence of length L sees positions j <= L - s + tq
                nvis = seq_len_clamped(a.seq_lens, it.seq, a.max_blocks) - a.s + tq + 1;
            }
            ok = sm100::warp_wait(&s_full[sb], (k >> 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            uint32_t sr[32];
            sm100::tmem_ld16(lane_base + sb * kTN, sr);       // lanes 16-31: logits of their row
            sm100::tmem_ld16(lane_base + sb * kTN + 16, sr + 16);
            sm100::tmem_wait_ld();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&s_free[sb]);
            float x[32];
            const int tok0 = it.tt * kTN;
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(sr[c]) * a.scale_log2;
            if (tok0 + kTN > nvis || !srow) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (!srow || tok0 + c >= nvis) x[c] = -INFINITY;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
                mt = fmaxf(mt, fmaxf(fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3])));
            // online softmax, log2 domain, lazy rescale
            const bool grow = (mt != -INFINITY) && (m_run == -INFINITY || mt > m_run + kRescaleThreshold);
            const bool need_rescale = grow && m_run != -INFINITY;
            const float m_new = grow ? mt : m_run;
            const float corr = grow ? (m_run == -INFINITY ? 0.f : ex2(m_run - m_new)) : 1.f;
            if (__any_sync(0xffffffffu, need_rescale)) {
                // O holds this segment's tiles up to k-1: let them retire, and
                // let S(k+1) land too, since the read-modify-write below also
                // passes over the logits lanes (they are stored back unchanged)
                const int kp = k - 1;
                ok = sm100::warp_wait(&o_done[kp & 1], (kp >> 1) & 1, abort_flag, a.err, lim);
                if (ok && k + 1 < hi - lo)
                    ok = sm100::warp_wait(&s_full[(k + 1) & 1], ((k + 1) >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float cr_row = __shfl_sync(0xffffffffu, need_rescale ? corr : 1.f, (lane & 15) + 16);
                const float f = srow ? 1.f : cr_row;
                for (int c = 0; c < 512; c += 16) {
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
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pw[16];
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ex2(x[2 * c] - mu), p1 = ex2(x[2 * c + 1] - mu);
                pw[c] = pack_bf162(p0, p1);
                lsum += p0 + p1;
            }
            l_run += lsum;
            // P buffer sb was last read by the P.C MMA of tile k-2
            if (k >= 2) {
                ok = sm100::warp_wait(&o_done[sb], ((k >> 1) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
            }
            if (srow) {
                // P row r: 64-byte row of 32 bf16, 16-byte chunk c at c ^ ((r >> 1) & 3) (64-byte swizzle)
                const uint32_t rowa = p_addr + sb * kPBytes + r * 64;
                const int sw = (r >> 1) & 3;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(rowa + ((c ^ sw) << 4), make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]));
            }
            fence_proxy_async_smem();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&p_full[sb]);
            if (it.last()) {
                // epilogue of the sequence segment: lanes 0-15 write their O rows
                ok = sm100::warp_wait(&o_done[sb], (k >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float l_tot = __shfl_sync(0xffffffffu, l_run, (lane & 15) + 16);
                const float m_fin = __shfl_sync(0xffffffffu, m_run, (lane & 15) + 16);
                const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
                const float lse2 = l_tot > 0.f ? m_fin + __log2f(l_tot) : -INFINITY;
                const long long orow = (long long)(it.seq * a.s + tq) * a.H + head;
                const long long slot = 2LL * rng + (it.seg == 0 ? 0 : 1);
                const bool writer = row_ok && !srow;
                for (int c = 0; c < 512; c += 16) {
                    uint32_t ov[16];
                    sm100::tmem_ld16(lane_base + kTmO + c, ov);
                    sm100::tmem_wait_ld();
                    if (!writer) continue;
                    if (it.complete) {
                        uint4 pk[2];
                        uint32_t *pp = reinterpret_cast<uint32_t *>(pk);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            pp[e] = pack_bf162(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
                        uint4 *d = reinterpret_cast<uint4 *>(a.out + orow * kDc + c);
                        d[0] = pk[0];
                        d[1] = pk[1];
                    } else {
                        float4 *d4 = reinterpret_cast<float4 *>(a.part_o + (slot * rows_per_seq + grow_row) * kDc + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d4[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                                __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
                    }
                }
                if (writer) {
                    if (it.complete) {
                        if (a.out_lse) a.out_lse[orow] = lse2 * kLn2;
                    } else {
                        a.part_lse2[slot * rows_per_seq + grow_row] = lse2;
                    }
                }
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(o_free);
            }
            it.advance();
        }
    }

    // ------------------------------------------------------------ teardown
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        // every MMA this CTA issued retires before its TMEM is released
        if (lane == 0) sm100::umma_commit(mma_done);
        __syncwarp();
        volatile int no_abort = 0;
        sm100::warp_wait(mma_done, 0, &no_abort, a.err, drain);
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 512);
    }
}

// -------------------------------------------------------------------- plan
// One CTA: `tile`-token tiles of every sequence (its last query sees all L
// tokens), their prefix sums, and the per-range quota.
// plan[0] = tiles per range, plan[1] = total tiles, plan[2] = ranges,
// plan[4 + b] = first tile of sequence b (b = 0..B).
__global__ void __launch_bounds__(1024)
dec_plan_kernel(const int32_t *__restrict__ seq_lens, int B, int s, int max_blocks, int ranges, int tile,
                int32_t *__restrict__ plan, uint32_t *err)
{
    __shared__ int part[1024];
    const int per = (B + 1023) / 1024;
    const int b0 = threadIdx.x * per, b1 = min(B, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) {
        int L = seq_lens[b];
        if (L < 0 || L > max_blocks * kBlock) {
            set_error(err, MLA_DEVERR_SEQ_LEN);
            L = L < 0 ? 0 : max_blocks * kBlock;
        }
        if (L < s) set_error(err, MLA_DEVERR_SEQ_LEN);  // some query sees no key
        sum += (L + tile - 1) / tile;
    }
    part[threadIdx.x] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = part[threadIdx.x] - sum;
    for (int b = b0; b < b1; ++b) {
        plan[4 + b] = run;
        int L = seq_lens[b];
        L = L < 0 ? 0 : min(L, max_blocks * kBlock);
        run += (L + tile - 1) / tile;
    }
    if (threadIdx.x == 1023) {
        const int total = part[1023];
        plan[4 + B] = total;
        plan[1] = total;
        plan[2] = ranges;
        plan[0] = total > 0 ? (total + ranges - 1) / ranges : 1;
    }
}

// ------------------------------------------------------------------ combine
// grid (B, row blocks): sequences cut by range ends are merged by
// log-sum-exp; sequences one range finished are already in place; queries
// with no visible key get a zero latent and lse = -inf.
__global__ void __launch_bounds__(128)
dec_combine_kernel(const int32_t *__restrict__ plan, const float *__restrict__ part_o,
                   const float *__restrict__ part_lse2, const int32_t *__restrict__ seq_lens, int max_blocks,
                   int s, int H, bf16 *__restrict__ out, float *__restrict__ out_lse)
{
    const int b = blockIdx.x, tid = threadIdx.x;
    const int rows = s * H;
    const int q = plan[0];
    const int a0 = plan[4 + b], a1 = plan[4 + b + 1];
    int L = seq_lens[b];
    L = L < 0 ? 0 : min(L, max_blocks * kBlock);
    const int c0 = a1 > a0 ? a0 / q : 0, c1 = a1 > a0 ? (a1 - 1) / q : 0;
    const bool split = a1 > a0 && c0 != c1;
    if (!split && L >= s) return;
    for (int rr = blockIdx.y; rr < rows; rr += gridDim.y) {
        const int t = rr / H;
        const long long orow = (long long)b * rows + rr;
        if (L - s + t + 1 <= 0) {
            reinterpret_cast<uint2 *>(out + orow * kDc)[tid] = make_uint2(0, 0);
            if (tid == 0 && out_lse) out_lse[orow] = -INFINITY;
            continue;
        }
        if (!split) continue;
        float M = -INFINITY;
        for (int c = c0; c <= c1; ++c) {
            const int slot = 2 * c + ((c == c0 && a0 != c * q) ? 1 : 0);
            M = fmaxf(M, part_lse2[(long long)slot * rows + rr]);
        }
        float den = 0.f;
        float4 acc = make_float4(0, 0, 0, 0);
        for (int c = c0; c <= c1; ++c) {
            const int slot = 2 * c + ((c == c0 && a0 != c * q) ? 1 : 0);
            const float l2 = part_lse2[(long long)slot * rows + rr];
            const float w = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
            den += w;
            const float4 v = reinterpret_cast<const float4 *>(part_o + ((long long)slot * rows + rr) * kDc)[tid];
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
}

}  // namespace mla
