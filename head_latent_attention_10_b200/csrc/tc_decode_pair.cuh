// tc_decode_pair.cuh -- absorbed-MLA decode for 128-row groups on a pair of
// CTAs (a 2-CTA cluster) that split the latent columns (sm_100a).
//
// What it computes (DeepSeek-V2 paper review, sections 2-3): for each query
// row (query token t of sequence b, head i), softmax_j(scale * q_abs . row_j)
// weighted sum of the latents c^KV_j, where row_j = [c^KV_j | k^R_j] is the
// 576-value cache row and q_abs = [(U^K_i)^T q^C | RoPE(q^R)].
//
// Why a pair: a group of 128 rows (128 heads of one query token) is the
// full-rate tcgen05 M, but its fp32 latent accumulator O (128 x 512) fills all
// of one SM's tensor memory.  So CTA c of the pair owns latent columns
// [256c, 256c+256) and RoPE dims [32c, 32c+32) of every row:
//   S_c(k) = Q_c C_c(k)^T     M=128, N=64, K=288 (16 + 2 steps)   partial logits
//   S      = S_0 + S_1        fp16-rounded partials swapped through distributed
//                             shared memory, summed in fp32 in both CTAs
//   P(k)   = online softmax of S (both CTAs compute the same bits)
//   O_c   += P(k) C_c(k)[:, latent half]  M=128, N=256, K=64 (P read from TMEM)
// Each CTA loads only its 288 columns of a page (36,864 B), so the pair reads
// every cache byte once, and every MMA runs at the M=128 rate.  The sum
// S_0 + S_1 is the same in both CTAs (fp32 addition is commutative), so both
// take the same softmax decisions and each rescales and normalizes its own O
// half; no other exchange is needed.  Rounding the partials to fp16 (11-bit
// significand) moves a logit by ~2^-12 of its partial (about 1e-3 after the
// 1/sqrt(192) scale for N(0,1) data); P itself is rounded to bf16 anyway.
//
// Shared memory (per CTA): Q_c (128 rows x 288 values: four 64-column chunks
// with 128-byte swizzle + the 32 RoPE columns with 64-byte swizzle), a 3-stage
// ring of page halves, and two 16 KB receive buffers for the peer's partial
// logits.  Tensor memory: O (columns 0-255), two logits buffers (256-383),
// two P buffers (bf16 pairs, 384-447).
//
// Warps (352 threads): 0 TMA pages; 1 logits MMAs; 2 TMA of each sequence's
// Q; 3-10 softmax (two warps per TMEM lane quarter, threads i and 16+i of a
// warp share a row); the softmax warp that completes P(k) issues the P.C MMAs.
// Every wait is bounded (a wait that gives up sets MLA_DEVERR_TIMEOUT and the
// CTA unwinds); the pair meets at a cluster barrier before exit, so neither
// CTA leaves while its peer may still write into its shared memory.
// No TMA load here uses cluster multicast.
#pragma once

#include "dec_common.cuh"

namespace mla {

constexpr int kPrT = 64;                          // tokens per tile (one page)
constexpr int kPrStages = 3;
constexpr int kPrThreads = 352;
constexpr int kPrChunk = 64 * 128;                // one 64-column latent chunk of a page half (8 KB)
constexpr int kPrRope = 64 * 64;                  // the page's 32 RoPE columns of this CTA (4 KB)
constexpr int kPrStage = 4 * kPrChunk + kPrRope;  // 36,864
constexpr int kPrQChunk = 128 * 128;              // 16 KB: one Q latent chunk, 128 rows
constexpr int kPrQ = 4 * kPrQChunk + 128 * 64;    // 73,728
constexpr int kPrXBuf = 128 * 128;                // 128 rows x 64 fp16 logits
constexpr int kPrOffQ = 0;
constexpr int kPrOffStage = kPrOffQ + kPrQ;                       // 73,728
constexpr int kPrOffX = kPrOffStage + kPrStages * kPrStage;       // 184,320
constexpr int kPrOffBar = kPrOffX + 2 * kPrXBuf;                  // 217,088
constexpr int kPrSmem = kPrOffBar + 256 + 1024;                   // + alignment slack
constexpr uint32_t kPrTmS = 256;                  // logits buffers: columns 256 + 64b
constexpr uint32_t kPrTmP = 384;                  // P buffers: columns 384 + 32b
constexpr int kPrAhead = 3;                       // tiles prefetched into L2 ahead of the load
constexpr int kPrSoftmaxWarps = 8;

struct PairMaps {
    CUtensorMap kv_lat;   // cache {576, rows}: box 64 x 64, 128-byte swizzle
    CUtensorMap kv_rope;  // cache {576, rows}: box 32 x 64, 64-byte swizzle
    CUtensorMap q_lat;    // q_abs {576, T*H}: box 64 x 128, 128-byte swizzle
    CUtensorMap q_rope;   // q_abs {576, T*H}: box 32 x 128, 64-byte swizzle
};

namespace pair {

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

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

__device__ __forceinline__ void remote_arrive(uint32_t cluster_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

__device__ __forceinline__ void st_cluster_v4(uint32_t a, uint4 v)
{
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// Bounded wait, with acquire at cluster scope, for a phase completed by the
// peer's remote arrivals.  It polls with test_wait, which never suspends the
// thread (a thread suspended in try_wait is not woken promptly by a remote
// arrive).  Same give-up rules as sm100::mbar_wait.
__device__ __forceinline__ bool wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *err,
                                             uint64_t limit_ns)
{
    const uint32_t a = sm100::smem_u32(bar);
    auto test = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (test()) return true;
    const uint64_t t0 = sm100::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (test()) return true;
        if ((i & 255u) == 0) {
            if (*abort) return false;
            if (sm100::globaltimer_ns() - t0 > limit_ns) {
                set_error(err, MLA_DEVERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

// Lane 0 polls; once the phase is seen complete every lane takes its own
// acquire of it (the phase cannot move on before this warp answers it), so
// each lane's later accesses are ordered after the peer's releases.
__device__ __forceinline__ bool warp_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  uint32_t *err, uint64_t limit_ns)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_cluster(bar, parity, abort, err, limit_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%0], %1;\n\t}"
            ::"r"(sm100::smem_u32(bar)), "r"(parity)
            : "memory");
    }
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t v)
{
    return __half22float2(*reinterpret_cast<__half2 *>(&v));
}

}  // namespace pair

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPrThreads, 1)
tc_decode_pair_kernel(const __grid_constant__ PairMaps maps, const DecArgs a)
{
    extern __shared__ uint8_t pr_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(pr_smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kPrOffBar);
    uint64_t *kv_full = bars + 0;    // [3] TMA -> logits issuer
    uint64_t *kv_empty = bars + 3;   // [3] P.C MMAs of the stage done -> TMA
    uint64_t *q_full = bars + 6;     // TMA of a sequence's Q -> logits issuer
    uint64_t *q_empty = bars + 7;    // last logits MMA of a segment done -> Q loader
    uint64_t *s_full = bars + 8;     // [2] logits issuer -> softmax
    uint64_t *s_free = bars + 10;    // [2] softmax (buffer read) -> logits issuer
    uint64_t *x_full = bars + 12;    // [2] the peer's partial logits have landed (256 remote arrivals)
    uint64_t *x_free = bars + 14;    // [2] the peer has read what we sent (256 remote arrivals)
    uint64_t *pv_done = bars + 16;   // [2] P.C MMAs of tile k done (buffer k & 1)
    uint64_t *mma_done = bars + 18;  // teardown: every MMA issued by this CTA has retired
    int *p_cnt = reinterpret_cast<int *>(bars + 19);  // [2] softmax warps done with P of tile k
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 20);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 21);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cr = pair::cluster_rank(), peer = cr ^ 1u;
    const int cid = blockIdx.x >> 1;
    const int group = cid % a.groups, rng = cid / a.groups;
    const int rows_per_seq = a.s * a.H;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kPrStages; ++i) {
            sm100::mbar_init(&kv_full[i], 1);
            sm100::mbar_init(&kv_empty[i], 1);
        }
        sm100::mbar_init(q_full, 1);
        sm100::mbar_init(q_empty, 1);
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&s_full[i], 1);
            sm100::mbar_init(&s_free[i], kPrSoftmaxWarps);
            sm100::mbar_init(&x_full[i], kPrSoftmaxWarps * 32);
            sm100::mbar_init(&x_free[i], kPrSoftmaxWarps * 32);
            sm100::mbar_init(&pv_done[i], 1);
            p_cnt[i] = 0;
        }
        sm100::mbar_init(mma_done, 1 + kPrSoftmaxWarps);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&maps.kv_lat);
        sm100::prefetch_tensormap(&maps.kv_rope);
        sm100::prefetch_tensormap(&maps.q_lat);
        sm100::prefetch_tensormap(&maps.q_rope);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    // the peer's barriers are initialized before anything is sent to them
    pair::cluster_sync();
    const uint32_t tmem = *tmem_slot;
    // everything above overlaps the plan kernel; its output is read below
    sm100::pdl_wait();
    const int32_t *seq_start = a.plan + 4;
    const int q_per = a.plan[0], total = a.plan[1];
    const int lo = rng * q_per, hi = min(lo + q_per, total);
    // both CTAs of the pair share the range: an empty one skips to the teardown
    const unsigned long long lim = a.limit_ns;
    const unsigned long long drain = lim > 200000000ull ? lim : 200000000ull;
    uint8_t *qs = smem + kPrOffQ;
    uint8_t *stages = smem + kPrOffStage;
    uint8_t *xbuf = smem + kPrOffX;
    const int xlat = 256 * (int)cr, xrope = kDc + 32 * (int)cr;   // this CTA's columns of a row

    auto page_of = [&](const TileIter &t) -> int {
        const int blk = a.block_table[(long long)t.seq * a.max_blocks + t.tt];
        return (blk < 0 || blk >= a.num_blocks) ? -1 : blk;
    };
    auto q_row0 = [&](int seq) { return seq * rows_per_seq + group * 128; };

    if (lo >= hi) {
        // no tiles
    } else if (warp == 0) {
        // ------------------------------------------------------ page TMA
        if (lane == 0) {
            TileIter it, ahead;
            it.init(seq_start, a.B, lo, hi);
            ahead = it;
            for (int i = 0; i < kPrAhead && ahead.ok; ++i) ahead.advance();
            int issued_k = 0;
            bool ok = true;
            while (ok && it.ok) {
                const int k = it.k, st = k % kPrStages;
                if (ahead.ok) {
                    const int pb = page_of(ahead);
                    if (pb >= 0) {
                        for (int j = 0; j < 4; ++j) sm100::tma_prefetch_3d(&maps.kv_lat, xlat + 64 * j, pb * kBlock, 0);
                        sm100::tma_prefetch_3d(&maps.kv_rope, xrope, pb * kBlock, 0);
                    }
                    ahead.advance();
                }
                if (k >= kPrStages)
                    ok = sm100::mbar_wait(&kv_empty[st], ((k / kPrStages) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                int blk = page_of(it);
                if (blk < 0) {
                    // never read outside the cache: load block 0 instead; the
                    // sequence's output is then unspecified and the error bit says so
                    set_error(a.err, MLA_DEVERR_BLOCK_ID);
                    blk = 0;
                }
                if (k == a.stall_tile) {
                    // test hook for failure detection: this page never arrives
                    it.advance();
                    continue;
                }
                uint8_t *dst = stages + st * kPrStage;
                sm100::mbar_arrive_expect_tx(&kv_full[st], kPrStage);
                for (int j = 0; j < 4; ++j)
                    sm100::tma_load_3d(&maps.kv_lat, &kv_full[st], dst + j * kPrChunk, xlat + 64 * j, blk * kBlock, 0);
                sm100::tma_load_3d(&maps.kv_rope, &kv_full[st], dst + 4 * kPrChunk, xrope, blk * kBlock, 0);
                issued_k = k + 1;
                it.advance();
            }
            if (*abort_flag) {  // wait for the copies still in flight
                volatile int no_abort = 0;
                for (int kk = issued_k - kPrStages < 0 ? 0 : issued_k - kPrStages; kk < issued_k; ++kk)
                    if (kk != a.stall_tile)
                        sm100::mbar_wait(&kv_full[kk % kPrStages], (kk / kPrStages) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 2) {
        // --------------------------------------------------------- Q TMA
        // one load of Q_c per sequence segment, once the previous segment's
        // logits MMAs (the readers of the Q buffer) have completed
        if (lane == 0) {
            TileIter it;
            it.init(seq_start, a.B, lo, hi);
            int seg = 0, loaded = 0;
            bool ok = true;
            while (ok && it.ok) {
                if (seg > 0) ok = sm100::mbar_wait(q_empty, (seg - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                const int y = q_row0(it.seq);
                sm100::mbar_arrive_expect_tx(q_full, kPrQ);
                for (int j = 0; j < 4; ++j)
                    sm100::tma_load_3d(&maps.q_lat, q_full, qs + j * kPrQChunk, xlat + 64 * j, y, 0);
                sm100::tma_load_3d(&maps.q_rope, q_full, qs + 4 * kPrQChunk, xrope, y, 0);
                loaded = seg + 1;
                // warm L2 with the next segment's Q
                TileIter nx = it;
                const int cur = it.seg;
                while (nx.ok && nx.seg == cur) nx.advance();
                if (nx.ok) {
                    for (int j = 0; j < 4; ++j) sm100::tma_prefetch_3d(&maps.q_lat, xlat + 64 * j, q_row0(nx.seq), 0);
                    sm100::tma_prefetch_3d(&maps.q_rope, xrope, q_row0(nx.seq), 0);
                }
                it = nx;
                ++seg;
            }
            if (*abort_flag && loaded > 0) {
                volatile int no_abort = 0;
                sm100::mbar_wait(q_full, (loaded - 1) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- logits MMAs
        const uint32_t idesc_s = sm100::idesc_bf16(128, kPrT, 0, 0);
        TileIter is;
        is.init(seq_start, a.B, lo, hi);
        bool ok = true;
        while (ok && is.ok) {
            const int kk = is.k, st = kk % kPrStages, b = kk & 1;
            if (is.first()) ok = sm100::warp_wait(q_full, is.seg & 1, abort_flag, a.err, lim);
            if (ok) ok = sm100::warp_wait(&kv_full[st], (kk / kPrStages) & 1, abort_flag, a.err, lim);
            if (ok && kk >= 2) ok = sm100::warp_wait(&s_free[b], ((kk >> 1) - 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            if (lane == 0) {
                const uint32_t sa = sm100::smem_u32(stages + st * kPrStage);
                const uint32_t qa = sm100::smem_u32(qs);
                const uint32_t d = tmem + kPrTmS + 64 * b;
#pragma unroll
                for (int step = 0; step < 16; ++step) {   // latent half: four 64-column chunks
                    const uint32_t off = (step & 3) * 32;
                    const uint64_t ad = sm100::desc_kmajor(qa + (step >> 2) * kPrQChunk + off, 128, sm100::kSw128);
                    const uint64_t bd = sm100::desc_kmajor(sa + (step >> 2) * kPrChunk + off, 128, sm100::kSw128);
                    sm100::umma_ss(d, ad, bd, idesc_s, step > 0);
                }
#pragma unroll
                for (int step = 0; step < 2; ++step) {    // the 32 RoPE columns
                    const uint64_t ad = sm100::desc_kmajor(qa + 4 * kPrQChunk + step * 32, 64, sm100::kSw64);
                    const uint64_t bd = sm100::desc_kmajor(sa + 4 * kPrChunk + step * 32, 64, sm100::kSw64);
                    sm100::umma_ss(d, ad, bd, idesc_s, 1);
                }
                sm100::umma_commit(&s_full[b]);
                if (is.last()) sm100::umma_commit(q_empty);
            }
            __syncwarp();
            is.advance();
        }
    } else {
        // -------------------------------------------------------- softmax
        // warp w (3..10): TMEM lane quarter q = w % 4, half `sub` of its 32
        // lanes; row r = 32q + 16 sub + i is read by threads i (logits 0-31)
        // and 16+i (logits 32-63)
        const int qd = warp & 3, sub = (warp - 3) >> 2;
        const int hc = lane >> 4;
        const int r = 32 * qd + 16 * sub + (lane & 15);
        const uint32_t lane_base = tmem + ((uint32_t)(32 * qd + 16 * sub) << 16);
        const int grow_row = group * 128 + r;          // index among the sequence's s*H rows
        const int tq = grow_row / a.H, head = grow_row % a.H;
        // this thread's 64 bytes of a receive buffer: row r, 16-byte chunks
        // 4hc .. 4hc+3, each XOR-ed with (r & 7) against bank conflicts
        uint32_t xoff[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xoff[i] = r * 128 + (((4 * hc + i) ^ (r & 7)) << 4);
        const uint32_t x_local = sm100::smem_u32(xbuf);
        const uint32_t x_remote = pair::peer_addr(x_local, peer);
        const uint32_t xfull_remote = pair::peer_addr(sm100::smem_u32(x_full), peer);
        const uint32_t xfree_remote = pair::peer_addr(sm100::smem_u32(x_free), peer);
        // Tile k+1's partial logits are fetched and sent before the softmax of
        // tile k, so the exchange latency overlaps that softmax.  Each lane
        // releases its own remote stores (and, on the receiving side, its own
        // reads) with a remote arrive: the exchange barriers count 256.
        uint32_t own_cur[16], own_nxt[16];
        auto fetch_send = [&](int kn) -> bool {   // tile kn's partials into own_nxt, and to the peer
            const int bn = kn & 1;
            if (!sm100::warp_wait(&s_full[bn], (kn >> 1) & 1, abort_flag, a.err, lim)) return false;
            sm100::tc_fence_after();
            uint32_t sv[32];
            sm100::tmem_ld16x2_32(lane_base + kPrTmS + 64 * bn, sv);
            sm100::tmem_wait_ld();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&s_free[bn]);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                own_nxt[c] = pair::pack_half2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
            // the peer's receive buffer bn is free once it has read tile kn-2
            if (kn >= 2 && !pair::warp_wait_cluster(&x_free[bn], ((kn >> 1) - 1) & 1, abort_flag, a.err, lim))
                return false;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pair::st_cluster_v4(x_remote + bn * kPrXBuf + xoff[i],
                                    make_uint4(own_nxt[4 * i], own_nxt[4 * i + 1], own_nxt[4 * i + 2],
                                               own_nxt[4 * i + 3]));
            pair::remote_arrive(xfull_remote + 8u * bn);
            return true;
        };
        TileIter it, nx;
        it.init(seq_start, a.B, lo, hi);
        nx = it;
        float m_run = -INFINITY, l_run = 0.f;
        int nvis = 0, nseq = 0;
        const uint32_t idesc_o = sm100::idesc_bf16(128, 256, 0, 1);
        bool ok = fetch_send(0);
#pragma unroll
        for (int c = 0; c < 16; ++c) own_cur[c] = own_nxt[c];
        if (nx.ok) nx.advance();
        while (ok && it.ok) {
            const int k = it.k, b = k & 1, st = k % kPrStages;
            if (it.first()) {
                m_run = -INFINITY;
                l_run = 0.f;
                // query tq of a sequence of length L sees positions j <= L - s + tq
                nseq = seq_len_clamped(a.seq_lens, it.seq, a.max_blocks);
                nvis = nseq - a.s + tq + 1;
            }
            if (nx.ok) {
                ok = fetch_send(nx.k);
                if (!ok) break;
            }
            // the peer's partials of tile k, same row and columns
            ok = pair::warp_wait_cluster(&x_full[b], (k >> 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            float x[32];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 v;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                             : "r"(x_local + b * kPrXBuf + xoff[i])
                             : "memory");
                const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 mine = pair::unpack_half2(own_cur[4 * i + e]);
                    const float2 theirs = pair::unpack_half2(pv[e]);
                    x[8 * i + 2 * e] = mine.x + theirs.x;       // the same sum in both CTAs
                    x[8 * i + 2 * e + 1] = mine.y + theirs.y;
                }
            }
            // every value read has been used: the buffer goes back to the peer
            pair::remote_arrive(xfree_remote + 8u * b);
#pragma unroll
            for (int c = 0; c < 16; ++c) own_cur[c] = own_nxt[c];
            if (nx.ok) nx.advance();

            const int tok0 = it.tt * kPrT + 32 * hc;
            if (tok0 + 32 > nvis) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (tok0 + c >= nvis) x[c] = -INFINITY;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; c += 4) mx = fmaxf(mx, fmaxf(fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            // online softmax, log2 domain, lazy rescale (both threads of a row,
            // and both CTAs of the pair, take the same decisions)
            const float mt = mx * a.scale_log2;
            const bool grow = (mt != -INFINITY) && (m_run == -INFINITY || mt > m_run + kRescaleThreshold);
            const bool need_rescale = grow && m_run != -INFINITY;
            const float m_new = grow ? mt : m_run;
            const float corr = grow ? (m_run == -INFINITY ? 0.f : ex2(m_run - m_new)) : 1.f;
            if (__any_sync(0xffffffffu, need_rescale)) {
                // O holds this segment's tiles up to k-1: let them retire, then
                // scale this warp's 16 rows of O
                const int kp = k - 1;
                ok = sm100::warp_wait(&pv_done[kp & 1], (kp >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float f = need_rescale ? corr : 1.f;
                for (int c = 0; c < 256; c += 64) {
                    uint32_t ov[32];
                    sm100::tmem_ld16x2_32(lane_base + c, ov);
                    sm100::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                    sm100::tmem_st16x2_32(lane_base + c, ov);
                }
                sm100::tmem_wait_st();
                sm100::tc_fence_before();
            }
            l_run *= corr;   // this thread's share of the row sum
            m_run = m_new;
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pw[16];
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ex2(fmaf(x[2 * c], a.scale_log2, -mu));
                const float p1 = ex2(fmaf(x[2 * c + 1], a.scale_log2, -mu));
                pw[c] = pack_bf162(p0, p1);
                lsum += p0 + p1;
            }
            l_run += lsum;
            // P(k) into TMEM buffer b, once the P.C MMAs of tile k-2 (its last
            // reader) have completed
            if (k >= 2) {
                const int kp = k - 2;
                ok = sm100::warp_wait(&pv_done[b], (kp >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
            }
            sm100::tmem_st16x2_16(lane_base + kPrTmP + 32 * b, pw);
            sm100::tmem_wait_st();
            {
                // a ragged last tile: zero the latent rows past the sequence end
                // so that 0 * (whatever the page holds there) stays 0; the 8
                // warps take the 4 chunks x (64 - valid) rows x 8 vectors in turn
                const int valid = min(kPrT, nseq - it.tt * kPrT);
                if (valid < kPrT) {
                    uint8_t *kvp = stages + st * kPrStage;
                    const int n = (kPrT - valid) * 4 * 8;
                    for (int e = (warp - 3) * 32 + lane; e < n; e += kPrSoftmaxWarps * 32) {
                        const int rr = valid + e / 32, j = (e >> 3) & 3, c16 = e & 7;
                        reinterpret_cast<uint4 *>(kvp + j * kPrChunk + rr * 128)[c16] = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            fence_proxy_async_smem();
            sm100::tc_fence_before();
            __syncwarp();
            {
                // the warp that completes P(k) issues O += P(k) C(k) (the MMAs of
                // O are thereby issued in tile order, each after every warp's P,
                // zeroing and earlier read or rescale of O)
                int last = 0;
                if (lane == 0) {
                    __threadfence_block();
                    last = atomicAdd(&p_cnt[b], 1) == kPrSoftmaxWarps - 1;
                    __threadfence_block();
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last && lane == 0) {
                    atomicExch(&p_cnt[b], 0);
                    sm100::tc_fence_after();
                    const uint64_t vd = sm100::desc_mnmajor_sw128(sm100::smem_u32(stages + st * kPrStage), kPrChunk);
                    const uint32_t acc0 = it.first() ? 0u : 1u;
#pragma unroll
                    for (int kq = 0; kq < kPrT / 16; ++kq)
                        sm100::umma_ts(tmem, tmem + kPrTmP + 32 * b + 8 * kq, vd + (uint64_t)((kq * 2048) >> 4),
                                       idesc_o, kq > 0 ? 1u : acc0);
                    sm100::umma_commit(&kv_empty[st]);
                    sm100::umma_commit(&pv_done[b]);
                }
                __syncwarp();
            }
            if (it.last()) {
                // epilogue of the sequence segment: threads i and 16+i write
                // the two halves of each 64-column block of this CTA's 256
                // columns of row r
                ok = sm100::warp_wait(&pv_done[b], (k >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
                const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
                const float lse2 = l_tot > 0.f ? m_run + __log2f(l_tot) : -INFINITY;
                const long long orow = (long long)(it.seq * a.s + tq) * a.H + head;
                const long long slot = 2LL * rng + (it.seg == 0 ? 0 : 1);
                for (int c = 0; c < 256; c += 64) {
                    uint32_t ov[32];
                    sm100::tmem_ld16x2_32(lane_base + c, ov);
                    sm100::tmem_wait_ld();
                    const int col = xlat + c + 32 * hc;
                    if (it.complete) {
                        uint4 *d = reinterpret_cast<uint4 *>(a.out + orow * kDc + col);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            d[e] = make_uint4(pack_bf162(__uint_as_float(ov[8 * e]) * inv, __uint_as_float(ov[8 * e + 1]) * inv),
                                              pack_bf162(__uint_as_float(ov[8 * e + 2]) * inv, __uint_as_float(ov[8 * e + 3]) * inv),
                                              pack_bf162(__uint_as_float(ov[8 * e + 4]) * inv, __uint_as_float(ov[8 * e + 5]) * inv),
                                              pack_bf162(__uint_as_float(ov[8 * e + 6]) * inv, __uint_as_float(ov[8 * e + 7]) * inv));
                    } else {
                        float4 *d4 = reinterpret_cast<float4 *>(a.part_o + (slot * rows_per_seq + grow_row) * kDc + col);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d4[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                                __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
                    }
                }
                if (cr == 0 && hc == 0) {
                    if (it.complete) {
                        if (a.out_lse) a.out_lse[orow] = lse2 * kLn2;
                    } else {
                        a.part_lse2[slot * rows_per_seq + grow_row] = lse2;
                    }
                }
                sm100::tc_fence_before();
                __syncwarp();
            }
            it.advance();
        }
    }

    // ------------------------------------------------------------ teardown
    sm100::pdl_trigger();   // the combine may start launching
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1 || warp >= 3) {
        // every MMA this CTA issued retires before its TMEM is released
        if (lane == 0) sm100::umma_commit(mma_done);
        __syncwarp();
    }
    if (warp == 1) {
        volatile int no_abort = 0;
        sm100::warp_wait(mma_done, 0, &no_abort, a.err, drain);
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 512);
    }
    // neither CTA leaves while its peer may still write into its shared
    // memory or arrive on its barriers
    pair::cluster_sync();
}

}  // namespace mla
