// tc_decode64.cuh -- absorbed-MLA decode on tcgen05 tensor cores (sm_100a),
// one 64-token cache page per tile, three logits-issuing warps.
//
// What it computes (DeepSeek-V2 paper review, sections 2-3): for every query
// row (query token t of sequence b, head i), softmax_j(scale * q_abs . row_j)
// weighted sum of the latents c^KV_j, where row_j = [c^KV_j | k^R_j] is the
// 576-value cache row and q_abs = [(U^K_i)^T q^C | RoPE(q^R)].  U^V is applied
// later.
//
// Work unit: 64 rows of one sequence (its s*H (query, head) pairs, cut in
// groups of 64; the MMA M dimension) against 64-token tiles of its cache.
// Why this shape on B200: a tcgen05.mma costs a fixed ~34 ns to issue from one
// thread whatever its size up to M=128, N=128, and M=64 runs at half rate, so
// the 36 K-steps of one tile's logits take ~1.2 us to issue from one thread.
// Three warps issue the logits of every third tile, each into its own buffer,
// so a tile's logits start as soon as its page lands; the P.C MMAs of a tile
// are issued by the softmax warp that completes its P (no hand-off):
//
//   S(k)  = Q C_k^T            M=64, N=64, K=576 (36 steps)   (warp 1 + k % 3)
//   O    += P(k) C_k[:, 0:512]  M=64, N=2 x 256, K=64          (last softmax warp)
//
// Each logits buffer has a single issuer and the P.C MMAs are issued in tile
// order (each after all four warps' P, tcgen05 fences around a shared-memory
// counter), so every sum is taken in a fixed order and the output does not
// depend on timing.
//
// TMEM (512 columns): a 64-row operand occupies one half of each 32-lane
// quarter (row m at lane 32*(m/16) + m%16, plus 16 for the upper half):
//   lanes 0-15:  S(k % 3 = 0, 1) (columns 0-127) | Q (128-415, bf16 pairs) | S(k % 3 = 2) (416-479)
//   lanes 16-31: O (columns 0-511)
// Q is the A operand of the logits MMAs, read from TMEM; an A operand in TMEM
// must sit in the same lanes as its accumulator, hence S and Q share a half.
// The softmax warps touch TMEM only with 16-lane accesses (tcgen05.ld/st
// .16x32bx2), so the logits/Q half and the O half are used independently: a
// rescale of O does not wait for the logits MMAs, and the next sequence's Q
// is written while this sequence's O is still being read out.
// Keeping Q out of shared memory leaves room for a 3-stage ring of 64-token
// tiles (73,728 B each; TMA loads one 64 x 64 box per chunk from the tile's
// page).  P of a tile (64 x 64 bf16, 128-byte swizzle, 8 KB) is written over
// the tile's RoPE chunk, which no MMA reads once the tile's logits are done,
// so P has one buffer per stage and is freed with the stage.  After each page
// load the loader prefetches the next page it will load into L2, so a freed
// stage refills from L2 (prefetching farther ahead competes with the other
// SMs' loads); when that tile starts a segment, the loader also
// bulk-prefetches the segment's Q rows, which the softmax warps read at the
// switch.
//
// Softmax: warps 4-7, one per TMEM quarter.  Threads i and 16+i of a warp
// share row 16q+i: each reads half of the row's 64 logits, frees the buffer
// for S(k+3), and does half of the exp work and half of the row's epilogue.
// Warp q also zeroes its quarter of a ragged tile's latent rows past the
// sequence end.
// Online softmax in the log2 domain with lazy rescaling (O and l are rescaled
// only when the running max grows by more than 8, a factor 256).
//
// Work split: the (sequence, tile) list of the batch is cut into contiguous
// ranges of equal cost per row group, a tile counting one and the start of a
// sequence four (plan_range, one warp of every CTA).  A sequence a range
// covers completely is normalized and written straight to the output.  A
// sequence cut by range ends leaves one fp32 partial per piece (normalized,
// with its log2-sum-exp), merged by dec_combine_kernel; a sequence cut into
// exactly two pieces is merged here instead, by the CTA whose range ends
// with its late piece (see the epilogue).  The epilogue stages each softmax
// warp's 16 output rows through shared memory, so that they leave in whole
// 128-byte lines.  Every wait is bounded; a wait that gives up sets
// MLA_DEVERR_TIMEOUT, the CTA unwinds, waits for its own copies in flight and
// frees its TMEM.
//
// FP8 cache (kFp8): a page is 576 E4M3 codes per token plus two fp32 scales
// per token (csrc/fp8.cuh).  TMA lands the codes, one 64-column box per
// chunk (4 KB each), in the upper half of the stage and the page's 512 B of
// scales in a side slot; four extra warps (8-11) widen them in place into the
// same f16 tile layout the bf16 path uses, with the token's larger scale
// s_j = max(sc_c, sc_r) factored out: the f16 values are code * sc / s_j
// (one part exact, the other scaled by <= 1), so the logits MMA gives l_j / s_j
// and the softmax multiplies its logits by s_j, and P_j s_j is the A operand
// of the latent sum.  Q and P are f16; the MMAs are kind::f16 with f16
// operands.  Chunk j's codes sit at 36,864 + 4,096 j and its f16 output at
// 8,192 j, so output chunk j overwrites the codes of chunks 2j-9 and 2j-8: the
// converters go in four groups (0-3 | 4-5 | 6 | 7-8) with a named barrier
// between groups, and chunk 8's codes are read before the last barrier.
#pragma once

#include "dec_common.cuh"
#include "fp8.cuh"

namespace mla {

constexpr int kT64 = 64;                          // tokens per tile (one page)
constexpr int kD64Stages = 3;
constexpr int kD64Threads = 256;
constexpr int kD64Chunk = kT64 * 128;             // one 64-column chunk of a tile (8 KB)
constexpr int kD64Stage = 9 * kD64Chunk;          // 73728
constexpr int kD64OffStage = 0;
constexpr int kD64OffBar = kD64OffStage + kD64Stages * kD64Stage;  // 221184
constexpr int kD64PChunk = 8 * kD64Chunk;         // P of a tile goes where its RoPE chunk was
// epilogue staging: per softmax warp 16 rows of kD64EpiRow bytes, so that the
// output rows leave in whole 128-byte lines (FP8 kernel: 64-byte rows)
constexpr int kD64EpiRow = 128, kD64EpiRowFp8 = 64;
constexpr int kD64OffEpi = kD64OffBar + 512;
constexpr int kD64Smem = kD64OffEpi + 4 * 16 * kD64EpiRow + 1024;  // + alignment slack
constexpr uint32_t kD64TmO = 16u << 16;           // O: lanes 16-31, columns 0-511
constexpr uint32_t kD64TmQ = 128;                 // Q: lanes 0-15, columns 128-415 (S: 0-127)
constexpr uint32_t kD64TmS2 = 416;                // third logits buffer: lanes 0-15, columns 416-479
constexpr int kD64Ahead = 1;                      // tiles prefetched into L2 ahead of the load
// FP8 cache: 128 more threads (the converters), per-stage scale slots
// ([64][2] fp32) and per-token factored scales s_j ([64] fp32) after the stages
constexpr int kD64Cvt = 128;                       // converter threads (warps 8-11)
constexpr int kD64ThreadsFp8 = kD64Threads + kD64Cvt;
constexpr int kD64CvtRows = kT64 * 4 / kD64Cvt;    // rows per converter thread (4 threads per row)
constexpr int kD64F8Codes = kT64 * kRow;          // 36,864 (one code per value): where the codes land
constexpr int kD64F8Box = kT64 * 64;              // one 64-column box of codes (4 KB)
constexpr int kD64OffScale = kD64Stages * kD64Stage;              // [3][64][2] fp32
constexpr int kD64OffSmax = kD64OffScale + kD64Stages * 512;      // [3][64] fp32
constexpr int kD64OffBarFp8 = kD64OffSmax + kD64Stages * 256;
constexpr int kD64OffEpiFp8 = kD64OffBarFp8 + 512;
constexpr int kD64SmemFp8 = kD64OffEpiFp8 + 4 * 16 * kD64EpiRowFp8 + 1024;

template <bool kFp8>
__global__ void __launch_bounds__(kFp8 ? kD64ThreadsFp8 : kD64Threads, 1)
tc_decode64_kernel(const __grid_constant__ CUtensorMap map_kv, const DecArgs a)
{
    extern __shared__ uint8_t d64_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(d64_smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (kFp8 ? kD64OffBarFp8 : kD64OffBar));
    uint64_t *cv_full = bars + 32;   // [3] FP8: the stage's codes widened to f16 (the converter warps)
    uint64_t *kv_full = bars + 18;   // [3] TMA -> MMA (bf16: chunks 5-8 of the page)
    uint64_t *kv_half = bars + 35;   // [3] bf16: chunks 0-4 of the page landed
    uint64_t *kv_empty = bars + 21;  // [3] P.C MMAs of the stage done -> TMA, softmax
    // Q of segment n is in TMEM once q_cnt >= 4 (n + 1) (each softmax warp adds
    // 1 per segment): a count rather than a barrier phase, so that an issuer
    // with no tile in some segments can never be two phases behind
    volatile int *q_cnt = reinterpret_cast<volatile int *>(bars + 4);
    uint64_t *s_full = bars + 26;    // [3] S issuer -> softmax (logits buffer b)
    uint64_t *s_free = bars + 29;    // [3] softmax (buffer b read) -> S issuer
    int *p_cnt = reinterpret_cast<int *>(bars + 24);  // [3] softmax warps done with P of the stage
    uint64_t *mma_done = bars + 14;  // every MMA-issuing thread at teardown
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 17);

    int *rplan = reinterpret_cast<int *>(bars + 40);   // this CTA's range (plan_range's out, 6 ints)
    uint64_t *early_in = bars + 44;  // [4] a late piece's merge: the early piece's rows landed (softmax warp q)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = blockIdx.x % a.groups, rng = blockIdx.x / a.groups;
    const int rows_per_seq = a.s * a.H;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kD64Stages; ++i) {
            sm100::mbar_init(&kv_full[i], 1);
            sm100::mbar_init(&kv_empty[i], 1);
            sm100::mbar_init(&kv_half[i], 1);
        }
        *q_cnt = 0;
        for (int i = 0; i < 3; ++i) {
            sm100::mbar_init(&s_full[i], 1);
            sm100::mbar_init(&s_free[i], 4);
        }
        for (int i = 0; i < kD64Stages; ++i) p_cnt[i] = 0;
        if constexpr (kFp8)
            for (int i = 0; i < kD64Stages; ++i) sm100::mbar_init(&cv_full[i], kD64Cvt / 32);
        sm100::mbar_init(mma_done, 7);
        for (int i = 0; i < 4; ++i) sm100::mbar_init(&early_in[i], 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&map_kv);
    }
    if (warp == 1) {
        sm100::tmem_alloc(tmem_slot, 512);
        sm100::tmem_relinquish();
    }
    // the sequence lengths and queries may come from the kernel before this one
    sm100::pdl_wait();
    if (warp == 2)
        plan_range(a.seq_lens, a.B, a.s, a.max_blocks, gridDim.x / a.groups, rng, blockIdx.x == 0,
                   !kFp8 && a.merges, a.plan, a.flags + 2 * a.B * a.groups * 4, a.err, rplan);
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int lo = rplan[0], hi = rplan[1];
    if (lo >= hi) {   // no tile for this CTA
        if (warp == 1) sm100::tmem_dealloc(tmem, 512);
        return;
    }
    const int seq0 = rplan[2], start0 = rplan[3];   // the sequence holding tile lo, its first tile
    const int qv = rplan[4], va0 = rplan[5];         // the plan's virtual quota, seq0's virtual start
    const unsigned long long lim = a.limit_ns;
    const unsigned long long drain = lim > 200000000ull ? lim : 200000000ull;
    uint8_t *stages = smem + kD64OffStage;

    auto page_of = [&](const TileIter &t) -> int {
        const int blk = a.block_table[(long long)t.seq * a.max_blocks + t.tt];
        return (blk < 0 || blk >= a.num_blocks) ? -1 : blk;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            TileIter it, ahead;
            it.init(a.seq_lens, a.max_blocks, a.B, lo, hi, seq0, start0, va0);
            ahead = it;
            for (int i = 0; i < kD64Ahead && ahead.ok; ++i) ahead.advance();
            // warm L2 with the page kD64Ahead tiles further on (and, when that tile
            // starts a segment, with the segment's Q rows, which the softmax warps
            // read at the switch: 64 rows of 1152 B at most); issued after each
            // page load, so the first loads of the range go out first
            auto prefetch_ahead = [&]() {
                if (ahead.ok) {
                    if (ahead.first() && ahead.seg > 0) {
                        const int r0 = group * kGroupRows, nr = min(kGroupRows, rows_per_seq - r0);
                        const char *q0 = reinterpret_cast<const char *>(a.q_abs + ((long long)ahead.seq * rows_per_seq + r0) * kRow);
                        for (int r = 0; r < nr; r += 8)
                            sm100::bulk_prefetch_l2(q0 + (long long)r * kRow * 2, min(8, nr - r) * kRow * 2);
                    }
                    const int pb = page_of(ahead);
                    if (pb >= 0) {
                        for (int j = 0; j < 9; ++j) sm100::tma_prefetch_3d(&map_kv, 64 * j, pb * kBlock, 0);
                        if constexpr (kFp8)
                            for (int e = 0; e < 4; ++e)
                                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.scales + (long long)pb * 128 + 32 * e));
                    }
                    ahead.advance();
                }
            };
            int issued_k = 0;
            bool ok = true;
            while (ok && it.ok) {
                const int k = it.k, st = k % kD64Stages;
                if (k >= kD64Stages)
                    ok = sm100::mbar_wait(&kv_empty[st], ((k / kD64Stages) - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                int blk = page_of(it);
                if (blk < 0) {
                    // never read outside the cache: load block 0 instead; the
                    // sequence's output is then unspecified and the error bit says so
                    set_error(a.err, MLA_DEVERR_BLOCK_ID);
                    blk = 0;
                }
                uint8_t *dst = stages + st * kD64Stage;
                if (k == a.stall_tile) {
                    // test hook for failure detection: this page never arrives, so the
                    // first wait on it runs out and the CTA unwinds
                    prefetch_ahead();
                    it.advance();
                    continue;
                }
                if constexpr (kFp8) {
                    sm100::mbar_arrive_expect_tx(&kv_full[st], 9 * kD64F8Box + 512);
                    for (int j = 0; j < 9; ++j)
                        sm100::tma_load_3d(&map_kv, &kv_full[st], dst + kD64F8Codes + j * kD64F8Box, 64 * j,
                                           blk * kBlock, 0);
                    sm100::bulk_load(smem + kD64OffScale + st * 512, a.scales + (long long)blk * 128, 512,
                                     &kv_full[st]);
                } else {
                    // two halves, so the logits can start on chunks 0-4 while 5-8 land
                    sm100::mbar_arrive_expect_tx(&kv_half[st], 5 * kD64Chunk);
                    sm100::mbar_arrive_expect_tx(&kv_full[st], 4 * kD64Chunk);
                    for (int j = 0; j < 9; ++j)
                        sm100::tma_load_3d(&map_kv, j < 5 ? &kv_half[st] : &kv_full[st], dst + j * kD64Chunk, 64 * j,
                                           blk * kBlock, 0);
                }
                issued_k = k + 1;
                prefetch_ahead();
                it.advance();
            }
            if (*abort_flag) {  // wait for the copies still in flight
                volatile int no_abort = 0;
                for (int kk = issued_k - kD64Stages < 0 ? 0 : issued_k - kD64Stages; kk < issued_k; ++kk)
                    if (kk != a.stall_tile) {
                        sm100::mbar_wait(&kv_full[kk % kD64Stages], (kk / kD64Stages) & 1, &no_abort, a.err, drain);
                        if (!kFp8)
                            sm100::mbar_wait(&kv_half[kk % kD64Stages], (kk / kD64Stages) & 1, &no_abort, a.err, drain);
                    }
            }
        }
    } else if (warp >= 1 && warp <= 3) {
        // --------------------------------------------------- logits MMAs
        // warp 1 + b takes the tiles k with k % 3 = b, each into its own
        // logits buffer, all 36 K steps
        const int b = warp - 1;
        const uint32_t scol = b < 2 ? 64u * b : kD64TmS2;
        const uint32_t idesc_s = kFp8 ? sm100::idesc_f16(kGroupRows, kT64, 0, 0) : sm100::idesc_bf16(kGroupRows, kT64, 0, 0);
        TileIter is;
        is.init(a.seq_lens, a.max_blocks, a.B, lo, hi, seq0, start0, va0);
        int q_seg = -1;
        bool ok = true;
        while (ok && is.ok) {
            const int kk = is.k, st = kk % kD64Stages;
            if (kk % 3 != b) {
                is.advance();
                continue;
            }
            // the Q rows of this tile's sequence are written into TMEM by the
            // softmax warps, which count the segments they have written
            if (q_seg < is.seg) {
                ok = wait_count(q_cnt, 4 * (is.seg + 1), abort_flag, a.err, lim);
                q_seg = is.seg;
            }
            if (!ok) break;
            ok = sm100::warp_wait(kFp8 ? &cv_full[st] : &kv_half[st], (kk / kD64Stages) & 1, abort_flag, a.err, lim);
            if (ok && kk >= 3) ok = sm100::warp_wait(&s_free[b], ((kk / 3) - 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            int ok2 = 1;
            if (lane == 0) {
                const uint64_t kd = sm100::desc_kmajor(sm100::smem_u32(stages + st * kD64Stage), 128, sm100::kSw128);
                const uint32_t d = tmem + scol;
#pragma unroll
                for (int step = 0; step < 36; ++step) {          // 16-column K steps
                    if (!kFp8 && step == 20) {
                        // chunks 5-8 (the bf16 page's second half)
                        if (!sm100::mbar_wait(&kv_full[st], (kk / kD64Stages) & 1, abort_flag, a.err, lim)) {
                            ok2 = 0;
                            break;
                        }
                        sm100::tc_fence_after();
                    }
                    const uint32_t off = (step >> 2) * kD64Chunk + (step & 3) * 32;
                    sm100::umma_ts(d, tmem + kD64TmQ + 8 * step, kd + (uint64_t)(off >> 4), idesc_s, step > 0);
                }
                if (ok2) sm100::umma_commit(&s_full[b]);
            }
            ok = __shfl_sync(0xffffffffu, ok2, 0) != 0;
            __syncwarp();
            is.advance();
        }
    } else if (kFp8 && warp >= 8) {
        // ----------------------------------------------- FP8 -> f16 (warps 8-11)
        // thread ct: rows rr_i = ct / 4 + 32 i (i = 0, 1), 16-code segment g =
        // ct % 4 of each 64-column chunk (a warp reads 512 contiguous bytes)
        const int ct = threadIdx.x - kD64Threads, g = ct & 3;
        TileIter it;
        it.init(a.seq_lens, a.max_blocks, a.B, lo, hi, seq0, start0, va0);
        bool ok = true;
        while (ok && it.ok) {
            const int k = it.k, st = k % kD64Stages;
            ok = sm100::warp_wait(&kv_full[st], (k / kD64Stages) & 1, abort_flag, a.err, lim);
            // the converter warps go on only if all saw the page land: they
            // meet at named barriers below, which none may skip
            {
                uint32_t both;
                asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
                             "bar.red.and.pred p, 3, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                             : "=r"(both) : "r"((uint32_t)ok) : "memory");
                ok = both != 0;
            }
            if (!ok) break;
            uint8_t *stg = stages + st * kD64Stage;
            const float2 *scl = reinterpret_cast<const float2 *>(smem + kD64OffScale + st * 512);
            float *smax = reinterpret_cast<float *>(smem + kD64OffSmax + st * 256);
            uint32_t rat_c[kD64CvtRows], rat_r[kD64CvtRows];   // f16x2 ratios sc / s_j of the thread's rows
            bool one_c[kD64CvtRows], one_r[kD64CvtRows];
#pragma unroll
            for (int i = 0; i < kD64CvtRows; ++i) {
                const int rr = (ct >> 2) + 32 * i;
                const float2 sc = scl[rr];
                const float m = fmaxf(sc.x, sc.y);
                const float fc = sc.x / m, fr = sc.y / m;
                one_c[i] = fc == 1.f;
                one_r[i] = fr == 1.f;
                const __half2 hc = __float2half2_rn(fc), hr = __float2half2_rn(fr);
                rat_c[i] = *reinterpret_cast<const uint32_t *>(&hc);
                rat_r[i] = *reinterpret_cast<const uint32_t *>(&hr);
                if (g == 0) smax[rr] = m;
            }
            auto read = [&](int j, uint4 *in) {
#pragma unroll
                for (int i = 0; i < kD64CvtRows; ++i)
                    in[i] = *reinterpret_cast<const uint4 *>(stg + kD64F8Codes + j * kD64F8Box +
                                                             64 * ((ct >> 2) + 32 * i) + 16 * g);
            };
            auto write = [&](int j, const uint4 *in, const uint32_t *rat, const bool *one) {
#pragma unroll
                for (int i = 0; i < kD64CvtRows; ++i) {
                    const int rr = (ct >> 2) + 32 * i;
                    const uint16_t *c = reinterpret_cast<const uint16_t *>(&in[i]);
                    uint32_t h[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) h[e] = e4m3x2_to_f16x2(c[e]);
                    if (!one[i]) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            __half2 v = *reinterpret_cast<__half2 *>(&h[e]);
                            v = __hmul2(v, *reinterpret_cast<const __half2 *>(&rat[i]));
                            h[e] = *reinterpret_cast<uint32_t *>(&v);
                        }
                    }
                    uint8_t *rowp = stg + j * kD64Chunk + rr * 128;
                    *reinterpret_cast<uint4 *>(rowp + (((2 * g) ^ (rr & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(rowp + (((2 * g + 1) ^ (rr & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
                }
            };
            auto group_sync = [] { asm volatile("bar.sync 3, 128;" ::: "memory"); };
            uint4 in[kD64CvtRows], in8[kD64CvtRows];
#pragma unroll 1
            for (int j = 0; j < 4; ++j) { read(j, in); write(j, in, rat_c, one_c); }
            group_sync();
#pragma unroll 1
            for (int j = 4; j < 6; ++j) { read(j, in); write(j, in, rat_c, one_c); }
            group_sync();
            read(6, in); write(6, in, rat_c, one_c);
            group_sync();
            read(7, in); read(8, in8); write(7, in, rat_c, one_c);
            group_sync();
            write(8, in8, rat_r, one_r);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&cv_full[st]);
            it.advance();
        }
    } else {
        // -------------------------------------------------------- softmax
        // warp q (0..3) owns group rows [16q, 16q+16): row 16q+i's logits and
        // Q sit at TMEM lane 32q+i, its O at lane 32q+16+i; threads i and 16+i
        // each take half of the row's columns in both
        const int qd = warp & 3;
        const bool srow = lane < 16;
        const int r = 16 * qd + (lane & 15);
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);        // logits and Q lanes
        const uint32_t o_base = tmem + ((uint32_t)(qd * 32 + 16) << 16);      // O lanes
        const uint32_t p_row0 = sm100::smem_u32(stages + kD64PChunk) + r * 128;
        const int grow_row = group * kGroupRows + r;  // index among the sequence's s*H rows
        const bool row_ok = grow_row < rows_per_seq;
        const int tq = row_ok ? grow_row / a.H : 0;   // query token of this row
        const int head = row_ok ? grow_row % a.H : 0;
        // Q rows of sequence `seq` into TMEM (16-lane stores: lanes 0-15 only, so
        // the O lanes are untouched and the previous sequence's epilogue can
        // still be running).  Thread i and thread 16+i each hold half of row r:
        // 32-column block j, columns 16 each.
        auto write_q = [&](int seq) {
            const uint4 *q4 = reinterpret_cast<const uint4 *>(
                a.q_abs + ((long long)seq * rows_per_seq + (row_ok ? grow_row : 0)) * kRow) + (srow ? 0 : 4);
            // all 36 loads in flight at once (one memory latency per switch),
            // through L2: the kernel that wrote the queries may have been
            // running when this one started, so the read-only path is out
            uint4 v[36];
#pragma unroll
            for (int e = 0; e < 36; ++e)
                v[e] = row_ok ? __ldcg(q4 + 8 * (e >> 2) + (e & 3)) : make_uint4(0, 0, 0, 0);
            if constexpr (kFp8) {
                // the FP8 path's MMAs take f16 operands
#pragma unroll
                for (int e = 0; e < 36; ++e) {
                    uint32_t *w = reinterpret_cast<uint32_t *>(&v[e]);
#pragma unroll
                    for (int f = 0; f < 4; ++f) {
                        const __half2 hh = __float22half2_rn(
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[f])));
                        w[f] = *reinterpret_cast<const uint32_t *>(&hh);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 9; ++j)
                sm100::tmem_st16x2_16(lane_base + kD64TmQ + 32 * j, reinterpret_cast<const uint32_t *>(v + 4 * j));
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                atomicAdd(const_cast<int *>(q_cnt), 1);
            }
        };
        TileIter it;
        it.init(a.seq_lens, a.max_blocks, a.B, lo, hi, seq0, start0, va0);
        float m_run = -INFINITY, l_run = 0.f;
        int nvis = 0, nseq = 0;
        const uint32_t idesc_o = kFp8 ? sm100::idesc_f16(kGroupRows, 256, 0, 1) : sm100::idesc_bf16(kGroupRows, 256, 0, 1);
        bool ok = true;
        if (it.ok) write_q(it.seq);
        while (ok && it.ok) {
            const int k = it.k;
            if (it.first()) {
                m_run = -INFINITY;
                l_run = 0.f;
                // query tq of a sequence of length L sees positions j <= L - s + tq
                nseq = seq_len_clamped(a.seq_lens, it.seq, a.max_blocks);
                nvis = nseq - a.s + tq + 1;
            }
            if (lane == 0 && (it.tt + 4 == it.t1 || (it.first() && it.t1 - it.t0 < 4))) {
                // a late piece (see the epilogue): bring the early piece's rows of
                // this warp's quarter into L2 before the merge reads them
                const int cf = (it.seq_v + kSwitchTiles) / qv, cl = (it.seq_v + kSwitchTiles + it.seq_t - 1) / qv;
                const int r0 = group * kGroupRows + 16 * qd;
                if (!kFp8 && a.merges && !it.complete && cl == cf + 1 && rng == cf && r0 < rows_per_seq) {
                    const char *e = reinterpret_cast<const char *>(a.part_o + (2LL * cl * rows_per_seq + r0) * kDc);
                    const int nr = min(16, rows_per_seq - r0);
                    for (int o = 0; o < nr * kDc * 4; o += 16384)
                        sm100::bulk_prefetch_l2(e + o, (uint32_t)min(16384, nr * kDc * 4 - o));
                }
            }
            const int sb = k % 3;
            ok = sm100::warp_wait(&s_full[sb], (k / 3) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            // raw logits of row r, columns [32h, 32h+32) (h = 0 for threads 0-15);
            // then the buffer is handed back for S(k+3)
            float x[32];
            {
                uint32_t sv[32];
                sm100::tmem_ld16x2_32(lane_base + (sb < 2 ? 64u * sb : kD64TmS2), sv);
                sm100::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(sv[c]);
                sm100::tc_fence_before();
                __syncwarp();
                if (lane == 0) sm100::mbar_arrive(&s_free[sb]);
            }
            const int tok0 = it.tt * kT64 + (srow ? 0 : 32);
            // FP8: the factored per-token scales s_j of this thread's 32 columns,
            // written by the converters before they released the stage
            const float *smx = reinterpret_cast<const float *>(smem + kD64OffSmax + (k % kD64Stages) * 256) +
                               (srow ? 0 : 32);
            if constexpr (kFp8) {
                ok = sm100::warp_wait(&cv_full[k % kD64Stages], (k / kD64Stages) & 1, abort_flag, a.err, lim);
                if (!ok) break;
#pragma unroll
                for (int c = 0; c < 32; ++c) x[c] *= smx[c];
            }
            if (tok0 + 32 > nvis) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (tok0 + c >= nvis) x[c] = -INFINITY;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; c += 4) mx = fmaxf(mx, fmaxf(fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            // online softmax, log2 domain, lazy rescale (both lanes of a row take
            // the same decisions: they hold the same max)
            const float mt = mx * a.scale_log2;
            const bool grow = (mt != -INFINITY) && (m_run == -INFINITY || mt > m_run + kRescaleThreshold);
            const bool need_rescale = grow && m_run != -INFINITY;
            const float m_new = grow ? mt : m_run;
            const float corr = grow ? (m_run == -INFINITY ? 0.f : ex2(m_run - m_new)) : 1.f;
            if (__any_sync(0xffffffffu, need_rescale)) {
                // O holds this segment's tiles up to k-1: let them retire, then
                // scale the O lanes (16-lane accesses: the logits and Q lanes,
                // which S(k+1) may be using, are not touched)
                const int kp = k - 1;
                ok = sm100::warp_wait(&kv_empty[kp % kD64Stages], (kp / kD64Stages) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float f = need_rescale ? corr : 1.f;
                for (int c = 0; c < 512; c += 64) {
                    uint32_t ov[32];
                    sm100::tmem_ld16x2_32(o_base + c, ov);
                    sm100::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                    sm100::tmem_st16x2_32(o_base + c, ov);
                }
                sm100::tmem_wait_st();
                sm100::tc_fence_before();
            }
            l_run *= corr;   // this lane's share of the row sum
            m_run = m_new;
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pw[16];
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ex2(fmaf(x[2 * c], a.scale_log2, -mu));
                const float p1 = ex2(fmaf(x[2 * c + 1], a.scale_log2, -mu));
                if constexpr (kFp8) {
                    // a masked column has p = 0 and may sit past the sequence
                    // end, where the scale can be NaN: keep its P exactly 0
                    const float2 sj = *reinterpret_cast<const float2 *>(smx + 2 * c);
                    const __half2 hh = __floats2half2_rn(p0 > 0.f ? p0 * sj.x : 0.f, p1 > 0.f ? p1 * sj.y : 0.f);
                    pw[c] = *reinterpret_cast<const uint32_t *>(&hh);
                } else {
                    pw[c] = pack_bf162(p0, p1);
                }
                lsum += p0 + p1;
            }
            l_run += lsum;
            {
                // P row r: 128-byte row of 64 bf16, 16-byte chunk c at c ^ (r & 7)
                // (128-byte swizzle); lanes 0-15 write chunks 0-3, lanes 16-31 chunks 4-7
                const int c0 = srow ? 0 : 4;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(p_row0 + (k % kD64Stages) * kD64Stage + (((c0 + c) ^ (r & 7)) << 4),
                                 make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]));
            }
            {
                // a ragged last tile: zero the latent rows past the sequence end so
                // that 0 * (whatever the page holds there) stays 0 (warp q: chunks 2q, 2q+1)
                const int valid = min(kT64, nseq - it.tt * kT64);
                uint8_t *kvp = stages + (k % kD64Stages) * kD64Stage;
                for (int e = lane; e < (kT64 - valid) * 16; e += 32) {
                    const int rr = valid + (e >> 4), j = 2 * qd + ((e >> 3) & 1), c16 = e & 7;
                    reinterpret_cast<uint4 *>(kvp + j * kD64Chunk + rr * 128)[c16] = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
            sm100::tc_fence_before();
            __syncwarp();
            {
                // the warp that completes P(k) issues O += P(k) C_k (the MMAs of
                // O are thereby issued in tile order, each after every warp's P,
                // V zeroing and previous read of O)
                const int st = k % kD64Stages;
                int last = 0;
                if (lane == 0) {
                    sm100::tc_fence_before();
                    __threadfence_block();
                    last = atomicAdd(&p_cnt[st], 1) == 3;
                    __threadfence_block();
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last && lane == 0) {
                    atomicExch(&p_cnt[st], 0);
                    sm100::tc_fence_after();
                    uint8_t *kvp = stages + st * kD64Stage;
                    const uint64_t vd = sm100::desc_mnmajor_sw128(sm100::smem_u32(kvp), kD64Chunk);
                    const uint64_t pd = sm100::desc_kmajor(sm100::smem_u32(kvp + kD64PChunk), 128, sm100::kSw128);
                    const uint32_t acc0 = it.first() ? 0u : 1u;
#pragma unroll
                    for (int kq = 0; kq < kT64 / 16; ++kq)
#pragma unroll
                        for (int jh = 0; jh < 2; ++jh)
                            sm100::umma_ss(tmem + kD64TmO + 256 * jh, pd + (uint64_t)((kq * 32) >> 4),
                                           vd + (uint64_t)((4 * jh * kD64Chunk + kq * 2048) >> 4), idesc_o,
                                           kq > 0 ? 1u : acc0);
                    sm100::umma_commit(&kv_empty[st]);
                }
                __syncwarp();
            }
            if (it.last()) {
                // every logits MMA of this segment has been read: the next
                // sequence's Q goes in now, so its logits overlap this epilogue
                TileIter nx = it;
                nx.advance();
                if (nx.ok) write_q(nx.seq);
                // epilogue of the sequence segment: threads i and 16+i write the
                // two halves of O row r
                ok = sm100::warp_wait(&kv_empty[k % kD64Stages], (k / kD64Stages) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
                const float m_fin = m_run;
                const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
                const float lse2 = l_tot > 0.f ? m_fin + __log2f(l_tot) : -INFINITY;
                const long long orow = (long long)(it.seq * a.s + tq) * a.H + head;
                const long long slot = 2LL * rng + (it.seg == 0 ? 0 : 1);
                // O row r leaves through the warp's staging rows: per 64-column
                // block, thread i / 16+i put their halves of row r in shared
                // memory (16-byte chunks XOR-swizzled by row), then each store
                // instruction of the warp writes whole rows of the block
                constexpr int RB = kFp8 ? kD64EpiRowFp8 : kD64EpiRow;
                constexpr int CPR = RB / 16;
                const uint32_t stg = sm100::smem_u32(smem + (kFp8 ? kD64OffEpiFp8 : kD64OffEpi)) + qd * 16 * RB;
                const int lr_me = lane & 15, hh = srow ? 0 : 1;
                auto swz = [](int row) { return (row * RB / 128) & (CPR - 1); };
                // stage pk (the thread's half of its row's block, HB bytes) and
                // write the warp's 16 rows of block c to base (EB-byte elements)
                auto store_block = [&](auto f32_tag, int c, const uint4 *pk, char *base) {
                    constexpr bool F32 = decltype(f32_tag)::value;
                    constexpr int EB = F32 ? 4 : 2;          // output element bytes
                    constexpr int HB = 32 * EB;              // a thread's half of a row's block
                    constexpr int NR = 2 * HB / RB;          // staging rounds per block
#pragma unroll
                    for (int q = 0; q < NR; ++q) {
                        // round q stages bytes [q RB, (q+1) RB) of the 16 rows' block
                        if constexpr (RB >= HB) {
                            if ((hh * HB) / RB == q) {
                                const int c0 = (hh * HB - q * RB) >> 4;
#pragma unroll
                                for (int j = 0; j < HB / 16; ++j)
                                    st_shared_v4(stg + lr_me * RB + (((c0 + j) ^ swz(lr_me)) << 4), pk[j]);
                            }
                        } else {
                            constexpr int W = HB / RB;   // rounds per half
                            if (q / W == hh) {
#pragma unroll
                                for (int j = 0; j < CPR; ++j)
                                    st_shared_v4(stg + lr_me * RB + ((j ^ swz(lr_me)) << 4), pk[(q % W) * CPR + j]);
                            }
                        }
                        __syncwarp();
#pragma unroll
                        for (int e = 0; e < RB / 32; ++e) {
                            const int f = e * 32 + lane, lr = f / CPR, ch = f % CPR;
                            const uint4 v = ld_shared_v4(stg + lr * RB + ((ch ^ swz(lr)) << 4));
                            const int grow = group * kGroupRows + 16 * qd + lr;
                            if (grow < rows_per_seq)
                                *reinterpret_cast<uint4 *>(base + ((long long)grow * kDc + c) * EB + q * RB + 16 * ch) = v;
                        }
                        __syncwarp();
                    }
                };
                auto drain = [&](auto f32_tag) {
                    constexpr bool F32 = decltype(f32_tag)::value;
                    char *base = F32 ? reinterpret_cast<char *>(a.part_o + slot * rows_per_seq * kDc)
                                     : reinterpret_cast<char *>(a.out + (long long)it.seq * rows_per_seq * kDc);
                    for (int c = 0; c < 512; c += 64) {
                        uint32_t ov[32];
                        sm100::tmem_ld16x2_32(o_base + c, ov);
                        sm100::tmem_wait_ld();
                        uint4 pk[F32 ? 8 : 4];
#pragma unroll
                        for (int j = 0; j < (F32 ? 8 : 4); ++j) {
                            if constexpr (F32) {
                                pk[j] = make_uint4(__float_as_uint(__uint_as_float(ov[4 * j]) * inv),
                                                   __float_as_uint(__uint_as_float(ov[4 * j + 1]) * inv),
                                                   __float_as_uint(__uint_as_float(ov[4 * j + 2]) * inv),
                                                   __float_as_uint(__uint_as_float(ov[4 * j + 3]) * inv));
                            } else {
                                pk[j] = make_uint4(pack_bf162(__uint_as_float(ov[8 * j]) * inv, __uint_as_float(ov[8 * j + 1]) * inv),
                                                   pack_bf162(__uint_as_float(ov[8 * j + 2]) * inv, __uint_as_float(ov[8 * j + 3]) * inv),
                                                   pack_bf162(__uint_as_float(ov[8 * j + 4]) * inv, __uint_as_float(ov[8 * j + 5]) * inv),
                                                   pack_bf162(__uint_as_float(ov[8 * j + 6]) * inv, __uint_as_float(ov[8 * j + 7]) * inv));
                            }
                        }
                        store_block(f32_tag, c, pk, base);
                    }
                };
                // A sequence cut into exactly two pieces: the piece that ends this
                // range (late) merges the next range's first piece (early, in slot
                // 2 c_last, finished long before) itself when that piece's rows of
                // this warp's quarter are written, and marks them merged so that
                // the combine leaves them; otherwise it writes its partial as any
                // cut piece.  The merge is the combine's arithmetic in the
                // combine's order, so the output bits do not depend on who merges.
                const int c_first = (it.seq_v + kSwitchTiles) / qv;
                const int c_last = (it.seq_v + kSwitchTiles + it.seq_t - 1) / qv;
                const bool two = a.merges && !it.complete && c_last == c_first + 1;
                int *qflag = a.flags + (it.seq * a.groups + group) * 4 + qd;   // early; merged at + B groups 4
                const int nq = a.B * a.groups * 4;
                bool merge = false;
                if (!kFp8 && two && rng == c_first) {   // (the FP8 kernel leaves every merge to the combine)
                    int rd = 0;
                    if (lane == 0) rd = ld_acquire_gpu(qflag);
                    merge = __shfl_sync(0xffffffffu, rd, 0) != 0;
                    __threadfence();
                }
                if (merge) {
                    const long long eslot = 2LL * c_last;
                    const float l2e = row_ok ? __ldcg(a.part_lse2 + eslot * rows_per_seq + grow_row) : -INFINITY;
                    const float mx = fmaxf(lse2, l2e);
                    const float w0 = lse2 == -INFINITY ? 0.f : exp2f(lse2 - mx);
                    const float w1 = l2e == -INFINITY ? 0.f : exp2f(l2e - mx);
                    float den = 0.f;
                    den += w0;
                    den += w1;
                    const float invd = den > 0.f ? 1.f / den : 0.f;
                    // the early piece's 16 rows of this quarter, one bulk copy per
                    // row into the stage memory (idle: this is the range's last
                    // segment, whose pages are all consumed), rows padded to
                    // 2,064 bytes so that the row-per-thread reads below spread
                    // over the banks
                    constexpr int kRowPad = kDc * 4 + 16;
                    uint8_t *erows = stages + qd * 16 * kRowPad;
                    const int r0 = group * kGroupRows + 16 * qd;
                    const int nr = max(0, min(16, rows_per_seq - r0));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        sm100::mbar_arrive_expect_tx(&early_in[qd], (uint32_t)(nr * kDc * 4));
                        for (int r = 0; r < nr; ++r)
                            sm100::bulk_load(erows + r * kRowPad, a.part_o + (eslot * rows_per_seq + r0 + r) * kDc, kDc * 4,
                                             &early_in[qd]);
                    }
                    ok = sm100::warp_wait(&early_in[qd], 0, abort_flag, a.err, lim);
                    if (!ok) {   // let the copies land before the CTA unwinds
                        volatile int no_abort = 0;
                        sm100::warp_wait(&early_in[qd], 0, &no_abort, a.err, lim > 200000000ull ? lim : 200000000ull);
                        break;
                    }
                    char *obase = reinterpret_cast<char *>(a.out + (long long)it.seq * rows_per_seq * kDc);
                    for (int c = 0; c < 512; c += 64) {
                        uint32_t ov[32];
                        sm100::tmem_ld16x2_32(o_base + c, ov);
                        sm100::tmem_wait_ld();
                        float ev[32];
                        const uint32_t esrc = sm100::smem_u32(erows + lr_me * kRowPad + (c + 32 * hh) * 4);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint4 v = ld_shared_v4(esrc + 16 * j);
                            ev[4 * j] = __uint_as_float(v.x);
                            ev[4 * j + 1] = __uint_as_float(v.y);
                            ev[4 * j + 2] = __uint_as_float(v.z);
                            ev[4 * j + 3] = __uint_as_float(v.w);
                        }
                        auto mv = [&](int i) {
                            return fmaf(w1, ev[i], fmaf(w0, __uint_as_float(ov[i]) * inv, 0.f)) * invd;
                        };
                        uint4 pk[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            pk[j] = make_uint4(pack_bf162(mv(8 * j), mv(8 * j + 1)), pack_bf162(mv(8 * j + 2), mv(8 * j + 3)),
                                               pack_bf162(mv(8 * j + 4), mv(8 * j + 5)), pack_bf162(mv(8 * j + 6), mv(8 * j + 7)));
                        store_block(std::false_type{}, c, pk, obase);
                    }
                    if (row_ok && srow && a.out_lse) a.out_lse[orow] = den > 0.f ? (mx + log2f(den)) * kLn2 : -INFINITY;
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) atomicExch(qflag + nq, 1);
                } else {
                    if (it.complete)
                        drain(std::false_type{});
                    else
                        drain(std::true_type{});
                    if (row_ok && srow) {
                        if (it.complete) {
                            if (a.out_lse) a.out_lse[orow] = lse2 * kLn2;
                        } else {
                            a.part_lse2[slot * rows_per_seq + grow_row] = lse2;
                        }
                    }
                    if (!kFp8 && two && rng == c_first && lane == 0)
                        atomicAdd(a.flags + 2 * nq, 1);   // this quarter falls back to the combine
                    if (!kFp8 && two && rng == c_last) {
                        // the early piece's rows of this quarter are written
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) atomicExch(qflag, 1);
                    }
                }
                __syncwarp();
            }
            it.advance();
        }
    }

    // ------------------------------------------------------------ teardown
    sm100::pdl_trigger();   // the combine may start launching
    sm100::tc_fence_before();
    __syncthreads();
    if (warp >= 1 && warp < 8) {
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
}

}  // namespace mla
