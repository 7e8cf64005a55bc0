// dec_common.cuh -- pieces shared by the decode kernels: the argument block,
// the walk over a range of the (sequence, tile) list, small device helpers
// and the plan kernel that cuts the batch's tiles into equal ranges.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace mla {

constexpr int kGroupRows = 64;                // rows of one work unit (the MMA M dimension)
constexpr int kSwitchTiles = 4;               // the planning weight of a sequence start, in tiles
constexpr int kMaxRanges = 148;               // ranges per row group at most (= CTAs / groups)
constexpr float kRescaleThreshold = 8.0f;     // lazy rescale of the running max, log2 units

struct DecArgs {
    const bf16 *q_abs;    // [B*s][H][576]
    const int32_t *block_table;
    const int32_t *seq_lens;
    int32_t *plan;        // written by CTA 0 for the combine (plan_range)
    int *flags;           // per (sequence, row group, warp quarter): [0, n) early piece written,
                          // [n, 2n) merged by the late piece's CTA (n = B * groups * 4); [2n] the
                          // combine's work count (0: nothing left to merge)
    bf16 *out;
    float *out_lse;
    float *part_o;        // [2*ranges][s*H][512] fp32
    float *part_lse2;     // [2*ranges][s*H]
    uint32_t *err;
    unsigned long long limit_ns;
    int stall_tile;       // test hook: the page load of this tile of every range is never issued (-1: none)
    int merges;           // merge two-piece sequences in the decode kernel (0: the combine merges all)
    const float *scales;  // FP8 cache only: [num_blocks][64][2] fp32 per-part scales
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

// Walks a range of the (sequence, tile) list one tile at a time.  Sequence
// r holds tiles [a_r, a_r + ceil(L_r / 64)); the walk starts in sequence r0,
// whose first tile a0 and virtual start v0 the range's plan gives, and takes
// the later starts from the sequence lengths.  seq_a, seq_t and seq_v are the
// current segment's sequence's first tile, tile count and virtual start.
struct TileIter {
    const int32_t *sl;
    int max_tok, n, pos, hi, r, ar, vr;
    int seq, t0, t1, seg, tt, k, seq_a, seq_t, seq_v;
    bool complete, ok;
    __device__ int tiles(int b) const
    {
        int L = sl[b];
        L = L < 0 ? 0 : min(L, max_tok);
        return (L + kBlock - 1) / kBlock;
    }
    __device__ bool next_seg()
    {
        if (pos >= hi) return false;
        int t;
        for (;;) {
            if (r >= n) return false;
            t = tiles(r);
            if (ar + t > pos) break;
            ar += t;   // an empty sequence, or one that ends before pos
            vr += t > 0 ? t + kSwitchTiles : 0;
            ++r;
        }
        const int e = ar + t, end = min(hi, e);
        seq = r; t0 = pos - ar; t1 = end - ar;
        seq_a = ar; seq_t = t; seq_v = vr;
        complete = (pos == ar) && (end == e);
        pos = end; ar = e; vr += t + kSwitchTiles; ++r; ++seg;
        return true;
    }
    __device__ void init(const int32_t *seq_lens, int max_blocks, int n_, int lo, int hi_, int r0, int a0, int v0)
    {
        sl = seq_lens; max_tok = max_blocks * kBlock; n = n_; pos = lo; hi = hi_; seg = -1; k = 0;
        r = r0; ar = a0; vr = v0;
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

// Warp-uniform bounded wait until *cnt >= target (a count other warps of the
// CTA raise with atomicAdd after their tcgen05 fences); lane 0 polls, and the
// verdict is broadcast.  Same give-up rules as sm100::mbar_wait.
__device__ __forceinline__ bool wait_count(volatile int *cnt, int target, volatile int *abort, uint32_t *err,
                                           unsigned long long limit_ns)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0 && *cnt < target) {
        const uint64_t t0 = sm100::globaltimer_ns();
        for (uint32_t i = 1; *cnt < target; ++i) {
            if ((i & 255u) == 0) {
                if (*abort) { ok = 0; break; }
                if (sm100::globaltimer_ns() - t0 > limit_ns) {
                    set_error(err, MLA_DEVERR_TIMEOUT);
                    *abort = 1;
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence_block();
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}


__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
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

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// -------------------------------------------------------------------- plan
// One warp of every decode CTA: the CTA's range of the batch's (sequence,
// tile) list.  The list holds the ceil(L_b / 64) tiles of every sequence b
// (its last query sees all L_b tokens) in sequence order.  Ranges are cut by
// cost: every non-empty sequence also weighs kSwitchTiles virtual tiles
// placed before its first tile (what a range pays to start a sequence: the
// previous sequence's epilogue and the next one's queries, about four tiles'
// time on every shape measured), and the ranges split the virtual list into
// equal parts of Qv = ceil(VT / ranges) virtual tiles.  A virtual position v
// inside sequence b (virtual start VA_b, real start A_b) maps to the real
// tile A_b + max(0, v - VA_b - kSwitchTiles); range r covers the real tiles
// [real(r Qv), real(min((r + 1) Qv, VT))), real(VT) = the total.  Lane l
// takes sequences [l per, (l+1) per); shuffle scans give the prefix sums.
// out = {first tile, end tile, the sequence holding the first tile, that
// sequence's first tile, Qv, that sequence's virtual start} (the third,
// fourth and sixth only when the range is not empty).
// With `publish` (CTA 0 of the grid), the warp also stores what the combine
// kernel reads, and flags invalid lengths:
//   plan[0] = Qv, plan[1] = total tiles, plan[2] = ranges, plan[3] = kSwitchTiles,
//   plan[4 + b] = first tile of sequence b (b = 0..B),
//   plan[5 + B] = n, the number of sequences the combine finishes (those
//   whose tiles span more than one range, and those with no tile), listed in
//   sequence order as int4 {b, VA_b, tiles, clamped length} from int
//   plan_list_off(B).  Sequence b's tiles lie in ranges
//   c0 = (VA_b + kSwitchTiles) / Qv .. c1 = (VA_b + kSwitchTiles + t_b - 1) / Qv.
__host__ __device__ inline int plan_list_off(int B) { return (B + 9) & ~3; }   // 16-byte aligned, after plan[5 + B]
__host__ __device__ inline int plan_ints(int B) { return plan_list_off(B) + 4 * B; }

// `work` (with `publish`): raised by the number of listed sequences the
// decode kernel does not merge itself (empty ones, those cut into three or
// more pieces, and with !merge_two the two-piece ones too).
__device__ void plan_range(const int32_t *seq_lens, int B, int s, int max_blocks, int ranges, int rng, bool publish,
                           bool merge_two, int32_t *plan, int *work, uint32_t *err, int *out)
{
    const int lane = threadIdx.x & 31;
    const int max_tok = max_blocks * kBlock;
    const int per = (B + 31) / 32;
    const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
    auto len_of = [&](int b) {
        const int L = seq_lens[b];
        return L < 0 ? 0 : min(L, max_tok);
    };
    int sum_t = 0, sum_v = 0;
    for (int b = b0; b < b1; ++b) {
        const int L = seq_lens[b];
        // out of range, or some query sees no key
        if (publish && (L < 0 || L > max_tok || L < s)) set_error(err, MLA_DEVERR_SEQ_LEN);
        const int t = (len_of(b) + kBlock - 1) / kBlock;
        sum_t += t;
        sum_v += t > 0 ? t + kSwitchTiles : 0;
    }
    int inc_t = sum_t, inc_v = sum_v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int vt = __shfl_up_sync(0xffffffffu, inc_t, o), vv = __shfl_up_sync(0xffffffffu, inc_v, o);
        if (lane >= o) {
            inc_t += vt;
            inc_v += vv;
        }
    }
    const int total = __shfl_sync(0xffffffffu, inc_t, 31), vtot = __shfl_sync(0xffffffffu, inc_v, 31);
    const int qv = vtot > 0 ? (vtot + ranges - 1) / ranges : 1;
    const int v_lo = rng * qv, v_hi = min(v_lo + qv, vtot);
    if (lane == 0) {   // a boundary at or past the end of the list
        out[0] = total;
        out[1] = total;
        out[4] = qv;
    }
    __syncwarp();
    int run_t = inc_t - sum_t, run_v = inc_v - sum_v;
    for (int b = b0; b < b1; ++b) {
        const int t = (len_of(b) + kBlock - 1) / kBlock;
        const int w = t > 0 ? t + kSwitchTiles : 0;
        if (v_lo >= run_v && v_lo < run_v + w) {
            out[0] = run_t + max(0, v_lo - run_v - kSwitchTiles);
            out[2] = b;
            out[3] = run_t;
            out[5] = run_v;
        }
        if (v_hi >= run_v && v_hi < run_v + w) out[1] = run_t + max(0, v_hi - run_v - kSwitchTiles);
        if (publish) plan[4 + b] = run_t;
        run_t += t;
        run_v += w;
    }
    if (publish) {
        if (lane == 0) {
            plan[0] = qv;
            plan[1] = total;
            plan[2] = ranges;
            plan[3] = kSwitchTiles;
            plan[4 + B] = total;
        }
        // the combine's list: sequences spanning more than one range, or with no tile
        auto listed = [&](int va, int t) {
            return t == 0 || (va + kSwitchTiles) / qv != (va + kSwitchTiles + t - 1) / qv;
        };
        int cnt = 0, left = 0;
        run_v = inc_v - sum_v;
        for (int b = b0; b < b1; ++b) {
            const int t = (len_of(b) + kBlock - 1) / kBlock;
            if (listed(run_v, t)) {
                ++cnt;
                const int pieces = t > 0 ? (run_v + kSwitchTiles + t - 1) / qv - (run_v + kSwitchTiles) / qv + 1 : 0;
                left += (pieces == 2 && merge_two) ? 0 : 1;
            }
            run_v += t > 0 ? t + kSwitchTiles : 0;
        }
        if (left) atomicAdd(work, left);
        int ci = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ci, o);
            if (lane >= o) ci += v;
        }
        int4 *list = reinterpret_cast<int4 *>(plan + plan_list_off(B));
        int at = ci - cnt;
        run_v = inc_v - sum_v;
        for (int b = b0; b < b1; ++b) {
            const int L = len_of(b);
            const int t = (L + kBlock - 1) / kBlock;
            if (listed(run_v, t)) list[at++] = make_int4(b, run_v, t, L);
            run_v += t > 0 ? t + kSwitchTiles : 0;
        }
        if (lane == 31) plan[5 + B] = ci;
    }
}


// ------------------------------------------------------------------ combine
// Sequences cut by range ends are merged by log-sum-exp; sequences one range
// finished are already in place; queries with no visible key get a zero
// latent and lse = -inf.  Only the sequences plan_range lists (cut by a range
// end, or with no tile) are visited, in blocks of 8 rows: a CTA takes one
// block of one listed sequence at a time.  Thread 0 copies the block's partial
// rows into shared memory, up to 4 pieces per round (the 8 rows of a piece
// are contiguous: one bulk copy of 16 KB), while each warp loads the
// log2-sum-exps of its row (lane i: piece i; pieces past 32 only enter the
// max).  Warp w then merges row 8 blk + w from shared memory, lane l owning
// the float4 columns l, 32 + l, 64 + l and 96 + l, so that the shared-memory
// reads are conflict-free and the output stores contiguous across the warp.
// Pieces are summed in range order.  Every partial slot lies in
// [2 c0, 2 c1 + 1] with c1 < ranges (plan_range gives c0, c1 and the slots).
constexpr int kCombineWarps = 8;                  // rows per block
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombinePieces = 4;                 // pieces per bulk round
constexpr int kCombineBuf = kCombinePieces * kCombineWarps * kDc * 4;   // 64 KB
constexpr int kCombineSmem = kCombineBuf + 16;
constexpr int kCombineCtasPerSm = 3;

__host__ __device__ inline int combine_blocks(int B, int s, int H)
{
    return B * ((s * H + kCombineWarps - 1) / kCombineWarps);
}


__global__ void __launch_bounds__(kCombineThreads, kCombineCtasPerSm)
dec_combine_kernel(const int32_t *plan, const int *flags, const float *part_o, const float *part_lse2, int B, int s,
                   int H, bf16 *__restrict__ out, float *__restrict__ out_lse, uint32_t *err,
                   unsigned long long limit_ns)
{
    extern __shared__ __align__(128) uint8_t cb_smem[];
    const float4 *buf = reinterpret_cast<const float4 *>(cb_smem);
    uint64_t *bar = reinterpret_cast<uint64_t *>(cb_smem + kCombineBuf);
    if (threadIdx.x == 0) {
        sm100::mbar_init(bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    // The decode kernel's partials, plan and flags are complete from here on.
    // This kernel starts while the decode kernel still runs, so what that
    // kernel writes is read only after the wait and only through L2 (__ldcg,
    // bulk copies), never through the read-only path, and the pointers carry
    // no __restrict__: either would let a load be served early or stale.
    sm100::pdl_wait();
    const int groups = (s * H + kGroupRows - 1) / kGroupRows;
    const int rows = s * H, nbr = (rows + kCombineWarps - 1) / kCombineWarps;
    const int4 *list = reinterpret_cast<const int4 *>(plan + plan_list_off(B));
    // L2 round trips follow one another here, so the loads go out in as few
    // rounds as they can: first the work count, the plan's quota and list
    // length and this CTA's first list entry (the grid has at most B nbr
    // CTAs, so the entry lies in the list area even past the list's end)
    const int work = __ldcg(flags + 2 * B * groups * 4);
    const int qv = __ldcg(plan), pw = __ldcg(plan + 3), nlist = __ldcg(plan + 5 + B);
    int4 seq = __ldcg(list + blockIdx.x / nbr);
    if (work == 0) return;   // the decode kernel merged every cut sequence
    const int nblk = nlist * nbr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int no_abort = 0;
    uint32_t phase = 0;
    auto copy_pieces = [&](int i0, int np, int slot0, int c0, int rr0, int nr) {
        if (threadIdx.x == 0) {
            sm100::mbar_arrive_expect_tx(bar, (uint32_t)(np * nr * kDc * 4));
            for (int u = 0; u < np; ++u)
                sm100::bulk_load(cb_smem + u * (kCombineWarps * kDc * 4),
                                 part_o + ((long long)(i0 + u == 0 ? slot0 : 2 * (c0 + i0 + u)) * rows + rr0) * kDc,
                                 (uint32_t)(nr * kDc * 4), bar);
        }
    };
    for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
        const int li = blk / nbr, rb = blk - li * nbr;
        if (blk != blockIdx.x) seq = __ldcg(list + li);
        const int b = seq.x, va = seq.y, tb = seq.z, L = seq.w;
        // the ranges holding the sequence's first and last tiles; the piece in
        // range c0 is that range's first segment only if the range starts with
        // the sequence (slot 2 c0), else its last (2 c0 + 1); every later piece
        // is its range's first segment (slot 2 c)
        const int c0 = tb > 0 ? (va + pw) / qv : 0, c1 = tb > 0 ? (va + pw + tb - 1) / qv : 0;
        const bool split = tb > 0 && c0 != c1;
        const int slot0 = 2 * c0 + (c0 * qv < va ? 1 : 0);
        const int rr0 = rb * kCombineWarps, nr = min(kCombineWarps, rows - rr0);
        const int rr = rr0 + warp;
        const bool row_ok = warp < nr;
        const bool visible = L - s + rr / H + 1 > 0;   // query rr / H sees some key
        const long long orow = (long long)b * rows + rr;
        uint2 *dst = reinterpret_cast<uint2 *>(out + orow * kDc) + lane;   // + 32 e: columns 4 (32 e + lane) ..
        const int n = c1 - c0 + 1;
        auto lse_of = [&](int i) { return __ldcg(part_lse2 + (long long)(i == 0 ? slot0 : 2 * (c0 + i)) * rows + rr); };
        const bool merge = split && row_ok && visible;
        // the second round: the first pieces' rows, their log2-sum-exps and
        // the merged flag together
        if (split) {
            __syncthreads();   // every warp is done with the previous block's rows
            copy_pieces(0, min(kCombinePieces, n), slot0, c0, rr0, nr);
        }
        const float l2_lane = (merge && lane < n) ? lse_of(lane) : -INFINITY;
        // a two-piece sequence whose late piece merged this block's quarter
        // itself (the decode kernel's epilogue) is already in place
        const int merged = (split && c1 == c0 + 1)
                               ? __ldcg(flags + B * groups * 4 + (b * groups + rr0 / kGroupRows) * 4 + (rr0 % kGroupRows) / 16)
                               : 0;
        if (merged) {
            // the copies land before their buffer is used again
            const bool ok = sm100::mbar_wait(bar, phase, &no_abort, err, limit_ns);
            if (!__syncthreads_and(ok)) {
                sm100::mbar_wait(bar, phase, &no_abort, err, limit_ns > 200000000ull ? limit_ns : 200000000ull);
                return;
            }
            phase ^= 1;
            continue;
        }
        if (!split) {
            // a sequence with no tile: every query row is zero
            if (row_ok && !visible) {
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[32 * e] = make_uint2(0, 0);
                if (lane == 0 && out_lse) out_lse[orow] = -INFINITY;
            }
            continue;   // uniform: the whole block belongs to one sequence
        }
        float M = l2_lane;
        if (merge)
            for (int i = lane + 32; i < n; i += 32) M = fmaxf(M, lse_of(i));
        M = warp_max(M);
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        float den = 0.f;
        for (int i0 = 0; i0 < n; i0 += kCombinePieces) {
            const int np = min(kCombinePieces, n - i0);
            if (i0 > 0) {
                __syncthreads();   // every warp is done with the previous round's rows
                copy_pieces(i0, np, slot0, c0, rr0, nr);
            }
            bool ok = sm100::mbar_wait(bar, phase, &no_abort, err, limit_ns);
            if (!__syncthreads_and(ok)) {
                // a copy that never lands: let the copies in flight finish
                // before the CTA leaves, and give up
                sm100::mbar_wait(bar, phase, &no_abort, err, limit_ns > 200000000ull ? limit_ns : 200000000ull);
                return;
            }
            phase ^= 1;
            if (merge) {
                for (int u = 0; u < np; ++u) {
                    const int i = i0 + u;
                    const float l2 = i < 32 ? __shfl_sync(0xffffffffu, l2_lane, i) : lse_of(i);
                    const float wgt = (l2 == -INFINITY) ? 0.f : exp2f(l2 - M);
                    den += wgt;
                    const float4 *row = buf + (u * kCombineWarps + warp) * (kDc / 4) + lane;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 v = row[32 * e];
                        acc[4 * e] = fmaf(wgt, v.x, acc[4 * e]);
                        acc[4 * e + 1] = fmaf(wgt, v.y, acc[4 * e + 1]);
                        acc[4 * e + 2] = fmaf(wgt, v.z, acc[4 * e + 2]);
                        acc[4 * e + 3] = fmaf(wgt, v.w, acc[4 * e + 3]);
                    }
                }
            }
        }
        if (!row_ok) continue;
        if (!visible) {
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[32 * e] = make_uint2(0, 0);
            if (lane == 0 && out_lse) out_lse[orow] = -INFINITY;
            continue;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            dst[32 * e] = make_uint2(pack_bf162(acc[4 * e] * inv, acc[4 * e + 1] * inv),
                                     pack_bf162(acc[4 * e + 2] * inv, acc[4 * e + 3] * inv));
        if (lane == 0 && out_lse) out_lse[orow] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
    }
}


}  // namespace mla
