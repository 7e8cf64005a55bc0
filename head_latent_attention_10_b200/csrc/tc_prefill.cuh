// tc_prefill.cuh -- prefill of a chunk of s new query tokens per sequence in
// the expanded form (sm_100a): every head's keys and values are materialised
// from the cached latents,
//   k_{j,i} = [U^K_i c_j ; k^R_j],  v_{j,i} = U^V_i c_j,
//   o_{t,i} = sum_j softmax_j(q_{t,i} . k_{j,i} * scale) v_{j,i}
// (DeepSeek-V2 paper review, section 2: k^C = W^UK c^KV, v^C = W^UV c^KV;
// section 3: the decoupled RoPE key shared by the heads and the scale
// 1/sqrt(d_h + d_R); DeepSeek-V3 report summary, Method 1:
// k_{t,i} = [k^C_{t,i}; k^R_t]).  Query t of a sequence of L cached tokens
// sits at position L - s + t and sees the keys j <= L - s + t.
//
// With many queries per sequence the expanded form costs fewer flops than the
// absorbed one (2 (192 + 128) per query, key and head against 2 (576 + 512)),
// and the step is bound by the tensor cores: a FlashAttention-style loop on
// tcgen05.  CTA (128-query tile, head i, sequence b), the tile as MMA M = 128,
// streams 128-key tiles of K = [K^C | k^R] and V^C:
//   S(k) = Q K_k^T    N=128, K=192: 12 MMAs, Q read from TMEM
//   P(k) = exp2(S(k) scale log2 e - m)           bf16, one thread per query row
//   O   += P(k) V_k   N=128, K=128: 8 MMAs, P read from TMEM
// TMEM (512 columns): S(k) in buffer k % 2 (columns 0-127, 128-255), P(k)
// written over the first 64 columns of its S buffer, O 256-383, Q 384-479
// (192 bf16 per row, written by the softmax warps at the start).
// With Q and P in TMEM, shared memory holds only key and value tiles: a
// 3-slot ring of K tiles (K^C 0-63, K^C 64-127, k^R; 48 KB each) and a 2-slot
// ring of V tiles (V^C 0-63, 64-127; 32 KB each), 208 KB, each ring fed by
// its own loader warp (0: K, 6: V) so that neither waits behind the other.
// Warp 1 keeps the logits one tile ahead: S(0), S(1), then S(k+2) into
// buffer k % 2 once P(k) V_k has completed (S(k+2) overwrites P(k)), so the
// softmax warps (2-5) find the next tile's logits ready when they finish this
// one; warp 7 issues P(k) V_k as soon as P(k) is written.  Two issuing
// threads, because a thread's tcgen05.mma issue blocks while the tensor pipe
// is busy, and one thread would hold P(k+1) V back behind S(k+2).  The causal mask applies to
// the tiles that straddle the diagonal; lazy rescaling as in the decode (O
// is rescaled in TMEM only when the running max grows by more than 8, after
// the previous P V has retired).  Every wait is bounded; no TMA load uses
// cluster multicast.
#pragma once

#include "dec_common.cuh"

namespace mla {

constexpr int kPfThreads = 256;                        // warps: 0 K loads, 1 S MMAs, 2-5 softmax, 6 V loads, 7 P V MMAs
constexpr int kPfChunk = 128 * 128;                    // [128 rows][64 bf16], 128-byte swizzle: 16 KB
constexpr int kPfKSlots = 3, kPfVSlots = 2;
constexpr int kPfOffK = 0;                             // K slot j: chunks 3j .. 3j+2
constexpr int kPfOffV = kPfKSlots * 3 * kPfChunk;      // V slot j: 2 chunks
constexpr int kPfOffBar = kPfOffV + kPfVSlots * 2 * kPfChunk;   // 212,992
constexpr int kPfSmem = kPfOffBar + 256 + 1024;        // barriers, alignment slack
constexpr uint32_t kPfTmS = 0, kPfTmO = 256, kPfTmQ = 384;   // S/P buffers at 0 and 128

// Tensor maps of one call.  Rows of K^C, V^C and the gathered latents are
// [B * Lpad] long (sequence b at rows b * Lpad ..); outputs are [B][s][H][128]
// with the sequence as the outermost dimension, so a 128-row tile is clipped
// at the end of its own sequence.
struct PrefillMaps {
    CUtensorMap kc;    // K^C   {128, H, B Lpad}, box {64, 1, 128}
    CUtensorMap vc;    // V^C   {128, H, B Lpad}, box {64, 1, 128}
    CUtensorMap kr;    // gathered rows {576, B Lpad, 1}, box {64, 128, 1}, read at x = 512
    CUtensorMap out;   // out   {128, H, s, B}, box {64, 1, 128, 1}
};

struct PrefillArgs {
    const bf16 *q_nope;           // [B*s][H][128]
    const bf16 *q_rot;            // [B*s][H][64], rotated
    const int32_t *seq_lens;
    int s, H, lpad, l_cap;        // l_cap: the largest valid sequence length
    float scale_log2;
    float *out_lse;               // [B][s][H] or null
    uint32_t *err;
    unsigned long long limit_ns;
};

// Number of 128-key tiles the query tile [q0, q0 + 128) of a sequence of L
// tokens sees (0 if the tile holds no query).
__device__ __forceinline__ int prefill_tiles(int q0, int s, int L)
{
    if (q0 >= s) return 0;
    const int last_q = min(q0 + 128, s) - 1;
    return (L - s + last_q) / 128 + 1;
}

__device__ __forceinline__ bool prefill_valid(int L, int s, int l_cap) { return L >= s && L <= l_cap; }

__global__ void __launch_bounds__(kPfThreads, 1)
tc_prefill_kernel(const __grid_constant__ PrefillMaps maps, const PrefillArgs a)
{
    extern __shared__ uint8_t pf_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kPfOffBar);
    uint64_t *k_full = bars;            // [3] K slot loaded
    uint64_t *k_free = bars + 3;        // [3] S of the slot's tile done
    uint64_t *v_full = bars + 6;        // [2] V slot loaded
    uint64_t *v_free = bars + 8;        // [2] P V of the slot's tile done
    uint64_t *q_ready = bars + 10;      // Q in TMEM (4 softmax warps)
    uint64_t *s_full = bars + 11;       // [2] S(k) in buffer k % 2
    uint64_t *p_full = bars + 13;       // [2] P(k) in TMEM and O rescaled (4 softmax warps)
    uint64_t *pv_done = bars + 15;      // [2] P(k) V_k done
    uint64_t *done = bars + 17;         // both issuers' last MMAs done (teardown)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 18);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 19);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = gridDim.x - 1 - blockIdx.x;   // the longest rows of the causal triangle first
    const int head = blockIdx.y, b = blockIdx.z;
    const int q0 = 128 * qb;
    const int L = a.seq_lens[b];
    const bool valid = prefill_valid(L, a.s, a.l_cap);
    const int nk = valid ? prefill_tiles(q0, a.s, L) : 0;
    const int row0 = b * a.lpad;                 // this sequence's first key row

    if (threadIdx.x == 0) {
        for (int i = 0; i < kPfKSlots; ++i) {
            sm100::mbar_init(&k_full[i], 1);
            sm100::mbar_init(&k_free[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&v_full[i], 1);
            sm100::mbar_init(&v_free[i], 1);
            sm100::mbar_init(&p_full[i], 4);
            sm100::mbar_init(&pv_done[i], 1);
        }
        sm100::mbar_init(q_ready, 4);
        sm100::mbar_init(&s_full[0], 1);
        sm100::mbar_init(&s_full[1], 1);
        sm100::mbar_init(done, 2);
        *abort_flag = 0;
        sm100::fence_mbar_init();
        sm100::prefetch_tensormap(&maps.kc);
        sm100::prefetch_tensormap(&maps.vc);
        sm100::prefetch_tensormap(&maps.kr);
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

    if (warp == 0) {
        // ----------------------------------------------------------- K loads
        if (lane == 0 && nk > 0) {
            int issued = 0;
            for (int k = 0; k < nk; ++k) {
                const int sl = k % kPfKSlots;
                if (k >= kPfKSlots &&
                    !sm100::mbar_wait(&k_free[sl], ((k / kPfKSlots) - 1) & 1, abort_flag, a.err, lim))
                    break;
                uint8_t *dst = smem + kPfOffK + 3 * sl * kPfChunk;
                const int r = row0 + 128 * k;
                sm100::mbar_arrive_expect_tx(&k_full[sl], 3 * kPfChunk);
                sm100::tma_load_3d(&maps.kc, &k_full[sl], dst, 0, head, r);
                sm100::tma_load_3d(&maps.kc, &k_full[sl], dst + kPfChunk, 64, head, r);
                sm100::tma_load_3d(&maps.kr, &k_full[sl], dst + 2 * kPfChunk, kDc, r, 0);
                issued = k + 1;
            }
            if (*abort_flag) {   // let the copies in flight land before the CTA can exit
                volatile int no_abort = 0;
                for (int k = issued - kPfKSlots < 0 ? 0 : issued - kPfKSlots; k < issued; ++k)
                    sm100::mbar_wait(&k_full[k % kPfKSlots], (k / kPfKSlots) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 6) {
        // ----------------------------------------------------------- V loads
        if (lane == 0 && nk > 0) {
            int issued = 0;
            for (int k = 0; k < nk; ++k) {
                const int sl = k & 1;
                if (k >= 2 && !sm100::mbar_wait(&v_free[sl], ((k >> 1) - 1) & 1, abort_flag, a.err, lim)) break;
                uint8_t *dst = smem + kPfOffV + 2 * sl * kPfChunk;
                const int r = row0 + 128 * k;
                sm100::mbar_arrive_expect_tx(&v_full[sl], 2 * kPfChunk);
                sm100::tma_load_3d(&maps.vc, &v_full[sl], dst, 0, head, r);
                sm100::tma_load_3d(&maps.vc, &v_full[sl], dst + kPfChunk, 64, head, r);
                issued = k + 1;
            }
            if (*abort_flag) {
                volatile int no_abort = 0;
                for (int k = issued - 2 < 0 ? 0 : issued - 2; k < issued; ++k)
                    sm100::mbar_wait(&v_full[k & 1], (k >> 1) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 1 || warp == 7) {
        // ------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t idesc_s = sm100::idesc_bf16(128, 128, 0, 0);
            const uint32_t idesc_o = sm100::idesc_bf16(128, 128, 0, 1);
            bool ok = nk == 0 || sm100::mbar_wait(q_ready, 0, abort_flag, a.err, lim);
            if (warp == 1) {
                // S(k) into buffer k % 2
                auto issue_s = [&](int k) -> bool {
                    const int sl = k % kPfKSlots;
                    if (!sm100::mbar_wait(&k_full[sl], (k / kPfKSlots) & 1, abort_flag, a.err, lim)) return false;
                    sm100::tc_fence_after();
                    const uint32_t ka = sm100::smem_u32(smem + kPfOffK + 3 * sl * kPfChunk);
#pragma unroll
                    for (int step = 0; step < 12; ++step)      // q^C 0-63, q^C 64-127, q^R
                        sm100::umma_ts(tmem + kPfTmS + 128 * (k & 1), tmem + kPfTmQ + 8 * step,
                                       sm100::desc_kmajor(ka + (step >> 2) * kPfChunk + (step & 3) * 32, 128,
                                                          sm100::kSw128),
                                       idesc_s, step > 0);
                    sm100::umma_commit(&s_full[k & 1]);
                    sm100::umma_commit(&k_free[sl]);
                    return true;
                };
                if (ok && nk > 0) ok = issue_s(0);
                if (ok && nk > 1) ok = issue_s(1);
                // S(k+2) overwrites P(k): that P V must have completed
                for (int k = 0; ok && k + 2 < nk; ++k)
                    ok = sm100::mbar_wait(&pv_done[k & 1], (k >> 1) & 1, abort_flag, a.err, lim) && issue_s(k + 2);
            } else {
                for (int k = 0; ok && k < nk; ++k) {
                    const int pb = k & 1;
                    ok = sm100::mbar_wait(&p_full[pb], (k >> 1) & 1, abort_flag, a.err, lim) &&
                         sm100::mbar_wait(&v_full[pb], (k >> 1) & 1, abort_flag, a.err, lim);
                    if (!ok) break;
                    sm100::tc_fence_after();
                    const uint64_t vd =
                        sm100::desc_mnmajor_sw128(sm100::smem_u32(smem + kPfOffV + 2 * pb * kPfChunk), kPfChunk);
#pragma unroll
                    for (int kq = 0; kq < 8; ++kq)           // 16 keys per MMA: 8 TMEM columns of P
                        sm100::umma_ts(tmem + kPfTmO, tmem + kPfTmS + 128 * pb + 8 * kq,
                                       vd + (uint64_t)((kq * 2048) >> 4), idesc_o, (k > 0 || kq > 0) ? 1u : 0u);
                    sm100::umma_commit(&pv_done[pb]);
                    sm100::umma_commit(&v_free[pb]);
                }
            }
            sm100::umma_commit(done);
        }
        __syncwarp();
    } else if (warp >= 2 && warp <= 5) {
        // ------------------------------------------------------ softmax
        // warp w owns TMEM lane quarter w % 4; thread = query row r
        const int qd = warp & 3;
        const int r = 32 * qd + lane, t = q0 + r;
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        const uint32_t tm_s = tmem + lane_off + kPfTmS;
        const uint32_t tm_o = tmem + lane_off + kPfTmO, tm_q = tmem + lane_off + kPfTmQ;
        const bool has_row = t < a.s;
        const int nvis = has_row ? L - a.s + t + 1 : 0;   // keys [0, nvis) visible to row t
        bool ok = true;
        if (nk > 0) {
            // this row's query [q^C | rotated q^R] into TMEM (192 bf16 = 96 columns)
            const long long qrow = ((long long)b * a.s + (has_row ? t : 0)) * a.H + head;
            const uint4 *qc = reinterpret_cast<const uint4 *>(a.q_nope + qrow * kDh);
            const uint4 *qr = reinterpret_cast<const uint4 *>(a.q_rot + qrow * kDr);
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                uint4 v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = 8 * c + e;   // 16-byte unit of the 384-byte row
                    v[e] = !has_row ? make_uint4(0, 0, 0, 0) : (u < 16 ? __ldg(qc + u) : __ldg(qr + (u - 16)));
                }
                sm100::tmem_st32(tm_q + 32 * c, reinterpret_cast<const uint32_t *>(v));
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(q_ready);
        }
        float m_run = -INFINITY, l_run = 0.f;
        for (int k = 0; ok && k < nk; ++k) {
            const int pb = k & 1;
            ok = sm100::warp_wait(&s_full[pb], (k >> 1) & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            uint32_t x[128];
#pragma unroll
            for (int c = 0; c < 128; c += 32) sm100::tmem_ld32(tm_s + 128 * pb + c, x + c);
            sm100::tmem_wait_ld();
            const int key0 = 128 * k;
            if (key0 + 128 > nvis) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (key0 + c >= nvis) x[c] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 4)
                mx = fmaxf(mx, fmaxf(fmaxf(__uint_as_float(x[c]), __uint_as_float(x[c + 1])),
                                     fmaxf(__uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]))));
            const float mt = mx * a.scale_log2;
            const bool grow = (mt != -INFINITY) && (m_run == -INFINITY || mt > m_run + kRescaleThreshold);
            const bool rescale = grow && m_run != -INFINITY;
            const float m_new = grow ? mt : m_run;
            const float corr = rescale ? ex2(m_run - m_new) : 1.f;
            l_run *= corr;
            m_run = m_new;
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = ex2(fmaf(__uint_as_float(x[2 * c]), a.scale_log2, -mu));
                const float p1 = ex2(fmaf(__uint_as_float(x[2 * c + 1]), a.scale_log2, -mu));
                lsum += p0 + p1;
                x[c] = pack_bf162(p0, p1);
            }
            l_run += lsum;
            // P(k) over the first 64 columns of S(k), already read by this thread
            sm100::tmem_st32(tm_s + 128 * pb, x);
            sm100::tmem_st32(tm_s + 128 * pb + 32, x + 32);
            if (__any_sync(0xffffffffu, rescale)) {
                // O holds the tiles before k: let P(k-1) V_{k-1} retire, then
                // scale this thread's row in place
                ok = sm100::warp_wait(&pv_done[(k - 1) & 1], ((k - 1) >> 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    uint32_t ov[32];
                    sm100::tmem_ld32(tm_o + c, ov);
                    sm100::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
                    sm100::tmem_st32(tm_o + c, ov);
                }
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            __syncwarp();
            if (lane == 0) sm100::mbar_arrive(&p_full[pb]);
        }
        // epilogue: O / l as bf16, staged over K slot 0 (free once the last
        // P V completed, which follows every S MMA) as two [128 rows][128 B]
        // chunks with 128-byte swizzle, stored with TMA
        if (ok && nk > 0) {
            ok = sm100::warp_wait(&pv_done[(nk - 1) & 1], ((nk - 1) >> 1) & 1, abort_flag, a.err, lim);
            sm100::tc_fence_after();
        }
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint8_t *stage = smem + kPfOffK;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
            uint32_t ov[32];
            if (ok && nk > 0) {
                sm100::tmem_ld32(tm_o + c, ov);
                sm100::tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) ov[e] = 0u;
            }
            uint8_t *chunk = stage + (c >> 6) * kPfChunk;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int unit = ((c & 63) >> 3) + q;        // 16-byte unit of the 128-byte row
                *reinterpret_cast<uint4 *>(chunk + r * 128 + ((unit ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf162(__uint_as_float(ov[8 * q]) * inv, __uint_as_float(ov[8 * q + 1]) * inv),
                               pack_bf162(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv),
                               pack_bf162(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv),
                               pack_bf162(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv));
            }
        }
        if (a.out_lse && has_row)
            a.out_lse[((long long)b * a.s + t) * a.H + head] =
                l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        fence_proxy_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");     // the 4 softmax warps
        if (warp == 2 && lane == 0) {
            sm100::tma_store_4d(&maps.out, stage, 0, head, q0, b);
            sm100::tma_store_4d(&maps.out, stage + kPfChunk, 64, head, q0, b);
            sm100::tma_store_commit();
            sm100::tma_store_wait_read();
        }
    }

    // ------------------------------------------------------------ teardown
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        volatile int no_abort = 0;
        sm100::warp_wait(done, 0, &no_abort, a.err, drain);
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 512);
    }
}

// Prefill set-up, one pass: each sequence's cached rows gathered through its
// block table into rows [b * lpad, b * lpad + lpad) of a contiguous [576]-wide
// buffer (rows at or past the sequence's length, and every row of an invalid
// sequence, are zero), and the chunk's RoPE queries rotated to q_pos (copied
// when q_pos is null).
__global__ void __launch_bounds__(256)
prefill_prepare_kernel(const bf16 *__restrict__ cache, int num_blocks, const int32_t *__restrict__ block_table,
                       int max_blocks, const int32_t *__restrict__ seq_lens, int B, int s, int H, int lpad,
                       int l_cap, bf16 *__restrict__ rows, const bf16 *__restrict__ q_rope,
                       const int32_t *__restrict__ q_pos, bf16 *__restrict__ q_rot, const RopeTable rope,
                       uint32_t *err)
{
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    constexpr int kUnits = kRow / 8;                            // 16-byte units per row
    const long long row_units = (long long)B * lpad * kUnits;
    for (long long w = tid; w < row_units; w += nthreads) {
        const long long row = w / kUnits;
        const int c = (int)(w % kUnits);
        const int b = (int)(row / lpad), j = (int)(row % lpad);
        const int L = seq_lens[b];
        const bool valid = prefill_valid(L, s, l_cap);
        if (!valid && j == 0 && c == 0) set_error(err, MLA_DEVERR_SEQ_LEN);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (valid && j < L) {
            const int blk = block_table[(long long)b * max_blocks + j / kBlock];
            if (blk >= 0 && blk < num_blocks)
                v = reinterpret_cast<const uint4 *>(cache + ((long long)blk * kBlock + j % kBlock) * kRow)[c];
            else if (c == 0)
                set_error(err, MLA_DEVERR_BLOCK_ID);
        }
        reinterpret_cast<uint4 *>(rows + row * kRow)[c] = v;
    }
    const long long units = (long long)B * s * (kDr / 2);
    for (long long w = tid; w < units; w += nthreads)
        rope_heads(q_rope, q_pos, w / (kDr / 2), (int)(w % (kDr / 2)), H, rope, q_rot, kDr, 0);
}

}  // namespace mla
