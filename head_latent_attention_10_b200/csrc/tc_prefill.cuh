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
// tcgen05.  CTA (block, head i, sequence b) owns two 128-query tiles of head
// i (MMA M = 128 each) and streams 128-key tiles of K = [K^C | k^R] and V^C:
//   S_u(k) = Q_u K_k^T    N=128, K=192 (12 MMAs)   fp32 in TMEM
//   P_u(k) = exp2(S_u(k) scale log2 e - m_u)       bf16, written over S_u(k)
//   O_u   += P_u(k) V_k   N=128, K=128 (8 MMAs, P read from TMEM)
// TMEM (512 columns): S_0/P_0 0-127, S_1/P_1 128-255, O_0 256-383, O_1
// 384-511.  Each tile u has its own issuing thread (warp 1 + u) and softmax
// warpgroup (warps 4-7, 8-11; thread = query row), so tile u's chain
// S_u(k) -> softmax -> P_u(k) V_k -> S_u(k+1) runs while the other tile's
// MMAs keep the tensor pipe busy.  S_u(k+1) overwrites P_u(k), so its issuer
// waits for P_u(k) V_k to complete first; that also means O_u is idle while
// the softmax rescales it.  Lazy rescaling as in the decode.
// Shared memory: Q_0, Q_1 (three 64-column chunks each, [128 rows][128 B],
// 128-byte swizzle: q^C 0-63, q^C 64-127, rotated q^R), two K slots (K^C
// 0-63, 64-127, k^R) and one V slot (V^C 0-63, 64-127): 224 KB.  Warp 0
// loads with TMA (no cluster multicast).  Every wait is bounded.
#pragma once

#include "dec_common.cuh"

namespace mla {

constexpr int kPfThreads = 384;
constexpr int kPfChunk = 128 * 128;                    // [128 rows][64 bf16]: 16 KB
constexpr int kPfOffQ = 0;                             // Q_u chunk c at (3u + c) * 16 KB
constexpr int kPfOffK = 6 * kPfChunk;                  // K slot j chunk c at +(3j + c) * 16 KB
constexpr int kPfOffV = 12 * kPfChunk;                 // V chunk c at +c * 16 KB
constexpr int kPfOffBar = 14 * kPfChunk;               // 229,376
constexpr int kPfSmem = kPfOffBar + 256 + 1024;        // barriers, alignment slack
constexpr uint32_t kPfTmS = 0, kPfTmO = 256;

// Tensor maps of one call.  Rows of K^C, V^C and the gathered latents are
// [B * Lpad] long (sequence b at rows b * Lpad ..); queries and outputs are
// [B][s][H][.] with the sequence as the outermost dimension, so a 128-row
// tile is clipped at the end of its own sequence.
struct PrefillMaps {
    CUtensorMap qc;    // q^C         {128, H, s, B}, box {64, 1, 128, 1}
    CUtensorMap qr;    // rotated q^R {64, H, s, B},  box {64, 1, 128, 1}
    CUtensorMap kc;    // K^C         {128, H, B Lpad}, box {64, 1, 128}
    CUtensorMap vc;    // V^C         {128, H, B Lpad}, box {64, 1, 128}
    CUtensorMap kr;    // gathered rows {576, B Lpad, 1}, box {64, 128, 1}, read at x = 512
    CUtensorMap out;   // out         {128, H, s, B}, box {64, 1, 128, 1}
};

struct PrefillArgs {
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
    uint64_t *q_full = bars;            // Q_0 and Q_1 loaded
    uint64_t *k_full = bars + 1;        // [2] K slot loaded
    uint64_t *v_full = bars + 3;        // V buffer loaded
    uint64_t *k_free = bars + 4;        // [2u + slot]: S_u of the slot's tile done
    uint64_t *v_free = bars + 8;        // [u]: P_u V of the buffer's tile done
    uint64_t *s_full = bars + 10;       // [u] S_u(k) in TMEM
    uint64_t *p_full = bars + 12;       // [u] P_u(k) in TMEM, O_u rescaled (4 softmax warps arrive)
    uint64_t *pv_done = bars + 14;      // [u] P_u(k) V_k done
    uint64_t *done = bars + 16;         // both issuers' last MMAs done (teardown)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 18);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = gridDim.x - 1 - blockIdx.x;   // the longest rows of the causal triangle first
    const int head = blockIdx.y, b = blockIdx.z;
    const int q0 = 256 * qb;
    const int L = a.seq_lens[b];
    const bool valid = prefill_valid(L, a.s, a.l_cap);
    const int nk0 = valid ? prefill_tiles(q0, a.s, L) : 0;
    const int nk1 = valid ? prefill_tiles(q0 + 128, a.s, L) : 0;
    const int nkmax = nk0 > nk1 ? nk0 : nk1;
    const int row0 = b * a.lpad;                 // this sequence's first key row

    if (threadIdx.x == 0) {
        sm100::mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            sm100::mbar_init(&k_full[i], 1);
            sm100::mbar_init(&s_full[i], 1);
            sm100::mbar_init(&p_full[i], 4);
            sm100::mbar_init(&pv_done[i], 1);
            sm100::mbar_init(&v_free[i], 1);
        }
        for (int i = 0; i < 4; ++i) sm100::mbar_init(&k_free[i], 1);
        sm100::mbar_init(v_full, 1);
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
        // ------------------------------------------------------------ loads
        if (lane == 0 && nkmax > 0) {
            auto load_k = [&](int k) {
                uint8_t *dst = smem + kPfOffK + 3 * (k & 1) * kPfChunk;
                const int r = row0 + 128 * k;
                sm100::mbar_arrive_expect_tx(&k_full[k & 1], 3 * kPfChunk);
                sm100::tma_load_3d(&maps.kc, &k_full[k & 1], dst, 0, head, r);
                sm100::tma_load_3d(&maps.kc, &k_full[k & 1], dst + kPfChunk, 64, head, r);
                sm100::tma_load_3d(&maps.kr, &k_full[k & 1], dst + 2 * kPfChunk, kDc, r, 0);
            };
            auto load_v = [&](int k) {
                const int r = row0 + 128 * k;
                sm100::mbar_arrive_expect_tx(v_full, 2 * kPfChunk);
                sm100::tma_load_3d(&maps.vc, v_full, smem + kPfOffV, 0, head, r);
                sm100::tma_load_3d(&maps.vc, v_full, smem + kPfOffV + kPfChunk, 64, head, r);
            };
            // a K slot (or the V buffer) is free once every query tile that
            // reads tile k is done with it; tile u reads the tiles [0, nk_u)
            auto wait_free = [&](uint64_t *bar0, uint64_t *bar1, int k, uint32_t parity) -> bool {
                if (k < nk0 && !sm100::mbar_wait(bar0, parity, abort_flag, a.err, lim)) return false;
                if (k < nk1 && !sm100::mbar_wait(bar1, parity, abort_flag, a.err, lim)) return false;
                return true;
            };
            sm100::mbar_arrive_expect_tx(q_full, 6 * kPfChunk);
            for (int u = 0; u < 2; ++u) {
                uint8_t *qd = smem + kPfOffQ + 3 * u * kPfChunk;
                sm100::tma_load_4d(&maps.qc, q_full, qd, 0, head, q0 + 128 * u, b);
                sm100::tma_load_4d(&maps.qc, q_full, qd + kPfChunk, 64, head, q0 + 128 * u, b);
                sm100::tma_load_4d(&maps.qr, q_full, qd + 2 * kPfChunk, 0, head, q0 + 128 * u, b);
            }
            load_k(0);
            int k_issued = 1, v_issued = 1;
            if (nkmax > 1) {
                load_k(1);
                k_issued = 2;
            }
            load_v(0);
            for (int k = 0; k < nkmax; ++k) {
                // K slot of tile k -> tile k + 2, once the S MMAs of tile k are done
                if (k + 2 < nkmax) {
                    if (!wait_free(&k_free[k & 1], &k_free[2 + (k & 1)], k, (k >> 1) & 1)) break;
                    load_k(k + 2);
                    k_issued = k + 3;
                }
                // V buffer of tile k -> tile k + 1, once the P V MMAs of tile k are done
                if (k + 1 < nkmax) {
                    if (!wait_free(&v_free[0], &v_free[1], k, k & 1)) break;
                    load_v(k + 1);
                    v_issued = k + 2;
                }
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA can exit
                volatile int no_abort = 0;
                sm100::mbar_wait(q_full, 0, &no_abort, a.err, drain);
                for (int k = k_issued - 2 < 0 ? 0 : k_issued - 2; k < k_issued; ++k)
                    sm100::mbar_wait(&k_full[k & 1], (k >> 1) & 1, &no_abort, a.err, drain);
                sm100::mbar_wait(v_full, (v_issued - 1) & 1, &no_abort, a.err, drain);
            }
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------- MMA issue, query tile u
        const int u = warp - 1;
        const int nk = u ? nk1 : nk0;
        if (lane == 0) {
            const uint32_t idesc_s = sm100::idesc_bf16(128, 128, 0, 0);
            const uint32_t idesc_o = sm100::idesc_bf16(128, 128, 0, 1);
            const uint32_t tm_s = tmem + kPfTmS + 128 * u, tm_o = tmem + kPfTmO + 128 * u;
            const uint32_t qa = sm100::smem_u32(smem + kPfOffQ + 3 * u * kPfChunk);
            const uint64_t vd = sm100::desc_mnmajor_sw128(sm100::smem_u32(smem + kPfOffV), kPfChunk);
            bool ok = nk == 0 || sm100::mbar_wait(q_full, 0, abort_flag, a.err, lim);
            for (int k = 0; ok && k < nk; ++k) {
                ok = sm100::mbar_wait(&k_full[k & 1], (k >> 1) & 1, abort_flag, a.err, lim);
                // S_u(k) overwrites P_u(k-1): its P V must have completed
                if (ok && k > 0) ok = sm100::mbar_wait(&pv_done[u], (k - 1) & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const uint32_t ka = sm100::smem_u32(smem + kPfOffK + 3 * (k & 1) * kPfChunk);
#pragma unroll
                for (int step = 0; step < 12; ++step) {      // q^C 0-63, q^C 64-127, q^R
                    const uint32_t off = (step >> 2) * kPfChunk + (step & 3) * 32;
                    sm100::umma_ss(tm_s, sm100::desc_kmajor(qa + off, 128, sm100::kSw128),
                                   sm100::desc_kmajor(ka + off, 128, sm100::kSw128), idesc_s, step > 0);
                }
                sm100::umma_commit(&s_full[u]);
                sm100::umma_commit(&k_free[2 * u + (k & 1)]);
                ok = sm100::mbar_wait(&p_full[u], k & 1, abort_flag, a.err, lim) &&
                     sm100::mbar_wait(v_full, k & 1, abort_flag, a.err, lim);
                if (!ok) break;
                sm100::tc_fence_after();
#pragma unroll
                for (int kq = 0; kq < 8; ++kq)               // 16 keys per MMA: 8 TMEM columns of P
                    sm100::umma_ts(tm_o, tm_s + 8 * kq, vd + (uint64_t)((kq * 2048) >> 4), idesc_o,
                                   (k > 0 || kq > 0) ? 1u : 0u);
                sm100::umma_commit(&pv_done[u]);
                sm100::umma_commit(&v_free[u]);
            }
            sm100::umma_commit(done);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------- softmax of query tile u
        const int u = (warp - 4) >> 2, qd = warp & 3;
        const int nk = u ? nk1 : nk0;
        const int r = 32 * qd + lane, t = q0 + 128 * u + r;
        const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
        const uint32_t tm_s = tmem + lane_off + kPfTmS + 128 * u, tm_o = tmem + lane_off + kPfTmO + 128 * u;
        const int nvis = (t < a.s) ? L - a.s + t + 1 : 0;    // keys [0, nvis) visible to row t
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int k = 0; ok && k < nk; ++k) {
            ok = sm100::warp_wait(&s_full[u], k & 1, abort_flag, a.err, lim);
            if (!ok) break;
            sm100::tc_fence_after();
            uint32_t x[128];
#pragma unroll
            for (int c = 0; c < 128; c += 32) sm100::tmem_ld32(tm_s + c, x + c);
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
            // P_u(k) over the first 64 columns of S_u(k) (this thread's own
            // lane, read above)
            sm100::tmem_st32(tm_s, x);
            sm100::tmem_st32(tm_s + 32, x + 32);
            // O_u holds the tiles before k, whose P V completed before S_u(k)
            // was issued: rescale this thread's row in place
            if (__any_sync(0xffffffffu, rescale)) {
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
            if (lane == 0) sm100::mbar_arrive(&p_full[u]);
        }
        // epilogue: O_u / l as bf16, staged over Q_u's q^C chunks (free once
        // the last P V completed, which follows the last S MMA) as [128
        // rows][128 B] with 128-byte swizzle, stored with TMA
        if (ok && nk > 0) {
            ok = sm100::warp_wait(&pv_done[u], (nk - 1) & 1, abort_flag, a.err, lim);
            sm100::tc_fence_after();
        }
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint8_t *stage = smem + kPfOffQ + 3 * u * kPfChunk;
        const bool has_rows = q0 + 128 * u < a.s;      // else nothing to store (and Q_u may still be landing)
#pragma unroll 1
        for (int c = 0; c < (has_rows ? 128 : 0); c += 32) {
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
        if (a.out_lse && t < a.s)
            a.out_lse[((long long)b * a.s + t) * a.H + head] =
                l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
        fence_proxy_async_smem();
        if (u == 0)
            asm volatile("bar.sync 1, 128;" ::: "memory");
        else
            asm volatile("bar.sync 2, 128;" ::: "memory");
        if (qd == 0 && lane == 0 && has_rows) {
            sm100::tma_store_4d(&maps.out, stage, 0, head, q0 + 128 * u, b);
            sm100::tma_store_4d(&maps.out, stage + kPfChunk, 64, head, q0 + 128 * u, b);
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
    const long long pairs = (long long)B * s * H * (kDr / 2);  // (token, head) rows x RoPE pairs
    for (long long w = tid; w < pairs; w += nthreads) {
        const long long qrow = w / (kDr / 2);
        const int k = (int)(w % (kDr / 2));
        const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162 *>(q_rope + qrow * kDr)[k];
        __nv_bfloat162 y = x;
        if (q_pos) {
            float y0, y1;
            rope_turn(__low2float(x), __high2float(x), q_pos[qrow / H], rope.theta[k], &y0, &y1);
            y = __floats2bfloat162_rn(y0, y1);
        }
        reinterpret_cast<__nv_bfloat162 *>(q_rot + qrow * kDr)[k] = y;
    }
}

}  // namespace mla
