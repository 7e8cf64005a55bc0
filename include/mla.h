/*
 * mla.h -- C ABI of the absorbed Multi-head Latent Attention (MLA) decode
 * library for NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V2; pages cited by title and section):
 *   - the KV cache keeps, per token, only the joint latent c^KV = W^DKV h
 *     (d_c = 512 values) and one decoupled RoPE key k^R = RoPE(W^KR h)
 *     (d_r = 64 values) shared by all heads
 *       [DeepSeek-V3 report summary (xyznot.com), Method 1 (MLA);
 *        DeepSeek-V2 paper review (jiphyeonjeon.kr), sections 2-3];
 *   - each head's content query is absorbed into the latent space,
 *     q~_i = (U^K_i)^T q^C_i, so the score against token j is
 *     (q~_i . c^KV_j + q^R_i . k^R_j) / sqrt(d_h + d_r)
 *       [DeepSeek-V2 paper review, section 2 (absorption identity) and
 *        section 3 (score and its 1/sqrt(128+64) scale)];
 *   - the attention-weighted latents are summed and U^V_i (then O_i) is
 *     applied once afterwards: o_i = U^V_i sum_j a_ij c^KV_j,
 *     u = sum_i O_i o_i   [DeepSeek-V2 paper review, section 2].
 *
 * Conventions shared by every call:
 *   - bf16 tensors are passed as pointers to 16-bit storage (IEEE bfloat16
 *     bit patterns), row-major, contiguous, 16-byte aligned.
 *   - Every pointer is caller-owned DEVICE memory unless stated otherwise.
 *     No call allocates device memory (no cudaMalloc, no allocating library
 *     routine).  mla_decode and mla_prefill keep their scratch in the
 *     caller's workspace; the other calls need none.  One call, mla_decode_noalloc, uses a fixed file-scope device
 *     array inside the library instead (MLA_NOALLOC_SCRATCH_BYTES, one per
 *     device, held until the process exits); calls of it that may overlap on
 *     one device race on that array (see its notes).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Inputs are never modified,
 *     except the cache by the append calls.
 *   - Argument errors are returned synchronously and launch nothing.  A
 *     failed launch returns MLA_ERR_CUDA.  Errors only the device can see
 *     (bad block-table entries, sequence lengths out of range, a bounded
 *     wait that gave up) set bits of a device error word (MLA_DEVERR_*);
 *     the offending access is skipped, never performed.
 *   - Supported shapes: d_c = 512, d_rope = 64, d_head = 128,
 *     block_size = 64, num_heads a multiple of 16 in [16, 128].  Anything
 *     else returns MLA_ERR_UNSUPPORTED.
 *
 * Paged latent cache layout (one model layer):
 *   cache[num_blocks][block_size][d_c + d_rope] bf16; a row is
 *   [c^KV (512) | k^R (64), already rotated] = 1152 bytes.  Logical position
 *   p of sequence b lives in block block_table[b * max_blocks + p / 64],
 *   slot p % 64.  The RoPE position of the token at logical position p is p.
 */
#ifndef MLA_H
#define MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer */
    MLA_ERR_UNSUPPORTED = 2, /* shape outside the supported set */
    MLA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    MLA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
    MLA_ERR_DEVICE = 5       /* device error word non-zero (MLA_SYNC_CHECK) */
} mla_status_t;

/* Bits of the device error word. */
#define MLA_DEVERR_BLOCK_ID 0x1u /* block-table entry outside [0, num_blocks) */
#define MLA_DEVERR_SEQ_LEN  0x2u /* seq_len > max_blocks*block_size, or a query
                                    with no visible key (seq_len < s), or a
                                    position / sequence index out of range */
#define MLA_DEVERR_TIMEOUT  0x4u /* a bounded device-side wait gave up */

/* mla_decode flags */
#define MLA_SYNC_CHECK   0x1u  /* synchronize the stream after the call and
                                  return MLA_ERR_DEVICE if the error word is
                                  non-zero */
#define MLA_FORCE_SIMPLE 0x2u  /* run the CUDA-core decode kernel instead of
                                  the tensor-core one (same results within
                                  rounding; used to cross-check) */
#define MLA_DEBUG_STALL  0x100u /* test hook for failure detection: every
                                  tensor-core decode CTA skips the page load
                                  of its first tile and the device waits give
                                  up after 20 ms, so the call records
                                  MLA_DEVERR_TIMEOUT and unwinds; the output is
                                  then unspecified.  Never set in production. */
#define MLA_DEBUG_COMBINE_ALL 0x200u /* test hook: every cut sequence is merged
                                  by the combine kernel, none inside the
                                  decode kernel; the results are the same bits
                                  either way (the two merges take the same
                                  steps in the same order). */

typedef struct {
    int32_t num_heads;   /* H */
    int32_t d_c;         /* latent width, 512 */
    int32_t d_rope;      /* RoPE key / query width, 64 */
    int32_t d_head;      /* per-head content width, 128 */
    int32_t block_size;  /* tokens per cache block, 64 */
    float softmax_scale; /* <= 0 selects 1/sqrt(d_head + d_rope); a caller
                            using YaRN passes its attention temperature here */
    float rope_base;     /* RoPE base; <= 0 selects 10000 */
    /* YaRN frequency scaling of RoPE [DeepSeek-V2 paper review, long-context
     * passage: the 4K pre-training context extended with YaRN, scale 40].
     * With rope_scaling = s > 1, pair k (base frequency theta_k = base^(-2k/d_rope))
     * makes r_k = L0 theta_k / (2 pi) turns over the original context L0; with
     * the ramp g = clamp((r_k - alpha) / (beta - alpha), 0, 1) it turns at
     * (1 - g) theta_k / s + g theta_k.  Used by every call that rotates (the
     * appends for k^R, mla_absorb_q for q^R).  rope_scaling <= 1: plain RoPE.
     * beta must exceed alpha (MLA_ERR_INVALID_ARG otherwise). */
    float rope_scaling;        /* s; <= 1 selects plain RoPE */
    int32_t rope_original_ctx; /* L0; <= 0 selects 4096 */
    float rope_yarn_alpha;     /* alpha; <= 0 selects 1 */
    float rope_yarn_beta;      /* beta; <= 0 selects 32 */
} mla_dims_t;

/* Human-readable name of a status code (static storage). */
const char *mla_status_string(mla_status_t status);

/*
 * mla_append_cache -- step a1: project new tokens into the latent cache.
 *   c^KV_t = W^DKV h_t,  k^R_t = RoPE(W^KR h_t, pos[t])
 *   [DeepSeek-V2 paper review, section 2 (c^KV = W^DKV h);
 *    DeepSeek-V3 report summary, Method 1 (k^R = RoPE(W^KR h), cache only
 *    c^KV and k^R)]
 * and writes row [c^KV | k^R] (rounded to bf16, fp32 accumulation) to the
 * slot of (seq_idx[t], pos[t]).
 *   h            [T][d_model] bf16
 *   w_dkv        [d_c][d_model] bf16      (W^DKV)
 *   w_kr         [d_rope][d_model] bf16   (W^KR)
 *   seq_idx, pos [T] int32                (device)
 *   block_table  [num_seqs][max_blocks] int32 (device)
 *   cache        [num_blocks][block_size][d_c+d_rope] bf16, written in place
 *   kv_norm_weight  optional [d_c] bf16 RMSNorm weight w; when given, the
 *                latent row is stored as c / sqrt(mean(c^2) + kv_norm_eps) * w
 *                (the RMSNorm after the compressed latent, DeepSeek-V2 paper
 *                review, section 2), taken on the bf16 projection output.
 *                NULL: no normalisation.  kv_norm_eps must be >= 0.
 *   err_word     optional device uint32; bits MLA_DEVERR_* are OR-ed in for
 *                tokens whose slot is invalid (those tokens are not written)
 * d_model must be a positive multiple of 64.  T = 0 is a no-op.
 * When d_model is a multiple of 512 the projection splits K over a cluster
 * of 8 CTAs per 64-column tile and sums their fp32 partials on chip in a
 * fixed order (deterministic, one launch, no scratch outside the kernel's
 * shared memory); other widths take one pass over K per 128-token tile.
 */
mla_status_t mla_append_cache(const mla_dims_t *dims, const void *h, int T, int d_model,
                              const void *w_dkv, const void *w_kr,
                              const int32_t *seq_idx, const int32_t *pos,
                              const int32_t *block_table, int num_seqs, int max_blocks,
                              void *cache, int num_blocks, const void *kv_norm_weight,
                              float kv_norm_eps, uint32_t *err_word, void *stream);

/*
 * mla_append_latent -- the RoPE-and-scatter half of step a1, for callers that
 * already hold the latent: writes [c_kv[t] | RoPE(k_rope[t], pos[t])] to the
 * slot of (seq_idx[t], pos[t]).  Same sources as mla_append_cache.
 *   c_kv   [T][d_c] bf16, copied bit for bit (or RMS-normalised when
 *          kv_norm_weight is given)
 *   k_rope [T][d_rope] bf16, the raw (unrotated) RoPE key W^KR h
 * Other arguments as for mla_append_cache.
 */
mla_status_t mla_append_latent(const mla_dims_t *dims, const void *c_kv, const void *k_rope,
                               int T, const int32_t *seq_idx, const int32_t *pos,
                               const int32_t *block_table, int num_seqs, int max_blocks,
                               void *cache, int num_blocks, const void *kv_norm_weight,
                               float kv_norm_eps, uint32_t *err_word, void *stream);

/*
 * mla_absorb_q -- step a2: absorb U^K into the query.
 *   q_abs[t][i][0:d_c]    = (U^K_i)^T q^C_{t,i}     (fp32 accumulation -> bf16)
 *   q_abs[t][i][d_c:]     = RoPE(q^R_{t,i}, q_pos[t]), or q^R copied if
 *                           q_pos == NULL (already rotated)
 *   [DeepSeek-V2 paper review, section 2: (q^C)^T U^K c = ((U^K)^T q^C)^T c;
 *    section 3: per-head RoPE query of 64 dims]
 *   q_nope [T][H][d_head] bf16, q_rope [T][H][d_rope] bf16,
 *   q_pos  [T] int32 or NULL, w_uk [H][d_head][d_c] bf16 (U^K_i),
 *   q_abs  [T][H][d_c+d_rope] bf16 (output).
 */
mla_status_t mla_absorb_q(const mla_dims_t *dims, const void *q_nope, const void *q_rope,
                          const int32_t *q_pos, const void *w_uk, int T, void *q_abs,
                          void *stream);

/*
 * mla_decode_workspace_size -- bytes of device workspace mla_decode needs for
 * B sequences of s query tokens whose lengths are at most max_seq_len.
 */
size_t mla_decode_workspace_size(const mla_dims_t *dims, int B, int s, int max_seq_len);

/*
 * mla_decode -- steps a3-a6: absorbed attention over the paged latent cache,
 * with split-KV partials merged by log-sum-exp.
 *   l_ij = softmax_scale * (q_abs[i] . cache_row_j)      (576-d dot product)
 *   out_latent[i] = sum_j softmax_j(l_ij) c^KV_j           (U^V not applied)
 *   [DeepSeek-V2 paper review, section 3 (score, scale, softmax over j) and
 *    section 2 (U^V pulled out of the weighted sum)]
 * Query t in [0,s) of sequence b sees the positions j <= seq_lens[b] - s + t.
 *   q_abs       [B*s][H][d_c+d_rope] bf16 (row = b*s + t)
 *   cache, num_blocks, block_table [B][max_blocks] int32, seq_lens [B] int32
 *   out_latent  [B*s][H][d_c] bf16
 *   out_lse     [B*s][H] fp32 natural-log softmax denominator of the scaled
 *               logits, or NULL.  A query with no visible key gets a zero
 *               latent and lse = -inf (and MLA_DEVERR_SEQ_LEN).
 *   workspace   device buffer of ws_bytes >= mla_decode_workspace_size();
 *               its first 4 bytes are the device error word (cleared by the
 *               call); the rest holds the split plan and partial results.
 *   flags       MLA_SYNC_CHECK, MLA_FORCE_SIMPLE (MLA_DEBUG_STALL,
 *               MLA_DEBUG_COMBINE_ALL: tests only).
 * Sequences are independent; calls that share a workspace must not overlap
 * on the GPU.  B = 0 is a no-op.  With B > 0, num_blocks and max_blocks must
 * be at least 1 (MLA_ERR_INVALID_ARG otherwise).
 */
mla_status_t mla_decode(const mla_dims_t *dims, const void *q_abs, const void *cache,
                        int num_blocks, const int32_t *block_table, int max_blocks,
                        const int32_t *seq_lens, int B, int s, void *out_latent,
                        float *out_lse, void *workspace, size_t ws_bytes, uint32_t flags,
                        void *stream);

/*
 * mla_decode_error -- copy the device error word of a workspace into
 * *err_host (blocking on `stream`), optionally clearing it.
 */
mla_status_t mla_decode_error(const void *workspace, uint32_t *err_host, int clear, void *stream);

/*
 * mla_decode_noalloc -- the same decode as mla_decode, for a caller that
 * cannot hand over a workspace.  The pages have no counterpart: it is a
 * packaging of the same computation, not a step of the method.
 *
 * Scratch: a file-scope device array of MLA_NOALLOC_SCRATCH_BYTES inside this
 * library, one per device.  Nothing is allocated: no cudaMalloc/cudaFree and
 * no allocating library call.  On the first call on a device (with that
 * device current) the library looks up the array's address with
 * cudaGetSymbolAddress and keeps it; make that first call before any stream
 * capture.  Nothing in the array has to start at zero: every call clears the
 * error word and rewrites the plan and the partials it reads.
 *
 * Arguments, layouts and the result are those of mla_decode without
 * `workspace` and `ws_bytes`.
 *
 * Errors:
 *   - MLA_ERR_WORKSPACE if the scratch this shape needs (the size
 *     mla_decode_workspace_size would report for the path the flags choose)
 *     exceeds MLA_NOALLOC_SCRATCH_BYTES.  This is checked before any device
 *     work.
 *   - MLA_ERR_CUDA if the address lookup fails.
 *   - Device-side errors are reported only through MLA_SYNC_CHECK, because
 *     the scratch is not visible to the caller.
 *
 * Concurrency: every call on a device shares the one array.  Calls ordered on
 * one stream are safe.  Calls that may overlap (different streams, or
 * different host threads without ordering) race on it.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (40u << 20)
mla_status_t mla_decode_noalloc(const mla_dims_t *dims, const void *q_abs, const void *cache,
                                int num_blocks, const int32_t *block_table, int max_blocks,
                                const int32_t *seq_lens, int B, int s, void *out_latent,
                                float *out_lse, uint32_t flags, void *stream);

/*
 * mla_up_v -- step a7: apply U^V (and optionally O) after the weighted sum.
 *   out_heads[t][i] = U^V_i latent[t][i]                 (bf16, fp32 accum.)
 *   out_model[t]    = sum_i O_i out_heads[t][i]          (if w_o != NULL)
 *   [DeepSeek-V2 paper review, section 2: u_t = sum_i O_i U^V_i (sum_j a_ij c_j)]
 *   latent    [T][H][d_c] bf16, w_uv [H][d_head][d_c] bf16 (U^V_i),
 *   w_o       [d_model][H*d_head] bf16 (column block i is O_i) or NULL,
 *   out_heads [T][H][d_head] bf16 (required), out_model [T][d_model] bf16.
 */
mla_status_t mla_up_v(const mla_dims_t *dims, const void *latent, int T, const void *w_uv,
                      const void *w_o, int d_model, void *out_heads, void *out_model,
                      void *stream);

/*
 * mla_prefill_workspace_size -- bytes of device workspace mla_prefill needs
 * for B sequences of s new query tokens whose lengths are at most
 * max_seq_len (0 for invalid dims or sizes).
 */
size_t mla_prefill_workspace_size(const mla_dims_t *dims, int B, int s, int max_seq_len);

/*
 * mla_prefill -- prefill of a chunk of s query tokens per sequence in the
 * expanded form: each head's keys and values are materialised from the cached
 * latents and attended to directly,
 *   k_{j,i} = [U^K_i c^KV_j ; k^R_j],   v_{j,i} = U^V_i c^KV_j,
 *   out[t][i] = sum_j softmax_j(softmax_scale * [q^C_{t,i} ; q^R_{t,i}] . k_{j,i}) v_{j,i}
 *   [DeepSeek-V2 paper review, section 2 (k^C = W^UK c^KV, v^C = W^UV c^KV)
 *    and section 3 (per-head query [q^C; q^R], the shared RoPE key, the
 *    1/sqrt(d_head + d_rope) scale); DeepSeek-V3 report summary, Method 1]
 * It gives what mla_absorb_q + mla_decode + mla_up_v give for the same
 * queries (the two forms are equal up to rounding) at fewer flops when s is
 * large.  The s tokens are the last s of each sequence: query t of sequence
 * b sits at position seq_lens[b] - s + t and sees the positions up to it.
 *   q_nope      [B*s][H][d_head] bf16 (row = b*s + t), q^C
 *   q_rope      [B*s][H][d_rope] bf16, q^R, rotated here to q_pos[b*s + t]
 *               (q_pos [B*s] int32), or taken as already rotated if q_pos
 *               is NULL
 *   w_uk, w_uv  [H][d_head][d_c] bf16 (U^K_i, U^V_i)
 *   cache, num_blocks, block_table [B][max_blocks], seq_lens [B]: as for
 *               mla_decode; the cache rows must hold the chunk's own tokens
 *   max_seq_len an upper bound of seq_lens (>= s); the call expands
 *               B * round_up(max_seq_len, 128) latent rows per head
 *   out         [B*s][H][d_head] bf16 (per-head outputs, O not applied)
 *   out_lse     [B*s][H] fp32 natural-log softmax denominator, or NULL
 *   workspace   ws_bytes >= mla_prefill_workspace_size(); its first 4 bytes
 *               are the device error word (cleared by the call, read with
 *               mla_decode_error); the rest holds the gathered latents, the
 *               rotated q^R and the expanded K^C and V^C.
 *   flags       MLA_SYNC_CHECK
 * A sequence with seq_lens[b] < s, > max_seq_len or > max_blocks * 64 gets
 * zero outputs, lse = -inf and MLA_DEVERR_SEQ_LEN.  B = 0 is a no-op; with
 * B > 0, num_blocks and max_blocks must be at least 1.  Calls that share a
 * workspace must not overlap on the GPU.
 */
mla_status_t mla_prefill(const mla_dims_t *dims, const void *q_nope, const void *q_rope,
                         const int32_t *q_pos, const void *w_uk, const void *w_uv, const void *cache,
                         int num_blocks, const int32_t *block_table, int max_blocks,
                         const int32_t *seq_lens, int B, int s, int max_seq_len, void *out,
                         float *out_lse, void *workspace, size_t ws_bytes, uint32_t flags,
                         void *stream);

/*
 * FP8 latent cache [DeepSeek-V2 paper review, sections 4 and 9: the deployed
 * model keeps its KV cache at about 6 bits per element; DeepSeek-V3 report
 * summary, the FP8 framework: E4M3 values with fine-grained scaling factors].
 * A token's row [c^KV (512) | k^R (64), rotated] is stored as 576 E4M3 codes
 * (OCP: bias 7, no infinities, 448 the largest finite value) plus one fp32
 * scale per part, scale = amax / 448 over the part (1 for an all-zero part),
 * code = E4M3(x / scale), the quotient in fp32, nearest-even, saturated.  A
 * code's value is E4M3(code) * scale.
 *   codes  [num_blocks][block_size][d_c + d_rope] uint8   (16-byte aligned)
 *   scales [num_blocks][block_size][2] fp32 (c^KV part, k^R part)
 *
 * mla_append_latent_fp8 -- mla_append_latent into the FP8 cache: forms the
 * same bf16 row (copy or RMSNorm of c_kv, RoPE of k_rope at pos), quantizes it
 * as above and writes codes and scales to the slot of (seq_idx[t], pos[t]).
 * Arguments as for mla_append_latent, with `codes` and `scales` in place of
 * `cache` (num_blocks pages of each); scales must be 8-byte aligned.
 */
mla_status_t mla_append_latent_fp8(const mla_dims_t *dims, const void *c_kv, const void *k_rope,
                                   int T, const int32_t *seq_idx, const int32_t *pos,
                                   const int32_t *block_table, int num_seqs, int max_blocks,
                                   void *codes, float *scales, int num_blocks,
                                   const void *kv_norm_weight, float kv_norm_eps,
                                   uint32_t *err_word, void *stream);

/*
 * mla_decode_fp8 -- mla_decode over the FP8 cache: the same attention with
 * each cache row taken as its codes' values times its scales.  The kernel
 * widens each page to f16 in shared memory (exactly: every E4M3 value is an
 * f16 value, one part of the row multiplied by the ratio of its scale to the
 * larger of the two) and runs the logits and the latent sum on f16 tensor
 * cores with fp32 accumulation; q_abs is read as bf16 and rounded to f16.
 * Arguments, workspace (mla_decode_workspace_size), outputs and errors as for
 * mla_decode, with `codes` and `scales` (16-byte aligned) in place of
 * `cache`.  flags: MLA_SYNC_CHECK, MLA_DEBUG_STALL; MLA_FORCE_SIMPLE returns
 * MLA_ERR_UNSUPPORTED.
 */
mla_status_t mla_decode_fp8(const mla_dims_t *dims, const void *q_abs, const void *codes,
                            const float *scales, int num_blocks, const int32_t *block_table,
                            int max_blocks, const int32_t *seq_lens, int B, int s,
                            void *out_latent, float *out_lse, void *workspace, size_t ws_bytes,
                            uint32_t flags, void *stream);

/*
 * Weight pre-absorption [DeepSeek-V2 paper review, section 2: at inference
 * W^UK can be absorbed into the query up-projection W^UQ and W^UV into the
 * output projection W^O; the query path compresses to c^Q = W^DQ h of width
 * d_q (1536 in V2) and q^C_i = W^UQ_i c^Q].
 *
 * mla_fold_weights -- one-time weight transform on the GPU (tensor cores,
 * fp32 accumulation, bf16 results):
 *   w_qk [H][d_c][d_q]       W^QK_i = (U^K_i)^T W^UQ_i
 *   w_ov [d_model][H*d_c]    block i (columns i*d_c ..) = O_i U^V_i
 * from w_uq [H][d_head][d_q], w_uk and w_uv [H][d_head][d_c] (as for
 * mla_absorb_q / mla_up_v) and w_o [d_model][H*d_head].  Either group
 * (w_uq, w_uk, w_qk) or (w_o, w_uv, w_ov) may be all NULL to skip it.
 * d_q and d_model must be positive multiples of 64.
 *
 * mla_absorb_q_folded -- step a2 from the compressed query:
 *   q_abs[t][i] = [ W^QK_i c_q[t] , RoPE(q_rope[t][i], q_pos[t]) ]
 * c_q [T][d_q] bf16, q_rope / q_pos / q_abs as for mla_absorb_q.  Equal to
 * mla_absorb_q on q^C_i = W^UQ_i c^Q up to rounding.
 *
 * mla_up_out_folded -- step a7 with the folded output weights:
 *   out_model[t] = sum_i W^OV_i latent[t][i]
 * latent [T][H][d_c] bf16 (mla_decode's output), out_model [T][d_model].
 * Equal to mla_up_v with w_o up to rounding.
 *
 * The folded forms trade memory traffic for fewer launches: at decode batch
 * sizes both steps read their weights once per call, and W^QK (H*d_c*d_q)
 * and W^OV (d_model*H*d_c) are larger than U^K + W^UQ and U^V + W^O
 * (for V2: 201 MB against 67 MB, and 671 MB against 185 MB).
 */
mla_status_t mla_fold_weights(const mla_dims_t *dims, int d_q, const void *w_uq, const void *w_uk,
                              void *w_qk, int d_model, const void *w_o, const void *w_uv,
                              void *w_ov, void *stream);
mla_status_t mla_absorb_q_folded(const mla_dims_t *dims, const void *c_q, int d_q,
                                 const void *q_rope, const int32_t *q_pos, const void *w_qk,
                                 int T, void *q_abs, void *stream);
mla_status_t mla_up_out_folded(const mla_dims_t *dims, const void *latent, int T,
                               const void *w_ov, int d_model, void *out_model, void *stream);

/*
 * mla_decode_ctas -- number of CTAs (the persistent grid) the tensor-core
 * decode launches on the current device for these dims and s query tokens
 * per sequence, or 0 if it cannot run.  A measurement aid.
 */
int mla_decode_ctas(const mla_dims_t *dims, int s);

/*
 * mla_kernel_launches -- number of CUDA kernels this library has launched in
 * the calling process (all devices, all entry points).  A measurement aid:
 * the difference across a region counts the library's launches in it.
 */
uint64_t mla_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H */
