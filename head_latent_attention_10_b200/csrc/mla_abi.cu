// mla_abi.cu -- the extern "C" entry points declared in include/mla.h:
// argument checks, workspace layout and kernel launches.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "k_simple.cuh"

using namespace mla;

unsigned long long mla::g_launches = 0;

namespace {

constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

mla_status_t check_dims(const mla_dims_t *d)
{
    if (!d) return MLA_ERR_INVALID_ARG;
    if (d->d_c != kDc || d->d_rope != kDr || d->d_head != kDh || d->block_size != kBlock)
        return MLA_ERR_UNSUPPORTED;
    if (d->num_heads < 16 || d->num_heads > 128 || d->num_heads % 16 != 0) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

inline float softmax_scale(const mla_dims_t *d)
{
    return d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)(d->d_head + d->d_rope));
}

inline double rope_base(const mla_dims_t *d)
{
    return d->rope_base > 0.f ? (double)d->rope_base : 10000.0;
}

inline mla_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Workspace of the decode: [error word | pad] [partial latents] [partial lse2]
struct SimpleWs {
    size_t off_o, off_lse, total;
    int nsplit;
};

SimpleWs simple_ws(int H, int T, int max_seq_len)
{
    SimpleWs w;
    w.nsplit = (max_seq_len + kSimpleSplit - 1) / kSimpleSplit;
    if (w.nsplit < 1) w.nsplit = 1;
    const size_t n = (size_t)T * w.nsplit * H;
    w.off_o = kWsAlign;
    w.off_lse = align_up(w.off_o + n * kDc * sizeof(float), kWsAlign);
    w.total = align_up(w.off_lse + n * sizeof(float), kWsAlign);
    return w;
}

}  // namespace

extern "C" {

uint64_t mla_kernel_launches(void) { return __atomic_load_n(&g_launches, __ATOMIC_RELAXED); }

const char *mla_status_string(mla_status_t s)
{
    switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: invalid argument";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: shape not supported";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: CUDA runtime or launch failure";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace missing or too small";
    case MLA_ERR_DEVICE: return "MLA_ERR_DEVICE: device error word set";
    }
    return "unknown mla_status_t";
}

mla_status_t mla_append_latent(const mla_dims_t *dims, const void *c_kv, const void *k_rope, int T,
                               const int32_t *seq_idx, const int32_t *pos,
                               const int32_t *block_table, int num_seqs, int max_blocks, void *cache,
                               int num_blocks, uint32_t *err_word, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || num_seqs < 0 || max_blocks < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!c_kv || !k_rope || !seq_idx || !pos || !block_table || !cache) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_kv) || !aligned16(cache) || ((uintptr_t)k_rope & 3u)) return MLA_ERR_INVALID_ARG;
    const int threads = 256, per = threads / 32;
    append_latent_kernel<<<(T + per - 1) / per, threads, 0, as_stream(stream)>>>(
        (const bf16 *)c_kv, (const bf16 *)k_rope, T, seq_idx, pos, block_table, num_seqs, max_blocks,
        (bf16 *)cache, num_blocks, rope_base(dims), err_word);
    count_launch();
    return cuda_status(cudaGetLastError());
}

mla_status_t mla_append_cache(const mla_dims_t *dims, const void *h, int T, int d_model,
                              const void *w_dkv, const void *w_kr, const int32_t *seq_idx,
                              const int32_t *pos, const int32_t *block_table, int num_seqs,
                              int max_blocks, void *cache, int num_blocks, uint32_t *err_word,
                              void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || num_seqs < 0 || max_blocks < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (d_model <= 0 || d_model % 64 != 0) return MLA_ERR_UNSUPPORTED;
    if (!h || !w_dkv || !w_kr || !seq_idx || !pos || !block_table || !cache) return MLA_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(w_kr) || !aligned16(cache))
        return MLA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    // c^KV = W^DKV h  (columns 0..511 of the row)
    GemmArgs g{T, kDc, d_model, (const bf16 *)h, 0, d_model, 1, (const bf16 *)w_dkv, 0, 1, d_model};
    EpiAppend e{(bf16 *)cache, seq_idx, pos, block_table, num_seqs, max_blocks, num_blocks, 0, false,
                rope_base(dims), err_word};
    cudaError_t ce = launch_gemm_simple(g, 1, e, s);
    if (ce != cudaSuccess) return MLA_ERR_CUDA;
    // k^R = RoPE(W^KR h)  (columns 512..575)
    GemmArgs g2{T, kDr, d_model, (const bf16 *)h, 0, d_model, 1, (const bf16 *)w_kr, 0, 1, d_model};
    EpiAppend e2{(bf16 *)cache, seq_idx, pos, block_table, num_seqs, max_blocks, num_blocks, kDc, true,
                 rope_base(dims), nullptr};
    return cuda_status(launch_gemm_simple(g2, 1, e2, s));
}

mla_status_t mla_absorb_q(const mla_dims_t *dims, const void *q_nope, const void *q_rope,
                          const int32_t *q_pos, const void *w_uk, int T, void *q_abs, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!q_nope || !q_rope || !w_uk || !q_abs) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(w_uk) || !aligned16(q_abs))
        return MLA_ERR_INVALID_ARG;
    const int H = dims->num_heads;
    cudaStream_t s = as_stream(stream);
    // per head i: q_abs[:, i, 0:512] = q_nope[:, i, :] (T x 128) . U^K_i (128 x 512)
    GemmArgs g{T, kDc, kDh, (const bf16 *)q_nope, kDh, (long long)H * kDh, 1,
               (const bf16 *)w_uk, (long long)kDh * kDc, kDc, 1};
    EpiStoreBf16 e{(bf16 *)q_abs, kRow, (long long)H * kRow};
    cudaError_t ce = launch_gemm_simple(g, H, e, s);
    if (ce != cudaSuccess) return MLA_ERR_CUDA;
    const int warps = T * H;
    rope_q_kernel<<<(warps + 7) / 8, 256, 0, s>>>((const bf16 *)q_rope, q_pos, T, H, (bf16 *)q_abs,
                                                  rope_base(dims));
    count_launch();
    return cuda_status(cudaGetLastError());
}

size_t mla_decode_workspace_size(const mla_dims_t *dims, int B, int s, int max_seq_len)
{
    if (check_dims(dims) != MLA_OK || B < 0 || s <= 0 || max_seq_len < 0) return 0;
    return simple_ws(dims->num_heads, B * s, max_seq_len).total;
}

mla_status_t mla_decode(const mla_dims_t *dims, const void *q_abs, const void *cache, int num_blocks,
                        const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int B,
                        int s, void *out_latent, float *out_lse, void *workspace, size_t ws_bytes,
                        uint32_t flags, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (B < 0 || s <= 0 || num_blocks < 0 || max_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (!q_abs || !cache || !block_table || !seq_lens || !out_latent) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_abs) || !aligned16(cache) || !aligned16(out_latent)) return MLA_ERR_INVALID_ARG;
    if (!workspace) return MLA_ERR_WORKSPACE;
    const int H = dims->num_heads, T = B * s;
    const SimpleWs w = simple_ws(H, T, max_blocks * kBlock);
    if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;
    cudaStream_t strm = as_stream(stream);
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), strm) != cudaSuccess) return MLA_ERR_CUDA;
    const float scale_log2 = softmax_scale(dims) * kLog2e;
    float *po = (float *)(ws + w.off_o);
    float *pl = (float *)(ws + w.off_lse);
    dim3 grid(T, H / kSimpleHeads, w.nsplit);
    if (cudaFuncSetAttribute(decode_simple_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSimpleSmem) != cudaSuccess)
        return MLA_ERR_CUDA;
    decode_simple_kernel<<<grid, 256, kSimpleSmem, strm>>>((const bf16 *)q_abs, (const bf16 *)cache, num_blocks,
                                                 block_table, max_blocks, seq_lens, s, H, scale_log2,
                                                 po, pl, w.nsplit, err);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    combine_simple_kernel<<<dim3(T, H), 128, 0, strm>>>(po, pl, w.nsplit, kSimpleSplit, seq_lens,
                                                        max_blocks, s, H, (bf16 *)out_latent, out_lse,
                                                        err);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    if (flags & MLA_SYNC_CHECK) {
        uint32_t host = 0;
        if (cudaMemcpyAsync(&host, err, sizeof host, cudaMemcpyDeviceToHost, strm) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (cudaStreamSynchronize(strm) != cudaSuccess) return MLA_ERR_CUDA;
        if (host) return MLA_ERR_DEVICE;
    }
    return MLA_OK;
}

mla_status_t mla_decode_error(const void *workspace, uint32_t *err_host, int clear, void *stream)
{
    if (!workspace || !err_host) return MLA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(err_host, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
    if (clear && cudaMemsetAsync((void *)workspace, 0, sizeof(uint32_t), s) != cudaSuccess)
        return MLA_ERR_CUDA;
    return MLA_OK;
}

mla_status_t mla_up_v(const mla_dims_t *dims, const void *latent, int T, const void *w_uv,
                      const void *w_o, int d_model, void *out_heads, void *out_model, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!latent || !w_uv || !out_heads) return MLA_ERR_INVALID_ARG;
    if (w_o && (!out_model || d_model <= 0 || d_model % 64 != 0)) return MLA_ERR_INVALID_ARG;
    if (!aligned16(latent) || !aligned16(w_uv) || !aligned16(out_heads)) return MLA_ERR_INVALID_ARG;
    const int H = dims->num_heads;
    cudaStream_t s = as_stream(stream);
    // per head i: out[:, i, :] = latent[:, i, :] (T x 512) . (U^V_i)^T (512 x 128)
    GemmArgs g{T, kDh, kDc, (const bf16 *)latent, kDc, (long long)H * kDc, 1,
               (const bf16 *)w_uv, (long long)kDh * kDc, 1, kDc};
    EpiStoreBf16 e{(bf16 *)out_heads, kDh, (long long)H * kDh};
    if (launch_gemm_simple(g, H, e, s) != cudaSuccess) return MLA_ERR_CUDA;
    if (w_o) {
        const int K = H * kDh;
        GemmArgs g2{T, d_model, K, (const bf16 *)out_heads, 0, K, 1, (const bf16 *)w_o, 0, 1, K};
        EpiStoreBf16 e2{(bf16 *)out_model, 0, d_model};
        if (launch_gemm_simple(g2, 1, e2, s) != cudaSuccess) return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

}  // extern "C"
