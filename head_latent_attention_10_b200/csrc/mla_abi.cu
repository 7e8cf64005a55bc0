// mla_abi.cu -- the extern "C" entry points declared in include/mla.h:
// argument checks, workspace layout and kernel launches.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "absorb.cuh"
#include "append_proj.cuh"
#include "common.cuh"
#include "k_simple.cuh"
#include "tc_decode64.cuh"
#include "tc_gemm.cuh"
#include "tc_prefill.cuh"
#include "tmap.cuh"

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
    if (d->rope_scaling > 1.f && d->rope_yarn_beta > 0.f &&
        d->rope_yarn_beta <= (d->rope_yarn_alpha > 0.f ? d->rope_yarn_alpha : 1.f))
        return MLA_ERR_INVALID_ARG;
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

// The frequency of each RoPE pair k: theta_k = base^(-2k/d_r), or with YaRN
// scaling s > 1 (DeepSeek-V2 paper review, long-context passage: scale 40
// over the 4K pre-training context) the NTK-by-parts interpolation: pair k
// makes r_k = L0 theta_k / (2 pi) turns over the original context L0; with
// the ramp g = clamp((r_k - alpha) / (beta - alpha), 0, 1) its frequency is
// (1 - g) theta_k / s + g theta_k.
RopeTable rope_table(const mla_dims_t *d)
{
    RopeTable t;
    const double base = rope_base(d), s = (double)d->rope_scaling;
    const double L0 = d->rope_original_ctx > 0 ? (double)d->rope_original_ctx : 4096.0;
    const double alpha = d->rope_yarn_alpha > 0.f ? (double)d->rope_yarn_alpha : 1.0;
    const double beta = d->rope_yarn_beta > 0.f ? (double)d->rope_yarn_beta : 32.0;
    const double pi = 3.14159265358979323846;
    for (int k = 0; k < kDr / 2; ++k) {
        const double th = pow(base, -2.0 * (double)k / (double)kDr);
        if (s <= 1.0) {
            t.theta[k] = th;
            continue;
        }
        double g = (L0 * th / (2.0 * pi) - alpha) / (beta - alpha);
        g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
        t.theta[k] = (1.0 - g) * th / s + g * th;
    }
    return t;
}

inline mla_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Bound of every device-side wait (ns).  With MLA_DEBUG_STALL (a test hook
// for failure detection) waits give up after 20 ms instead.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr unsigned long long kStallWaitLimitNs = 20000000ull;

// Per-device state that is filled once, on the first call that needs it:
// lock-free reads, filled under one mutex, so that concurrent first calls
// from several host threads are safe.
std::mutex g_dev_mu;
constexpr int kMaxDevices = 64;

inline int current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) of `kern` once per device,
// so that later launches can be captured into a graph.
template <class K>
cudaError_t ensure_smem_attr(K kern, int bytes, std::atomic<bool> *done)
{
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
    return e;
}

// Device address of a file-scope __device__ array on the current device,
// looked up once per device (host code only holds a stand-in for it).
template <class T>
void *symbol_address(const T &sym, std::atomic<void *> *addr)
{
    const int dev = current_device();
    if (dev < 0) return nullptr;
    void *p = addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    std::lock_guard<std::mutex> g(g_dev_mu);
    p = addr[dev].load(std::memory_order_relaxed);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, sym) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    addr[dev].store(p, std::memory_order_release);
    return p;
}

// A bf16 tensor map over a row-major 2-D or batched 3-D operand.
//   rows x inner elements per batch entry, row stride and batch stride in elements.
bool tmap(CUtensorMap *m, const void *p, uint64_t inner, uint64_t rows, uint64_t batch, uint64_t row_stride,
          uint64_t batch_stride, uint32_t box_inner, uint32_t box_rows)
{
    const uint64_t s1 = row_stride * 2, s2 = (batch > 1 ? batch_stride : row_stride * rows) * 2;
    return make_tmap_3d(m, p, inner, rows, batch, s1, s2, box_inner, box_rows, 1, swizzle_for(box_inner * 2));
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream runs, and waits for it with pdl_wait().
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// C = A B on tcgen05; `c` is the output tensor map of the staged (TMA store)
// epilogue, unused by the others.
template <int BN, bool kBmn, class Epi, bool kAmn = false>
cudaError_t launch_tc_gemm(const CUtensorMap &a, const CUtensorMap &b, int M, int N, int K, int Z, const Epi &epi,
                           uint32_t *err, cudaStream_t st, const CUtensorMap *c = nullptr)
{
    using S = GemmSmem<BN>;
    auto kern = tc_gemm_kernel<BN, kBmn, Epi, kAmn>;
    static std::atomic<bool> attr_set[kMaxDevices];
    const cudaError_t e = ensure_smem_attr(kern, S::BYTES, attr_set);
    if (e != cudaSuccess) return e;
    dim3 grid((N + BN - 1) / BN, (M + 127) / 128, Z);
    const cudaError_t le = launch_pdl(kern, grid, dim3(kGemmThreads), S::BYTES, st, a, b, c ? *c : a, M, N, K, epi,
                                      err, kWaitLimitNs);
    count_launch();
    return le;
}

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

// Tensor-core decode workspace: [error word][plan][partial latents][partial lse2]
// [merge flags][partial latents][partial lse2]; the first off_zero_end bytes
// are zeroed per call
struct TcWs {
    size_t off_plan, off_flags, off_zero_end, off_o, off_lse, total;
};

inline int dec_groups(int H, int s) { return (s * H + kGroupRows - 1) / kGroupRows; }

TcWs tc_ws(int H, int s, int B)
{
    TcWs w;
    const int groups = dec_groups(H, s);
    const int ranges = kMaxRanges / groups > 0 ? kMaxRanges / groups : 1;
    w.off_plan = kWsAlign;
    w.off_flags = align_up(w.off_plan + (size_t)plan_ints(B) * sizeof(int32_t), 16);
    w.off_zero_end = w.off_flags + (2 * (size_t)B * groups * 4 + 1) * sizeof(int);
    w.off_o = align_up(w.off_zero_end, kWsAlign);
    const size_t slots = 2 * (size_t)ranges * s * H;
    w.off_lse = align_up(w.off_o + slots * kDc * sizeof(float), kWsAlign);
    w.total = align_up(w.off_lse + slots * sizeof(float), kWsAlign);
    return w;
}

// Prefill workspace: [error word][gathered rows [B Lpad][576]][rotated q^R
// [B s][H][64]][K^C [B Lpad][H][128]][V^C [B Lpad][H][128]]
struct PfWs {
    size_t off_rows, off_qr, off_kc, off_vc, total;
    int lpad;
};

PfWs pf_ws(int H, int B, int s, int max_seq_len)
{
    PfWs w;
    w.lpad = (max_seq_len + 127) / 128 * 128;
    const size_t rows = (size_t)B * w.lpad;
    w.off_rows = kWsAlign;
    w.off_qr = align_up(w.off_rows + rows * kRow * 2, kWsAlign);
    w.off_kc = align_up(w.off_qr + (size_t)B * s * H * kDr * 2, kWsAlign);
    w.off_vc = align_up(w.off_kc + rows * H * kDh * 2, kWsAlign);
    w.total = align_up(w.off_vc + rows * H * kDh * 2, kWsAlign);
    return w;
}

int sm_count()
{
    static std::atomic<int> sms_cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return 0;
    int sms = sms_cache[dev].load(std::memory_order_acquire);
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 0;
        sms_cache[dev].store(sms, std::memory_order_release);
    }
    return sms;
}

// Ranges (persistent CTAs per row group) of the decode on the current device.
int decode_ranges(int H, int s)
{
    static std::atomic<bool> attr64[kMaxDevices];
    const int sms = sm_count();
    if (sms <= 0) return 0;
    if (ensure_smem_attr(tc_decode64_kernel<false>, kD64Smem, attr64) != cudaSuccess) return 0;
    const int groups = dec_groups(H, s);
    int r = sms / groups;
    const int cap = kMaxRanges / groups;
    if (r > cap) r = cap;
    return r > 0 ? r : 1;
}

// The tensor-core decode (plan, decode kernel, combine) on a bf16 cache, or
// on an FP8 cache (codes + per-part scales) with kFp8.
template <bool kFp8>
mla_status_t run_tc_decode(const mla_dims_t *dims, const void *q_abs, const void *cache, const float *scales,
                           int num_blocks, const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                           int B, int s, void *out_latent, float *out_lse, char *ws, size_t ws_bytes,
                           uint32_t flags, cudaStream_t strm)
{
    const int H = dims->num_heads;
    uint32_t *err = (uint32_t *)ws;
    const TcWs w = tc_ws(H, s, B);
    if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;
    const int groups = dec_groups(H, s);
    const int ranges = decode_ranges(H, s);
    if (ranges <= 0) return MLA_ERR_CUDA;
    CUtensorMap mkv;
    if (kFp8) {
        if (!make_tmap_3d_u8(&mkv, cache, kRow, (uint64_t)num_blocks * kBlock, 1, kRow, (uint64_t)num_blocks * kBlock * kRow,
                             64, kT64, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
            return MLA_ERR_CUDA;
        static std::atomic<bool> attr8[kMaxDevices];
        if (ensure_smem_attr(tc_decode64_kernel<true>, kD64SmemFp8, attr8) != cudaSuccess) return MLA_ERR_CUDA;
    } else {
        if (!tmap(&mkv, cache, kRow, (uint64_t)num_blocks * kBlock, 1, kRow, 0, 64, kT64)) return MLA_ERR_CUDA;
    }
    // the error word, the plan and the merge flags
    if (cudaMemsetAsync(ws, 0, w.off_zero_end, strm) != cudaSuccess) return MLA_ERR_CUDA;
    int32_t *plan = (int32_t *)(ws + w.off_plan);
    DecArgs da;
    da.flags = (int *)(ws + w.off_flags);
    da.q_abs = (const bf16 *)q_abs;
    da.block_table = block_table;
    da.seq_lens = seq_lens;
    da.plan = plan;
    da.out = (bf16 *)out_latent;
    da.out_lse = out_lse;
    da.part_o = (float *)(ws + w.off_o);
    da.part_lse2 = (float *)(ws + w.off_lse);
    da.err = err;
    da.limit_ns = (flags & MLA_DEBUG_STALL) ? kStallWaitLimitNs : kWaitLimitNs;
    da.stall_tile = (flags & MLA_DEBUG_STALL) ? 0 : -1;
    da.merges = (flags & MLA_DEBUG_COMBINE_ALL) ? 0 : 1;
    da.scales = scales;
    da.scale_log2 = softmax_scale(dims) * kLog2e;
    da.max_blocks = max_blocks;
    da.num_blocks = num_blocks;
    da.s = s;
    da.H = H;
    da.B = B;
    da.groups = groups;
    // the decode kernel sets itself up while the kernel before it ends, and
    // the combine launches while the decode's last CTAs finish
    cudaError_t e = launch_pdl(tc_decode64_kernel<kFp8>, dim3(ranges * groups),
                               dim3(kFp8 ? kD64ThreadsFp8 : kD64Threads), kFp8 ? kD64SmemFp8 : kD64Smem, strm, mkv,
                               da);
    count_launch();
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    static std::atomic<bool> attr_cb[kMaxDevices];
    if (ensure_smem_attr(dec_combine_kernel, kCombineSmem, attr_cb) != cudaSuccess) return MLA_ERR_CUDA;
    const int blocks = combine_blocks(B, s, H);
    const int cgrid = blocks < kCombineCtasPerSm * sm_count() ? blocks : kCombineCtasPerSm * sm_count();
    e = launch_pdl(dec_combine_kernel, dim3(cgrid), dim3(kCombineThreads), kCombineSmem, strm, (const int32_t *)plan,
                   (const int *)da.flags, (const float *)da.part_o, (const float *)da.part_lse2, B, s, H,
                   (bf16 *)out_latent, out_lse, err, da.limit_ns);
    count_launch();
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Decode scratch for callers that pass no workspace: one array per device,
// its address looked up once per device.
__device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

void *noalloc_scratch()
{
    static std::atomic<void *> addr[kMaxDevices];
    return symbol_address(g_noalloc_scratch, addr);
}

// The projection half of mla_append_cache: c^KV = W^DKV h and k^R =
// RoPE(W^KR h) written as bf16 rows to the tokens' page slots.
mla_status_t append_project(const mla_dims_t *dims, const void *h, int T, int d_model, const void *w_dkv,
                            const void *w_kr, const int32_t *seq_idx, const int32_t *pos,
                            const int32_t *block_table, int num_seqs, int max_blocks, void *cache,
                            int num_blocks, uint32_t *err_word, cudaStream_t s)
{
    if (d_model % (64 * kApSlices) == 0) {
        // K split over a cluster of CTAs, partials reduced on chip, one launch
        CUtensorMap mh, md, mr;
        if (!tmap(&mh, h, d_model, T, 1, d_model, 0, 64, 128) ||
            !tmap(&md, w_dkv, d_model, kDc, 1, d_model, 0, 64, 64) ||
            !tmap(&mr, w_kr, d_model, kDr, 1, d_model, 0, 64, 64))
            return MLA_ERR_CUDA;
        static std::atomic<bool> attr_set[kMaxDevices];
        if (ensure_smem_attr(append_proj_kernel, kApSmem, attr_set) != cudaSuccess) return MLA_ERR_CUDA;
        AppendArgs aa{(bf16 *)cache, seq_idx, pos, block_table, T, d_model, num_seqs, max_blocks, num_blocks,
                      rope_table(dims), err_word, kWaitLimitNs};
        append_proj_kernel<<<dim3(9, (T + 127) / 128, kApSlices), kApThreads, kApSmem, s>>>(mh, md, mr, aa);
        count_launch();
        return cuda_status(cudaGetLastError());
    }
    // other widths: one pass over K per 128-token tile
    CUtensorMap ma, mb1, mb2;
    if (!tmap(&ma, h, d_model, T, 1, d_model, 0, 64, 128) ||
        !tmap(&mb1, w_dkv, d_model, kDc, 1, d_model, 0, 64, 256) ||
        !tmap(&mb2, w_kr, d_model, kDr, 1, d_model, 0, 64, 64))
        return MLA_ERR_CUDA;
    // c^KV = W^DKV h  (columns 0..511 of the row)
    TcEpiAppend e{(bf16 *)cache, seq_idx, pos, block_table, num_seqs, max_blocks, num_blocks, 0, 0,
                  rope_table(dims), err_word};
    if (launch_tc_gemm<256, false>(ma, mb1, T, kDc, d_model, 1, e, err_word, s) != cudaSuccess)
        return MLA_ERR_CUDA;
    // k^R = RoPE(W^KR h)  (columns 512..575)
    TcEpiAppend e2{(bf16 *)cache, seq_idx, pos, block_table, num_seqs, max_blocks, num_blocks, kDc, 1,
                   rope_table(dims), nullptr};
    return cuda_status(launch_tc_gemm<64, false>(ma, mb2, T, kDr, d_model, 1, e2, err_word, s));
}

}  // namespace

extern "C" {

int mla_decode_ctas(const mla_dims_t *dims, int s)
{
    if (check_dims(dims) != MLA_OK || s <= 0) return 0;
    const int H = dims->num_heads;
    return decode_ranges(H, s) * dec_groups(H, s);
}

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
                               int num_blocks, const void *kv_norm_weight, float kv_norm_eps,
                               uint32_t *err_word, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || num_seqs < 0 || max_blocks < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!c_kv || !k_rope || !seq_idx || !pos || !block_table || !cache) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_kv) || !aligned16(cache) || ((uintptr_t)k_rope & 3u)) return MLA_ERR_INVALID_ARG;
    if (kv_norm_weight && (!aligned16(kv_norm_weight) || !(kv_norm_eps >= 0.f))) return MLA_ERR_INVALID_ARG;
    const int threads = 256, per = threads / 32;
    append_latent_kernel<<<(T + per - 1) / per, threads, 0, as_stream(stream)>>>(
        (const bf16 *)c_kv, (const bf16 *)k_rope, T, seq_idx, pos, block_table, num_seqs, max_blocks,
        (bf16 *)cache, num_blocks, rope_table(dims), (const bf16 *)kv_norm_weight, kv_norm_eps, err_word);
    count_launch();
    return cuda_status(cudaGetLastError());
}

mla_status_t mla_append_cache(const mla_dims_t *dims, const void *h, int T, int d_model,
                              const void *w_dkv, const void *w_kr, const int32_t *seq_idx,
                              const int32_t *pos, const int32_t *block_table, int num_seqs,
                              int max_blocks, void *cache, int num_blocks, const void *kv_norm_weight,
                              float kv_norm_eps, uint32_t *err_word, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || num_seqs < 0 || max_blocks < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (d_model <= 0 || d_model % 64 != 0) return MLA_ERR_UNSUPPORTED;
    if (!h || !w_dkv || !w_kr || !seq_idx || !pos || !block_table || !cache) return MLA_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(w_kr) || !aligned16(cache))
        return MLA_ERR_INVALID_ARG;
    if (kv_norm_weight && (!aligned16(kv_norm_weight) || !(kv_norm_eps >= 0.f))) return MLA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const mla_status_t pst = append_project(dims, h, T, d_model, w_dkv, w_kr, seq_idx, pos, block_table, num_seqs,
                                            max_blocks, cache, num_blocks, err_word, s);
    if (pst != MLA_OK || !kv_norm_weight) return pst;
    // RMSNorm of the latent rows just written (their columns come from
    // different CTAs of the projection, so the row's norm is taken after it)
    latent_rmsnorm_kernel<<<(T + 7) / 8, 256, 0, s>>>(T, seq_idx, pos, block_table, num_seqs, max_blocks,
                                                      (bf16 *)cache, num_blocks, (const bf16 *)kv_norm_weight,
                                                      kv_norm_eps);
    count_launch();
    return cuda_status(cudaGetLastError());
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
    // per head i: q_abs[:, i, 0:512] = q_nope[:, i, :] (T x 128) . U^K_i (128 x 512),
    // and the RoPE part, in one launch
    CUtensorMap ma, mb, mo;
    if (!tmap(&ma, q_nope, kDh, T, H, (uint64_t)H * kDh, kDh, 64, 128) ||
        !tmap(&mb, w_uk, kDc, kDh, H, kDc, (uint64_t)kDh * kDc, 64, 64) ||
        !make_tmap_3d(&mo, q_abs, kRow, H, T, (uint64_t)kRow * 2, (uint64_t)H * kRow * 2, 64, 1, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))   // q_abs as {576, H, T}: box 64 columns x 1 head x 128 tokens
        return MLA_ERR_CUDA;
    static std::atomic<bool> attr_set[kMaxDevices];
    if (ensure_smem_attr(absorb_kernel, kAbSmem, attr_set) != cudaSuccess) return MLA_ERR_CUDA;
    absorb_kernel<<<dim3(H, (T + 127) / 128, kAbParts), kAbThreads, kAbSmem, s>>>(ma, mb, mo, (const bf16 *)q_rope, q_pos, T, H,
                                                                         (bf16 *)q_abs, rope_table(dims), nullptr,
                                                                         kWaitLimitNs);
    count_launch();
    return cuda_status(cudaGetLastError());
}

size_t mla_decode_workspace_size(const mla_dims_t *dims, int B, int s, int max_seq_len)
{
    if (check_dims(dims) != MLA_OK || B < 0 || s <= 0 || max_seq_len < 0) return 0;
    const size_t a = simple_ws(dims->num_heads, B * s, max_seq_len).total;
    const size_t b = tc_ws(dims->num_heads, s, B).total;
    return a > b ? a : b;
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
    if (num_blocks == 0 || max_blocks == 0) return MLA_ERR_INVALID_ARG;
    if (!q_abs || !cache || !block_table || !seq_lens || !out_latent) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_abs) || !aligned16(cache) || !aligned16(out_latent)) return MLA_ERR_INVALID_ARG;
    if (!workspace) return MLA_ERR_WORKSPACE;
    const int H = dims->num_heads, T = B * s;
    cudaStream_t strm = as_stream(stream);
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    const float scale_log2 = softmax_scale(dims) * kLog2e;
    if (flags & MLA_FORCE_SIMPLE) {
        const SimpleWs w = simple_ws(H, T, max_blocks * kBlock);
        if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;
        if (cudaMemsetAsync(err, 0, sizeof(uint32_t), strm) != cudaSuccess) return MLA_ERR_CUDA;
        float *po = (float *)(ws + w.off_o);
        float *pl = (float *)(ws + w.off_lse);
        dim3 grid(T, H / kSimpleHeads, w.nsplit);
        static std::atomic<bool> attr_set[kMaxDevices];
        if (ensure_smem_attr(decode_simple_kernel, kSimpleSmem, attr_set) != cudaSuccess) return MLA_ERR_CUDA;
        decode_simple_kernel<<<grid, 256, kSimpleSmem, strm>>>((const bf16 *)q_abs, (const bf16 *)cache,
                                                               num_blocks, block_table, max_blocks, seq_lens, s,
                                                               H, scale_log2, po, pl, w.nsplit, err);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
        combine_simple_kernel<<<dim3(T, H), 128, 0, strm>>>(po, pl, w.nsplit, kSimpleSplit, seq_lens,
                                                            max_blocks, s, H, (bf16 *)out_latent, out_lse, err);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    } else {
        const mla_status_t r = run_tc_decode<false>(dims, q_abs, cache, nullptr, num_blocks, block_table, max_blocks,
                                                    seq_lens, B, s, out_latent, out_lse, ws, ws_bytes, flags, strm);
        if (r != MLA_OK) return r;
    }
    if (flags & MLA_SYNC_CHECK) {
        uint32_t host = 0;
        if (cudaMemcpyAsync(&host, err, sizeof host, cudaMemcpyDeviceToHost, strm) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (cudaStreamSynchronize(strm) != cudaSuccess) return MLA_ERR_CUDA;
        if (host) return MLA_ERR_DEVICE;
    }
    return MLA_OK;
}

mla_status_t mla_decode_noalloc(const mla_dims_t *dims, const void *q_abs, const void *cache,
                                int num_blocks, const int32_t *block_table, int max_blocks,
                                const int32_t *seq_lens, int B, int s, void *out_latent, float *out_lse,
                                uint32_t flags, void *stream)
{
    const mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (B < 0 || s <= 0 || num_blocks < 0 || max_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    const size_t need = (flags & MLA_FORCE_SIMPLE)
                            ? simple_ws(dims->num_heads, B * s, max_blocks * kBlock).total
                            : tc_ws(dims->num_heads, s, B).total;
    if (need > (size_t)MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
    void *scratch = noalloc_scratch();
    if (!scratch) return MLA_ERR_CUDA;
    return mla_decode(dims, q_abs, cache, num_blocks, block_table, max_blocks, seq_lens, B, s, out_latent,
                      out_lse, scratch, MLA_NOALLOC_SCRATCH_BYTES, flags, stream);
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
    if (w_o && (!aligned16(w_o) || !aligned16(out_model))) return MLA_ERR_INVALID_ARG;
    if (!aligned16(latent) || !aligned16(w_uv) || !aligned16(out_heads)) return MLA_ERR_INVALID_ARG;
    const int H = dims->num_heads;
    cudaStream_t s = as_stream(stream);
    // per head i: out[:, i, :] = latent[:, i, :] (T x 512) . (U^V_i)^T (512 x 128)
    CUtensorMap ma, mb, mo;
    if (!tmap(&ma, latent, kDc, T, H, (uint64_t)H * kDc, kDc, 64, 128) ||
        !tmap(&mb, w_uv, kDc, kDh, H, kDc, (uint64_t)kDh * kDc, 64, 128) ||
        !make_tmap_3d(&mo, out_heads, kDh, H, T, (uint64_t)kDh * 2, (uint64_t)H * kDh * 2, 64, 1, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))   // out_heads as {128, H, T}
        return MLA_ERR_CUDA;
    if (launch_tc_gemm<128, false>(ma, mb, T, kDh, kDc, H, TcEpiTmaStore{}, nullptr, s, &mo) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (w_o) {
        // out_model = out_heads (T x H*128) . W^O^T
        const int K = H * kDh;
        CUtensorMap ma2, mb2;
        if (!tmap(&ma2, out_heads, K, T, 1, K, 0, 64, 128) || !tmap(&mb2, w_o, K, d_model, 1, K, 0, 64, 256))
            return MLA_ERR_CUDA;
        TcEpiStore e2{(bf16 *)out_model, 0, d_model};
        if (launch_tc_gemm<256, false>(ma2, mb2, T, d_model, K, 1, e2, nullptr, s) != cudaSuccess)
            return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

size_t mla_prefill_workspace_size(const mla_dims_t *dims, int B, int s, int max_seq_len)
{
    if (check_dims(dims) != MLA_OK || B < 0 || s <= 0 || max_seq_len < s) return 0;
    return pf_ws(dims->num_heads, B, s, max_seq_len).total;
}

mla_status_t mla_prefill(const mla_dims_t *dims, const void *q_nope, const void *q_rope, const int32_t *q_pos,
                         const void *w_uk, const void *w_uv, const void *cache, int num_blocks,
                         const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int B, int s,
                         int max_seq_len, void *out, float *out_lse, void *workspace, size_t ws_bytes,
                         uint32_t flags, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (B < 0 || s <= 0 || num_blocks < 0 || max_blocks < 0 || max_seq_len < s) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (num_blocks == 0 || max_blocks == 0) return MLA_ERR_INVALID_ARG;
    if (!q_nope || !q_rope || !w_uk || !w_uv || !cache || !block_table || !seq_lens || !out)
        return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(cache) ||
        !aligned16(out))
        return MLA_ERR_INVALID_ARG;
    if (!workspace) return MLA_ERR_WORKSPACE;
    const int H = dims->num_heads;
    const PfWs w = pf_ws(H, B, s, max_seq_len);
    if (ws_bytes < w.total) return MLA_ERR_WORKSPACE;
    const long long rows_total = (long long)B * w.lpad;
    if (rows_total > (1ll << 31) - 1 || (long long)B * s * H > (1ll << 31) - 1) return MLA_ERR_UNSUPPORTED;
    const int M = (int)rows_total;
    cudaStream_t strm = as_stream(stream);
    char *ws = (char *)workspace;
    uint32_t *err = (uint32_t *)ws;
    bf16 *rows = (bf16 *)(ws + w.off_rows), *q_rot = (bf16 *)(ws + w.off_qr);
    bf16 *kc = (bf16 *)(ws + w.off_kc), *vc = (bf16 *)(ws + w.off_vc);
    const long long cap_blocks = (long long)max_blocks * kBlock;
    const int l_cap = cap_blocks < max_seq_len ? (int)cap_blocks : max_seq_len;

    // tensor maps: the expansions, one GEMM each over all heads,
    // K^C [M][H*128] = rows [M][512] . [U^K_0; ..; U^K_{H-1}]^T (the stacked
    // [H*128][512] weights are K-major as stored), and the attention
    CUtensorMap ma, muk, muv, mkc, mvc, skc, svc;
    if (!tmap(&ma, rows, kDc, M, 1, kRow, 0, 64, 128) ||
        !tmap(&muk, w_uk, kDc, (uint64_t)H * kDh, 1, kDc, 0, 64, 256) ||
        !tmap(&muv, w_uv, kDc, (uint64_t)H * kDh, 1, kDc, 0, 64, 256) ||
        !make_tmap_3d(&skc, kc, (uint64_t)H * kDh, 1, M, (uint64_t)H * kDh * 2, (uint64_t)H * kDh * 2, 64, 1, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_3d(&svc, vc, (uint64_t)H * kDh, 1, M, (uint64_t)H * kDh * 2, (uint64_t)H * kDh * 2, 64, 1, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_3d(&mkc, kc, kDh, H, M, kDh * 2, (uint64_t)H * kDh * 2, 64, 1, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_3d(&mvc, vc, kDh, H, M, kDh * 2, (uint64_t)H * kDh * 2, 64, 1, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return MLA_ERR_CUDA;
    PrefillMaps pm;
    {
        const uint64_t odims[4] = {(uint64_t)kDh, (uint64_t)H, (uint64_t)s, (uint64_t)B};
        const uint64_t ostr[3] = {(uint64_t)kDh * 2, (uint64_t)H * kDh * 2, (uint64_t)s * H * kDh * 2};
        const uint32_t obox[4] = {64, 1, 128, 1};
        if (!make_tmap_4d(&pm.out, out, odims, ostr, obox, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tmap_3d(&pm.kr, rows, kRow, M, 1, kRow * 2, (uint64_t)M * kRow * 2, 64, 128, 1,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return MLA_ERR_CUDA;
        pm.kc = mkc;
        pm.vc = mvc;
    }
    if (cudaMemsetAsync(err, 0, sizeof(uint32_t), strm) != cudaSuccess) return MLA_ERR_CUDA;
    {
        const long long work = rows_total * (kRow / 8) + (long long)B * s * (kDr / 2);
        long long blocks = (work + 255) / 256;
        if (blocks > 8ll * sm_count()) blocks = 8ll * sm_count();
        prefill_prepare_kernel<<<(int)blocks, 256, 0, strm>>>((const bf16 *)cache, num_blocks, block_table,
                                                              max_blocks, seq_lens, B, s, H, w.lpad, l_cap, rows,
                                                              (const bf16 *)q_rope, q_pos, q_rot, rope_table(dims),
                                                              err);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    }
    if (launch_tc_gemm<256, false, TcEpiTmaStore>(ma, muk, M, H * kDh, kDc, 1, TcEpiTmaStore{}, err, strm, &skc) !=
            cudaSuccess ||
        launch_tc_gemm<256, false, TcEpiTmaStore>(ma, muv, M, H * kDh, kDc, 1, TcEpiTmaStore{}, err, strm, &svc) !=
            cudaSuccess)
        return MLA_ERR_CUDA;
    PrefillArgs pa;
    pa.q_nope = (const bf16 *)q_nope;
    pa.q_rot = q_rot;
    pa.seq_lens = seq_lens;
    pa.s = s;
    pa.H = H;
    pa.lpad = w.lpad;
    pa.l_cap = l_cap;
    pa.scale_log2 = softmax_scale(dims) * kLog2e;
    pa.out_lse = out_lse;
    pa.err = err;
    pa.limit_ns = kWaitLimitNs;
    static std::atomic<bool> attr_set[kMaxDevices];
    if (ensure_smem_attr(tc_prefill_kernel, kPfSmem, attr_set) != cudaSuccess) return MLA_ERR_CUDA;
    tc_prefill_kernel<<<dim3((s + 127) / 128, H, B), kPfThreads, kPfSmem, strm>>>(pm, pa);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    if (flags & MLA_SYNC_CHECK) {
        uint32_t h = 0;
        if (cudaMemcpyAsync(&h, err, sizeof h, cudaMemcpyDeviceToHost, strm) != cudaSuccess ||
            cudaStreamSynchronize(strm) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (h) return MLA_ERR_DEVICE;
    }
    return MLA_OK;
}

mla_status_t mla_append_latent_fp8(const mla_dims_t *dims, const void *c_kv, const void *k_rope, int T,
                                   const int32_t *seq_idx, const int32_t *pos, const int32_t *block_table,
                                   int num_seqs, int max_blocks, void *codes, float *scales, int num_blocks,
                                   const void *kv_norm_weight, float kv_norm_eps, uint32_t *err_word, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || num_seqs < 0 || max_blocks < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!c_kv || !k_rope || !seq_idx || !pos || !block_table || !codes || !scales) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_kv) || !aligned16(codes) || ((uintptr_t)k_rope & 3u) || ((uintptr_t)scales & 7u))
        return MLA_ERR_INVALID_ARG;
    if (kv_norm_weight && (!aligned16(kv_norm_weight) || !(kv_norm_eps >= 0.f))) return MLA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    append_latent_fp8_kernel<<<(T + 7) / 8, 256, 0, s>>>((const bf16 *)c_kv, (const bf16 *)k_rope, T, seq_idx, pos,
                                                         block_table, num_seqs, max_blocks, (uint8_t *)codes, scales,
                                                         num_blocks, rope_table(dims), (const bf16 *)kv_norm_weight,
                                                         kv_norm_eps, err_word);
    count_launch();
    return cuda_status(cudaGetLastError());
}

mla_status_t mla_decode_fp8(const mla_dims_t *dims, const void *q_abs, const void *codes, const float *scales,
                            int num_blocks, const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                            int B, int s, void *out_latent, float *out_lse, void *workspace, size_t ws_bytes,
                            uint32_t flags, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (B < 0 || s <= 0 || num_blocks < 0 || max_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (num_blocks == 0 || max_blocks == 0) return MLA_ERR_INVALID_ARG;
    if (flags & MLA_FORCE_SIMPLE) return MLA_ERR_UNSUPPORTED;
    if (!q_abs || !codes || !scales || !block_table || !seq_lens || !out_latent) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_abs) || !aligned16(codes) || !aligned16(scales) || !aligned16(out_latent))
        return MLA_ERR_INVALID_ARG;
    if (!workspace) return MLA_ERR_WORKSPACE;
    cudaStream_t strm = as_stream(stream);
    char *ws = (char *)workspace;
    const mla_status_t r = run_tc_decode<true>(dims, q_abs, codes, scales, num_blocks, block_table, max_blocks,
                                               seq_lens, B, s, out_latent, out_lse, ws, ws_bytes, flags, strm);
    if (r != MLA_OK) return r;
    if (flags & MLA_SYNC_CHECK) {
        uint32_t host = 0;
        if (cudaMemcpyAsync(&host, ws, sizeof host, cudaMemcpyDeviceToHost, strm) != cudaSuccess ||
            cudaStreamSynchronize(strm) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (host) return MLA_ERR_DEVICE;
    }
    return MLA_OK;
}

mla_status_t mla_fold_weights(const mla_dims_t *dims, int d_q, const void *w_uq, const void *w_uk, void *w_qk,
                              int d_model, const void *w_o, const void *w_uv, void *w_ov, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    const bool qk = w_uq || w_uk || w_qk, ov = w_o || w_uv || w_ov;
    if (qk && (!w_uq || !w_uk || !w_qk || d_q <= 0 || d_q % 64 != 0)) return MLA_ERR_INVALID_ARG;
    if (ov && (!w_o || !w_uv || !w_ov || d_model <= 0 || d_model % 64 != 0)) return MLA_ERR_INVALID_ARG;
    if ((w_uq && !aligned16(w_uq)) || (w_uk && !aligned16(w_uk)) || (w_qk && !aligned16(w_qk)) ||
        (w_o && !aligned16(w_o)) || (w_uv && !aligned16(w_uv)) || (w_ov && !aligned16(w_ov)))
        return MLA_ERR_INVALID_ARG;
    const int H = dims->num_heads;
    cudaStream_t s = as_stream(stream);
    if (qk) {
        // W^QK_i [512][d_q] = (U^K_i)^T [512][128] . W^UQ_i [128][d_q]: A = U^K_i
        // read MN-major (stored [128][512]), B = W^UQ_i MN-major (stored [128][d_q])
        CUtensorMap ma, mb, mc;
        if (!tmap(&ma, w_uk, kDc, kDh, H, kDc, (uint64_t)kDh * kDc, 64, 64) ||
            !tmap(&mb, w_uq, d_q, kDh, H, d_q, (uint64_t)kDh * d_q, 64, 64) ||
            !make_tmap_3d(&mc, w_qk, d_q, H, kDc, (uint64_t)kDc * d_q * 2, (uint64_t)d_q * 2, 64, 1, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return MLA_ERR_CUDA;
        if (launch_tc_gemm<256, true, TcEpiTmaStore, true>(ma, mb, kDc, d_q, kDh, H, TcEpiTmaStore{}, nullptr, s,
                                                           &mc) != cudaSuccess)
            return MLA_ERR_CUDA;
    }
    if (ov) {
        // W^OV [d_model][H*512], block i = O_i [d_model][128] . U^V_i [128][512]:
        // A = the 128 columns of head i in W^O (K-major), B = U^V_i MN-major
        CUtensorMap ma, mb, mc;
        if (!tmap(&ma, w_o, kDh, d_model, H, (uint64_t)H * kDh, kDh, 64, 128) ||
            !tmap(&mb, w_uv, kDc, kDh, H, kDc, (uint64_t)kDh * kDc, 64, 64) ||
            !make_tmap_3d(&mc, w_ov, kDc, H, d_model, (uint64_t)kDc * 2, (uint64_t)H * kDc * 2, 64, 1, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return MLA_ERR_CUDA;
        if (launch_tc_gemm<256, true, TcEpiTmaStore>(ma, mb, d_model, kDc, kDh, H, TcEpiTmaStore{}, nullptr, s, &mc) !=
            cudaSuccess)
            return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

mla_status_t mla_absorb_q_folded(const mla_dims_t *dims, const void *c_q, int d_q, const void *q_rope,
                                 const int32_t *q_pos, const void *w_qk, int T, void *q_abs, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || d_q <= 0 || d_q % 64 != 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!c_q || !q_rope || !w_qk || !q_abs) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_q) || !aligned16(w_qk) || !aligned16(q_abs) || ((uintptr_t)q_rope & 3u))
        return MLA_ERR_INVALID_ARG;
    const int H = dims->num_heads;
    cudaStream_t s = as_stream(stream);
    // q_abs[t][i][0:512] = W^QK_i c_q[t]: one GEMM over all heads, C [T][H*512]
    // = c_q [T][d_q] . W^QK^T (W^QK stored [H*512][d_q], K-major), each
    // 512-column head block stored into its q_abs row
    CUtensorMap ma, mb, mc;
    if (!tmap(&ma, c_q, d_q, T, 1, d_q, 0, 64, 128) ||
        !tmap(&mb, w_qk, d_q, (uint64_t)H * kDc, 1, d_q, 0, 64, 256) ||
        !make_tmap_3d(&mc, q_abs, kDc, H, T, (uint64_t)kRow * 2, (uint64_t)H * kRow * 2, 64, 1, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return MLA_ERR_CUDA;
    TcEpiTmaStore e;
    e.split_n = kDc;
    if (launch_tc_gemm<256, false, TcEpiTmaStore>(ma, mb, T, H * kDc, d_q, 1, e, nullptr, s, &mc) != cudaSuccess)
        return MLA_ERR_CUDA;
    long long blocks = ((long long)T * (kDr / 2) + 255) / 256;
    if (blocks > 8ll * sm_count()) blocks = 8ll * sm_count();
    rope_q_kernel<<<(int)blocks, 256, 0, s>>>((const bf16 *)q_rope, q_pos, T, H, (bf16 *)q_abs, kRow, kDc,
                                              rope_table(dims));
    count_launch();
    return cuda_status(cudaGetLastError());
}

mla_status_t mla_up_out_folded(const mla_dims_t *dims, const void *latent, int T, const void *w_ov, int d_model,
                               void *out_model, void *stream)
{
    mla_status_t st = check_dims(dims);
    if (st != MLA_OK) return st;
    if (T < 0 || d_model <= 0 || d_model % 64 != 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!latent || !w_ov || !out_model) return MLA_ERR_INVALID_ARG;
    if (!aligned16(latent) || !aligned16(w_ov) || !aligned16(out_model)) return MLA_ERR_INVALID_ARG;
    const int K = dims->num_heads * kDc;
    cudaStream_t s = as_stream(stream);
    // out_model [T][d_model] = latent [T][H*512] . W^OV^T (W^OV [d_model][H*512], K-major)
    CUtensorMap ma, mb;
    if (!tmap(&ma, latent, K, T, 1, K, 0, 64, 128) || !tmap(&mb, w_ov, K, d_model, 1, K, 0, 64, 256))
        return MLA_ERR_CUDA;
    TcEpiStore e{(bf16 *)out_model, 0, d_model};
    if (launch_tc_gemm<256, false>(ma, mb, T, d_model, K, 1, e, nullptr, s) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

}  // extern "C"
