"""Python binding of the MLA decode library (include/mla.h).

Argument marshalling only: every call takes torch tensors that already live
on the GPU, passes their device pointers and the current CUDA stream to the
C entry point of the same name in libmla_b200.so, and raises MLAError on a
non-zero status.  Every step of the computation runs in the library's CUDA
kernels; there is no fallback of any kind.  If libmla_b200.so has not been
built (python head_latent_attention_10_b200/build.py) the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmla_b200.so")

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_WORKSPACE, MLA_ERR_DEVICE = range(6)
MLA_DEVERR_BLOCK_ID, MLA_DEVERR_SEQ_LEN, MLA_DEVERR_TIMEOUT = 0x1, 0x2, 0x4
MLA_SYNC_CHECK, MLA_FORCE_SIMPLE, MLA_DEBUG_STALL, MLA_DEBUG_COMBINE_ALL = 0x1, 0x2, 0x100, 0x200

EXPORTED = ("mla_status_string", "mla_append_cache", "mla_append_latent", "mla_absorb_q",
            "mla_decode_workspace_size", "mla_decode", "mla_decode_error", "mla_up_v",
            "mla_kernel_launches", "mla_decode_ctas", "mla_decode_noalloc",
            "mla_prefill_workspace_size", "mla_prefill", "mla_append_latent_fp8", "mla_decode_fp8",
            "mla_fold_weights", "mla_absorb_q_folded", "mla_up_out_folded")


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mla_status_string(status)}")


class mla_dims_t(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("d_head", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("rope_scaling", ctypes.c_float), ("rope_original_ctx", ctypes.c_int32),
                ("rope_yarn_alpha", ctypes.c_float), ("rope_yarn_beta", ctypes.c_float)]


def dims(num_heads: int, softmax_scale: float = 0.0, rope_base: float = 10000.0, d_c: int = 512,
         d_rope: int = 64, d_head: int = 128, block_size: int = 64, rope_scaling: float = 0.0,
         rope_original_ctx: int = 0, rope_yarn_alpha: float = 0.0, rope_yarn_beta: float = 0.0) -> mla_dims_t:
    """Shape descriptor; softmax_scale <= 0 selects 1/sqrt(d_head + d_rope);
    rope_scaling > 1 selects YaRN-scaled RoPE frequencies."""
    return mla_dims_t(num_heads, d_c, d_rope, d_head, block_size, softmax_scale, rope_base, rope_scaling,
                      rope_original_ctx, rope_yarn_alpha, rope_yarn_beta)


_LIB = None
_vp, _i = ctypes.c_void_p, ctypes.c_int


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with "
                           "python head_latent_attention_10_b200/build.py")
    lib = ctypes.CDLL(path)
    D = ctypes.POINTER(mla_dims_t)
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_status_string.argtypes = [_i]
    _f = ctypes.c_float
    lib.mla_append_cache.argtypes = [D, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _f, _vp, _vp]
    lib.mla_append_latent.argtypes = [D, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _f, _vp, _vp]
    lib.mla_absorb_q.argtypes = [D, _vp, _vp, _vp, _vp, _i, _vp, _vp]
    lib.mla_decode_workspace_size.argtypes = [D, _i, _i, _i]
    lib.mla_decode_workspace_size.restype = ctypes.c_size_t
    lib.mla_decode.argtypes = [D, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _vp, _vp, _vp, ctypes.c_size_t,
                               ctypes.c_uint32, _vp]
    lib.mla_decode_noalloc.argtypes = [D, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _vp, _vp, ctypes.c_uint32, _vp]
    lib.mla_decode_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32), _i, _vp]
    lib.mla_up_v.argtypes = [D, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp]
    lib.mla_decode_ctas.argtypes = [D, _i]
    lib.mla_decode_ctas.restype = _i
    lib.mla_prefill_workspace_size.argtypes = [D, _i, _i, _i]
    lib.mla_prefill_workspace_size.restype = ctypes.c_size_t
    lib.mla_prefill.argtypes = [D, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp, _vp,
                                _vp, ctypes.c_size_t, ctypes.c_uint32, _vp]
    lib.mla_append_latent_fp8.argtypes = [D, _vp, _vp, _i, _vp, _vp, _vp, _i, _i, _vp, _vp, _i, _vp, _f, _vp, _vp]
    lib.mla_decode_fp8.argtypes = [D, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _vp, _vp, _vp, ctypes.c_size_t,
                                   ctypes.c_uint32, _vp]
    lib.mla_fold_weights.argtypes = [D, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp]
    lib.mla_absorb_q_folded.argtypes = [D, _vp, _i, _vp, _vp, _vp, _i, _vp, _vp]
    lib.mla_up_out_folded.argtypes = [D, _vp, _i, _vp, _i, _vp, _vp]
    lib.mla_kernel_launches.argtypes = []
    lib.mla_kernel_launches.restype = ctypes.c_uint64
    for name in EXPORTED:
        if name not in ("mla_status_string", "mla_decode_workspace_size", "mla_kernel_launches",
                        "mla_decode_ctas", "mla_prefill_workspace_size"):
            getattr(lib, name).restype = _i
    _LIB = lib
    return lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MLAError(status, where)


def mla_status_string(status: int) -> str:
    return load_library().mla_status_string(status).decode()


def mla_append_cache(d, h, w_dkv, w_kr, seq_idx, pos, block_table, cache, err_word=None, stream=None,
                     kv_norm_weight=None, kv_norm_eps=1e-6):
    """c^KV = W^DKV h (RMS-normalised with kv_norm_weight if given) and
    k^R = RoPE(W^KR h, pos) written to the paged cache."""
    T, d_model = h.shape
    _check(load_library().mla_append_cache(
        ctypes.byref(d), _ptr(h), T, d_model, _ptr(w_dkv), _ptr(w_kr), _ptr(seq_idx), _ptr(pos),
        _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(cache), cache.shape[0],
        _ptr(kv_norm_weight), kv_norm_eps, _ptr(err_word), _stream(stream)), "mla_append_cache")


def mla_append_latent(d, c_kv, k_rope, seq_idx, pos, block_table, cache, err_word=None, stream=None,
                      kv_norm_weight=None, kv_norm_eps=1e-6):
    """[c_kv (RMS-normalised with kv_norm_weight if given) | RoPE(k_rope, pos)]
    written to the paged cache."""
    _check(load_library().mla_append_latent(
        ctypes.byref(d), _ptr(c_kv), _ptr(k_rope), c_kv.shape[0], _ptr(seq_idx), _ptr(pos),
        _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(cache), cache.shape[0],
        _ptr(kv_norm_weight), kv_norm_eps, _ptr(err_word), _stream(stream)), "mla_append_latent")


def mla_absorb_q(d, q_nope, q_rope, q_pos, w_uk, q_abs, stream=None):
    """q_abs = [(U^K_i)^T q^C_i | RoPE(q^R_i, q_pos)]."""
    _check(load_library().mla_absorb_q(
        ctypes.byref(d), _ptr(q_nope), _ptr(q_rope), _ptr(q_pos), _ptr(w_uk), q_nope.shape[0],
        _ptr(q_abs), _stream(stream)), "mla_absorb_q")


def mla_kernel_launches() -> int:
    """Kernels the library has launched in this process."""
    return int(load_library().mla_kernel_launches())


def mla_decode_ctas(d, s: int = 1) -> int:
    """CTAs of the tensor-core decode's persistent grid on the current device."""
    return int(load_library().mla_decode_ctas(ctypes.byref(d), s))


def mla_decode_workspace_size(d, B: int, s: int, max_seq_len: int) -> int:
    return int(load_library().mla_decode_workspace_size(ctypes.byref(d), B, s, max_seq_len))


def mla_decode(d, q_abs, cache, block_table, seq_lens, s, out_latent, out_lse, workspace,
               flags: int = 0, stream=None):
    """Absorbed attention over the paged latent cache; writes out_latent and out_lse."""
    B = seq_lens.shape[0]
    _check(load_library().mla_decode(
        ctypes.byref(d), _ptr(q_abs), _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, s, _ptr(out_latent), _ptr(out_lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), flags, _stream(stream)),
        "mla_decode")


MLA_NOALLOC_SCRATCH_BYTES = 40 << 20


def mla_decode_noalloc(d, q_abs, cache, block_table, seq_lens, s, out_latent, out_lse,
                       flags: int = 0, stream=None):
    """mla_decode on the library's own per-device scratch array (no workspace)."""
    B = seq_lens.shape[0]
    _check(load_library().mla_decode_noalloc(
        ctypes.byref(d), _ptr(q_abs), _ptr(cache), cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, s, _ptr(out_latent), _ptr(out_lse), flags,
        _stream(stream)), "mla_decode_noalloc")


def mla_decode_error(workspace, clear: bool = False, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(load_library().mla_decode_error(_ptr(workspace), ctypes.byref(v), int(clear),
                                           _stream(stream)), "mla_decode_error")
    return int(v.value)


def mla_prefill_workspace_size(d, B: int, s: int, max_seq_len: int) -> int:
    return int(load_library().mla_prefill_workspace_size(ctypes.byref(d), B, s, max_seq_len))


def mla_prefill(d, q_nope, q_rope, q_pos, w_uk, w_uv, cache, block_table, seq_lens, s, max_seq_len,
                out, out_lse, workspace, flags: int = 0, stream=None):
    """Expanded-form attention of the last s tokens of each sequence over its
    cached latents; writes the per-head outputs out [B*s][H][d_head]."""
    B = seq_lens.shape[0]
    _check(load_library().mla_prefill(
        ctypes.byref(d), _ptr(q_nope), _ptr(q_rope), _ptr(q_pos), _ptr(w_uk), _ptr(w_uv), _ptr(cache),
        cache.shape[0], _ptr(block_table), block_table.shape[1], _ptr(seq_lens), B, s, max_seq_len,
        _ptr(out), _ptr(out_lse), _ptr(workspace), workspace.numel() * workspace.element_size(), flags,
        _stream(stream)), "mla_prefill")


def mla_append_latent_fp8(d, c_kv, k_rope, seq_idx, pos, block_table, codes, scales, err_word=None,
                          stream=None, kv_norm_weight=None, kv_norm_eps=1e-6):
    """The row [c_kv | RoPE(k_rope, pos)] (RMS-normalised latent if
    kv_norm_weight is given) quantized to E4M3 codes [num_blocks][64][576]
    uint8 with per-part fp32 scales [num_blocks][64][2]."""
    _check(load_library().mla_append_latent_fp8(
        ctypes.byref(d), _ptr(c_kv), _ptr(k_rope), c_kv.shape[0], _ptr(seq_idx), _ptr(pos),
        _ptr(block_table), block_table.shape[0], block_table.shape[1], _ptr(codes), _ptr(scales),
        codes.shape[0], _ptr(kv_norm_weight), kv_norm_eps, _ptr(err_word), _stream(stream)),
        "mla_append_latent_fp8")


def mla_decode_fp8(d, q_abs, codes, scales, block_table, seq_lens, s, out_latent, out_lse, workspace,
                   flags: int = 0, stream=None):
    """Absorbed attention over the FP8 latent cache; writes out_latent and out_lse."""
    B = seq_lens.shape[0]
    _check(load_library().mla_decode_fp8(
        ctypes.byref(d), _ptr(q_abs), _ptr(codes), _ptr(scales), codes.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), B, s, _ptr(out_latent), _ptr(out_lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), flags, _stream(stream)), "mla_decode_fp8")


def mla_fold_weights(d, w_uq=None, w_uk=None, w_qk=None, w_o=None, w_uv=None, w_ov=None, stream=None):
    """W^QK_i = (U^K_i)^T W^UQ_i into w_qk [H][512][d_q]; W^OV block i = O_i U^V_i
    into w_ov [d_model][H*512].  Either group may be left out."""
    d_q = 0 if w_uq is None else w_uq.shape[-1]
    d_model = 0 if w_o is None else w_o.shape[0]
    _check(load_library().mla_fold_weights(
        ctypes.byref(d), d_q, _ptr(w_uq), _ptr(w_uk), _ptr(w_qk), d_model, _ptr(w_o), _ptr(w_uv), _ptr(w_ov),
        _stream(stream)), "mla_fold_weights")


def mla_absorb_q_folded(d, c_q, q_rope, q_pos, w_qk, q_abs, stream=None):
    """q_abs = [W^QK_i c_q | RoPE(q^R_i, q_pos)]."""
    _check(load_library().mla_absorb_q_folded(
        ctypes.byref(d), _ptr(c_q), c_q.shape[1], _ptr(q_rope), _ptr(q_pos), _ptr(w_qk), c_q.shape[0],
        _ptr(q_abs), _stream(stream)), "mla_absorb_q_folded")


def mla_up_out_folded(d, latent, w_ov, out_model, stream=None):
    """out_model = sum_i W^OV_i latent_i."""
    _check(load_library().mla_up_out_folded(
        ctypes.byref(d), _ptr(latent), latent.shape[0], _ptr(w_ov), w_ov.shape[0], _ptr(out_model),
        _stream(stream)), "mla_up_out_folded")


def mla_up_v(d, latent, w_uv, out_heads, w_o=None, out_model=None, stream=None):
    """out_heads = U^V_i latent_i; out_model = sum_i O_i out_heads_i if w_o is given."""
    d_model = 0 if w_o is None else w_o.shape[0]
    _check(load_library().mla_up_v(
        ctypes.byref(d), _ptr(latent), latent.shape[0], _ptr(w_uv), _ptr(w_o), d_model,
        _ptr(out_heads), _ptr(out_model), _stream(stream)), "mla_up_v")
