"""fp64 CPU oracle for absorbed-MLA decode -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product library (head_latent_attention_10_b200) never does,
and the two share no code.

Each function wraps one C routine of mla_oracle.c (plain loops, fp64).  Arrays
holding bf16 storage are passed as uint16 bit patterns (numpy uint16 or torch
bfloat16 on the CPU); the C side widens them to double exactly.  Everything
else is float64.

Sources the routines follow (page title, section):
  * DeepSeek-V2 paper review (jiphyeonjeon.kr), section 2: c^KV = W^DKV h,
    k^C = W^UK c^KV, v^C = W^UV c^KV, and the absorption identities.
  * same page, section 3: decoupled RoPE, score (q^C.k^C + q^R.k^R)/sqrt(128+64),
    softmax over j.
  * DeepSeek-V3 report summary (xyznot.com), Method 1: k^R = RoPE(W^KR h),
    k_{t,i} = [k^C_{t,i}; k^R_t], only c^KV and k^R are cached.

Parity status: every routine here has pins of its own in
tests/test_oracle_pins.py, none is "parity unpinned":
  * decode_expanded, decode_latent: brute force on tiny integer inputs, the
    absorption identity between the two, softmax rows summing to 1, the
    single-token, uniform-attention and one-hot closed forms, the scale guard,
    causal masking, paging invariances;
  * decode_latent_rows: bit-identical to decode_latent, plus the single-token
    and uniform-attention closed forms;
  * rope, rope_rows: the identity at position 0, closed forms for unit
    vectors, norm preservation, relative-position invariance, and each row of
    rope_rows equal to rope of that row;
  * kv_project: identity weights at position 0, a NumPy matmul;
  * absorb_q: a NumPy matmul, U^K = [I | 0] returning q^C exactly;
  * up_v, out_proj: a NumPy matmul, U^V = [I | 0] returning the first 128
    latent columns exactly;
  * the cache accounting figures the review prints (section 4);
  * e4m3_values, e4m3_encode: the values the OCP FP8 specification prints
    (1, 448, 2^-6, 2^-9, NaN), torch's own float8_e4m3fn conversion on every
    code and on in-range values, round-to-nearest-even ties;
  * quantize_rows: scales equal amax / 448, every code within half a step of
    x / scale, the largest element of each part maps to 448 exactly;
  * decode_latent_fp8_rows: bit-identical to decode_latent_rows on a cache of
    E4M3-representable values with unit scales, and a brute-force NumPy
    softmax on tiny inputs;
  * rmsnorm_rows: unit root-mean-square output with unit weights, scale
    invariance, the constant-row closed form;
  * yarn_theta, rope_rows_theta: scale 1 gives the plain RoPE frequencies and
    rotations, pairs far below the ramp are divided by s and pairs far above
    it are unchanged, the ramp is continuous, the rotation preserves norms;
  * fold_qk, fold_ov: identity W^UQ (or W^O) returning (U^K)^T (or the U^V
    blocks) exactly, and brute-force dot products on tiny integer inputs;
  * absorb_q_folded, up_out_folded: equal to the pinned two-step path
    (absorb_q of W^UQ c^Q; out_proj of up_v) on the same inputs.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_LIB = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def load(path: str):
    """Load an oracle shared library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    lib.mla_oracle_num_threads.restype = ctypes.c_int
    lib.mla_oracle_rope.argtypes = [_f64p, ctypes.c_int, ctypes.c_double, ctypes.c_double, _f64p]
    lib.mla_oracle_rope_rows.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _i32p, ctypes.c_double, _f64p]
    lib.mla_oracle_kv_project.argtypes = [ctypes.c_int] * 4 + [_u16p, _u16p, _u16p, _i32p,
                                                             ctypes.c_double, _f64p, _f64p]
    lib.mla_oracle_absorb_q.argtypes = [ctypes.c_int] * 5 + [_f64p, _f64p, _i32p, _f64p,
                                                            ctypes.c_double, _f64p]
    lib.mla_oracle_decode_expanded.argtypes = (
        [ctypes.c_int] * 7 + [ctypes.c_double, _u16p, ctypes.c_int, _i32p, ctypes.c_int, _i32p,
                              _f64p, _f64p, _i32p, _f64p, _f64p, ctypes.c_int, _i32p, _i32p,
                              _f64p, _f64p, _f64p, ctypes.c_int])
    lib.mla_oracle_decode_expanded.restype = ctypes.c_int
    lib.mla_oracle_decode_latent.argtypes = (
        [ctypes.c_int] * 7 + [ctypes.c_double, _u16p, ctypes.c_int, _i32p, ctypes.c_int, _i32p,
                              _f64p, ctypes.c_int, _i32p, _i32p, _f64p, _f64p])
    lib.mla_oracle_decode_latent.restype = ctypes.c_int
    lib.mla_oracle_decode_latent_rows.argtypes = (
        [ctypes.c_int] * 7 + [ctypes.c_double, _u16p, ctypes.c_int, _i32p, ctypes.c_int, _i32p,
                              _f64p, ctypes.c_int, _i32p, _f64p, _f64p])
    lib.mla_oracle_decode_latent_rows.restype = ctypes.c_int
    _u8p = ctypes.POINTER(ctypes.c_uint8)
    _f32p = ctypes.POINTER(ctypes.c_float)
    lib.mla_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.mla_oracle_e4m3_value.restype = ctypes.c_double
    lib.mla_oracle_e4m3_values.argtypes = [ctypes.c_int, _u8p, _f64p]
    lib.mla_oracle_e4m3_encode_n.argtypes = [ctypes.c_int, _f32p, _u8p]
    lib.mla_oracle_quantize_rows.argtypes = [ctypes.c_int] * 3 + [_f32p, _u8p, _f32p]
    lib.mla_oracle_decode_latent_fp8_rows.argtypes = (
        [ctypes.c_int] * 7 + [_u8p, _f32p, ctypes.c_int, _i32p, ctypes.c_int, _i32p, _f64p, ctypes.c_int,
                              _i32p, _f64p, _f64p])
    lib.mla_oracle_decode_latent_fp8_rows.restype = ctypes.c_int
    lib.mla_oracle_rmsnorm_rows.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _f64p, ctypes.c_double, _f64p]
    lib.mla_oracle_yarn_theta.argtypes = [ctypes.c_int] + [ctypes.c_double] * 5 + [_f64p]
    lib.mla_oracle_rope_rows_theta.argtypes = [ctypes.c_int, ctypes.c_int, _f64p, _i32p, _f64p, _f64p]
    lib.mla_oracle_up_v.argtypes = [ctypes.c_int] * 4 + [_f64p, _f64p, _f64p]
    lib.mla_oracle_out_proj.argtypes = [ctypes.c_int] * 4 + [_f64p, _f64p, _f64p]
    lib.mla_oracle_fold_qk.argtypes = [ctypes.c_int] * 4 + [_f64p, _f64p, _f64p]
    lib.mla_oracle_fold_ov.argtypes = [ctypes.c_int] * 4 + [_f64p, _f64p, _f64p]
    lib.mla_oracle_absorb_q_folded.argtypes = [ctypes.c_int] * 5 + [_f64p, _f64p, _i32p, _f64p, ctypes.c_double,
                                                                   _f64p]
    lib.mla_oracle_up_out_folded.argtypes = [ctypes.c_int] * 4 + [_f64p, _f64p, _f64p]
    return lib


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def num_threads() -> int:
    """OpenMP threads the oracle uses (the CPU baseline's core count)."""
    return int(_lib().mla_oracle_num_threads())


# ---------------------------------------------------------------- marshalling
def _bits(a) -> np.ndarray:
    """bf16 storage as a contiguous uint16 array (torch bf16 or numpy uint16)."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        a = a.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 storage must be passed as uint16 bit patterns")
    return a


def _f64(a) -> np.ndarray:
    if hasattr(a, "dtype") and str(a.dtype).startswith("torch."):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "dtype") and str(a.dtype).startswith("torch."):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a, t):
    return None if a is None else a.ctypes.data_as(t)


def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = _bits(bits)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ routines
def rope(x, pos: float, base: float = 10000.0) -> np.ndarray:
    """RoPE of one vector (adjacent pairs, theta_k = base^(-2k/d_r))."""
    x = _f64(x)
    y = np.empty_like(x)
    _lib().mla_oracle_rope(_p(x, _f64p), x.shape[-1], float(pos), float(base), _p(y, _f64p))
    return y


def rope_rows(x, pos, base: float = 10000.0) -> np.ndarray:
    """RoPE of each row x[n] at position pos[n]."""
    x, pos = _f64(x), _i32(pos)
    y = np.empty_like(x)
    _lib().mla_oracle_rope_rows(x.shape[0], x.shape[1], _p(x, _f64p), _p(pos, _i32p), float(base),
                                _p(y, _f64p))
    return y


def kv_project(h, w_dkv, w_kr, pos, base: float = 10000.0):
    """Append projection: (c^KV [T][d_c], rotated k^R [T][d_r]) in fp64."""
    h, w_dkv, w_kr, pos = _bits(h), _bits(w_dkv), _bits(w_kr), _i32(pos)
    T, d = h.shape
    d_c, d_r = w_dkv.shape[0], w_kr.shape[0]
    c = np.empty((T, d_c)); kr = np.empty((T, d_r))
    _lib().mla_oracle_kv_project(T, d, d_c, d_r, _p(h, _u16p), _p(w_dkv, _u16p), _p(w_kr, _u16p),
                                 _p(pos, _i32p), float(base), _p(c, _f64p), _p(kr, _f64p))
    return c, kr


def absorb_q(q_nope, q_rope, w_uk, q_pos=None, base: float = 10000.0) -> np.ndarray:
    """q_abs [T][H][d_c+d_r]: (U^K_i)^T q^C_{t,i} followed by RoPE(q^R_{t,i}, q_pos[t])."""
    q_nope, q_rope, w_uk = _f64(q_nope), _f64(q_rope), _f64(w_uk)
    T, H, d_h = q_nope.shape
    d_r = q_rope.shape[-1]
    d_c = w_uk.shape[-1]
    qp = None if q_pos is None else _i32(q_pos)
    out = np.empty((T, H, d_c + d_r))
    _lib().mla_oracle_absorb_q(T, H, d_h, d_c, d_r, _p(q_nope, _f64p), _p(q_rope, _f64p),
                               _p(qp, _i32p), _p(w_uk, _f64p), float(base), _p(out, _f64p))
    return out


def _pairs(rows, heads, T, H):
    if rows is None:
        rr, hh = np.meshgrid(np.arange(T), np.arange(H), indexing="ij")
        return _i32(rr.ravel()), _i32(hh.ravel())
    return _i32(rows), _i32(heads)


def decode_expanded(cache, block_table, seq_lens, s, q_nope, q_rope, w_uk, w_uv, q_pos=None,
                    rows=None, heads=None, block_size=64, d_r=64, base=10000.0,
                    probs_stride=0):
    """Expanded-form MLA decode for (row, head) pairs (all pairs if rows is None).

    Returns (o [n][d_h], lse [n], probs [n][probs_stride] or None).
    """
    cache, bt, sl = _bits(cache), _i32(block_table), _i32(seq_lens)
    q_nope, q_rope, w_uk, w_uv = _f64(q_nope), _f64(q_rope), _f64(w_uk), _f64(w_uv)
    T, H, d_h = q_nope.shape
    D = cache.shape[-1]
    d_c = D - d_r
    B = sl.shape[0]
    num_blocks = cache.size // (block_size * D)
    max_blocks = bt.shape[-1] if bt.ndim > 1 else bt.size // max(B, 1)
    pr, ph = _pairs(rows, heads, T, H)
    n = pr.size
    out = np.zeros((n, d_h)); lse = np.zeros(n)
    probs = np.zeros((n, probs_stride)) if probs_stride else None
    qp = None if q_pos is None else _i32(q_pos)
    rc = _lib().mla_oracle_decode_expanded(
        B, s, H, d_c, d_r, d_h, block_size, float(base), _p(cache, _u16p), num_blocks,
        _p(bt, _i32p), max_blocks, _p(sl, _i32p), _p(q_nope, _f64p), _p(q_rope, _f64p),
        _p(qp, _i32p), _p(w_uk, _f64p), _p(w_uv, _f64p), n, _p(pr, _i32p), _p(ph, _i32p),
        _p(out, _f64p), _p(lse, _f64p), _p(probs, _f64p), int(probs_stride))
    if rc != 0:
        raise ValueError("block table entry out of range")
    return out, lse, probs


def decode_latent(cache, block_table, seq_lens, s, q_abs, rows=None, heads=None,
                  block_size=64, d_r=64, d_h=128, base=10000.0):
    """Absorbed-form decode: (latent output [n][d_c], lse [n]) for (row, head) pairs."""
    cache, bt, sl = _bits(cache), _i32(block_table), _i32(seq_lens)
    q_abs = _f64(q_abs)
    T, H, D = q_abs.shape
    d_c = D - d_r
    B = sl.shape[0]
    num_blocks = cache.size // (block_size * D)
    max_blocks = bt.shape[-1] if bt.ndim > 1 else bt.size // max(B, 1)
    pr, ph = _pairs(rows, heads, T, H)
    n = pr.size
    out = np.zeros((n, d_c)); lse = np.zeros(n)
    rc = _lib().mla_oracle_decode_latent(
        B, s, H, d_c, d_r, d_h, block_size, float(base), _p(cache, _u16p), num_blocks,
        _p(bt, _i32p), max_blocks, _p(sl, _i32p), _p(q_abs, _f64p), n, _p(pr, _i32p),
        _p(ph, _i32p), _p(out, _f64p), _p(lse, _f64p))
    if rc != 0:
        raise ValueError("block table entry out of range")
    return out, lse


def decode_latent_rows(cache, block_table, seq_lens, s, q_abs, rows=None, block_size=64, d_r=64, d_h=128,
                       base=10000.0):
    """Absorbed-form decode of every head of the given rows (all rows if None):
    (latent [n_rows][H][d_c], lse [n_rows][H]).  The same arithmetic, in the same
    order, as decode_latent (bit-identical results); each key's RoPE part is
    turned once per group of 16 heads, so whole batches stay affordable."""
    cache, bt, sl = _bits(cache), _i32(block_table), _i32(seq_lens)
    q_abs = _f64(q_abs)
    T, H, D = q_abs.shape
    d_c = D - d_r
    B = sl.shape[0]
    num_blocks = cache.size // (block_size * D)
    max_blocks = bt.shape[-1] if bt.ndim > 1 else bt.size // max(B, 1)
    rr = _i32(np.arange(T) if rows is None else rows)
    out = np.zeros((rr.size, H, d_c)); lse = np.zeros((rr.size, H))
    rc = _lib().mla_oracle_decode_latent_rows(
        B, s, H, d_c, d_r, d_h, block_size, float(base), _p(cache, _u16p), num_blocks, _p(bt, _i32p),
        max_blocks, _p(sl, _i32p), _p(q_abs, _f64p), rr.size, _p(rr, _i32p), _p(out, _f64p), _p(lse, _f64p))
    if rc != 0:
        raise ValueError("block table entry out of range")
    return out, lse


# ------------------------------------------------------------- FP8 cache
def e4m3_values(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> their values (float64; NaN for the NaN codes)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _lib().mla_oracle_e4m3_values(c.size, c.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), _p(out, _f64p))
    return out


def e4m3_encode(x) -> np.ndarray:
    """float32 values -> nearest E4M3 codes (ties to even, saturating at 448)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _lib().mla_oracle_e4m3_encode_n(x.size, x.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                    out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def quantize_rows(rows, d_c=512):
    """Cache rows [N][d_c + d_r] (float32) -> (codes uint8 [N][D], scales float32
    [N][2]): scale = amax / 448 per part (c^KV, k^R), code = E4M3(x / scale)."""
    r = np.ascontiguousarray(rows, dtype=np.float32)
    N, D = r.shape
    codes = np.empty((N, D), np.uint8)
    scales = np.empty((N, 2), np.float32)
    _lib().mla_oracle_quantize_rows(N, d_c, D - d_c, r.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                    codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                    scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return codes, scales


def decode_latent_fp8_rows(codes, scales, block_table, seq_lens, s, q_abs, rows=None, block_size=64, d_r=64,
                           d_h=128):
    """Absorbed decode over the FP8 cache (codes [num_blocks][64][576] uint8,
    scales [num_blocks][64][2] float32, k^R already rotated): (latent
    [n_rows][H][d_c], lse [n_rows][H])."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    bt, sl = _i32(block_table), _i32(seq_lens)
    q_abs = _f64(q_abs)
    T, H, D = q_abs.shape
    d_c = D - d_r
    B = sl.shape[0]
    num_blocks = codes.size // (block_size * D)
    max_blocks = bt.shape[-1] if bt.ndim > 1 else bt.size // max(B, 1)
    rr = _i32(np.arange(T) if rows is None else rows)
    out = np.zeros((rr.size, H, d_c)); lse = np.zeros((rr.size, H))
    rc = _lib().mla_oracle_decode_latent_fp8_rows(
        B, s, H, d_c, d_r, d_h, block_size, codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
        scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), num_blocks, _p(bt, _i32p), max_blocks,
        _p(sl, _i32p), _p(q_abs, _f64p), rr.size, _p(rr, _i32p), _p(out, _f64p), _p(lse, _f64p))
    if rc != 0:
        raise ValueError("block table entry out of range")
    return out, lse


# ------------------------------------------------------------ append extras
def rmsnorm_rows(x, w, eps=1e-6) -> np.ndarray:
    """x [N][d] -> x / sqrt(mean(x^2) + eps) * w, row by row."""
    x, w = _f64(x), _f64(w)
    y = np.empty_like(x)
    _lib().mla_oracle_rmsnorm_rows(x.shape[0], x.shape[1], _p(x, _f64p), _p(w, _f64p), float(eps), _p(y, _f64p))
    return y


def yarn_theta(d_r=64, base=10000.0, s=40.0, L0=4096.0, alpha=1.0, beta=32.0) -> np.ndarray:
    """The RoPE frequency of each of the d_r / 2 pairs under YaRN scaling s."""
    th = np.empty(d_r // 2)
    _lib().mla_oracle_yarn_theta(d_r, float(base), float(s), float(L0), float(alpha), float(beta), _p(th, _f64p))
    return th


def rope_rows_theta(x, pos, theta) -> np.ndarray:
    """RoPE of each row x[n] at position pos[n] with the frequencies theta."""
    x, pos, theta = _f64(x), _i32(pos), _f64(theta)
    y = np.empty_like(x)
    _lib().mla_oracle_rope_rows_theta(x.shape[0], x.shape[1], _p(x, _f64p), _p(pos, _i32p), _p(theta, _f64p),
                                      _p(y, _f64p))
    return y


def up_v(latent, w_uv) -> np.ndarray:
    """o [T][H][d_h] = U^V_i latent[t][i]."""
    latent, w_uv = _f64(latent), _f64(w_uv)
    T, H, d_c = latent.shape
    d_h = w_uv.shape[1]
    out = np.empty((T, H, d_h))
    _lib().mla_oracle_up_v(T, H, d_h, d_c, _p(latent, _f64p), _p(w_uv, _f64p), _p(out, _f64p))
    return out


def out_proj(heads, w_o) -> np.ndarray:
    """u [T][d_model] = sum_i O_i o_{t,i} with W^O [d_model][H*d_h]."""
    heads, w_o = _f64(heads), _f64(w_o)
    T, H, d_h = heads.shape
    d_model = w_o.shape[0]
    u = np.empty((T, d_model))
    _lib().mla_oracle_out_proj(T, H, d_h, d_model, _p(heads, _f64p), _p(w_o, _f64p), _p(u, _f64p))
    return u


# ------------------------------------------------ weight pre-absorption (f3)
def fold_qk(w_uq, w_uk) -> np.ndarray:
    """W^QK [H][d_c][d_q], W^QK_i = (U^K_i)^T W^UQ_i."""
    w_uq, w_uk = _f64(w_uq), _f64(w_uk)
    H, d_h, d_q = w_uq.shape
    d_c = w_uk.shape[-1]
    out = np.empty((H, d_c, d_q))
    _lib().mla_oracle_fold_qk(H, d_h, d_c, d_q, _p(w_uq, _f64p), _p(w_uk, _f64p), _p(out, _f64p))
    return out


def fold_ov(w_o, w_uv) -> np.ndarray:
    """W^OV [d_model][H*d_c], block i = O_i U^V_i."""
    w_o, w_uv = _f64(w_o), _f64(w_uv)
    H, d_h, d_c = w_uv.shape
    d_model = w_o.shape[0]
    out = np.empty((d_model, H * d_c))
    _lib().mla_oracle_fold_ov(H, d_h, d_c, d_model, _p(w_o, _f64p), _p(w_uv, _f64p), _p(out, _f64p))
    return out


def absorb_q_folded(c_q, q_rope, w_qk, q_pos=None, base: float = 10000.0) -> np.ndarray:
    """q_abs [T][H][d_c+d_r] = [W^QK_i c_q[t] | RoPE(q^R_{t,i}, q_pos[t])]."""
    c_q, q_rope, w_qk = _f64(c_q), _f64(q_rope), _f64(w_qk)
    T, d_q = c_q.shape
    H, d_c, _ = w_qk.shape
    d_r = q_rope.shape[-1]
    qp = None if q_pos is None else _i32(q_pos)
    out = np.empty((T, H, d_c + d_r))
    _lib().mla_oracle_absorb_q_folded(T, H, d_c, d_q, d_r, _p(c_q, _f64p), _p(q_rope, _f64p), _p(qp, _i32p),
                                      _p(w_qk, _f64p), float(base), _p(out, _f64p))
    return out


def up_out_folded(latent, w_ov) -> np.ndarray:
    """u [T][d_model] = sum_i W^OV_i latent[t][i]."""
    latent, w_ov = _f64(latent), _f64(w_ov)
    T, H, d_c = latent.shape
    d_model = w_ov.shape[0]
    u = np.empty((T, d_model))
    _lib().mla_oracle_up_out_folded(T, H, d_c, d_model, _p(latent, _f64p), _p(w_ov, _f64p), _p(u, _f64p))
    return u
