"""Seeded synthetic workloads for MLA decode, shared by the tests, the oracle
side and the GPU side.

This module holds no arithmetic of the method: it draws random numbers, rounds
them to bf16, and lays tokens out in the paged latent cache (a data layout).
RoPE, projections, absorption and attention all live elsewhere: the oracle
applies RoPE to the raw keys itself, and the GPU path applies it when it
writes the cache.

Shapes follow the pages' models: DeepSeek-V2 (128 heads, hidden 5120) and
DeepSeek-V2-Lite (16 heads, hidden 2048), each with a 512-d joint latent, a
64-d decoupled RoPE key and a 128-d head (DeepSeek-V2 paper review,
jiphyeonjeon.kr, sections 3-4; DeepSeek-Lite page, axforge.ai, section 5).

Distributions (the stated workload recipe): c^KV, raw k^R, q^C and raw q^R are
N(0,1); U^K and U^V are N(0, 1/512) (1/512 is the variance); h is N(0,1) and
W^DKV, W^KR are N(0, 1/d_model); W^O is N(0, 1/(H*d_h)).  All values are
rounded to bf16 with round-to-nearest-even.  Each tensor is drawn from its own
child stream of numpy.random.SeedSequence(seed), so a tensor's values do not
depend on the sizes of the others.

Paged layout: 64-token blocks.  N_phys = sum_b ceil(L_b/64) physical blocks;
the block table is a seeded random permutation of 0..N_phys-1 filled
sequence-major (identity for contiguous workloads); unused table entries are
-1; cache slots past a sequence's end hold bf16 NaN so that any read of them
shows up in the output.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Sequence, Tuple, Union

import numpy as np

BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)
D_C, D_R, D_H, BLOCK = 512, 64, 128, 64

_STREAMS = ("w_uk", "w_uv", "c_kv", "k_rope", "q_nope", "q_rope", "block_perm", "seq_lens",
            "h", "w_dkv", "w_kr", "w_o", "q_abs_nope", "q_abs_rope", "latent", "fp8_codes", "fp8_scales",
            "w_uq", "c_q")


@dataclass(frozen=True)
class MLAConfig:
    """One decode workload.  L is an int (all sequences) or (lo, hi) drawn
    uniformly per sequence from the seed; seq_lens overrides both."""
    name: str
    B: int
    s: int
    H: int
    L: Union[int, Tuple[int, int]]
    paged: bool
    seed: int
    d_model: int
    seq_lens: Optional[Tuple[int, ...]] = None
    d_c: int = D_C
    d_r: int = D_R
    d_h: int = D_H
    block_size: int = BLOCK
    describe: str = field(default="", compare=False)

    @property
    def T(self) -> int:
        return self.B * self.s

    def with_(self, **kw) -> "MLAConfig":
        return replace(self, **kw)


CONFIGS: Dict[str, MLAConfig] = {
    "tiny": MLAConfig("tiny", B=1, s=1, H=16, L=256, paged=False, seed=1001, d_model=2048,
                      describe="B=1, s=1, H=16, L=256, contiguous cache"),
    "v2lite": MLAConfig("v2lite", B=64, s=1, H=16, L=4096, paged=True, seed=1002, d_model=2048,
                        describe="DeepSeek-V2-Lite-shaped decode: B=64, H=16, L=4096, paged"),
    "v2": MLAConfig("v2", B=128, s=1, H=128, L=4096, paged=True, seed=1003, d_model=5120,
                    describe="DeepSeek-V2-shaped decode: B=128, H=128, L=4096, paged"),
    "longctx": MLAConfig("longctx", B=8, s=1, H=128, L=131072, paged=True, seed=1004, d_model=5120,
                         describe="long-context split-KV decode: B=8, H=128, L=131072, paged"),
    "mtp": MLAConfig("mtp", B=128, s=2, H=128, L=(512, 16384), paged=True, seed=1005, d_model=5120,
                     describe="ragged 2-token causal decode: B=128, s=2, H=128, L~U[512,16384]"),
}


# ---------------------------------------------------------------- primitives
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even), returned as uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _streams(seed: int) -> Dict[str, np.random.Generator]:
    children = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return {n: np.random.default_rng(c) for n, c in zip(_STREAMS, children)}


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def seq_lens_of(cfg: MLAConfig) -> np.ndarray:
    if cfg.seq_lens is not None:
        sl = np.asarray(cfg.seq_lens, dtype=np.int32)
        assert sl.shape == (cfg.B,)
        return sl
    if isinstance(cfg.L, tuple):
        lo, hi = cfg.L
        return _streams(cfg.seed)["seq_lens"].integers(lo, hi + 1, size=cfg.B).astype(np.int32)
    return np.full(cfg.B, int(cfg.L), dtype=np.int32)


def paging(cfg: MLAConfig, seq_lens: np.ndarray):
    """(block_table [B][max_blocks] int32, num_blocks, logical->physical map)."""
    bs = cfg.block_size
    nblk = (seq_lens.astype(np.int64) + bs - 1) // bs
    n_phys = int(nblk.sum())
    max_blocks = int(max(1, nblk.max() if nblk.size else 1))
    if cfg.paged:
        perm = _streams(cfg.seed)["block_perm"].permutation(n_phys).astype(np.int32)
    else:
        perm = np.arange(n_phys, dtype=np.int32)
    table = np.full((cfg.B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(cfg.B):
        table[b, : nblk[b]] = perm[off: off + nblk[b]]
        off += int(nblk[b])
    return table, max(n_phys, 1), perm


def token_index(seq_lens: np.ndarray):
    """Logical token list (seq index, position) in sequence-major order."""
    sl = seq_lens.astype(np.int64)
    seq = np.repeat(np.arange(sl.size, dtype=np.int32), sl)
    starts = np.concatenate([[0], np.cumsum(sl)[:-1]]) if sl.size else np.zeros(0, np.int64)
    pos = (np.arange(int(sl.sum()), dtype=np.int64) - np.repeat(starts, sl)).astype(np.int32)
    return seq, pos


def scatter_to_pages(cfg: MLAConfig, table: np.ndarray, num_blocks: int, tok_seq, tok_pos,
                     rows: np.ndarray) -> np.ndarray:
    """Place token rows [N][576] (bf16 bits) into a NaN-filled paged cache."""
    D = cfg.d_c + cfg.d_r
    cache = np.full((num_blocks, cfg.block_size, D), BF16_NAN, dtype=np.uint16)
    blk = table[tok_seq, tok_pos // cfg.block_size]
    cache[blk, tok_pos % cfg.block_size] = rows
    return cache


# ------------------------------------------------------------------ workloads
def make_decode_inputs(cfg: MLAConfig, with_cache_pages: bool = True) -> dict:
    """All decode inputs of a workload (bf16 as uint16 bits).

    Keys: seq_lens [B], block_table [B][max_blocks], num_blocks,
    tok_seq/tok_pos [N], c_kv [N][512], k_rope [N][64] (raw, unrotated),
    cache [num_blocks][64][576] (c^KV | raw k^R; NaN in unused slots; only if
    with_cache_pages), q_nope [T][H][128], q_rope [T][H][64] (raw),
    q_pos [T] (= L_b - s + 1 + t), w_uk, w_uv [H][128][512].
    """
    st = _streams(cfg.seed)
    sl = seq_lens_of(cfg)
    table, nphys, _ = paging(cfg, sl)
    tok_seq, tok_pos = token_index(sl)
    N = tok_seq.size
    out = dict(cfg=cfg, seq_lens=sl, block_table=table, num_blocks=nphys,
               tok_seq=tok_seq, tok_pos=tok_pos)
    out["w_uk"] = _normal_bf16(st["w_uk"], (cfg.H, cfg.d_h, cfg.d_c), (1.0 / 512) ** 0.5)
    out["w_uv"] = _normal_bf16(st["w_uv"], (cfg.H, cfg.d_h, cfg.d_c), (1.0 / 512) ** 0.5)
    out["c_kv"] = _normal_bf16(st["c_kv"], (N, cfg.d_c), 1.0)
    out["k_rope"] = _normal_bf16(st["k_rope"], (N, cfg.d_r), 1.0)
    out["q_nope"] = _normal_bf16(st["q_nope"], (cfg.T, cfg.H, cfg.d_h), 1.0)
    out["q_rope"] = _normal_bf16(st["q_rope"], (cfg.T, cfg.H, cfg.d_r), 1.0)
    t = np.tile(np.arange(cfg.s, dtype=np.int32), cfg.B)
    out["q_pos"] = (np.repeat(sl, cfg.s) - cfg.s + 1 + t).astype(np.int32)
    if with_cache_pages:
        rows = np.concatenate([out["c_kv"], out["k_rope"]], axis=1)
        out["cache"] = scatter_to_pages(cfg, table, nphys, tok_seq, tok_pos, rows)
    return out


def make_q_abs(cfg: MLAConfig) -> np.ndarray:
    """A random absorbed query [T][H][576] (bf16 bits) for testing the decode
    call on its own: latent part N(0, 1/4) (the spread of (U^K)^T q^C for the
    distributions above), RoPE part N(0,1) taken as already rotated."""
    st = _streams(cfg.seed)
    a = _normal_bf16(st["q_abs_nope"], (cfg.T, cfg.H, cfg.d_c), 0.5)
    r = _normal_bf16(st["q_abs_rope"], (cfg.T, cfg.H, cfg.d_r), 1.0)
    return np.concatenate([a, r], axis=2)


def make_latent(cfg: MLAConfig) -> np.ndarray:
    """A random latent attention output [T][H][512] (bf16 bits), N(0, 1/64)."""
    return _normal_bf16(_streams(cfg.seed)["latent"], (cfg.T, cfg.H, cfg.d_c), 0.125)


def make_append_inputs(cfg: MLAConfig, T: int) -> dict:
    """h [T][d_model], W^DKV [512][d_model], W^KR [64][d_model] (bf16 bits)."""
    st = _streams(cfg.seed)
    d = cfg.d_model
    return dict(h=_normal_bf16(st["h"], (T, d), 1.0),
                w_dkv=_normal_bf16(st["w_dkv"], (cfg.d_c, d), (1.0 / d) ** 0.5),
                w_kr=_normal_bf16(st["w_kr"], (cfg.d_r, d), (1.0 / d) ** 0.5))


def make_query_latent_inputs(cfg: MLAConfig, T: int, d_q: int = 1536) -> dict:
    """The compressed query path: c^Q [T][d_q] N(0,1) and W^UQ [H][d_h][d_q]
    N(0, 1/d_q), so that q^C = W^UQ c^Q is about N(0,1) like q^C above
    (bf16 bits).  d_q = 1536 is DeepSeek-V2's query latent width."""
    st = _streams(cfg.seed)
    return dict(c_q=_normal_bf16(st["c_q"], (T, d_q), 1.0),
                w_uq=_normal_bf16(st["w_uq"], (cfg.H, cfg.d_h, d_q), (1.0 / d_q) ** 0.5))


def make_w_o(cfg: MLAConfig) -> np.ndarray:
    """W^O [d_model][H*d_h] (bf16 bits)."""
    return _normal_bf16(_streams(cfg.seed)["w_o"], (cfg.d_model, cfg.H * cfg.d_h),
                        (1.0 / (cfg.H * cfg.d_h)) ** 0.5)


def sample_pairs(cfg: MLAConfig, seq_lens: np.ndarray, n_rows: int, n_heads: int,
                 seed: int = 7) -> Tuple[np.ndarray, np.ndarray]:
    """(row, head) pairs for sampled checks at full size: always includes the
    shortest and the longest sequence's rows, plus random others."""
    rng = np.random.default_rng(seed)
    order = np.argsort(seq_lens, kind="stable")
    seqs = {int(order[0]), int(order[-1])}
    while len(seqs) < min(n_rows, cfg.B):
        seqs.add(int(rng.integers(cfg.B)))
    rows, heads = [], []
    for b in sorted(seqs):
        for t in range(cfg.s):
            hs = rng.choice(cfg.H, size=min(n_heads, cfg.H), replace=False)
            for h in sorted(hs):
                rows.append(b * cfg.s + t)
                heads.append(int(h))
    return np.asarray(rows, np.int32), np.asarray(heads, np.int32)


def make_fp8_cache(cfg: MLAConfig, table: np.ndarray, num_blocks: int, tok_seq, tok_pos):
    """A random FP8 latent cache for testing the FP8 decode on its own, drawn
    as bit patterns (no quantization here): every token's 576 E4M3 codes have
    a random sign, an exponent field uniform in 5..9 (values 2^-2 .. 2^2 times
    1 + m/8) and a uniform 3-bit mantissa; its two fp32 scales (c^KV part,
    k^R part) are uniform in [0.1, 0.3].  Slots no token maps to hold the NaN
    code 0x7F and NaN scales.  Returns (codes [num_blocks][64][576] uint8,
    scales [num_blocks][64][2] float32)."""
    st = _streams(cfg.seed)
    D = cfg.d_c + cfg.d_r
    N = tok_seq.size
    g = st["fp8_codes"]
    sign = g.integers(0, 2, size=(N, D), dtype=np.uint8) << np.uint8(7)
    expo = g.integers(5, 10, size=(N, D), dtype=np.uint8) << np.uint8(3)
    mant = g.integers(0, 8, size=(N, D), dtype=np.uint8)
    rows = (sign | expo | mant).astype(np.uint8)
    sc = st["fp8_scales"].uniform(0.1, 0.3, size=(N, 2)).astype(np.float32)
    codes = np.full((num_blocks, cfg.block_size, D), E4M3_NAN, dtype=np.uint8)
    scales = np.full((num_blocks, cfg.block_size, 2), np.nan, dtype=np.float32)
    blk = table[tok_seq, tok_pos // cfg.block_size]
    codes[blk, tok_pos % cfg.block_size] = rows
    scales[blk, tok_pos % cfg.block_size] = sc
    return codes, scales
