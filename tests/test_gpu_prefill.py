"""GPU parity of the expanded-form prefill (mla_prefill) against the oracle.

Each case prefills a chunk of s query tokens per sequence over a paged cache
written by the library's own cache writer.  Every output (all rows, all
heads) is compared with the oracle's absorbed path (absorb_q ->
decode_latent_rows -> up_v, fp64), which the oracle pins tie to the expanded
form; a sample of (row, head) pairs is also compared with the oracle's
textbook expanded form (k^C = U^K c, v^C = U^V c per key).  The bar is the
decode's (assert_parity: max-abs <= 2e-2, relative L2 <= 1e-2); the lse is
held to 1e-2 absolute, like the decode's.

The cases span: chunks that are not a multiple of the 128-query tile, two
query tiles per CTA with the second one partly or wholly empty, a sequence
whose whole length is the chunk (L = s), long ragged tails, several 128-key
tiles, H = 16 .. 128, contiguous and permuted pages.
"""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits, i32, torch_bits

pytestmark = pytest.mark.gpu

CASES = [
    W.MLAConfig("pf_h16_ragged", B=3, s=200, H=16, L=0, paged=True, seed=301, d_model=2048,
                seq_lens=(520, 200, 333)),
    W.MLAConfig("pf_h128", B=1, s=300, H=128, L=0, paged=True, seed=302, d_model=5120,
                seq_lens=(1000,)),
    W.MLAConfig("pf_h32_short_and_long", B=2, s=64, H=32, L=0, paged=False, seed=303, d_model=2048,
                seq_lens=(64, 2000)),
    W.MLAConfig("pf_h64_three_blocks", B=1, s=513, H=64, L=0, paged=True, seed=304, d_model=4096,
                seq_lens=(700,)),
    W.MLAConfig("pf_h16_one_token", B=2, s=1, H=16, L=0, paged=True, seed=305, d_model=2048,
                seq_lens=(1, 129)),
]


@pytest.fixture(scope="module")
def lib():
    import head_latent_attention_10_b200 as M
    M.load_library()
    return M


def prefill(g: GpuWorkload, q_pos=True, seq_lens=None, block_table=None, flags=0, max_seq_len=None):
    import torch
    import head_latent_attention_10_b200 as M
    cfg = g.cfg
    msl = max_seq_len or int(g.d["seq_lens"].max())
    ws = torch.empty(M.mla_prefill_workspace_size(g.dims, cfg.B, cfg.s, msl), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((cfg.T, cfg.H, cfg.d_h), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    M.mla_prefill(g.dims, g.q_nope, g.q_rope, g.q_pos if q_pos else None, g.w_uk, g.w_uv, g.cache,
                  g.block_table if block_table is None else block_table,
                  g.seq_lens if seq_lens is None else seq_lens, cfg.s, msl, out, lse, ws, flags=flags)
    torch.cuda.synchronize()
    err = M.mla_decode_error(ws)
    return W.bf16_bits_to_f32(host_bits(out)).astype(np.float64), lse.cpu().numpy().astype(np.float64), err


def oracle_rows(g: GpuWorkload, rows):
    """The oracle's absorbed path for every head of the given rows."""
    import oracle
    d, f = g.d, oracle.bf16_to_f64
    q_abs = oracle.absorb_q(f(d["q_nope"][rows]), f(d["q_rope"][rows]), f(d["w_uk"]), q_pos=d["q_pos"][rows])
    full = np.zeros((g.cfg.T,) + q_abs.shape[1:])
    full[rows] = q_abs
    lat, lse = oracle.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], g.cfg.s, full, rows=rows)
    return oracle.up_v(lat, f(d["w_uv"])), lse


def check_rows(cfg):
    """All rows when the oracle's absorbed path stays within seconds, else the
    first and last rows of every 128-query tile plus a seeded sample."""
    if cfg.T * cfg.H <= 16 * 1200:
        return np.arange(cfg.T)
    rng = np.random.default_rng(cfg.seed + 5)
    rows = set()
    for b in range(cfg.B):
        for q0 in range(0, cfg.s, 128):
            rows.update({b * cfg.s + q0, b * cfg.s + min(q0 + 127, cfg.s - 1)})
        rows.update((b * cfg.s + rng.choice(cfg.s, size=min(cfg.s, 12), replace=False)).tolist())
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_prefill_against_oracle(lib, cfg):
    import oracle
    g = GpuWorkload(cfg)
    got, lse, err = prefill(g)
    assert err == 0
    rows = check_rows(cfg)
    want, wlse = oracle_rows(g, rows)
    assert_parity(got[rows], want, what=f"{cfg.name} out ({rows.size} rows x {cfg.H} heads)")
    np.testing.assert_allclose(lse[rows], wlse, atol=1e-2, rtol=0)
    # the textbook expanded form on a sample of pairs, covering the first
    # and last query of each sequence
    rng = np.random.default_rng(cfg.seed + 9)
    pr = [b * cfg.s for b in range(cfg.B)] + [b * cfg.s + cfg.s - 1 for b in range(cfg.B)]
    pr += rng.integers(cfg.T, size=12).tolist()
    ph = rng.integers(cfg.H, size=len(pr))
    pr = np.asarray(pr, np.int32)
    d, f = g.d, oracle.bf16_to_f64
    ref, rl, _ = oracle.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]),
                                        f(d["q_rope"]), f(d["w_uk"]), f(d["w_uv"]), q_pos=d["q_pos"],
                                        rows=pr, heads=ph)
    assert_parity(got[pr, ph], ref, what=f"{cfg.name} expanded pairs")
    np.testing.assert_allclose(lse[pr, ph], rl, atol=1e-2, rtol=0)


def test_prefill_matches_the_absorbed_decode_on_the_gpu(lib):
    """The two forms of the same attention agree on the GPU too."""
    cfg = CASES[0]
    g = GpuWorkload(cfg)
    got, lse, _ = prefill(g)
    lat, dlse = g.decode(g.absorb())
    dec = W.bf16_bits_to_f32(host_bits(g.up_v(lat))).astype(np.float64)
    assert_parity(got, dec, what="prefill vs absorb+decode+up_v")
    np.testing.assert_allclose(lse, dlse.cpu().numpy(), atol=1e-2, rtol=0)


def test_prefill_with_pre_rotated_queries(lib):
    """q_pos = NULL takes q^R as already rotated."""
    import oracle
    import torch
    cfg = CASES[0]
    g = GpuWorkload(cfg)
    d, f = g.d, oracle.bf16_to_f64
    rot = oracle.rope_rows(f(d["q_rope"]).reshape(-1, cfg.d_r), np.repeat(d["q_pos"], cfg.H))
    rot_bits = W.f32_to_bf16_bits(rot.astype(np.float32)).reshape(d["q_rope"].shape)
    g.q_rope = torch_bits(rot_bits)
    got, lse, err = prefill(g, q_pos=False)
    assert err == 0
    rng = np.random.default_rng(cfg.seed + 13)
    pr = rng.integers(cfg.T, size=24).astype(np.int32)
    ph = rng.integers(cfg.H, size=24).astype(np.int32)
    ref, rl, _ = oracle.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]),
                                        f(rot_bits), f(d["w_uk"]), f(d["w_uv"]), q_pos=None, rows=pr, heads=ph)
    assert_parity(got[pr, ph], ref, what="pre-rotated q^R")
    np.testing.assert_allclose(lse[pr, ph], rl, atol=1e-2, rtol=0)


def test_prefill_is_bit_reproducible(lib):
    cfg = CASES[3]
    g = GpuWorkload(cfg)
    a, la, _ = prefill(g)
    b, lb, _ = prefill(g)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_prefill_invalid_sequences_get_zero_rows_and_an_error(lib):
    """A sequence shorter than the chunk (or past max_seq_len) gets zero
    outputs and lse = -inf with MLA_DEVERR_SEQ_LEN; the others are unaffected."""
    import head_latent_attention_10_b200 as M
    cfg = CASES[0]
    g = GpuWorkload(cfg)
    good, glse, _ = prefill(g)
    sl = g.d["seq_lens"].copy()
    sl[1] = cfg.s - 1
    got, lse, err = prefill(g, seq_lens=i32(sl))
    assert err & M.MLA_DEVERR_SEQ_LEN
    s = cfg.s
    assert np.all(got[s:2 * s] == 0) and np.all(np.isneginf(lse[s:2 * s]))
    keep = np.r_[0:s, 2 * s:3 * s]
    assert np.array_equal(got[keep], good[keep]) and np.array_equal(lse[keep], glse[keep])
    sl = g.d["seq_lens"].copy()
    sl[2] = int(g.d["seq_lens"].max()) + 1
    got, lse, err = prefill(g, seq_lens=i32(sl))
    assert err & M.MLA_DEVERR_SEQ_LEN
    assert np.all(got[2 * s:] == 0) and np.all(np.isneginf(lse[2 * s:]))


def test_prefill_bad_block_entry_sets_the_error_word(lib):
    import head_latent_attention_10_b200 as M
    cfg = CASES[0]
    g = GpuWorkload(cfg)
    bt = g.d["block_table"].copy()
    bt[0, 2] = g.d["num_blocks"] + 5
    got, lse, err = prefill(g, block_table=i32(bt))
    assert err & M.MLA_DEVERR_BLOCK_ID
    assert np.isfinite(got).all()


def test_prefill_larger_max_seq_len_changes_nothing(lib):
    """The padding of the expanded rows (max_seq_len rounded up) does not
    change any result."""
    cfg = CASES[0]
    g = GpuWorkload(cfg)
    a, la, _ = prefill(g)
    b, lb, _ = prefill(g, max_seq_len=2000)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
