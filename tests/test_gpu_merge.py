"""The two-piece cut sequences the decode kernel merges itself against the
same call with every merge left to the combine kernel (MLA_DEBUG_COMBINE_ALL):
the outputs must be the same bits, and they must match the oracle.  The
batches are built so that the cost-balanced plan cuts sequences into two
pieces (merged in the decode kernel) and into more (left to the combine),
which is checked on the host with the plan's own arithmetic
(test_combine_indices.Plan, 148 SMs)."""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits
from test_combine_indices import SWITCH, Plan

pytestmark = pytest.mark.gpu


def lens(seed, B, lo, hi):
    return tuple(int(x) for x in np.random.default_rng(seed).integers(lo, hi, size=B))


CASES = [
    # 16 rows: two-piece sequences merged in the decode kernel, three-piece ones by the combine
    (W.MLAConfig("h16_many_pieces", B=30, s=1, H=16, L=0, paged=True, seed=601, d_model=2048,
                 seq_lens=lens(601, 30, 200, 900)), {2, 3}),
    # 16 rows, long sequences: many pieces, all left to the combine
    (W.MLAConfig("h16_long", B=4, s=1, H=16, L=0, paged=True, seed=602, d_model=2048,
                 seq_lens=lens(602, 4, 3000, 4000)), {8}),
    # 128 heads, short sequences: two-piece merges, the other sequences whole
    (W.MLAConfig("h128_two_pieces", B=100, s=1, H=128, L=0, paged=True, seed=603, d_model=5120,
                 seq_lens=lens(603, 100, 600, 800)), {2}),
    # two queries of 16 heads (32 rows)
    (W.MLAConfig("h16_s2", B=40, s=2, H=16, L=0, paged=True, seed=604, d_model=2048,
                 seq_lens=lens(604, 40, 200, 900)), {2, 3}),
]


def pieces(cfg):
    """Pieces of every sequence under the decode's plan on a 148-SM B200."""
    groups = (cfg.s * cfg.H + 63) // 64
    ranges = 148 // groups
    sl = np.asarray(W.seq_lens_of(cfg), np.int32)
    p = Plan(sl, int((sl.max() + 63) // 64), ranges)
    out = []
    for b in range(cfg.B):
        t, va = int(p.tiles[b]), int(p.vstart[b])
        out.append(0 if t == 0 else (va + SWITCH + t - 1) // p.qv - (va + SWITCH) // p.qv + 1)
    return np.asarray(out)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_in_kernel_merges_equal_the_combine_bit_for_bit(case):
    import torch
    import oracle
    import head_latent_attention_10_b200 as M
    cfg, want_at_least = case
    npc = pieces(cfg)
    # the batch exercises the piece counts it is meant to
    for n in want_at_least:
        assert (npc >= n).any() if n == 8 else (npc == n).any(), (cfg.name, n, np.bincount(npc))
    M.load_library()
    g = GpuWorkload(cfg)
    q_abs = g.absorb()
    lat_k, lse_k = g.decode(q_abs)
    lat_c, lse_c = g.decode(q_abs, flags=M.MLA_DEBUG_COMBINE_ALL)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(lat_k), host_bits(lat_c)), cfg.name
    assert np.array_equal(lse_k.cpu().numpy().view(np.uint32), lse_c.cpu().numpy().view(np.uint32)), cfg.name
    # the merged rows against the oracle: every row of up to 12 cut sequences
    cut = np.nonzero(npc >= 2)[0][:12]
    rows = np.concatenate([np.arange(b * cfg.s, (b + 1) * cfg.s) for b in cut]).astype(np.int64)
    d = g.d
    q64 = oracle.bf16_to_f64(host_bits(q_abs))
    want, wlse = oracle.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], cfg.s, q64, rows=rows)
    got = W.bf16_bits_to_f32(host_bits(lat_k))[rows].astype(np.float64)
    assert_parity(got, want, what=f"{cfg.name}: {cut.size} cut sequences")
    np.testing.assert_allclose(lse_k.cpu().numpy()[rows], wlse, atol=1e-2, rtol=0)


RACING = [
    # 16 heads: one warp quarter of one row group holds every row
    W.MLAConfig("h16_two_ranges", B=74, s=1, H=16, L=4096, paged=True, seed=605, d_model=2048),
    # 128 heads: two row groups, all four quarters of each
    W.MLAConfig("h128_two_ranges", B=37, s=1, H=128, L=4096, paged=True, seed=606, d_model=5120),
]


@pytest.mark.parametrize("cfg", RACING, ids=lambda c: c.name)
def test_repeated_calls_with_fallbacks_to_the_combine(cfg):
    """Sequences of 4096 tokens, as many as give each one two ranges of its
    own: the second (the early piece, 34 tiles) is no shorter than the first
    (the late piece, 30 tiles and the switch), so the late piece often finds
    the early one unfinished and leaves the sequence to the combine at the
    very end of the decode kernel.  The combine starts while the decode
    kernel still runs (programmatic dependent launch) and must see that late
    work: every call gives the combine-only bits, and over the calls some
    sequences are left to the combine."""
    import torch
    import head_latent_attention_10_b200 as M
    npc = pieces(cfg)
    assert (npc == 2).all(), np.bincount(npc)
    M.load_library()
    g = GpuWorkload(cfg)
    q_abs = g.absorb()
    lat_c, lse_c = g.decode(q_abs, flags=M.MLA_DEBUG_COMBINE_ALL)
    want, wlse = host_bits(lat_c), lse_c.cpu().numpy().view(np.uint32)
    B, groups = cfg.B, (cfg.s * cfg.H + 63) // 64
    # the work count: after the plan (16-byte aligned) and two flag arrays
    plan_ints = ((B + 9) & ~3) + 4 * B
    off_flags = (256 + 4 * plan_ints + 15) // 16 * 16
    work_at = off_flags + 4 * (2 * B * groups * 4)
    left = 0
    for _ in range(24):
        lat, lse = g.decode(q_abs)
        torch.cuda.synchronize()
        left += int(g.ws[work_at:work_at + 4].view(torch.int32).item())
        assert np.array_equal(host_bits(lat), want)
        assert np.array_equal(lse.cpu().numpy().view(np.uint32), wlse)
    assert left > 0, "no call left a sequence to the combine"
