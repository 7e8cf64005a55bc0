"""Parity at the full workload sizes, in the launch configuration bench.py
times.  Each whole batch is decoded on the GPU and checked against the fp64
oracle:
- every (row, head) latent output and lse, against the absorbed fp64 form
  (oracle.decode_latent_rows) on the same bf16 absorbed queries the GPU used,
  so the decode is checked on its own; this covers every sequence, including
  those the split plan cuts across CTAs (merged by the combine kernel);
- the absorbed queries themselves at full size (oracle.absorb_q);
- the per-head output o = U^V latent of the whole GPU path (absorb -> decode
  -> up_v) against the textbook expanded fp64 form (k^C = U^K c, v^C = U^V c,
  no absorption), on sampled pairs, at least four of them from cut
  sequences.  The expanded form costs ~1e5 fp64 MACs per (pair, key), so it
  is sampled: 32 pairs per workload, 8 on the long-context batch."""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits, rel_l2

pytestmark = pytest.mark.gpu

FULL = ["v2lite", "v2", "longctx", "mtp"]


@pytest.fixture(scope="module", params=FULL)
def run(request):
    """One resident workload, decoded once and shared by the tests below
    (module scope with a parameter: pytest runs every test of one workload
    before building the next)."""
    import head_latent_attention_10_b200 as M
    M.load_library()
    g = GpuWorkload(W.CONFIGS[request.param])
    q_abs = g.absorb()
    lat, lse = g.decode(q_abs, flags=M.MLA_SYNC_CHECK)
    yield request.param, g, q_abs, lat, lse
    del g, q_abs, lat, lse


def cut_sequences(g):
    """Sequences the decode's split plan cut across CTAs, from the plan the
    call left in its workspace (int32 words after the 256-byte error-word
    slot: virtual tiles per range, total tiles, ranges, the switch weight in
    tiles, then the first tile of each sequence).  A sequence with t tiles and
    virtual start VA (its first tile's start plus the weight of the non-empty
    sequences before it) spans ranges (VA + w) // q .. (VA + w + t - 1) // q;
    the outputs of those spanning more than one come from the combine."""
    import torch
    B = g.cfg.B
    plan = g.ws[256:256 + 4 * (4 + B + 1)].view(torch.int32).cpu().numpy()
    q, total, w = int(plan[0]), int(plan[1]), int(plan[3])
    start = plan[4:4 + B + 1].astype(np.int64)
    assert start[-1] == total
    tiles = np.diff(start)
    vstart = np.concatenate([[0], np.cumsum(np.where(tiles > 0, tiles + w, 0))])
    cut = [b for b in range(B)
           if tiles[b] > 0 and (vstart[b] + w) // q != (vstart[b] + w + tiles[b] - 1) // q]
    return np.asarray(cut, np.int64)


def test_full_size_decode_matches_oracle_on_every_output(run):
    import oracle
    name, g, q_abs, lat, lse = run
    cfg, d = g.cfg, g.d
    ref, rlse = oracle.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], cfg.s,
                                          oracle.bf16_to_f64(host_bits(q_abs)))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(ref.shape)
    assert_parity(got, ref, what=f"{name} latent (all {cfg.T * cfg.H} rows)")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(rlse.shape), rlse, atol=1e-2, rtol=0)
    # the bar holds sequence by sequence too, and on the cut ones as a group
    per_seq = got.reshape(cfg.B, -1)
    ref_seq = ref.reshape(cfg.B, -1)
    worst = max(rel_l2(per_seq[b], ref_seq[b]) for b in range(cfg.B))
    assert worst <= 1e-2, f"{name}: worst per-sequence rel-L2 {worst:.3e}"
    cut = cut_sequences(g)
    if name != "v2lite" or cut.size:
        assert cut.size > 0, f"{name}: the plan cut no sequence"
        assert_parity(per_seq[cut], ref_seq[cut], what=f"{name} latent of {cut.size} cut sequences")


def test_full_size_absorb_q(run):
    import oracle
    name, g, q_abs, _, _ = run
    d = g.d
    ref = oracle.absorb_q(oracle.bf16_to_f64(d["q_nope"]), oracle.bf16_to_f64(d["q_rope"]),
                          oracle.bf16_to_f64(d["w_uk"]), q_pos=d["q_pos"])
    assert_parity(W.bf16_bits_to_f32(host_bits(q_abs)), ref, what=f"{name} q_abs")


def test_full_size_path_against_expanded_oracle(run):
    """absorb -> decode -> up_v on the GPU against the textbook expanded form,
    which shares nothing with the GPU path but the bf16 inputs."""
    import oracle
    name, g, _, lat, _ = run
    cfg, d = g.cfg, g.d
    o = W.bf16_bits_to_f32(host_bits(g.up_v(lat)))
    n_pairs = 8 if name == "longctx" else 32
    rng = np.random.default_rng(cfg.seed + 77)
    cut = cut_sequences(g)
    order = np.argsort(d["seq_lens"], kind="stable")
    seqs = list(rng.choice(cut, size=min(4, cut.size), replace=False)) if cut.size else []
    for b in (order[0], order[-1]):             # the shortest and the longest
        if b not in seqs:
            seqs.append(b)
    while len(seqs) < min(cfg.B, n_pairs // 2):
        b = int(rng.integers(cfg.B))
        if b not in seqs:
            seqs.append(b)
    rows, heads = [], []
    while len(rows) < n_pairs:
        b = seqs[len(rows) % len(seqs)]
        rows.append(int(b) * cfg.s + int(rng.integers(cfg.s)))
        heads.append(int(rng.integers(cfg.H)))
    rows, heads = np.asarray(rows, np.int32), np.asarray(heads, np.int32)
    assert np.isin(rows // cfg.s, cut).sum() >= min(4, cut.size * cfg.s)
    f = oracle.bf16_to_f64
    want, _, _ = oracle.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]),
                                        f(d["q_rope"]), f(d["w_uk"]), f(d["w_uv"]), q_pos=d["q_pos"],
                                        rows=rows, heads=heads)
    assert_parity(o[rows, heads], want, what=f"{name} per-head output ({n_pairs} pairs)")
