"""GPU parity: every library call against the fp64 oracle on seeded inputs.

Sizes are ones the oracle finishes in seconds while still spanning several
64-token blocks, several KV splits and ragged tails.  The bar (written in
assert_parity): max-abs error <= 2e-2 and relative L2 error <= 1e-2 for
floating point; bit-exact for the cache placement.
"""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits, i32, rel_l2, torch_bits

pytestmark = pytest.mark.gpu

SMALL = [
    W.MLAConfig("h16_ragged", B=3, s=1, H=16, L=0, paged=True, seed=201, d_model=2048,
                seq_lens=(1000, 65, 1)),
    W.MLAConfig("h128_ragged", B=3, s=1, H=128, L=0, paged=True, seed=202, d_model=5120,
                seq_lens=(700, 129, 63)),
    W.MLAConfig("h128_two_queries", B=3, s=2, H=128, L=0, paged=True, seed=203, d_model=5120,
                seq_lens=(300, 2, 1500)),
    W.MLAConfig("h64_many_splits", B=2, s=1, H=64, L=0, paged=True, seed=204, d_model=4096,
                seq_lens=(2500, 1100)),
    W.MLAConfig("h32_contiguous", B=2, s=1, H=32, L=0, paged=False, seed=205, d_model=2048,
                seq_lens=(257, 64)),
    W.CONFIGS["tiny"],
]


@pytest.fixture(scope="module")
def lib():
    import head_latent_attention_10_b200 as M
    M.load_library()
    return M


def _oracle():
    import oracle
    return oracle


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_cache_writer_places_rows_bit_exactly(lib, cfg):
    o = _oracle()
    g = GpuWorkload(cfg)
    d = g.d
    got = host_bits(g.cache)
    # latent part: bit for bit at the slot the block table names; every
    # slot no token maps to is still NaN
    assert np.array_equal(got[..., :cfg.d_c], d["cache"][..., :cfg.d_c])
    # RoPE part: the rotated raw key, within bf16 rounding of the fp64 rotation
    bt = d["block_table"]
    blk = bt[d["tok_seq"], d["tok_pos"] // 64]
    slot = d["tok_pos"] % 64
    kr_gpu = W.bf16_bits_to_f32(got[blk, slot, cfg.d_c:]).astype(np.float64)
    kr_ref = o.rope_rows(o.bf16_to_f64(d["k_rope"]), d["tok_pos"])
    assert np.max(np.abs(kr_gpu - kr_ref) / (np.abs(kr_ref) + 1e-2)) < 2 ** -7
    mask = np.ones(got.shape[:2], bool)
    mask[blk, slot] = False
    assert np.all(got[mask] == d["cache"][mask])
    assert int(g.err.item()) == 0


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_absorb_q(lib, cfg):
    o = _oracle()
    g = GpuWorkload(cfg)
    got = W.bf16_bits_to_f32(host_bits(g.absorb()))
    ref = o.absorb_q(o.bf16_to_f64(g.d["q_nope"]), o.bf16_to_f64(g.d["q_rope"]),
                     o.bf16_to_f64(g.d["w_uk"]), q_pos=g.d["q_pos"])
    assert_parity(got, ref, what="absorb_q")


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
@pytest.mark.parametrize("flags", [0, 2], ids=["default", "simple"])
def test_decode_latent(lib, cfg, flags):
    o = _oracle()
    g = GpuWorkload(cfg)
    q_abs_bits = W.make_q_abs(cfg)
    lat, lse = g.decode(torch_bits(q_abs_bits), flags=flags)
    ref, rlse = o.decode_latent(g.d["cache"], g.d["block_table"], g.d["seq_lens"], cfg.s,
                                o.bf16_to_f64(q_abs_bits))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(ref.shape)
    assert_parity(got, ref, what="latent")
    # lse moves with the logits: the cache holds the rotated k^R rounded to
    # bf16 (relative 2^-9 per element), so a logit can move by up to
    # scale * sum_m |q^R_m| |k^R_m| 2^-9 ~ 1e-2 for N(0,1) data.
    np.testing.assert_allclose(lse.cpu().numpy().ravel(), rlse, atol=1e-2, rtol=0)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_full_path_against_expanded_oracle(lib, cfg):
    """absorb -> decode -> up_v on the GPU against the textbook expanded form."""
    o = _oracle()
    g = GpuWorkload(cfg)
    out = g.up_v(g.decode(g.absorb())[0])
    got = W.bf16_bits_to_f32(host_bits(out)).astype(np.float64)
    rng = np.random.default_rng(cfg.seed)
    heads = np.sort(rng.choice(cfg.H, size=min(cfg.H, 16), replace=False))
    rows = np.repeat(np.arange(cfg.T), heads.size)
    hh = np.tile(heads, cfg.T)
    f = o.bf16_to_f64
    ref, _, _ = o.decode_expanded(g.d["cache"], g.d["block_table"], g.d["seq_lens"], cfg.s,
                                  f(g.d["q_nope"]), f(g.d["q_rope"]), f(g.d["w_uk"]), f(g.d["w_uv"]),
                                  q_pos=g.d["q_pos"], rows=rows, heads=hh)
    assert_parity(got[rows, hh], ref, what="o")


@pytest.mark.parametrize("cfg", SMALL[:3], ids=lambda c: c.name)
def test_up_v_and_out_proj(lib, cfg):
    import torch
    o = _oracle()
    g = GpuWorkload(cfg)
    lat_bits = W.make_latent(cfg)
    w_o = W.make_w_o(cfg)
    out_h = torch.empty(cfg.T, cfg.H, cfg.d_h, dtype=torch.bfloat16, device="cuda")
    out_m = torch.empty(cfg.T, cfg.d_model, dtype=torch.bfloat16, device="cuda")
    lib.mla_up_v(g.dims, torch_bits(lat_bits), g.w_uv, out_h, w_o=torch_bits(w_o), out_model=out_m)
    ref_h = o.up_v(o.bf16_to_f64(lat_bits), o.bf16_to_f64(g.d["w_uv"]))
    assert_parity(W.bf16_bits_to_f32(host_bits(out_h)), ref_h, what="heads")
    ref_m = o.out_proj(ref_h, o.bf16_to_f64(w_o))
    assert_parity(W.bf16_bits_to_f32(host_bits(out_m)), ref_m, what="model")


@pytest.mark.parametrize("cfg", SMALL[:2], ids=lambda c: c.name)
def test_append_cache_projection(lib, cfg):
    import torch
    o = _oracle()
    g = GpuWorkload(cfg)
    T = 37
    a = W.make_append_inputs(cfg, T)
    rng = np.random.default_rng(3)
    seq = rng.integers(0, cfg.B, T).astype(np.int32)
    maxpos = g.d["block_table"].shape[1] * 64
    pos = np.array([rng.integers(0, min(maxpos, int(g.d["seq_lens"][b]) + 1)) if g.d["seq_lens"][b] > 0
                    else 0 for b in seq], np.int32)
    # one token per slot so that the writes do not collide
    _, uniq = np.unique(seq.astype(np.int64) * maxpos + pos, return_index=True)
    seq, pos = seq[np.sort(uniq)], pos[np.sort(uniq)]
    h = a["h"][: seq.size]
    cache0 = host_bits(g.cache)
    lib.mla_append_cache(g.dims, torch_bits(h), torch_bits(a["w_dkv"]), torch_bits(a["w_kr"]),
                         i32(seq), i32(pos), g.block_table, g.cache, err_word=g.err)
    got = host_bits(g.cache)
    c_ref, kr_ref = o.kv_project(h, a["w_dkv"], a["w_kr"], pos)
    bt = g.d["block_table"]
    blk, slot = bt[seq, pos // 64], pos % 64
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, :512]), c_ref, what="c_kv")
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, 512:]), kr_ref, what="k_rope")
    mask = np.ones(got.shape[:2], bool); mask[blk, slot] = False
    assert np.array_equal(got[mask], cache0[mask])


@pytest.mark.parametrize("d_model", [576, 1024], ids=["one_pass", "cluster_split_k"])
def test_append_cache_identity_weights_are_bit_exact(lib, d_model):
    """W^DKV = [I 0], W^KR = [0 I 0] at position 0 copies the first 576
    columns of h bit for bit (projection by I is exact in fp32, also when
    the K sum is split over the CTAs of a cluster; RoPE at 0 is the
    identity).  576 runs the GEMM in one pass over K, 1024 the cluster
    split-K kernel."""
    import torch
    cfg = W.MLAConfig("ident", B=2, s=1, H=16, L=0, paged=True, seed=301, d_model=d_model,
                      seq_lens=(5, 70))
    g = GpuWorkload(cfg)
    h = W.f32_to_bf16_bits(np.random.default_rng(1).standard_normal((2, d_model)).astype(np.float32))
    eye = np.eye(576, d_model, dtype=np.float32)
    wd, wr = W.f32_to_bf16_bits(eye[:512]), W.f32_to_bf16_bits(eye[512:])
    seq = np.array([0, 1], np.int32); pos = np.array([0, 0], np.int32)
    lib.mla_append_cache(g.dims, torch_bits(h), torch_bits(wd), torch_bits(wr), i32(seq), i32(pos),
                         g.block_table, g.cache)
    got = host_bits(g.cache)
    bt = g.d["block_table"]
    assert np.array_equal(got[bt[0, 0], 0], h[0, :576]) and np.array_equal(got[bt[1, 0], 0], h[1, :576])


def test_block_permutation_gives_bitwise_identical_outputs(lib):
    cfg = W.MLAConfig("perm", B=4, s=2, H=128, L=0, paged=True, seed=401, d_model=5120,
                      seq_lens=(900, 64, 65, 333))
    q = torch_bits(W.make_q_abs(cfg))
    a = GpuWorkload(cfg).decode(q)
    b = GpuWorkload(cfg.with_(paged=False)).decode(q)
    assert np.array_equal(host_bits(a[0]), host_bits(b[0]))
    assert np.array_equal(a[1].cpu().numpy(), b[1].cpu().numpy())


def test_decode_is_bit_reproducible(lib):
    """Every accumulator has one issuing thread and the P.C MMAs run in tile
    order, so repeated calls on the same inputs give identical bits (latent
    and lse), including sequences split across CTAs and merged by the
    combine."""
    cfg = W.MLAConfig("repro", B=6, s=2, H=128, L=0, paged=True, seed=408, d_model=5120,
                      seq_lens=(2000, 70, 1500, 1, 900, 3100))
    g = GpuWorkload(cfg)
    q = torch_bits(W.make_q_abs(cfg))
    first = g.decode(q)
    ref_lat, ref_lse = host_bits(first[0]), first[1].cpu().numpy()
    for _ in range(4):
        lat, lse = g.decode(q)
        assert np.array_equal(host_bits(lat), ref_lat)
        assert np.array_equal(lse.cpu().numpy().view(np.uint32), ref_lse.view(np.uint32))


def test_heads_with_distinct_queries_get_distinct_outputs(lib):
    cfg = W.MLAConfig("heads", B=1, s=1, H=16, L=300, paged=True, seed=402, d_model=2048)
    g = GpuWorkload(cfg)
    lat, _ = g.decode(torch_bits(W.make_q_abs(cfg)))
    x = W.bf16_bits_to_f32(host_bits(lat))[0]
    assert min(np.max(np.abs(x[i] - x[j])) for i in range(16) for j in range(i)) > 1e-3


def test_single_token_returns_the_latent_exactly(lib):
    cfg = W.MLAConfig("one", B=3, s=1, H=128, L=1, paged=True, seed=403, d_model=5120)
    g = GpuWorkload(cfg)
    lat, lse = g.decode(torch_bits(W.make_q_abs(cfg)))
    got = host_bits(lat)
    for b in range(3):
        assert np.all(got[b] == g.d["c_kv"][b][None, :])


def test_bad_block_table_entry_sets_device_error(lib):
    import torch
    cfg = W.MLAConfig("bad", B=2, s=1, H=16, L=0, paged=True, seed=404, d_model=2048, seq_lens=(130, 40))
    g = GpuWorkload(cfg)
    g.block_table[0, 1] = g.cache.shape[0] + 5
    with pytest.raises(lib.MLAError) as e:
        g.decode(torch_bits(W.make_q_abs(cfg)), flags=lib.MLA_SYNC_CHECK)
    assert e.value.status == lib.MLA_ERR_DEVICE
    assert lib.mla_decode_error(g.ws) & lib.MLA_DEVERR_BLOCK_ID
    torch.cuda.synchronize()
    # the other sequence is unaffected and the context still works
    lat, _ = g.decode(torch_bits(W.make_q_abs(cfg)))
    assert np.isfinite(W.bf16_bits_to_f32(host_bits(lat))[1]).all()


def test_max_jump_on_the_last_tile_of_each_sequence(lib):
    """Each sequence ends in two tokens that score far above the rest, so the
    running max jumps (and O is rescaled) on a sequence's last tile, while
    further sequences follow in the same CTA's range: short sequences, s*H =
    256 rows (four row groups, so few ranges, each spanning several
    sequences)."""
    o = _oracle()
    rng = np.random.default_rng(406)
    lens = tuple(int(x) for x in rng.integers(40, 200, 64))
    cfg = W.MLAConfig("late_max", B=64, s=2, H=128, L=0, paged=True, seed=406, d_model=5120,
                      seq_lens=lens)
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    # heads share a per-sequence direction v, so one row can outscore all others
    v = rng.standard_normal((cfg.B, 1, 1, cfg.d_c + cfg.d_r)).astype(np.float32) * 0.5
    q = v + 0.25 * W.bf16_bits_to_f32(W.make_q_abs(cfg)).reshape(cfg.B, cfg.s, cfg.H, -1)
    q_bits = W.f32_to_bf16_bits(q.reshape(cfg.T, cfg.H, -1))
    sl = d["seq_lens"]
    spike = d["tok_pos"] >= sl[d["tok_seq"]] - 2          # the last two tokens
    d["c_kv"][spike] = W.f32_to_bf16_bits(2.0 * v[d["tok_seq"][spike], 0, 0, :cfg.d_c])
    d["k_rope"][spike] = 0
    d["cache"] = W.scatter_to_pages(cfg, d["block_table"], d["num_blocks"], d["tok_seq"], d["tok_pos"],
                                    np.concatenate([d["c_kv"], d["k_rope"]], axis=1))
    g = GpuWorkload(cfg, d=d)
    lat, lse = g.decode(torch_bits(q_bits), flags=lib.MLA_SYNC_CHECK)
    ref, rlse = o.decode_latent(d["cache"], d["block_table"], sl, cfg.s, o.bf16_to_f64(q_bits))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(ref.shape)
    assert_parity(got, ref, what="latent")
    np.testing.assert_allclose(lse.cpu().numpy().ravel(), rlse, atol=1e-2, rtol=0)
    # the spike dominates: lse sits far above that of the N(0,1) rows
    assert np.min(rlse) > 10.0


@pytest.mark.parametrize("flags", [0, 2], ids=["default", "simple"])
def test_empty_sequences_get_zero_rows(lib, flags):
    """Sequences with no cache token have no tile, so no decode CTA visits
    them: their rows must still come out as a zero latent with lse = -inf
    (the oracle's empty softmax), between sequences that are split across
    several CTAs."""
    o = _oracle()
    cfg = W.MLAConfig("empty", B=5, s=1, H=16, L=0, paged=True, seed=407, d_model=2048,
                      seq_lens=(0, 3000, 0, 70, 0))
    g = GpuWorkload(cfg)
    q = W.make_q_abs(cfg)
    lat, lse = g.decode(torch_bits(q), flags=flags)
    ref, rlse = o.decode_latent(g.d["cache"], g.d["block_table"], g.d["seq_lens"], cfg.s, o.bf16_to_f64(q))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(ref.shape)
    assert_parity(got, ref, what="latent")
    lse = lse.cpu().numpy().ravel()
    empty = np.repeat(np.asarray(cfg.seq_lens) == 0, cfg.H)
    assert np.all(got[empty] == 0) and np.all(np.isneginf(lse[empty]))
    np.testing.assert_allclose(lse[~empty], rlse[~empty], atol=1e-2, rtol=0)


def test_seq_len_beyond_table_and_short_rows(lib):
    import torch
    cfg = W.MLAConfig("short", B=2, s=2, H=16, L=0, paged=True, seed=405, d_model=2048, seq_lens=(1, 50))
    g = GpuWorkload(cfg)
    lat, lse = g.decode(torch_bits(W.make_q_abs(cfg)))
    err = lib.mla_decode_error(g.ws, clear=True)
    assert err & lib.MLA_DEVERR_SEQ_LEN
    x = W.bf16_bits_to_f32(host_bits(lat))
    assert np.all(x[0] == 0) and np.all(np.isneginf(lse[0].cpu().numpy()))
    assert np.isfinite(x[1:]).all()
    g.seq_lens[1] = g.block_table.shape[1] * 64 + 1
    with pytest.raises(lib.MLAError):
        g.decode(torch_bits(W.make_q_abs(cfg)), flags=lib.MLA_SYNC_CHECK)
    torch.cuda.synchronize()


def test_empty_batch_is_a_no_op(lib):
    import torch
    d = lib.dims(128)
    z = torch.empty(0, dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    q = torch.empty(0, 128, 576, dtype=torch.bfloat16, device="cuda")
    cache = torch.empty(1, 64, 576, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, 128, 512, dtype=torch.bfloat16, device="cuda")
    lib.mla_decode(d, q, cache, z.view(0, 1), z, 1, out, None, ws)


@pytest.mark.parametrize("d_model", [2048, 5120])
def test_append_cache_many_tokens(lib, d_model):
    """More than one 128-token tile of the cluster split-K projection (T = 300,
    a ragged last tile) against the fp64 projection, with every token in a
    slot of its own."""
    o = _oracle()
    cfg = W.MLAConfig("app_many", B=4, s=1, H=16, L=0, paged=True, seed=311, d_model=d_model,
                      seq_lens=(400, 130, 64, 700))
    g = GpuWorkload(cfg)
    a = W.make_append_inputs(cfg, 300)
    rng = np.random.default_rng(12)
    slots = rng.choice(int(np.sum(g.d["seq_lens"])), size=300, replace=False)
    seq = g.d["tok_seq"][slots].astype(np.int32)
    pos = g.d["tok_pos"][slots].astype(np.int32)
    cache0 = host_bits(g.cache)
    lib.mla_append_cache(g.dims, torch_bits(a["h"]), torch_bits(a["w_dkv"]), torch_bits(a["w_kr"]),
                         i32(seq), i32(pos), g.block_table, g.cache, err_word=g.err)
    got = host_bits(g.cache)
    c_ref, kr_ref = o.kv_project(a["h"], a["w_dkv"], a["w_kr"], pos)
    bt = g.d["block_table"]
    blk, slot = bt[seq, pos // 64], pos % 64
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, :512]), c_ref, what="c_kv")
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, 512:]), kr_ref, what="k_rope")
    mask = np.ones(got.shape[:2], bool); mask[blk, slot] = False
    assert np.array_equal(got[mask], cache0[mask])
    assert int(g.err.item()) == 0


def test_absorb_q_many_tokens_and_rotated_copy(lib):
    """Several 128-token tiles per head (T = 300, ragged), and with no
    positions the RoPE part is the input copied bit for bit."""
    import torch
    o = _oracle()
    cfg = W.MLAConfig("abs_many", B=150, s=2, H=32, L=64, paged=True, seed=312, d_model=2048)
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    dims = lib.dims(cfg.H)
    q_abs = torch.empty(cfg.T, cfg.H, 576, dtype=torch.bfloat16, device="cuda")
    lib.mla_absorb_q(dims, torch_bits(d["q_nope"]), torch_bits(d["q_rope"]), i32(d["q_pos"]), torch_bits(d["w_uk"]),
                     q_abs)
    ref = o.absorb_q(o.bf16_to_f64(d["q_nope"]), o.bf16_to_f64(d["q_rope"]), o.bf16_to_f64(d["w_uk"]),
                     q_pos=d["q_pos"])
    assert_parity(W.bf16_bits_to_f32(host_bits(q_abs)), ref, what="absorb_q, 300 tokens")
    lib.mla_absorb_q(dims, torch_bits(d["q_nope"]), torch_bits(d["q_rope"]), None, torch_bits(d["w_uk"]), q_abs)
    assert np.array_equal(host_bits(q_abs)[..., 512:], d["q_rope"])


# ------------------------------------------------- append extras (row f4)
YARN = dict(rope_scaling=40.0, rope_original_ctx=4096, rope_yarn_alpha=1.0, rope_yarn_beta=32.0)


def _norm_weight(seed):
    rng = np.random.default_rng(seed)
    return W.f32_to_bf16_bits((1.0 + 0.1 * rng.standard_normal(512)).astype(np.float32))


def test_append_latent_rmsnorm_and_yarn(lib):
    """mla_append_latent with an RMSNorm weight and YaRN-scaled RoPE (scale 40
    over a 4096-token original context) against the fp64 RMSNorm of the bf16
    latent and the fp64 rotation at the YaRN frequencies."""
    o = _oracle()
    cfg = W.MLAConfig("f4_lat", B=3, s=1, H=16, L=0, paged=True, seed=501, d_model=2048,
                      seq_lens=(5000, 70, 131))
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    dims = lib.dims(cfg.H, **YARN)
    import torch
    cache = torch.full((d["num_blocks"], 64, 576), float("nan"), dtype=torch.bfloat16, device="cuda")
    bt = i32(d["block_table"])
    w = _norm_weight(502)
    lib.mla_append_latent(dims, torch_bits(d["c_kv"]), torch_bits(d["k_rope"]), i32(d["tok_seq"]), i32(d["tok_pos"]),
                          bt, cache, kv_norm_weight=torch_bits(w), kv_norm_eps=1e-6)
    got = host_bits(cache)
    blk = d["block_table"][d["tok_seq"], d["tok_pos"] // 64]
    slot = d["tok_pos"] % 64
    c_ref = o.rmsnorm_rows(o.bf16_to_f64(d["c_kv"]), o.bf16_to_f64(w), 1e-6)
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, :512]), c_ref, what="RMS-normalised latent")
    th = o.yarn_theta(s=40.0, L0=4096.0, alpha=1.0, beta=32.0)
    kr_ref = o.rope_rows_theta(o.bf16_to_f64(d["k_rope"]), d["tok_pos"], th)
    assert_parity(W.bf16_bits_to_f32(got[blk, slot, 512:]), kr_ref, what="YaRN-rotated k^R")
    # YaRN moved the slow pairs: far positions differ from plain RoPE
    plain = o.rope_rows(o.bf16_to_f64(d["k_rope"]), d["tok_pos"])
    far = d["tok_pos"] > 2000
    assert np.max(np.abs(kr_ref[far] - plain[far])) > 0.1


@pytest.mark.parametrize("d_model", [5120, 576], ids=["cluster_split_k", "one_pass"])
def test_append_cache_rmsnorm_and_yarn(lib, d_model):
    """The projection path with RMSNorm and YaRN: the oracle projects in fp64,
    rounds the latent to bf16 (the projection's output precision), normalises
    it in fp64 and rotates the raw k^R at the YaRN frequencies."""
    import torch
    o = _oracle()
    cfg = W.MLAConfig("f4_app", B=3, s=1, H=16, L=0, paged=True, seed=503, d_model=d_model,
                      seq_lens=(3000, 64, 700))
    g = GpuWorkload(cfg)
    a = W.make_append_inputs(cfg, 150)
    rng = np.random.default_rng(504)
    slots = rng.choice(int(np.sum(g.d["seq_lens"])), size=150, replace=False)
    seq = g.d["tok_seq"][slots].astype(np.int32)
    pos = g.d["tok_pos"][slots].astype(np.int32)
    dims = lib.dims(cfg.H, **YARN)
    w = _norm_weight(505)
    lib.mla_append_cache(dims, torch_bits(a["h"]), torch_bits(a["w_dkv"]), torch_bits(a["w_kr"]), i32(seq), i32(pos),
                         g.block_table, g.cache, err_word=g.err, kv_norm_weight=torch_bits(w), kv_norm_eps=1e-6)
    got = host_bits(g.cache)
    c, kr_raw = o.kv_project(a["h"], a["w_dkv"], a["w_kr"], np.zeros_like(pos))   # RoPE at 0: the raw key
    c_bf16 = W.bf16_bits_to_f32(W.f32_to_bf16_bits(c.astype(np.float32))).astype(np.float64)
    c_ref = o.rmsnorm_rows(c_bf16, o.bf16_to_f64(w), 1e-6)
    kr_ref = o.rope_rows_theta(kr_raw, pos, o.yarn_theta(s=40.0, L0=4096.0, alpha=1.0, beta=32.0))
    bt = g.d["block_table"]
    blk, sl = bt[seq, pos // 64], pos % 64
    assert_parity(W.bf16_bits_to_f32(got[blk, sl, :512]), c_ref, what="RMS-normalised projected latent")
    assert_parity(W.bf16_bits_to_f32(got[blk, sl, 512:]), kr_ref, what="YaRN-rotated projected k^R")
    assert int(g.err.item()) == 0


def test_absorb_q_yarn(lib):
    """mla_absorb_q with YaRN-scaled RoPE at query positions up to 131071
    against the fp64 rotation at the YaRN frequencies; the latent part is the
    plain absorption."""
    import torch
    o = _oracle()
    rng = np.random.default_rng(506)
    T, H = 40, 64
    q_nope = W.f32_to_bf16_bits(rng.standard_normal((T, H, 128)).astype(np.float32))
    q_rope = W.f32_to_bf16_bits(rng.standard_normal((T, H, 64)).astype(np.float32))
    w_uk = W.f32_to_bf16_bits((rng.standard_normal((H, 128, 512)) / np.sqrt(512)).astype(np.float32))
    q_pos = rng.integers(0, 131072, T).astype(np.int32)
    dims = lib.dims(H, **YARN)
    q_abs = torch.empty(T, H, 576, dtype=torch.bfloat16, device="cuda")
    lib.mla_absorb_q(dims, torch_bits(q_nope), torch_bits(q_rope), i32(q_pos), torch_bits(w_uk), q_abs)
    got = W.bf16_bits_to_f32(host_bits(q_abs))
    th = o.yarn_theta(s=40.0, L0=4096.0, alpha=1.0, beta=32.0)
    qr = o.bf16_to_f64(q_rope)
    ref_r = o.rope_rows_theta(qr.reshape(-1, 64), np.repeat(q_pos, H), th).reshape(qr.shape)
    assert_parity(got[..., 512:], ref_r, what="YaRN-rotated q^R")
    ref = o.absorb_q(o.bf16_to_f64(q_nope), qr, o.bf16_to_f64(w_uk))
    assert_parity(got[..., :512], ref[..., :512], what="absorbed latent query")
