"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with a copy of itself.  Each pin is one of:
a figure the pages print (tests/golden/), a closed form, an invariant, a
special case that reduces to a library routine (numpy), or a brute-force
pure-Python evaluation on tiny inputs.  test_planted_mistakes_are_caught
plants plausible mistakes in a copy of the oracle's C source and checks that
these pins catch every one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import mla_workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ------------------------------------------------------------ tiny workloads
def tiny_case(rng, B=2, s=1, H=2, d_c=4, d_r=2, d_h=2, bs=2, lens=(3, 2), ints=True, paged=True):
    """Small-integer MLA inputs (exact in bf16) with a random block table."""
    lens = np.asarray(lens, np.int32)
    D = d_c + d_r
    nblk = [(int(L) + bs - 1) // bs for L in lens]
    nphys = sum(nblk)
    perm = rng.permutation(nphys) if paged else np.arange(nphys)
    maxb = max(nblk)
    table = np.full((B, maxb), -1, np.int32)
    off = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[off:off + nblk[b]]
        off += nblk[b]
    draw = (lambda *sh: rng.integers(-3, 4, size=sh).astype(np.float32)) if ints else \
        (lambda *sh: rng.standard_normal(sh).astype(np.float32))
    logical = [draw(int(L), D) for L in lens]
    cache = np.full((nphys, bs, D), W.BF16_NAN, np.uint16)
    for b in range(B):
        for j in range(lens[b]):
            cache[table[b, j // bs], j % bs] = bits(logical[b][j])
    T = B * s
    q_nope = W.bf16_bits_to_f32(bits(draw(T, H, d_h))).astype(np.float64)
    q_rope = W.bf16_bits_to_f32(bits(draw(T, H, d_r))).astype(np.float64)
    w_uk = W.bf16_bits_to_f32(bits(draw(H, d_h, d_c))).astype(np.float64)
    w_uv = W.bf16_bits_to_f32(bits(draw(H, d_h, d_c))).astype(np.float64)
    t = np.tile(np.arange(s), B)
    q_pos = (np.repeat(lens, s) - s + 1 + t).astype(np.int32)
    logical = [W.bf16_bits_to_f32(bits(x)).astype(np.float64) for x in logical]
    return dict(lens=lens, table=table, cache=cache, logical=logical, q_nope=q_nope,
                q_rope=q_rope, w_uk=w_uk, w_uv=w_uv, q_pos=q_pos, s=s, B=B, H=H,
                d_c=d_c, d_r=d_r, d_h=d_h, bs=bs)


# -------------------------------------------------- brute force (pure Python)
def py_rope(x, pos, base=10000.0):
    d = len(x)
    y = [0.0] * d
    for k in range(d // 2):
        ang = pos * base ** (-2.0 * k / d)
        y[2 * k] = x[2 * k] * math.cos(ang) - x[2 * k + 1] * math.sin(ang)
        y[2 * k + 1] = x[2 * k] * math.sin(ang) + x[2 * k + 1] * math.cos(ang)
    return y


def brute_force(c, scale_dims=None):
    """Textbook MLA decode straight from the pages' formulas, plain Python."""
    d_c, d_r, d_h, s, H = c["d_c"], c["d_r"], c["d_h"], c["s"], c["H"]
    scale = 1.0 / math.sqrt(scale_dims if scale_dims else d_h + d_r)
    outs, lses, probs = {}, {}, {}
    for b in range(c["B"]):
        L = int(c["lens"][b])
        rows = c["logical"][b]
        for t in range(s):
            row = b * s + t
            nvis = L - s + t + 1
            for i in range(H):
                if nvis <= 0:
                    outs[row, i] = [0.0] * d_h
                    lses[row, i] = -math.inf
                    continue
                qc = list(c["q_nope"][row, i])
                qr = py_rope(list(c["q_rope"][row, i]), int(c["q_pos"][row]))
                scores = []
                for j in range(nvis):
                    cj = list(rows[j][:d_c])
                    kr = py_rope(list(rows[j][d_c:]), j)
                    kc = [sum(c["w_uk"][i, k, m] * cj[m] for m in range(d_c)) for k in range(d_h)]
                    scores.append((sum(qc[k] * kc[k] for k in range(d_h)) +
                                   sum(qr[m] * kr[m] for m in range(d_r))) * scale)
                mx = max(scores)
                e = [math.exp(x - mx) for x in scores]
                den = sum(e)
                a = [x / den for x in e]
                o = [0.0] * d_h
                for j in range(nvis):
                    cj = list(rows[j][:d_c])
                    for k in range(d_h):
                        o[k] += a[j] * sum(c["w_uv"][i, k, m] * cj[m] for m in range(d_c))
                outs[row, i] = o
                lses[row, i] = mx + math.log(den)
                probs[row, i] = a
    return outs, lses, probs


def run_expanded(o, c, probs_stride=0):
    return o.decode_expanded(c["cache"], c["table"], c["lens"], c["s"], c["q_nope"], c["q_rope"],
                             c["w_uk"], c["w_uv"], q_pos=c["q_pos"], block_size=c["bs"],
                             d_r=c["d_r"], probs_stride=probs_stride)


def check_brute(o, c, tol=1e-13):
    out, lse, _ = run_expanded(o, c)
    ref, rlse, _ = brute_force(c)
    n = 0
    for row in range(c["B"] * c["s"]):
        for i in range(c["H"]):
            np.testing.assert_allclose(out[n], ref[row, i], rtol=tol, atol=tol)
            if math.isinf(rlse[row, i]):
                assert math.isinf(lse[n])
            else:
                assert abs(lse[n] - rlse[row, i]) < tol * max(1, abs(rlse[row, i]))
            n += 1


# ------------------------------------------------------------------- pins
def test_golden_cache_accounting():
    """The row layout (576 values, 1152 bytes in bf16) reproduces every
    cache-size figure the pages print."""
    g = json.load(open(os.path.join(GOLD, "cache_accounting.json")))
    row = W.D_C + W.D_R
    assert row == g["mla_elements_per_token_per_layer"]["value"]
    assert row * g["v2_layers"]["value"] == g["v2_elements_per_token"]["value"]
    assert row / (2 * 128) == g["gqa_equivalent_groups"]["value"]
    assert round(100 * row / (2 * 128 * 128), 2) == g["mha_ratio_percent"]["value"]
    b67 = 95 * 2 * 8 * 128 * 2
    assert b67 == g["dense67b_bytes_per_token"]["value"]
    b6 = 60 * row * 6 // 8
    assert b6 == g["v2_bytes_per_token_6bit"]["value"]
    assert round(100 * (1 - b6 / b67), 2) == g["reduction_percent_6bit"]["value"]
    b16 = 60 * row * 2
    assert b16 == g["v2_bytes_per_token_16bit"]["value"]
    assert round(100 * (1 - b16 / b67), 2) == g["reduction_percent_16bit"]["value"]
    assert round(27 * row / 1000, 1) == g["table9_small_mla_elements_k"]["value"]
    assert round(2 * 16 * 128 * 27 / 1000, 1) == g["table9_small_mha_elements_k"]["value"]
    assert round(60 * row / 1000, 1) == g["table9_large_mla_elements_k"]["value"]
    assert W.D_H + W.D_R == g["score_scale_dims"]["value"]
    lite = g["v2lite_shapes"]["value"]
    c2 = W.CONFIGS["v2lite"]
    assert (c2.H, c2.d_h, c2.d_c, c2.d_r, c2.d_model) == (
        lite["heads"], lite["head_dim"], lite["d_c"], lite["d_r"], lite["hidden"])


def test_rope_identity_at_zero(oracle_mod):
    x = np.random.default_rng(0).standard_normal(64)
    assert np.array_equal(oracle_mod.rope(x, 0.0), x)


def test_rope_closed_forms(oracle_mod):
    # pair 0 turns by exactly pos radians
    e0 = np.zeros(64); e0[0] = 1.0
    y = oracle_mod.rope(e0, math.pi / 2)
    np.testing.assert_allclose(y[:2], [0.0, 1.0], atol=1e-15)
    # pair 16 of 32 has theta = 10000^(-1/2) = 1/100, so position 100 turns it by 1 rad
    e32 = np.zeros(64); e32[32] = 1.0
    y = oracle_mod.rope(e32, 100.0)
    np.testing.assert_allclose(y[32:34], [math.cos(1.0), math.sin(1.0)], atol=1e-14)
    assert np.count_nonzero(np.abs(np.delete(y, [32, 33])) > 0) == 0
    # the last pair turns slowest: theta_31 = 10000^(-62/64) < theta_30
    e62 = np.zeros(64); e62[62] = 1.0
    e60 = np.zeros(64); e60[60] = 1.0
    a62 = math.atan2(oracle_mod.rope(e62, 1.0)[63], 1.0)
    a60 = math.atan2(oracle_mod.rope(e60, 1.0)[61], 1.0)
    assert 0 < a62 < a60 < 1e-3


def test_rope_norm_and_relative_position(oracle_mod):
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m in (0, 5, 1000, 131071):
        np.testing.assert_allclose(np.linalg.norm(oracle_mod.rope(q, m)), np.linalg.norm(q), rtol=1e-14)
    for m, n, dlt in ((3, 10, 7), (100, 4000, 123), (0, 9, 50000)):
        a = oracle_mod.rope(q, m) @ oracle_mod.rope(k, n)
        b = oracle_mod.rope(q, m + dlt) @ oracle_mod.rope(k, n + dlt)
        assert abs(a - b) < 1e-10 * (1 + abs(a))
    # composition: R_m R_n = R_{m+n}
    np.testing.assert_allclose(oracle_mod.rope(oracle_mod.rope(q, 17), 25), oracle_mod.rope(q, 42),
                               atol=1e-12)


@pytest.mark.parametrize("seed,s,lens", [(0, 1, (3, 2)), (1, 2, (3, 4)), (2, 1, (1, 5)), (3, 2, (2, 1))])
def test_brute_force_tiny(oracle_mod, seed, s, lens):
    c = tiny_case(np.random.default_rng(seed), B=2, s=s, lens=lens)
    check_brute(oracle_mod, c)


def test_brute_force_tiny_gaussian(oracle_mod):
    c = tiny_case(np.random.default_rng(11), B=2, s=2, H=3, d_c=6, d_r=4, d_h=3, bs=3,
                  lens=(7, 4), ints=False)
    check_brute(oracle_mod, c)


def test_scale_guard(oracle_mod):
    """The scale is 1/sqrt(d_h + d_r) (192 for the real shapes), not
    1/sqrt(d_c + d_r) (576): the two give clearly different outputs."""
    c = tiny_case(np.random.default_rng(5), B=1, s=1, H=2, d_c=16, d_r=4, d_h=8, bs=4,
                  lens=(6,), ints=False)
    c["w_uk"] = c["w_uk"] / 4.0  # keep the logits O(1), where the scale matters most
    out, _, _ = run_expanded(oracle_mod, c)
    good, _, _ = brute_force(c)
    wrong, _, _ = brute_force(c, scale_dims=c["d_c"] + c["d_r"])
    for i in range(2):
        np.testing.assert_allclose(out[i], good[0, i], atol=1e-13)
        assert np.max(np.abs(np.asarray(wrong[0, i]) - out[i])) > 2e-2


def test_softmax_rows_sum_to_one(oracle_mod):
    c = tiny_case(np.random.default_rng(2), B=2, s=2, lens=(6, 3), ints=False)
    _, _, probs = run_expanded(oracle_mod, c, probs_stride=8)
    n = 0
    for b in range(2):
        for t in range(2):
            nvis = c["lens"][b] - 2 + t + 1
            for i in range(c["H"]):
                p = probs[n]
                assert np.all(p >= 0)
                assert abs(p.sum() - 1.0) < 1e-14
                assert np.all(p[nvis:] == 0)
                n += 1


def _absorbed_vs_expanded(o, cfg_inputs, rows=None, heads=None):
    d = cfg_inputs
    cfg = d["cfg"]
    q_abs = o.absorb_q(o.bf16_to_f64(d["q_nope"]), o.bf16_to_f64(d["q_rope"]),
                       o.bf16_to_f64(d["w_uk"]), q_pos=d["q_pos"])
    lat, lse_a = o.decode_latent(d["cache"], d["block_table"], d["seq_lens"], cfg.s, q_abs,
                                 rows=rows, heads=heads)
    exp, lse_e, _ = o.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], cfg.s,
                                      o.bf16_to_f64(d["q_nope"]), o.bf16_to_f64(d["q_rope"]),
                                      o.bf16_to_f64(d["w_uk"]), o.bf16_to_f64(d["w_uv"]),
                                      q_pos=d["q_pos"], rows=rows, heads=heads)
    pr = rows if rows is not None else np.repeat(np.arange(cfg.T), cfg.H)
    ph = heads if heads is not None else np.tile(np.arange(cfg.H), cfg.T)
    w_uv = o.bf16_to_f64(d["w_uv"])
    o_abs = np.einsum("nkm,nm->nk", w_uv[ph], lat)
    return exp, o_abs, lse_e, lse_a


def test_absorbed_equals_expanded_tiny_config(oracle_mod):
    """The absorption identities (DeepSeek-V2 paper review, section 2) hold in
    fp64 on the tiny decode workload (H=16, L=256)."""
    d = W.make_decode_inputs(W.CONFIGS["tiny"])
    exp, o_abs, lse_e, lse_a = _absorbed_vs_expanded(oracle_mod, d)
    assert np.max(np.abs(exp - o_abs)) <= 1e-12 * np.max(np.abs(exp))
    np.testing.assert_allclose(lse_e, lse_a, rtol=1e-12)


def test_absorbed_equals_expanded_paged_ragged(oracle_mod):
    cfg = W.MLAConfig("t", B=3, s=2, H=4, L=0, paged=True, seed=77, d_model=64,
                      seq_lens=(130, 2, 64))
    d = W.make_decode_inputs(cfg)
    exp, o_abs, lse_e, lse_a = _absorbed_vs_expanded(oracle_mod, d)
    assert np.max(np.abs(exp - o_abs)) <= 1e-12 * np.max(np.abs(exp))
    np.testing.assert_allclose(lse_e, lse_a, rtol=1e-12)


def test_absorb_q_matches_library_matmul(oracle_mod):
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 3, 128)); qr = rng.standard_normal((5, 3, 64))
    U = rng.standard_normal((3, 128, 512))
    out = oracle_mod.absorb_q(q, qr, U)
    np.testing.assert_allclose(out[..., :512], np.einsum("hkm,thk->thm", U, q), rtol=1e-12, atol=1e-12)
    assert np.array_equal(out[..., 512:], qr)
    # the score identity: ((U^K)^T q)^T c == q^T (U^K c)
    c = rng.standard_normal(512)
    for t in range(5):
        for h in range(3):
            assert abs(out[t, h, :512] @ c - q[t, h] @ (U[h] @ c)) < 1e-9
    # with positions, the RoPE part is rotated
    pos = np.array([0, 1, 2, 3, 4], np.int32)
    out2 = oracle_mod.absorb_q(q, qr, U, q_pos=pos)
    assert np.array_equal(out2[0, :, 512:], qr[0])
    assert abs(np.linalg.norm(out2[3, 1, 512:]) - np.linalg.norm(qr[3, 1])) < 1e-12


def test_single_token_closed_form(oracle_mod):
    """With one visible key the softmax weight is 1: o = U^V c_0 and the
    latent output is c_0 exactly."""
    cfg = W.MLAConfig("t", B=2, s=1, H=4, L=1, paged=True, seed=5, d_model=64)
    d = W.make_decode_inputs(cfg)
    q_abs = oracle_mod.absorb_q(oracle_mod.bf16_to_f64(d["q_nope"]), oracle_mod.bf16_to_f64(d["q_rope"]),
                                oracle_mod.bf16_to_f64(d["w_uk"]), q_pos=d["q_pos"])
    lat, _ = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 1, q_abs)
    c0 = oracle_mod.bf16_to_f64(d["c_kv"])  # token 0 of each sequence, sequence-major
    for b in range(2):
        for h in range(4):
            assert np.array_equal(lat[b * 4 + h], c0[b])
    exp, _, _ = oracle_mod.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], 1,
                                           oracle_mod.bf16_to_f64(d["q_nope"]),
                                           oracle_mod.bf16_to_f64(d["q_rope"]),
                                           oracle_mod.bf16_to_f64(d["w_uk"]),
                                           oracle_mod.bf16_to_f64(d["w_uv"]), q_pos=d["q_pos"])
    Uv = oracle_mod.bf16_to_f64(d["w_uv"])
    for b in range(2):
        for h in range(4):
            np.testing.assert_allclose(exp[b * 4 + h], Uv[h] @ c0[b], rtol=1e-12, atol=1e-14)


def test_uniform_attention_closed_form(oracle_mod):
    """q^C = 0 and q^R = 0 make every logit 0: the latent output is the mean
    of the visible latents."""
    cfg = W.MLAConfig("t", B=2, s=2, H=2, L=0, paged=True, seed=9, d_model=64, seq_lens=(70, 5))
    d = W.make_decode_inputs(cfg)
    q_abs = np.zeros((cfg.T, cfg.H, 576))
    lat, lse = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 2, q_abs)
    c = oracle_mod.bf16_to_f64(d["c_kv"])
    starts = [0, 70]
    n = 0
    for b, L in enumerate((70, 5)):
        for t in range(2):
            nvis = L - 2 + t + 1
            for h in range(2):
                np.testing.assert_allclose(lat[n], c[starts[b]:starts[b] + nvis].mean(0), atol=1e-14)
                assert abs(lse[n] - math.log(nvis)) < 1e-14
                n += 1


def test_one_hot_limit(oracle_mod):
    """A query aligned with one key and scaled up puts all weight on it."""
    cfg = W.MLAConfig("t", B=1, s=1, H=1, L=40, paged=True, seed=13, d_model=64)
    d = W.make_decode_inputs(cfg)
    c = oracle_mod.bf16_to_f64(d["c_kv"])
    kr = oracle_mod.bf16_to_f64(d["k_rope"])
    k = 17
    key = np.concatenate([c[k], oracle_mod.rope(kr[k], k)])
    q_abs = (60.0 * key / np.linalg.norm(key))[None, None, :] * math.sqrt(192)
    lat, _ = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 1, q_abs)
    np.testing.assert_allclose(lat[0], c[k], atol=1e-9)


def test_heads_are_independent(oracle_mod):
    """Permuting the heads of q, U^K and U^V permutes the outputs (each head
    has its own a_ij; DeepSeek-V2 paper review, section 2)."""
    cfg = W.MLAConfig("t", B=2, s=1, H=5, L=0, paged=True, seed=21, d_model=64, seq_lens=(33, 8))
    d = W.make_decode_inputs(cfg)
    f = oracle_mod.bf16_to_f64
    perm = np.array([3, 0, 4, 1, 2])
    a, _, _ = oracle_mod.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], 1, f(d["q_nope"]),
                                         f(d["q_rope"]), f(d["w_uk"]), f(d["w_uv"]), q_pos=d["q_pos"])
    b, _, _ = oracle_mod.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], 1,
                                         f(d["q_nope"])[:, perm], f(d["q_rope"])[:, perm],
                                         f(d["w_uk"])[perm], f(d["w_uv"])[perm], q_pos=d["q_pos"])
    assert np.array_equal(a.reshape(2, 5, -1)[:, perm], b.reshape(2, 5, -1))
    # and heads really differ
    assert np.max(np.abs(a.reshape(2, 5, -1)[:, 0] - a.reshape(2, 5, -1)[:, 1])) > 1e-3


def test_block_permutation_invariance(oracle_mod):
    """The result depends only on the logical token order, not on where the
    blocks sit physically."""
    base = W.MLAConfig("t", B=3, s=1, H=2, L=0, paged=True, seed=31, d_model=64, seq_lens=(200, 65, 1))
    d1 = W.make_decode_inputs(base)
    d2 = W.make_decode_inputs(base.with_(paged=False))
    assert not np.array_equal(d1["block_table"], d2["block_table"])
    q_abs = oracle_mod.bf16_to_f64(W.make_q_abs(base))
    l1, s1 = oracle_mod.decode_latent(d1["cache"], d1["block_table"], d1["seq_lens"], 1, q_abs)
    l2, s2 = oracle_mod.decode_latent(d2["cache"], d2["block_table"], d2["seq_lens"], 1, q_abs)
    assert np.array_equal(l1, l2) and np.array_equal(s1, s2)


def test_nan_tail_slots_never_read(oracle_mod):
    cfg = W.MLAConfig("t", B=2, s=2, H=2, L=0, paged=True, seed=41, d_model=64, seq_lens=(67, 3))
    d = W.make_decode_inputs(cfg)
    assert np.isnan(W.bf16_bits_to_f32(d["cache"])).any()
    lat, lse = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 2,
                                        oracle_mod.bf16_to_f64(W.make_q_abs(cfg)))
    assert np.isfinite(lat).all() and np.isfinite(lse).all()


def test_causal_mask_two_queries(oracle_mod):
    """With s=2, query 0 of a length-L sequence sees exactly what a single
    query sees in the same sequence cut to length L-1."""
    cfg = W.MLAConfig("t", B=1, s=2, H=3, L=50, paged=True, seed=51, d_model=64)
    d = W.make_decode_inputs(cfg)
    q_abs = oracle_mod.bf16_to_f64(W.make_q_abs(cfg))
    lat2, lse2 = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 2, q_abs)
    lat1, lse1 = oracle_mod.decode_latent(d["cache"], d["block_table"], np.array([49], np.int32), 1,
                                          q_abs[0:1])
    assert np.array_equal(lat2[:3], lat1) and np.array_equal(lse2[:3], lse1)


def test_empty_row(oracle_mod):
    cfg = W.MLAConfig("t", B=2, s=1, H=2, L=0, paged=True, seed=61, d_model=64, seq_lens=(0, 4))
    d = W.make_decode_inputs(cfg)
    lat, lse = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], 1,
                                        oracle_mod.bf16_to_f64(W.make_q_abs(cfg)))
    assert np.all(lat[:2] == 0) and np.all(np.isneginf(lse[:2])) and np.isfinite(lse[2:]).all()


def test_bad_block_table_is_rejected(oracle_mod):
    cfg = W.MLAConfig("t", B=1, s=1, H=1, L=10, paged=True, seed=71, d_model=64)
    d = W.make_decode_inputs(cfg)
    bt = d["block_table"].copy(); bt[0, 0] = 5
    with pytest.raises(ValueError):
        oracle_mod.decode_latent(d["cache"], bt, d["seq_lens"], 1, np.zeros((1, 1, 576)))


def test_kv_project_matches_library_and_identity(oracle_mod):
    rng = np.random.default_rng(8)
    T, d = 6, 96
    h = bits(rng.standard_normal((T, d)))
    wd = bits(rng.standard_normal((512, d)) / 10)
    wr = bits(rng.standard_normal((64, d)) / 10)
    pos = np.array([0, 1, 7, 100, 4095, 131071], np.int32)
    c, kr = oracle_mod.kv_project(h, wd, wr, pos)
    hf, wdf, wrf = (oracle_mod.bf16_to_f64(x) for x in (h, wd, wr))
    np.testing.assert_allclose(c, hf @ wdf.T, rtol=1e-12, atol=1e-12)
    raw = hf @ wrf.T
    np.testing.assert_allclose(kr[0], raw[0], atol=1e-12)               # RoPE at 0 is the identity
    np.testing.assert_allclose(np.linalg.norm(kr, axis=1), np.linalg.norm(raw, axis=1), rtol=1e-12)
    # identity projection reproduces the input exactly
    hh = bits(rng.standard_normal((3, 576)))
    eye_c = bits(np.eye(576)[:512]); eye_r = bits(np.eye(576)[512:])
    c2, kr2 = oracle_mod.kv_project(hh, eye_c, eye_r, np.zeros(3, np.int32))
    assert np.array_equal(c2, oracle_mod.bf16_to_f64(hh)[:, :512])
    assert np.array_equal(kr2, oracle_mod.bf16_to_f64(hh)[:, 512:])


def test_up_v_and_out_proj_match_library(oracle_mod):
    rng = np.random.default_rng(9)
    lat = rng.standard_normal((4, 3, 512)); U = rng.standard_normal((3, 128, 512))
    o = oracle_mod.up_v(lat, U)
    np.testing.assert_allclose(o, np.einsum("hkm,thm->thk", U, lat), rtol=1e-12, atol=1e-11)
    Wo = rng.standard_normal((40, 3 * 128))
    u = oracle_mod.out_proj(o, Wo)
    np.testing.assert_allclose(u, o.reshape(4, -1) @ Wo.T, rtol=1e-12, atol=1e-10)


def test_generator_bf16_rounding_matches_torch():
    import torch
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    mine = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_generator_is_deterministic_and_paged():
    cfg = W.MLAConfig("t", B=3, s=2, H=2, L=(10, 200), paged=True, seed=99, d_model=64)
    a, b = W.make_decode_inputs(cfg), W.make_decode_inputs(cfg)
    for k in ("cache", "block_table", "q_nope", "w_uk", "seq_lens"):
        assert np.array_equal(a[k], b[k])
    bt = a["block_table"]
    used = bt[bt >= 0]
    assert sorted(used.tolist()) == list(range(a["num_blocks"]))
    for bb in range(3):
        n = (a["seq_lens"][bb] + 63) // 64
        assert np.all(bt[bb, :n] >= 0) and np.all(bt[bb, n:] == -1)


# ------------------------------------------------------ planted mistakes
MUTATIONS = {
    "drop_rope_term": ("for (int m = 0; m < d_r; ++m) dot += qr[m] * kr[m];", ""),
    "rope_sign": ("y[2 * k] = x0 * c - x1 * s;", "y[2 * k] = x0 * c + x1 * s;"),
    "transposed_uk": ("acc += Uk[(size_t)k * d_c + m] * c[m];", "acc += Uk[(size_t)(m % d_h) * d_c + k] * c[m];"),
    "latent_scale": ("const double scale = 1.0 / sqrt((double)(d_h + d_r));\n    int bad = 0;\n    (void)B;\n#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)\n    for (int p = 0; p < n_pairs; ++p) {\n        const int row = pair_row[p], i = pair_head[p];\n        const int b = row / s, t = row % s;\n        const int L",
                     "const double scale = 1.0 / sqrt((double)(d_c + d_r));\n    int bad = 0;\n    (void)B;\n#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)\n    for (int p = 0; p < n_pairs; ++p) {\n        const int row = pair_row[p], i = pair_head[p];\n        const int b = row / s, t = row % s;\n        const int L"),
    "mask_off_by_one": ("const int n_vis = L - s + t + 1;", "const int n_vis = L - s + t;"),
    "key_position": ("mla_oracle_rope(kr_raw, d_r, (double)j, rope_base, kr);\n            for (int k = 0; k < d_h; ++k) {",
                     "mla_oracle_rope(kr_raw, d_r, (double)(j + 1), rope_base, kr);\n            for (int k = 0; k < d_h; ++k) {"),
    "no_max_subtract_den": ("lse[p] = mx + log(den);\n        /* o = sum", "lse[p] = log(den);\n        /* o = sum"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(oracle_mod, tmp_path, name):
    """Plant one plausible mistake in a copy of the oracle source and check
    that the brute-force pin rejects the mutant."""
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle_mod.__file__), "mla_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, name
    mutant = tmp_path / "m.c"
    mutant.write_text(src.replace(old, new, 1))
    so = tmp_path / "m.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(mutant), "-lm"],
                   check=True)
    saved = oracle_mod._LIB
    oracle_mod._LIB = oracle_mod.load(str(so))
    try:
        caught = False
        for seed, s, lens in ((0, 1, (3, 2)), (1, 2, (3, 4)), (4, 2, (5, 6))):
            c = tiny_case(np.random.default_rng(seed), B=2, s=s, lens=lens, ints=False)
            try:
                check_brute(oracle_mod, c, tol=1e-9)
            except AssertionError:
                caught = True
                break
        assert caught, f"mutation {name} was not caught"
    finally:
        oracle_mod._LIB = saved


# ------------------------------------------------- pins added for the batch forms
def test_rope_rows_equal_rope_of_each_row_and_closed_forms(oracle_mod):
    """rope_rows is rope applied to each row at its own position: checked row
    by row, and against the closed form of a unit vector (pair k turns by
    pos * 10000^(-2k/64))."""
    rng = np.random.default_rng(21)
    pos = np.array([0, 1, 63, 64, 4095, 131071, 7, 7], np.int32)
    x = rng.standard_normal((pos.size, 64))
    y = oracle_mod.rope_rows(x, pos)
    for n in range(pos.size):
        assert np.array_equal(y[n], oracle_mod.rope(x[n], float(pos[n])))
    assert np.array_equal(y[0], x[0])                       # position 0: identity
    e = np.zeros((pos.size, 64)); k = 5
    e[:, 2 * k] = 1.0
    ye = oracle_mod.rope_rows(e, pos)
    ang = pos.astype(np.float64) * 10000.0 ** (-2 * k / 64)
    np.testing.assert_allclose(ye[:, 2 * k], np.cos(ang), atol=1e-12)
    np.testing.assert_allclose(ye[:, 2 * k + 1], np.sin(ang), atol=1e-12)
    assert np.count_nonzero(np.delete(ye, [2 * k, 2 * k + 1], axis=1)) == 0


def test_up_v_identity_returns_the_latent_columns_exactly(oracle_mod):
    """U^V_i = [I_128 | 0]: o_i is the first 128 latent columns, exactly."""
    rng = np.random.default_rng(22)
    lat = rng.standard_normal((5, 3, 512))
    U = np.zeros((3, 128, 512)); U[:, :, :128] = np.eye(128)
    assert np.array_equal(oracle_mod.up_v(lat, U), lat[:, :, :128])
    # a permutation of columns picks them out in that order
    perm = rng.permutation(512)[:128]
    P = np.zeros((3, 128, 512)); P[:, np.arange(128), perm] = 1.0
    assert np.array_equal(oracle_mod.up_v(lat, P), lat[:, :, perm])


def test_absorb_q_identity_returns_q_exactly(oracle_mod):
    """U^K_i = [I_128 | 0]: (U^K_i)^T q^C puts q^C in the first 128 columns
    and zeros elsewhere."""
    rng = np.random.default_rng(23)
    q = rng.standard_normal((4, 2, 128)); qr = rng.standard_normal((4, 2, 64))
    U = np.zeros((2, 128, 512)); U[:, :, :128] = np.eye(128)
    out = oracle_mod.absorb_q(q, qr, U)
    assert np.array_equal(out[..., :128], q)
    assert np.all(out[..., 128:512] == 0)


@pytest.mark.parametrize("seed,s,lens,H", [(31, 1, (130, 1, 64, 0), 16), (32, 2, (70, 2, 129), 32),
                                           (33, 1, (200,), 20)])
def test_decode_latent_rows_is_bit_identical_to_decode_latent(oracle_mod, seed, s, lens, H):
    """The batch form reorders only the loops: every output is the same bits
    as the per-pair form, for head counts that do and do not fill whole groups
    of 16, ragged and empty rows."""
    cfg = W.MLAConfig("rows", B=len(lens), s=s, H=H, L=0, paged=True, seed=seed, d_model=64,
                      seq_lens=lens)
    d = W.make_decode_inputs(cfg)
    q = oracle_mod.bf16_to_f64(W.make_q_abs(cfg))
    a, la = oracle_mod.decode_latent(d["cache"], d["block_table"], d["seq_lens"], s, q)
    b, lb = oracle_mod.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], s, q)
    assert np.array_equal(a.reshape(b.shape), b)
    assert np.array_equal(la.reshape(lb.shape), lb)
    rows = np.array([cfg.T - 1, 0], np.int32)
    c, lc = oracle_mod.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], s, q, rows=rows)
    assert np.array_equal(c, b[rows]) and np.array_equal(lc, lb[rows])


def test_decode_latent_rows_closed_forms(oracle_mod):
    """One visible key returns its latent exactly; zero queries return the
    plain mean of the visible latents (uniform weights)."""
    cfg = W.MLAConfig("rows1", B=2, s=1, H=17, L=1, paged=True, seed=24, d_model=64)
    d = W.make_decode_inputs(cfg)
    q = oracle_mod.bf16_to_f64(W.make_q_abs(cfg))
    lat, lse = oracle_mod.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], 1, q)
    c0 = oracle_mod.bf16_to_f64(d["c_kv"])
    assert np.array_equal(lat, np.repeat(c0[:, None, :], cfg.H, axis=1))
    cfg = W.MLAConfig("rows2", B=2, s=1, H=16, L=0, paged=True, seed=25, d_model=64, seq_lens=(90, 7))
    d = W.make_decode_inputs(cfg)
    lat, lse = oracle_mod.decode_latent_rows(d["cache"], d["block_table"], d["seq_lens"], 1,
                                             np.zeros((cfg.T, cfg.H, 576)))
    c = oracle_mod.bf16_to_f64(d["c_kv"])
    starts = np.concatenate([[0], np.cumsum(d["seq_lens"])])
    for b in range(2):
        mean = c[starts[b]:starts[b + 1]].mean(axis=0)
        np.testing.assert_allclose(lat[b], np.repeat(mean[None], cfg.H, axis=0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[b], np.log(d["seq_lens"][b]), rtol=1e-14)


# ------------------------------------------------------------- FP8 cache pins
def test_e4m3_values_the_specification_prints(oracle_mod):
    """OCP 8-bit floating point, E4M3: 0x38 = 1, 0x7E = 448 (largest finite),
    0x08 = 2^-6 (smallest normal), 0x07 = 7/8 * 2^-6 (largest subnormal), 0x01 =
    2^-9 (smallest subnormal), 0xC0 = -2, 0x7F and 0xFF are NaN, 0x80 = -0."""
    v = oracle_mod.e4m3_values(np.array([0x38, 0x7E, 0x08, 0x07, 0x01, 0xC0, 0x00, 0x80], np.uint8))
    assert list(v) == [1.0, 448.0, 2.0 ** -6, 0.875 * 2.0 ** -6, 2.0 ** -9, -2.0, 0.0, -0.0]
    assert np.isnan(oracle_mod.e4m3_values(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_matches_torch_on_every_code_and_in_range_values(oracle_mod):
    """torch's float8_e4m3fn is an independent implementation of the same
    format: every code decodes to the same value, and in-range floats
    (|x| <= 448, where torch does not saturate) encode to the same code."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = oracle_mod.e4m3_values(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    rng = np.random.default_rng(40)
    x = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(20000) * 1e-2,
                        rng.uniform(-448, 448, 20000), oracle_mod.e4m3_values(codes[ok & (np.abs(ref) <= 448)]),
                        # exact midpoints between neighbouring values: ties go to the even code
                        (ref[1:0x7E] + ref[2:0x7F]) / 2]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle_mod.e4m3_encode(x), want)


def test_e4m3_encode_saturates_and_rounds_ties_to_even(oracle_mod):
    codes = oracle_mod.e4m3_encode(np.array([448.0, 449.0, 464.0, 1e6, -1e6, 2.0 ** -10, 1.5 * 2.0 ** -9,
                                             1.0625, 1.1875], np.float32))
    # 464 is midway between 448 and the next step (480, not finite): it stays
    # at the even 448; 2^-10 is midway between 0 and 2^-9: 0 (even);
    # 1.0625 is midway between 1 (0x38) and 1.125 (0x39): 0x38; 1.1875
    # between 1.125 (0x39) and 1.25 (0x3A): 0x3A
    assert list(codes) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x02, 0x38, 0x3A]


def test_quantize_rows_scales_and_codes(oracle_mod):
    rng = np.random.default_rng(41)
    rows = (rng.standard_normal((50, 576)) * rng.uniform(0.01, 30, (50, 1))).astype(np.float32)
    rows[3, :512] = 0.0                                   # an all-zero part gets scale 1
    codes, scales = oracle_mod.quantize_rows(rows)
    amax_c = np.abs(rows[:, :512]).max(1)
    amax_r = np.abs(rows[:, 512:]).max(1)
    np.testing.assert_array_equal(scales[:, 0], np.where(amax_c > 0, amax_c / np.float32(448), 1).astype(np.float32))
    np.testing.assert_array_equal(scales[:, 1], (amax_r / np.float32(448)).astype(np.float32))
    assert np.all(codes[3, :512] == 0)
    vals = oracle_mod.e4m3_values(codes)
    q = rows / np.repeat(scales, [512, 64], axis=1)
    # every code is the nearest value (within half a step of its neighbours)
    err = np.abs(vals - q)
    step = np.maximum(np.abs(vals) * 2.0 ** -3, 2.0 ** -9)
    assert np.all(err <= step / 2 + 1e-6 * np.abs(q))
    # the element of largest magnitude lands on +-448
    i = np.argmax(np.abs(rows[0, :512]))
    assert abs(vals[0, i]) == 448.0


def _fp8_tiny_cache(oracle_mod, cfg, rng, unit_scales=False):
    """An FP8 cache for a workload: random E4M3-representable latents and
    rotated keys, pages and table from the workload's paging."""
    sl = W.seq_lens_of(cfg)
    table, nphys, _ = W.paging(cfg, sl)
    tok_seq, tok_pos = W.token_index(sl)
    codes_tok = rng.integers(0, 0x7F, size=(tok_seq.size, 576)).astype(np.uint8)   # finite, non-negative
    codes_tok |= (rng.integers(0, 2, size=codes_tok.shape).astype(np.uint8) << 7)  # signs
    codes_tok[:, :] = np.where((codes_tok & 0x7F) == 0x7F, 0x7E, codes_tok)
    scales_tok = np.ones((tok_seq.size, 2), np.float32) if unit_scales else \
        rng.uniform(1e-3, 1e-2, (tok_seq.size, 2)).astype(np.float32)
    codes = np.zeros((nphys, 64, 576), np.uint8)
    scales = np.zeros((nphys, 64, 2), np.float32)
    blk = table[tok_seq, tok_pos // 64]
    codes[blk, tok_pos % 64] = codes_tok
    scales[blk, tok_pos % 64] = scales_tok
    return sl, table, codes, scales, codes_tok, scales_tok, tok_seq


def test_decode_fp8_equals_bf16_decode_on_representable_values(oracle_mod):
    """With unit scales and no RoPE part (zero codes, which rotate to zero in
    the bf16 path too), an FP8 cache of E4M3 values holds exactly the values
    of a bf16 cache: the two decodes agree bit for bit."""
    rng = np.random.default_rng(42)
    cfg = W.MLAConfig("f8", B=3, s=2, H=20, L=0, paged=True, seed=43, d_model=64, seq_lens=(130, 2, 65))
    sl, table, codes, scales, codes_tok, _, tok_seq = _fp8_tiny_cache(oracle_mod, cfg, rng, unit_scales=True)
    codes[..., 512:] = 0
    vals = oracle_mod.e4m3_values(codes).astype(np.float32)        # exact in bf16 (3-bit mantissa)
    bf = W.f32_to_bf16_bits(vals)
    assert np.array_equal(W.bf16_bits_to_f32(bf), vals)
    q = oracle_mod.bf16_to_f64(W.make_q_abs(cfg))
    a, la = oracle_mod.decode_latent_fp8_rows(codes, scales, table, sl, cfg.s, q)
    b, lb = oracle_mod.decode_latent_rows(bf, table, sl, cfg.s, q)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_decode_fp8_brute_force_tiny(oracle_mod):
    """A textbook NumPy softmax over the dequantized rows (codes times their
    part's scale, the RoPE key taken as already rotated)."""
    rng = np.random.default_rng(44)
    cfg = W.MLAConfig("f8b", B=2, s=1, H=3, L=0, paged=True, seed=45, d_model=64, seq_lens=(70, 9))
    sl, table, codes, scales, codes_tok, scales_tok, tok_seq = _fp8_tiny_cache(oracle_mod, cfg, rng)
    q = rng.standard_normal((cfg.T, cfg.H, 576))
    got, lse = oracle_mod.decode_latent_fp8_rows(codes, scales, table, sl, cfg.s, q)
    x = oracle_mod.e4m3_values(codes_tok) * np.repeat(scales_tok.astype(np.float64), [512, 64], axis=1)
    starts = np.concatenate([[0], np.cumsum(sl)])
    for b in range(cfg.B):
        X = x[starts[b]:starts[b + 1]]
        for h in range(cfg.H):
            l = X @ q[b, h] / math.sqrt(192.0)
            p = np.exp(l - l.max())
            np.testing.assert_allclose(got[b, h], (p / p.sum()) @ X[:, :512], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(lse[b, h], l.max() + math.log(p.sum()), rtol=1e-13)


FP8_MUTATIONS = {
    "exponent_bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "subnormal_scale": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "ties_to_odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "wrong_max": ("const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;",
                  "const float sc = amax > 0.0f ? amax / 240.0f : 1.0f;"),
    "rope_part_with_latent_scale": ("* (double)scales[2 * slot + (m < d_c ? 0 : 1)];", "* (double)scales[2 * slot];"),
}


@pytest.mark.parametrize("name", sorted(FP8_MUTATIONS))
def test_planted_fp8_mistakes_are_caught(oracle_mod, tmp_path, name):
    """One plausible mistake in the FP8 routines of a copy of the oracle must
    make one of the FP8 pins fail."""
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle_mod.__file__), "mla_oracle.c")).read()
    old, new = FP8_MUTATIONS[name]
    assert src.count(old) == 1, name
    mutant = tmp_path / "m.c"
    mutant.write_text(src.replace(old, new, 1))
    so = tmp_path / "m.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(mutant), "-lm"], check=True)
    saved = oracle_mod._LIB
    oracle_mod._LIB = oracle_mod.load(str(so))
    pins = (test_e4m3_values_the_specification_prints, test_e4m3_matches_torch_on_every_code_and_in_range_values,
            test_e4m3_encode_saturates_and_rounds_ties_to_even, test_quantize_rows_scales_and_codes,
            test_decode_fp8_brute_force_tiny)
    try:
        caught = False
        for pin in pins:
            try:
                pin(oracle_mod)
            except AssertionError:
                caught = True
                break
        assert caught, f"mutation {name} was not caught"
    finally:
        oracle_mod._LIB = saved


# ------------------------------------------------------- append extras pins
def test_rmsnorm_rows_closed_forms(oracle_mod):
    rng = np.random.default_rng(50)
    x = rng.standard_normal((20, 512)) * rng.uniform(0.1, 30, (20, 1))
    ones = np.ones(512)
    y = oracle_mod.rmsnorm_rows(x, ones, eps=0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(1)), 1.0, rtol=1e-14)       # unit RMS
    np.testing.assert_allclose(oracle_mod.rmsnorm_rows(7.5 * x, ones, eps=0.0), y, rtol=1e-13)  # scale invariant
    c = np.full((1, 512), -3.0)                                                  # constant row: sign * w
    w = rng.standard_normal(512)
    np.testing.assert_allclose(oracle_mod.rmsnorm_rows(c, w, eps=0.0)[0], -w, rtol=1e-15)
    # eps enters under the root: a zero row stays zero, a tiny row is damped
    assert np.all(oracle_mod.rmsnorm_rows(np.zeros((1, 512)), w, eps=1e-6) == 0)
    t = np.full((1, 512), 1e-3)
    np.testing.assert_allclose(oracle_mod.rmsnorm_rows(t, ones, eps=1e-6)[0], 1e-3 / math.sqrt(1e-6 + 1e-6),
                               rtol=1e-14)


def test_yarn_theta_reduces_to_rope_and_interpolates(oracle_mod):
    base = 10000.0
    plain = base ** (-2.0 * np.arange(32) / 64)
    np.testing.assert_allclose(oracle_mod.yarn_theta(s=1.0), plain, rtol=5e-16)  # numpy and libm pow: an ulp apart at most
    th = oracle_mod.yarn_theta(s=40.0, L0=4096.0, alpha=1.0, beta=32.0)
    rot = 4096.0 * plain / (2 * math.pi)                 # rotations over the original context
    hi, lo = rot > 32.0, rot < 1.0
    assert hi.any() and lo.any()
    np.testing.assert_allclose(th[hi], plain[hi], rtol=1e-15)        # fast pairs unchanged
    np.testing.assert_allclose(th[lo], plain[lo] / 40.0, rtol=1e-15)  # slow pairs interpolated by s
    mid = ~(hi | lo)
    g = (rot[mid] - 1.0) / 31.0
    np.testing.assert_allclose(th[mid], (1 - g) * plain[mid] / 40.0 + g * plain[mid], rtol=1e-14)
    assert np.all(np.diff(th) < 0)                       # still strictly decreasing with k


def test_rope_rows_theta_matches_plain_rope_and_preserves_norms(oracle_mod):
    rng = np.random.default_rng(51)
    pos = np.array([0, 1, 4095, 65536, 131071], np.int32)
    x = rng.standard_normal((pos.size, 64))
    plain = oracle_mod.rope_rows_theta(x, pos, oracle_mod.yarn_theta(s=1.0))
    np.testing.assert_allclose(plain, oracle_mod.rope_rows(x, pos), rtol=0, atol=1e-12)
    y = oracle_mod.rope_rows_theta(x, pos, oracle_mod.yarn_theta(s=40.0))
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    assert np.array_equal(y[0], x[0])
    # relative positions: <R_m q, R_n k> depends on n - m only, also with YaRN
    th = oracle_mod.yarn_theta(s=40.0)
    q, k = rng.standard_normal((1, 64)), rng.standard_normal((1, 64))
    a = oracle_mod.rope_rows_theta(q, np.array([7], np.int32), th) @ oracle_mod.rope_rows_theta(k, np.array([900], np.int32), th).T
    b = oracle_mod.rope_rows_theta(q, np.array([7007], np.int32), th) @ oracle_mod.rope_rows_theta(k, np.array([7900], np.int32), th).T
    assert abs(a - b) < 1e-10


# ------------------------------------------------ weight pre-absorption pins
def test_fold_identities_return_the_factors_exactly(oracle_mod):
    """W^UQ_i = I (d_q = d_h) makes W^QK_i = (U^K_i)^T; W^O = I (d_model =
    H d_h) makes the blocks of W^OV the U^V_i, placed block-diagonally."""
    rng = np.random.default_rng(31)
    H, d_h, d_c = 3, 8, 12
    w_uk = rng.standard_normal((H, d_h, d_c))
    w_uv = rng.standard_normal((H, d_h, d_c))
    eye = np.broadcast_to(np.eye(d_h), (H, d_h, d_h)).copy()
    got = oracle_mod.fold_qk(eye, w_uk)
    assert np.array_equal(got, np.transpose(w_uk, (0, 2, 1)))
    got = oracle_mod.fold_ov(np.eye(H * d_h), w_uv)
    want = np.zeros((H * d_h, H * d_c))
    for i in range(H):
        want[i * d_h:(i + 1) * d_h, i * d_c:(i + 1) * d_c] = w_uv[i]
    assert np.array_equal(got, want)


def test_fold_brute_force_tiny_integers(oracle_mod):
    """Each entry of W^QK and W^OV is one dot product, checked one by one on
    small integers (exact in fp64)."""
    rng = np.random.default_rng(32)
    H, d_h, d_c, d_q, d_model = 2, 3, 4, 5, 6
    w_uq = rng.integers(-3, 4, (H, d_h, d_q)).astype(np.float64)
    w_uk = rng.integers(-3, 4, (H, d_h, d_c)).astype(np.float64)
    w_uv = rng.integers(-3, 4, (H, d_h, d_c)).astype(np.float64)
    w_o = rng.integers(-3, 4, (d_model, H * d_h)).astype(np.float64)
    qk = oracle_mod.fold_qk(w_uq, w_uk)
    ov = oracle_mod.fold_ov(w_o, w_uv)
    for i in range(H):
        for c in range(d_c):
            for q in range(d_q):
                assert qk[i, c, q] == sum(w_uk[i, k, c] * w_uq[i, k, q] for k in range(d_h))
    for m in range(d_model):
        for i in range(H):
            for c in range(d_c):
                assert ov[m, i * d_c + c] == sum(w_o[m, i * d_h + k] * w_uv[i, k, c] for k in range(d_h))


def test_folded_paths_equal_the_two_step_paths(oracle_mod):
    """The identities the folding rests on, against the pinned routines:
    absorb_q_folded(c^Q) = absorb_q(q^C = W^UQ c^Q) and up_out_folded(õ) =
    out_proj(up_v(õ))."""
    rng = np.random.default_rng(33)
    T, H, d_h, d_c, d_r, d_q, d_model = 3, 4, 8, 16, 8, 24, 20
    w_uq = rng.standard_normal((H, d_h, d_q))
    w_uk = rng.standard_normal((H, d_h, d_c))
    w_uv = rng.standard_normal((H, d_h, d_c))
    w_o = rng.standard_normal((d_model, H * d_h))
    c_q = rng.standard_normal((T, d_q))
    q_rope = rng.standard_normal((T, H, d_r))
    q_pos = np.array([0, 7, 300], np.int32)
    q_c = np.einsum("ikq,tq->tik", w_uq, c_q)
    want = oracle_mod.absorb_q(q_c, q_rope, w_uk, q_pos=q_pos)
    got = oracle_mod.absorb_q_folded(c_q, q_rope, oracle_mod.fold_qk(w_uq, w_uk), q_pos=q_pos)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(got[..., d_c:],
                                  oracle_mod.absorb_q_folded(c_q, q_rope, np.zeros((H, d_c, d_q)),
                                                             q_pos=q_pos)[..., d_c:])
    lat = rng.standard_normal((T, H, d_c))
    want = oracle_mod.out_proj(oracle_mod.up_v(lat, w_uv), w_o)
    got = oracle_mod.up_out_folded(lat, oracle_mod.fold_ov(w_o, w_uv))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


FOLD_MUTATIONS = {
    "qk_untransposed": ("const double u = w_uk[((size_t)i * d_h + k) * d_c + c];",
                        "const double u = w_uk[((size_t)i * d_h + c % d_h) * d_c + k];"),
    "ov_wrong_head_block": ("const double o = w_o[(size_t)m * H * d_h + (size_t)i * d_h + k];",
                            "const double o = w_o[(size_t)m * H * d_h + (size_t)((i + 1) % H) * d_h + k];"),
    "absorb_folded_drops_rope": ("mla_oracle_rope(r, d_r, (double)q_pos[t], base, o + d_c);",
                                 "for (int m = 0; m < d_r; ++m) o[d_c + m] = r[m];"),
    "up_out_folded_skips_last_head": ("for (int j = 0; j < H * d_c; ++j) acc += w[j] * x[j];",
                                      "for (int j = 0; j < (H - 1) * d_c; ++j) acc += w[j] * x[j];"),
}


@pytest.mark.parametrize("name", sorted(FOLD_MUTATIONS))
def test_planted_fold_mistakes_are_caught(oracle_mod, tmp_path, name):
    """One plausible mistake in the folding routines of a copy of the oracle
    must make one of the folding pins fail."""
    import subprocess
    src = open(os.path.join(os.path.dirname(oracle_mod.__file__), "mla_oracle.c")).read()
    old, new = FOLD_MUTATIONS[name]
    assert src.count(old) == 1, name
    mutant = tmp_path / "m.c"
    mutant.write_text(src.replace(old, new, 1))
    so = tmp_path / "m.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(mutant), "-lm"], check=True)
    saved = oracle_mod._LIB
    oracle_mod._LIB = oracle_mod.load(str(so))
    pins = (test_fold_identities_return_the_factors_exactly, test_fold_brute_force_tiny_integers,
            test_folded_paths_equal_the_two_step_paths)
    try:
        caught = False
        for pin in pins:
            try:
                pin(oracle_mod)
            except AssertionError:
                caught = True
                break
        assert caught, f"mutation {name} was not caught"
    finally:
        oracle_mod._LIB = saved
