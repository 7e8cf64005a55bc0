"""GPU parity of the FP8 (E4M3) latent cache: the cache writer bit for bit
against the oracle's quantizer, and the FP8 decode against the oracle's
FP8 decode on the same codes and scales.

The decode tests feed both sides one random FP8 cache drawn as bit patterns
by the workload generator (mla_workloads.make_fp8_cache), so neither side's
quantizer is involved; the end-to-end test runs the GPU writer and the GPU
decode and compares with the oracle's quantizer and decode from the raw bf16
inputs.  Bars: bit-exact for codes and scales; for the decode the bf16 path's
bar (assert_parity: max-abs <= 2e-2, relative L2 <= 1e-2; lse 1e-2 absolute):
the kernel rounds q_abs and P to f16 (finer than bf16) and widens codes
exactly.
"""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import assert_parity, host_bits, i32, rel_l2, torch_bits

pytestmark = pytest.mark.gpu

CASES = [
    W.MLAConfig("f8_h16_ragged", B=3, s=1, H=16, L=0, paged=True, seed=401, d_model=2048,
                seq_lens=(1000, 65, 1)),
    W.MLAConfig("f8_h128_ragged", B=3, s=1, H=128, L=0, paged=True, seed=402, d_model=5120,
                seq_lens=(700, 129, 63)),
    W.MLAConfig("f8_h128_two_queries", B=3, s=2, H=128, L=0, paged=True, seed=403, d_model=5120,
                seq_lens=(300, 2, 1500)),
    W.MLAConfig("f8_h64_many_splits", B=2, s=1, H=64, L=0, paged=True, seed=404, d_model=4096,
                seq_lens=(2500, 1100)),
    W.MLAConfig("f8_h32_contiguous", B=2, s=1, H=32, L=0, paged=False, seed=405, d_model=2048,
                seq_lens=(257, 64)),
]


@pytest.fixture(scope="module")
def lib():
    import head_latent_attention_10_b200 as M
    M.load_library()
    return M


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def fp8_decode(M, cfg, d, codes, scales, q_abs, flags=0, seq_lens=None):
    import torch
    dims = M.dims(cfg.H)
    lat = torch.empty(cfg.T, cfg.H, cfg.d_c, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
    ws = torch.empty(M.mla_decode_workspace_size(dims, cfg.B, cfg.s, d["block_table"].shape[1] * 64),
                     dtype=torch.uint8, device="cuda")
    M.mla_decode_fp8(dims, torch_bits(q_abs), _dev(codes), _dev(scales), _dev(d["block_table"]),
                     _dev(d["seq_lens"] if seq_lens is None else seq_lens), cfg.s, lat, lse, ws, flags=flags)
    torch.cuda.synchronize()
    err = M.mla_decode_error(ws)
    return W.bf16_bits_to_f32(host_bits(lat)).astype(np.float64), lse.cpu().numpy().astype(np.float64), err


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fp8_decode_against_oracle(lib, cfg):
    import oracle
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    codes, scales = W.make_fp8_cache(cfg, d["block_table"], d["num_blocks"], d["tok_seq"], d["tok_pos"])
    q_abs = W.make_q_abs(cfg)
    got, lse, err = fp8_decode(lib, cfg, d, codes, scales, q_abs)
    assert err == 0
    ref, rlse = oracle.decode_latent_fp8_rows(codes, scales, d["block_table"], d["seq_lens"], cfg.s,
                                              oracle.bf16_to_f64(q_abs))
    assert_parity(got, ref, what=f"{cfg.name} latent")
    np.testing.assert_allclose(lse, rlse, atol=1e-2, rtol=0)


def test_fp8_writer_is_bit_exact_against_the_oracle_quantizer(lib):
    """Tokens at position 0 (RoPE is the identity there), one per sequence:
    the GPU's codes and scales equal the oracle quantizer's on the same bf16
    rows, bit for bit; untouched slots keep their fill."""
    import oracle
    import torch
    cfg = W.MLAConfig("f8_writer", B=200, s=1, H=16, L=1, paged=True, seed=406, d_model=2048)
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    assert np.all(d["tok_pos"] == 0)
    nb = d["num_blocks"]
    codes = torch.full((nb, 64, 576), 0x7F, dtype=torch.uint8, device="cuda")
    scales = torch.full((nb, 64, 2), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dims = lib.dims(cfg.H)
    lib.mla_append_latent_fp8(dims, torch_bits(d["c_kv"]), torch_bits(d["k_rope"]), i32(d["tok_seq"]),
                              i32(d["tok_pos"]), i32(d["block_table"]), codes, scales, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = np.concatenate([W.bf16_bits_to_f32(d["c_kv"]), W.bf16_bits_to_f32(d["k_rope"])], axis=1)
    want_c, want_s = oracle.quantize_rows(rows)
    blk = d["block_table"][d["tok_seq"], 0]
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(gc[blk, 0], want_c)
    assert np.array_equal(gs[blk, 0].view(np.uint32), want_s.view(np.uint32))
    assert np.all(gc[:, 1:] == 0x7F) and np.all(np.isnan(gs[:, 1:]))


def test_fp8_writer_rotates_the_key(lib):
    """Real positions: latent codes and scales bit-exact against the oracle
    quantizer (the latent is not rotated); the dequantized RoPE part within
    E4M3's half-step (plus the bf16 rounding) of the oracle's fp64 rotation."""
    import oracle
    import torch
    cfg = W.CONFIGS["tiny"].with_(name="f8_writer_rot", seq_lens=(300,), L=300, seed=407)
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    nb = d["num_blocks"]
    codes = torch.full((nb, 64, 576), 0x7F, dtype=torch.uint8, device="cuda")
    scales = torch.full((nb, 64, 2), float("nan"), dtype=torch.float32, device="cuda")
    dims = lib.dims(cfg.H)
    lib.mla_append_latent_fp8(dims, torch_bits(d["c_kv"]), torch_bits(d["k_rope"]), i32(d["tok_seq"]),
                              i32(d["tok_pos"]), i32(d["block_table"]), codes, scales)
    torch.cuda.synchronize()
    blk = d["block_table"][d["tok_seq"], d["tok_pos"] // 64]
    slot = d["tok_pos"] % 64
    gc, gs = codes.cpu().numpy()[blk, slot], scales.cpu().numpy()[blk, slot]
    # latent part: exact (no rotation)
    lat = W.bf16_bits_to_f32(d["c_kv"])
    wc, ws_ = oracle.quantize_rows(np.concatenate([lat, np.zeros((lat.shape[0], 64), np.float32)], axis=1))
    assert np.array_equal(gc[:, :512], wc[:, :512])
    assert np.array_equal(gs[:, 0].view(np.uint32), ws_[:, 0].view(np.uint32))
    # RoPE part: value within half an E4M3 step (2^-4 relative) plus bf16 rounding
    kr_ref = oracle.rope_rows(oracle.bf16_to_f64(d["k_rope"]), d["tok_pos"])
    kr_gpu = oracle.e4m3_values(gc[:, 512:]) * gs[:, 1:2].astype(np.float64)
    tol = (2.0 ** -4 + 2.0 ** -8) * np.abs(kr_ref) + gs[:, 1:2] * 2.0 ** -9
    assert np.all(np.abs(kr_gpu - kr_ref) <= tol)


def test_fp8_end_to_end_against_the_oracle(lib):
    """GPU writer -> GPU FP8 decode against the oracle's quantizer -> oracle
    FP8 decode from the same raw inputs (the rotated RoPE keys may differ by a
    bf16 rounding, hence one code, on either side)."""
    import oracle
    import torch
    cfg = CASES[1]
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    nb = d["num_blocks"]
    codes = torch.full((nb, 64, 576), 0x7F, dtype=torch.uint8, device="cuda")
    scales = torch.full((nb, 64, 2), float("nan"), dtype=torch.float32, device="cuda")
    dims = lib.dims(cfg.H)
    lib.mla_append_latent_fp8(dims, torch_bits(d["c_kv"]), torch_bits(d["k_rope"]), i32(d["tok_seq"]),
                              i32(d["tok_pos"]), i32(d["block_table"]), codes, scales)
    q_abs = W.make_q_abs(cfg)
    got, lse, err = fp8_decode(lib, cfg, d, codes.cpu().numpy(), scales.cpu().numpy(), q_abs)
    assert err == 0
    kr = oracle.rope_rows(oracle.bf16_to_f64(d["k_rope"]), d["tok_pos"])
    kr_bf16 = W.bf16_bits_to_f32(W.f32_to_bf16_bits(kr.astype(np.float32)))
    rows = np.concatenate([W.bf16_bits_to_f32(d["c_kv"]), kr_bf16], axis=1)
    oc, osc = oracle.quantize_rows(rows)
    ocodes = np.full((nb, 64, 576), 0x7F, np.uint8)
    oscales = np.full((nb, 64, 2), np.nan, np.float32)
    blk = d["block_table"][d["tok_seq"], d["tok_pos"] // 64]
    ocodes[blk, d["tok_pos"] % 64] = oc
    oscales[blk, d["tok_pos"] % 64] = osc
    ref, rlse = oracle.decode_latent_fp8_rows(ocodes, oscales, d["block_table"], d["seq_lens"], cfg.s,
                                              oracle.bf16_to_f64(q_abs))
    assert_parity(got, ref, what="fp8 end to end")
    np.testing.assert_allclose(lse, rlse, atol=1e-2, rtol=0)


def test_fp8_decode_is_bit_reproducible_and_page_order_free(lib):
    """Two runs give the same bits; the same cache laid out contiguously
    (identity block table) gives the same bits as the permuted pages."""
    cfg = CASES[3]
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    codes, scales = W.make_fp8_cache(cfg, d["block_table"], d["num_blocks"], d["tok_seq"], d["tok_pos"])
    q_abs = W.make_q_abs(cfg)
    a, la, _ = fp8_decode(lib, cfg, d, codes, scales, q_abs)
    b, lb, _ = fp8_decode(lib, cfg, d, codes, scales, q_abs)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    # the same logical cache with pages in logical order
    bt = d["block_table"]
    order = bt[bt >= 0]
    d2 = dict(d)
    ident = np.full_like(bt, -1)
    k = 0
    for s in range(bt.shape[0]):
        n = int((bt[s] >= 0).sum())
        ident[s, :n] = np.arange(k, k + n)
        k += n
    d2["block_table"] = ident
    c2 = np.full_like(codes, 0x7F)
    s2 = np.full_like(scales, np.nan)
    c2[:order.size] = codes[order]
    s2[:order.size] = scales[order]
    c, lc, _ = fp8_decode(lib, cfg, d2, c2, s2, q_abs)
    assert np.array_equal(a, c) and np.array_equal(la, lc)


def test_fp8_decode_bad_block_and_short_sequences(lib):
    import head_latent_attention_10_b200 as M
    cfg = CASES[0]
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    codes, scales = W.make_fp8_cache(cfg, d["block_table"], d["num_blocks"], d["tok_seq"], d["tok_pos"])
    q_abs = W.make_q_abs(cfg)
    good, glse, _ = fp8_decode(lib, cfg, d, codes, scales, q_abs)
    d2 = dict(d)
    bt = d["block_table"].copy()
    bt[0, 3] = d["num_blocks"] + 7
    d2["block_table"] = bt
    _, _, err = fp8_decode(lib, cfg, d2, codes, scales, q_abs)
    assert err & M.MLA_DEVERR_BLOCK_ID
    sl = d["seq_lens"].copy()
    sl[2] = 0
    got, lse, err = fp8_decode(lib, cfg, d, codes, scales, q_abs, seq_lens=sl)
    assert err & M.MLA_DEVERR_SEQ_LEN
    assert np.all(got[2] == 0) and np.all(np.isneginf(lse[2]))
    assert np.array_equal(got[:2], good[:2])


def test_fp8_decode_stall_hook_reports_a_timeout(lib):
    import head_latent_attention_10_b200 as M
    cfg = CASES[1]
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    codes, scales = W.make_fp8_cache(cfg, d["block_table"], d["num_blocks"], d["tok_seq"], d["tok_pos"])
    q_abs = W.make_q_abs(cfg)
    _, _, err = fp8_decode(lib, cfg, d, codes, scales, q_abs, flags=M.MLA_DEBUG_STALL)
    assert err & M.MLA_DEVERR_TIMEOUT
    # the context is still usable afterwards
    good, _, err = fp8_decode(lib, cfg, d, codes, scales, q_abs)
    assert err == 0 and np.isfinite(good).all()
