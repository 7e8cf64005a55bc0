"""GPU parity of weight pre-absorption (mla_fold_weights, mla_absorb_q_folded,
mla_up_out_folded) against the oracle.

The folded weights are compared with the oracle's fp64 fold (their entries
are single dot products of length 128, rounded once to bf16: relative L2
<= 4e-3, about twice bf16's half-ulp); the folded steps are fed folded
weights the oracle computed and rounded to bf16 (never the GPU's), and held
to the decode's bar (assert_parity).  The end-to-end case checks that the
folded path on GPU-folded weights and the two-step path agree with the
oracle's two-step path on the same raw inputs.
"""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import assert_parity, host_bits, i32, rel_l2, torch_bits

pytestmark = pytest.mark.gpu

CASES = [
    W.MLAConfig("fold_h16", B=1, s=1, H=16, L=64, paged=False, seed=501, d_model=2048),
    W.MLAConfig("fold_h128", B=1, s=1, H=128, L=64, paged=False, seed=502, d_model=5120),
]


@pytest.fixture(scope="module")
def lib():
    import head_latent_attention_10_b200 as M
    M.load_library()
    return M


def _bf(x):
    """fp64 -> bf16 bits (through fp32, nearest-even)."""
    return W.f32_to_bf16_bits(np.asarray(x, np.float32))


def _f(t):
    return W.bf16_bits_to_f32(host_bits(t)).astype(np.float64)


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fold_weights_against_oracle(lib, cfg):
    import oracle
    import torch
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    qi = W.make_query_latent_inputs(cfg, T=4)
    w_o = W.make_w_o(cfg)
    dims = lib.dims(cfg.H)
    w_qk = torch.empty(cfg.H, 512, 1536, dtype=torch.bfloat16, device="cuda")
    w_ov = torch.empty(cfg.d_model, cfg.H * 512, dtype=torch.bfloat16, device="cuda")
    lib.mla_fold_weights(dims, torch_bits(qi["w_uq"]), torch_bits(d["w_uk"]), w_qk, torch_bits(w_o),
                         torch_bits(d["w_uv"]), w_ov)
    torch.cuda.synchronize()
    f = oracle.bf16_to_f64
    ref_qk = oracle.fold_qk(f(qi["w_uq"]), f(d["w_uk"]))
    got_qk = _f(w_qk)
    assert rel_l2(got_qk, ref_qk) <= 4e-3
    assert np.max(np.abs(got_qk - ref_qk)) <= 1e-2 * np.max(np.abs(ref_qk))
    ref_ov = oracle.fold_ov(f(w_o), f(d["w_uv"]))
    got_ov = _f(w_ov)
    assert rel_l2(got_ov, ref_ov) <= 4e-3
    assert np.max(np.abs(got_ov - ref_ov)) <= 1e-2 * np.max(np.abs(ref_ov))


@pytest.mark.parametrize("T", [1, 128, 300])
def test_absorb_q_folded_against_oracle(lib, T):
    import oracle
    import torch
    cfg = CASES[0]
    d = W.make_decode_inputs(cfg.with_(B=T, s=1, L=64), with_cache_pages=False)
    qi = W.make_query_latent_inputs(cfg, T=T)
    f = oracle.bf16_to_f64
    w_qk = _bf(oracle.fold_qk(f(qi["w_uq"]), f(d["w_uk"])))
    q_rope = d["q_rope"][:T]
    q_pos = d["q_pos"][:T]
    dims = lib.dims(cfg.H)
    q_abs = torch.empty(T, cfg.H, 576, dtype=torch.bfloat16, device="cuda")
    lib.mla_absorb_q_folded(dims, torch_bits(qi["c_q"]), torch_bits(q_rope), i32(q_pos), torch_bits(w_qk), q_abs)
    torch.cuda.synchronize()
    ref = oracle.absorb_q_folded(f(qi["c_q"]), f(q_rope), f(w_qk), q_pos=q_pos)
    assert_parity(_f(q_abs), ref, what=f"absorb_q_folded T={T}")


@pytest.mark.parametrize("T", [1, 128, 300])
def test_up_out_folded_against_oracle(lib, T):
    import oracle
    import torch
    cfg = CASES[0]
    lat = W.make_latent(cfg.with_(B=T, s=1))
    w_o = W.make_w_o(cfg)
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    f = oracle.bf16_to_f64
    w_ov = _bf(oracle.fold_ov(f(w_o), f(d["w_uv"])))
    dims = lib.dims(cfg.H)
    out = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device="cuda")
    lib.mla_up_out_folded(dims, torch_bits(lat), torch_bits(w_ov), out)
    torch.cuda.synchronize()
    ref = oracle.up_out_folded(f(lat), f(w_ov))
    assert_parity(_f(out), ref, what=f"up_out_folded T={T}")


def test_folded_and_two_step_paths_agree_end_to_end(lib):
    """GPU fold -> folded absorb and folded output projection, against the
    oracle's two-step path (absorb_q of W^UQ c^Q; out_proj of up_v) on the
    same raw weights and inputs."""
    import oracle
    import torch
    cfg = CASES[1]
    T = 128
    d = W.make_decode_inputs(cfg, with_cache_pages=False)
    qi = W.make_query_latent_inputs(cfg, T=T)
    w_o = W.make_w_o(cfg)
    lat = W.make_latent(cfg.with_(B=T, s=1))
    dims = lib.dims(cfg.H)
    w_qk = torch.empty(cfg.H, 512, 1536, dtype=torch.bfloat16, device="cuda")
    w_ov = torch.empty(cfg.d_model, cfg.H * 512, dtype=torch.bfloat16, device="cuda")
    lib.mla_fold_weights(dims, torch_bits(qi["w_uq"]), torch_bits(d["w_uk"]), w_qk, torch_bits(w_o),
                         torch_bits(d["w_uv"]), w_ov)
    q_pos = np.arange(T, dtype=np.int32) * 7
    q_rope = np.ascontiguousarray(np.resize(d["q_rope"], (T, cfg.H, 64)))
    q_abs = torch.empty(T, cfg.H, 576, dtype=torch.bfloat16, device="cuda")
    lib.mla_absorb_q_folded(dims, torch_bits(qi["c_q"]), torch_bits(q_rope), i32(q_pos), w_qk, q_abs)
    out = torch.empty(T, cfg.d_model, dtype=torch.bfloat16, device="cuda")
    lib.mla_up_out_folded(dims, torch_bits(lat), w_ov, out)
    torch.cuda.synchronize()
    f = oracle.bf16_to_f64
    q_c = np.einsum("ikq,tq->tik", f(qi["w_uq"]), f(qi["c_q"]))
    ref_q = oracle.absorb_q(q_c, f(q_rope), f(d["w_uk"]), q_pos=q_pos)
    assert_parity(_f(q_abs), ref_q, what="folded absorb vs two-step oracle")
    ref_u = oracle.out_proj(oracle.up_v(f(lat), f(d["w_uv"])), f(w_o))
    assert_parity(_f(out), ref_u, what="folded output projection vs two-step oracle")
