"""Parity at the full workload sizes, in the launch configuration bench.py
times.  Each whole batch is decoded on the GPU.  The oracle, which cannot
afford every output, checks a sample of (row, head) outputs:
- the latent output and lse of each sampled pair, in the absorbed fp64 form;
- the per-head output o = U^V latent, in the textbook expanded fp64 form, for
  a few pairs.  The long-context batch is left out of this part: each pair
  there costs tens of GFLOP in fp64.
The sample always holds the shortest and the longest sequence (see
mla_workloads.sample_pairs)."""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits

pytestmark = pytest.mark.gpu

FULL = ["v2lite", "v2", "longctx", "mtp"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_decode_on_sampled_outputs(name):
    import head_latent_attention_10_b200 as M
    import oracle
    M.load_library()
    cfg = W.CONFIGS[name]
    g = GpuWorkload(cfg)
    q_abs = g.absorb()
    lat, lse = g.decode(q_abs, flags=M.MLA_SYNC_CHECK)
    d = g.d
    rows, heads = W.sample_pairs(cfg, d["seq_lens"], n_rows=3, n_heads=6)
    ref, rlse = oracle.decode_latent(d["cache"], d["block_table"], d["seq_lens"], cfg.s,
                                     oracle.bf16_to_f64(host_bits(q_abs)), rows=rows, heads=heads)
    got = W.bf16_bits_to_f32(host_bits(lat))[rows, heads]
    assert_parity(got, ref, what=f"{name} latent")
    np.testing.assert_allclose(lse.cpu().numpy()[rows, heads], rlse, atol=1e-2, rtol=0)
    if name == "longctx":
        return
    o = W.bf16_bits_to_f32(host_bits(g.up_v(lat)))
    r2, h2 = W.sample_pairs(cfg, d["seq_lens"], n_rows=2, n_heads=2, seed=11)
    f = oracle.bf16_to_f64
    want, _, _ = oracle.decode_expanded(d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]),
                                        f(d["q_rope"]), f(d["w_uk"]), f(d["w_uv"]), q_pos=d["q_pos"],
                                        rows=r2, heads=h2)
    assert_parity(o[r2, h2], want, what=f"{name} per-head output")
