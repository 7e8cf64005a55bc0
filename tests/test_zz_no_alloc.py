"""mla_decode_noalloc: the decode on the library's own per-device scratch
array must give the same bits as mla_decode with a caller workspace, on two
different calls in a row (the second call finds the first call's plan and
partials in the scratch and must not depend on them).  Named so that it is
collected last; it also passes on its own."""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits

pytestmark = pytest.mark.gpu

CASES = [
    W.MLAConfig("na_h128", B=3, s=1, H=128, L=0, paged=True, seed=301, d_model=5120,
                seq_lens=(900, 130, 17)),
    W.MLAConfig("na_h16_two_queries", B=4, s=2, H=16, L=0, paged=True, seed=302, d_model=2048,
                seq_lens=(2, 700, 1400, 65)),
]


def _noalloc(M, w, q_abs, flags):
    import torch
    cfg = w.cfg
    lat = torch.empty(cfg.T, cfg.H, cfg.d_c, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
    M.mla_decode_noalloc(w.dims, q_abs, w.cache, w.block_table, w.seq_lens, cfg.s, lat, lse, flags=flags)
    return lat, lse


@pytest.mark.parametrize("flags", [0, 2], ids=["tensor_core", "simple"])
def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row(flags):
    import torch
    import head_latent_attention_10_b200 as M
    import oracle
    M.load_library()
    loads = [GpuWorkload(c) for c in CASES]
    for w in loads:                     # two different calls in a row, then the first again
        q_abs = w.absorb()
        ref_lat, ref_lse = w.decode(q_abs, flags=flags | M.MLA_SYNC_CHECK)
        lat, lse = _noalloc(M, w, q_abs, flags | M.MLA_SYNC_CHECK)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(lat), host_bits(ref_lat)), w.cfg.name
        assert np.array_equal(lse.cpu().numpy().view(np.uint32), ref_lse.cpu().numpy().view(np.uint32))
    w = loads[0]
    q_abs = w.absorb()
    lat, _ = _noalloc(M, w, q_abs, flags)
    torch.cuda.synchronize()
    # and the result is the method's: the absorbed fp64 oracle on the same bf16 inputs
    d = w.d
    want, _ = oracle.decode_latent(d["cache"], d["block_table"], d["seq_lens"], w.cfg.s,
                                   oracle.bf16_to_f64(host_bits(q_abs)))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(want.shape)
    assert_parity(got, want, what="noalloc latent")


def test_noalloc_rejects_a_shape_beyond_its_scratch():
    import torch
    import head_latent_attention_10_b200 as M
    M.load_library()
    w = GpuWorkload(CASES[0])
    q_abs = w.absorb()
    # the CUDA-core path keeps per-split partials for every query row: 5000 rows
    # of a 128-head batch at 64K context need far more than the scratch holds
    bt = torch.zeros(5000, 1024, dtype=torch.int32, device="cuda")
    sl = torch.ones(5000, dtype=torch.int32, device="cuda")
    lat = torch.empty(5000, 128, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MLAError) as e:
        M.mla_decode_noalloc(w.dims, q_abs, w.cache, bt, sl, 1, lat, None, flags=M.MLA_FORCE_SIMPLE)
    assert "WORKSPACE" in str(e.value)


def test_noalloc_rejects_a_tensor_core_shape_beyond_its_scratch_before_any_launch():
    """The tensor-core path's partials grow with s*H: 200 query tokens of 128
    heads form 400 row groups, one range each, and their 51,200 partial rows
    (105 MB) exceed the 40 MB array.  The call must refuse before launching."""
    import torch
    import head_latent_attention_10_b200 as M
    M.load_library()
    w = GpuWorkload(CASES[0])
    s = 200
    q_abs = torch.zeros(s, 128, 576, dtype=torch.bfloat16, device="cuda")
    lat = torch.empty(s, 128, 512, dtype=torch.bfloat16, device="cuda")
    sl = torch.full((1,), 900, dtype=torch.int32, device="cuda")
    bt = w.block_table[:1].contiguous()
    torch.cuda.synchronize()
    n0 = M.mla_kernel_launches()
    with pytest.raises(M.MLAError) as e:
        M.mla_decode_noalloc(w.dims, q_abs, w.cache, bt, sl, s, lat, None)
    assert "WORKSPACE" in str(e.value)
    assert M.mla_kernel_launches() == n0
