"""Failure detection without a GPU fault: every wait in the decode kernel is
bounded.  The test hook flag MLA_DEBUG_STALL makes each CTA skip the page
load of its first tile (a barrier that nothing completes) and cuts the bound
to 20 ms.  The kernel must record
MLA_DEVERR_TIMEOUT in the workspace error word, unwind (its copies in flight
drained, its TMEM freed) and leave the context usable: the next call,
without the hook, must return the right answer."""
import numpy as np
import pytest

import mla_workloads as W
from _gpu_setup import GpuWorkload, assert_parity, host_bits

pytestmark = pytest.mark.gpu

CFG = W.MLAConfig("timeout", B=3, s=1, H=128, L=0, paged=True, seed=601, d_model=5120,
                  seq_lens=(700, 129, 63))


def test_wait_bound_reports_timeout_and_context_survives():
    import head_latent_attention_10_b200 as M
    import oracle
    M.load_library()
    g = GpuWorkload(CFG)
    q_abs = g.absorb()
    with pytest.raises(M.MLAError) as e:
        g.decode(q_abs, flags=M.MLA_SYNC_CHECK | M.MLA_DEBUG_STALL)
    assert e.value.status == M.MLA_ERR_DEVICE
    assert M.mla_decode_error(g.ws, clear=True) & M.MLA_DEVERR_TIMEOUT
    lat, _ = g.decode(q_abs, flags=M.MLA_SYNC_CHECK)
    d = g.d
    want, _ = oracle.decode_latent(d["cache"], d["block_table"], d["seq_lens"], CFG.s,
                                   oracle.bf16_to_f64(host_bits(q_abs)))
    got = W.bf16_bits_to_f32(host_bits(lat)).reshape(want.shape)
    assert_parity(got, want, what="after a timed-out call")
