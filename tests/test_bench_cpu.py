"""Host logic of bench.py's N-GPU replica mode, run as world-size-2 gloo ranks
on the CPU: the per-rank workloads are independent batches of one shape, and
every rank ends with the max over ranks of its timings."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    import mla_workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        mine = [10.0 + rank, 3.0 - rank, 7.0 * (rank + 1)]
        got = bench.max_over_ranks(mine, world, "cpu")
        cfg = bench.replica_config(W.CONFIGS["tiny"], rank)
        d = W.make_decode_inputs(cfg, with_cache_pages=False)
        np.save(os.path.join(out_dir, f"q{rank}.npy"), d["q_nope"])
        np.save(os.path.join(out_dir, f"got{rank}.npy"), np.array(got + [cfg.B, cfg.H, cfg.s]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_max_and_draw_independent_batches(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    g0, g1 = np.load(tmp_path / "got0.npy"), np.load(tmp_path / "got1.npy")
    # max over ranks of [10+r, 3-r, 7(r+1)] = [11, 3, 14], the same on both ranks
    assert g0[:3].tolist() == [11.0, 3.0, 14.0]
    assert g1[:3].tolist() == g0[:3].tolist()
    # same shape on every rank, different values
    assert g0[3:].tolist() == g1[3:].tolist()
    q0, q1 = np.load(tmp_path / "q0.npy"), np.load(tmp_path / "q1.npy")
    assert q0.shape == q1.shape and not np.array_equal(q0, q1)


def test_single_rank_is_the_plain_workload():
    sys.path.insert(0, ROOT)
    import bench
    import mla_workloads as W
    cfg = W.CONFIGS["v2"]
    assert bench.replica_config(cfg, 0) is cfg
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]


def test_prefill_flop_count_matches_brute_force():
    """The prefill's algorithmic flops: visible (query, key) pairs counted one
    by one on small shapes, and the expansion over the padded rows."""
    import bench
    for B, s, L, H in [(1, 1, 1, 16), (2, 5, 9, 16), (1, 200, 520, 32), (3, 130, 130, 16)]:
        vis = sum(L - s + t + 1 for t in range(s))
        att, exp_ = bench.prefill_flops(B, s, L, H)
        assert att == 2.0 * B * H * vis * (192 + 128)
        lpad = -(-L // 128) * 128
        assert exp_ == 2.0 * 2 * B * lpad * H * 128 * 512
