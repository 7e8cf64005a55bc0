"""Benchmark: one MLA decode step of the whole hot path on synthetic inputs.

A step = append the newest latent of every sequence from its hidden state
(mla_append_cache) -> absorb U^K into the queries (mla_absorb_q) -> attention
over the paged latent cache with split-KV combine (mla_decode) -> U^V
up-projection (mla_up_v).  Default workload: the DeepSeek-V2-shaped decode
batch (B=128 sequences, 1 query token each, H=128 heads, L=4096, d_c=512,
d_r=64, 64-token paged cache with a random block table), bf16 storage with
fp32 accumulation.  Every rank (one per GPU) runs its own copy of the batch:
sequences are independent, so there is no collective (weak scaling).

Prints one JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
on the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mla_workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), tc=float(d["bf16_tflops"]),
                    tc_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, source="fallback")


def algorithmic(cfg: W.MLAConfig, seq_lens: np.ndarray, max_blocks: int):
    """Bytes and FLOPs one mla_decode call must move and compute.
    Bytes: visible cache rows (1152 B/token, read once for all heads), the
    absorbed queries, the latent outputs and lse, the block table and lengths.
    FLOPs: 2*(576 + 512) per (head, query, visible key)."""
    s = cfg.s
    vis = sum(max(0, int(L) - s + t + 1) for L in seq_lens for t in range(s))
    # a sequence's cache rows are read once even with several queries
    rows_read = int(np.sum(seq_lens))
    D = cfg.d_c + cfg.d_r
    byts = rows_read * D * 2 + cfg.T * cfg.H * D * 2 + cfg.T * cfg.H * (cfg.d_c * 2 + 4) \
        + cfg.B * max_blocks * 4 + cfg.B * 4
    flops = 2 * (D + cfg.d_c) * cfg.H * vis
    return byts, flops, rows_read


def algorithmic_fp8(cfg: W.MLAConfig, seq_lens: np.ndarray, max_blocks: int):
    """As `algorithmic`, for the FP8 cache: a cache row is 576 one-byte codes
    plus two fp32 scales (584 B/token)."""
    byts, flops, rows_read = algorithmic(cfg, seq_lens, max_blocks)
    D = cfg.d_c + cfg.d_r
    return byts - rows_read * D * 2 + rows_read * (D + 8), flops, rows_read


# DRAM bytes (read + write) the current decode kernel moves per cache token,
# from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of
# tc_decode64_kernel on the V2-shaped batch cut to 32 sequences (157.7 MB read
# + 7.5 MB written for 131,072 tokens).  Set to None whenever the decode kernel
# changes.
DECODE_DRAM_BYTES_PER_TOKEN = (157.684992e6 + 7.459840e6) / (32 * 4096)


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------ replicas (N GPUs)
def replica_config(cfg: W.MLAConfig, rank: int) -> W.MLAConfig:
    """Rank r times its own batch of the same shape: independent sequences,
    drawn from a seed of its own (rank 0 keeps the single-GPU workload)."""
    if rank == 0:
        return cfg
    return cfg.with_(seed=cfg.seed + 7919 * rank)


def max_over_ranks(vals, world: int, device: str):
    """Every rank gets the element-wise max of `vals` over all ranks (a job
    is as slow as its slowest replica).  One collective, same on every rank."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


# -------------------------------------------------------------- our arm
class Step:
    """Device-resident workload plus the four library calls of one step."""

    def __init__(self, cfg: W.MLAConfig, dev: int, flags: int):
        import torch
        import head_latent_attention_10_b200 as M
        self.M, self.torch, self.cfg, self.flags = M, torch, cfg, flags
        M.load_library()
        torch.cuda.set_device(dev)
        d = W.make_decode_inputs(cfg, with_cache_pages=False)
        self.seq_lens_np = d["seq_lens"]
        self.max_blocks = d["block_table"].shape[1]
        cu = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        self.dims = M.dims(cfg.H)
        self.block_table = cu(d["block_table"])
        self.seq_lens = cu(d["seq_lens"])
        D = cfg.d_c + cfg.d_r
        self.cache = torch.full((d["num_blocks"], cfg.block_size, D), float("nan"),
                                dtype=torch.bfloat16, device="cuda")
        N, chunk = d["tok_seq"].size, 1 << 20
        for a in range(0, N, chunk):
            b = min(N, a + chunk)
            M.mla_append_latent(self.dims, bf(d["c_kv"][a:b]), bf(d["k_rope"][a:b]), cu(d["tok_seq"][a:b]),
                                cu(d["tok_pos"][a:b]), self.block_table, self.cache)
        del d["c_kv"], d["k_rope"]
        self.w_uk, self.w_uv = bf(d["w_uk"]), bf(d["w_uv"])
        a = W.make_append_inputs(cfg, cfg.T)
        self.w_dkv, self.w_kr = bf(a["w_dkv"]), bf(a["w_kr"])
        # per-step inputs: new hidden states, their slots (the newest s
        # positions of each sequence), and the queries
        T = cfg.T
        t = np.tile(np.arange(cfg.s), cfg.B)
        app_pos = (np.repeat(d["seq_lens"], cfg.s) - cfg.s + t).astype(np.int32)
        self.host = dict(h=a["h"], q_nope=d["q_nope"], q_rope=d["q_rope"], q_pos=d["q_pos"],
                         app_seq=np.repeat(np.arange(cfg.B, dtype=np.int32), cfg.s), app_pos=app_pos)
        self.dev = {k: (bf(v) if v.dtype == np.uint16 else cu(v)) for k, v in self.host.items()}
        self.q_abs = torch.empty(T, cfg.H, D, dtype=torch.bfloat16, device="cuda")
        self.lat = torch.empty(T, cfg.H, cfg.d_c, dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty(T, cfg.H, dtype=torch.float32, device="cuda")
        self.out = torch.empty(T, cfg.H, cfg.d_h, dtype=torch.bfloat16, device="cuda")
        self.ws = torch.empty(M.mla_decode_workspace_size(self.dims, cfg.B, cfg.s, self.max_blocks * 64),
                              dtype=torch.uint8, device="cuda")
        self.stream = torch.cuda.current_stream()
        # the append and the absorption are independent: the absorption runs
        # on a side stream, forked from and joined back into the main one
        self.side = torch.cuda.Stream()
        self.ev_fork, self.ev_join = torch.cuda.Event(), torch.cuda.Event()
        torch.cuda.synchronize()

    def run(self, inp=None, dec_events=None, out=None, serial_events=None):
        """One step.  With `serial_events` (five events) every call runs on the
        main stream, one after the other, with an event between calls."""
        M, x = self.M, (inp if inp is not None else self.dev)
        main = self.torch.cuda.current_stream()
        ev = serial_events
        if ev is not None:
            ev[0].record(main)
            M.mla_append_cache(self.dims, x["h"], self.w_dkv, self.w_kr, x["app_seq"], x["app_pos"],
                               self.block_table, self.cache)
            ev[1].record(main)
            M.mla_absorb_q(self.dims, x["q_nope"], x["q_rope"], x["q_pos"], self.w_uk, self.q_abs)
            ev[2].record(main)
        else:
            self.ev_fork.record(main)
            self.side.wait_event(self.ev_fork)
            with self.torch.cuda.stream(self.side):
                M.mla_absorb_q(self.dims, x["q_nope"], x["q_rope"], x["q_pos"], self.w_uk, self.q_abs)
                self.ev_join.record(self.side)
            M.mla_append_cache(self.dims, x["h"], self.w_dkv, self.w_kr, x["app_seq"], x["app_pos"],
                               self.block_table, self.cache)
            main.wait_event(self.ev_join)
        if dec_events is not None:
            dec_events[0].record(main)
        M.mla_decode(self.dims, self.q_abs, self.cache, self.block_table, self.seq_lens, self.cfg.s,
                     self.lat, self.lse, self.ws, flags=self.flags)
        if dec_events is not None:
            dec_events[1].record(main)
        if ev is not None:
            ev[3].record(main)
        M.mla_up_v(self.dims, self.lat, self.w_uv, self.out if out is None else out)
        if ev is not None:
            ev[4].record(main)


def run_ours(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    cfg = W.CONFIGS[args.config]
    if args.batch:
        cfg = cfg.with_(B=args.batch, describe=cfg.describe + f" (batch cut to {args.batch})")
    import head_latent_attention_10_b200 as M
    st = Step(replica_config(cfg, rank), local, flags=(M.MLA_FORCE_SIMPLE if args.simple else 0))
    E = torch.cuda.Event

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # --- device-resident timing (inputs already in HBM)
    for _ in range(args.warmup):
        st.run()
    barrier()
    # One step captured as a CUDA graph (the same library calls, kernels and
    # arguments; replays save the launch gaps between the step's kernels).
    graph, per_step, launch_mode = None, 0, "stream"
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            c0 = M.mla_kernel_launches()
            with torch.cuda.graph(g):
                st.run()
            per_step = M.mla_kernel_launches() - c0
            for _ in range(args.warmup):
                g.replay()
            graph, launch_mode = g, "cuda graph of one step"
        except Exception as e:  # capture unsupported here: time the stream launches
            launch_mode = f"stream (graph capture failed: {type(e).__name__})"
            torch.cuda.synchronize()
    barrier()
    clock = ClockSampler(local)
    clock.start()
    time.sleep(0.3)
    barrier()
    l0 = M.mla_kernel_launches()
    t0, t1 = E(enable_timing=True), E(enable_timing=True)
    t0.record()
    for k in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            st.run()
    t1.record()
    barrier()
    launches = per_step * args.steps if graph is not None else M.mla_kernel_launches() - l0
    clocks = clock.stop()
    ms = t0.elapsed_time(t1) / args.steps
    # the decode call alone (plan + decode + combine), stream-launched, events
    # on the launching stream around each call
    n_dec = min(args.steps, 200)
    dec = [(E(enable_timing=True), E(enable_timing=True)) for _ in range(n_dec)]
    for k in range(n_dec):
        st.run(dec_events=dec[k])
    barrier()
    dec_ms = float(np.mean([a.elapsed_time(b) for a, b in dec]))
    # the same calls one after the other on one stream, timed call by call
    ser = [[E(enable_timing=True) for _ in range(5)] for _ in range(n_dec)]
    for k in range(n_dec):
        st.run(serial_events=ser[k])
    barrier()
    parts = [float(np.mean([e[i].elapsed_time(e[i + 1]) for e in ser])) for i in range(4)]
    ms, dec_ms = max_over_ranks([ms, dec_ms], world, "cuda")
    parts = max_over_ranks(parts, world, "cuda")
    if graph is not None:
        del graph
        barrier()

    # --- end to end: pinned host inputs copied in and the output copied out,
    # every step.  Steps are pipelined over two input and two output buffers:
    # step i+1's inputs cross PCIe (h2d stream) while step i computes, and step
    # i's result comes back (d2h stream) while step i+1 computes.
    pin = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16 else v)
           .pin_memory() for k, v in st.host.items()}
    out_host = [torch.empty(st.out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    stage = [{k: torch.empty_like(v) for k, v in st.dev.items()} for _ in range(2)]
    out_dev = [torch.empty_like(st.out) for _ in range(2)]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [E() for _ in range(2)]
    ev_done = [E() for _ in range(2)]
    ev_out = [E() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(ev_done[b])      # step i-2 has read stage[b]
            with torch.cuda.stream(s_in):
                for k, v in pin.items():
                    dst = stage[b][k]
                    dst.view(torch.int16 if dst.dtype == torch.bfloat16 else dst.dtype).copy_(v, non_blocking=True)
                ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_out[b])       # step i-2's result has left out_dev[b]
            st.run(stage[b], out=out_dev[b])
            ev_done[b].record(comp)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
                ev_out[b].record(s_out)
        for b in range(min(n, 2)):
            comp.wait_event(ev_out[b])

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = E(enable_timing=True), E(enable_timing=True)
    e0.record()
    e2e_steps(args.steps)
    e1.record()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    e2e_ms, = max_over_ranks([e2e_ms], world, "cuda")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    tok = cfg.T * world
    byts, flops, rows = algorithmic(cfg, st.seq_lens_np, st.max_blocks)
    pk = peaks()
    hbm_t, tc_t = byts / (pk["hbm"] * 1e9), flops / (pk["tc"] * 1e12)
    bound = "hbm" if hbm_t >= tc_t else "tensor"
    dec_s = dec_ms / 1e3
    if bound == "hbm":
        achieved, peak, unit = byts / dec_s / 1e9, pk["hbm"], "GB/s"
    else:
        achieved, peak, unit = flops / dec_s / 1e12, pk["tc"], "TFLOP/s"
    line = {
        "metric": "MLA decode tokens/s, latent-cache GB/s & TFLOP/s (H=128,B=128,L=4K) vs roofline",
        "value": tok / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, N(0,1) latents/queries, "
        "N(0,1/512) up-projections, random block table)",
        "config": {"workload": cfg.describe, "B": cfg.B, "s": cfg.s, "H": cfg.H,
                   "L": cfg.L if not isinstance(cfg.L, tuple) else list(cfg.L),
                   "d_c": cfg.d_c, "d_r": cfg.d_r, "d_h": cfg.d_h, "block_size": cfg.block_size,
                   "parallelism": f"replicas x{world} (independent sequences, no collective)",
                   "l2": "inputs larger than L2 (%.0f MB of cache read per step)" % (rows * 1152 / 1e6),
                   "decode_path": "simple" if args.simple else "default",
                   "launch": launch_mode,
                   "decode_ctas": M.mla_decode_ctas(st.dims, cfg.s)},
        "decode": {"ms": dec_ms, "cache_gbs": rows * 1152 / dec_s / 1e9, "bytes": byts,
                   "gbs": byts / dec_s / 1e9, "flops": flops, "tflops": flops / dec_s / 1e12,
                   "roofline_us": max(hbm_t, tc_t) * 1e6,
                   "roofline_frac": max(hbm_t, tc_t) / dec_s},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "traffic": (DECODE_DRAM_BYTES_PER_TOKEN * rows
                                 if (cfg.name == "v2" and not args.simple and DECODE_DRAM_BYTES_PER_TOKEN)
                                 else None),
                     "peak_source": pk["source"] + (" burst" if bound == "tensor" else "")},
        "step_calls_us": {"note": "each call timed on its own (stream launches, one after the other); "
                                  "the timed step overlaps the append with the absorption on a side stream",
                          "append": parts[0] * 1e3, "absorb": parts[1] * 1e3, "decode": parts[2] * 1e3,
                          "up_v": parts[3] * 1e3},
        "e2e": {"value": tok / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if not args.no_per_config and world == 1:
        line["per_config"] = per_config(M, [n for n in ("tiny", "v2lite", "v2", "longctx", "mtp")])
        line["per_config_fp8"] = per_config(M, [n for n in ("v2lite", "v2", "longctx", "mtp")], fp8=True)
    if not args.no_prefill and world == 1:
        line["prefill"] = prefill_bench(M)
        line["folded_weights"] = fold_bench(M)
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------- every config's decode
def per_config(M, names, iters=30, fp8=False):
    """The decode call (plan + decode + combine) on each named workload: its
    CUDA-event time on the launching stream (mean of `iters` back-to-back
    calls after 3 warm-ups), latent-cache GB/s, TFLOP/s and roofline
    fraction.  Inputs are generated on the device (seeded torch draws with
    the workloads' distributions: cache and RoPE query N(0,1), absorbed
    latent query N(0,1/4), a random block permutation, the workload's own
    sequence lengths); timing does not depend on their values.  Workloads
    whose cache fits in L2 are timed with a 256 MB L2 flush before each call
    and also warm (no flush).  `graph_us` is the same call captured once as a
    CUDA graph and replayed (the flush, if any, outside the timed replay)."""
    import torch
    out = {}
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    E = torch.cuda.Event
    for name in names:
        cfg = W.CONFIGS[name]
        sl = W.seq_lens_of(cfg)
        table, nphys, _ = W.paging(cfg, sl)
        g = torch.Generator(device="cuda")
        g.manual_seed(cfg.seed)
        D = cfg.d_c + cfg.d_r
        if fp8:
            # E4M3 bit patterns with a random sign, exponent field 5..9 and
            # mantissa (no NaN code), scales uniform in [0.1, 0.3]
            bits = torch.randint(0, 1 << 30, (nphys, cfg.block_size, D), generator=g, device="cuda")
            codes = ((bits & 0x80) | (((bits >> 8) % 5 + 5) << 3) | ((bits >> 16) & 7)).to(torch.uint8)
            scales = torch.rand((nphys, cfg.block_size, 2), generator=g, device="cuda") * 0.2 + 0.1
            cache = None
        else:
            cache = torch.randn((nphys, cfg.block_size, D), generator=g, device="cuda").to(torch.bfloat16)
        q = torch.randn((cfg.T, cfg.H, D), generator=g, device="cuda")
        q[..., :cfg.d_c] *= 0.5
        q = q.to(torch.bfloat16)
        bt = torch.from_numpy(table).cuda()
        slt = torch.from_numpy(sl).cuda()
        dims = M.dims(cfg.H)
        lat = torch.empty(cfg.T, cfg.H, cfg.d_c, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
        ws = torch.empty(M.mla_decode_workspace_size(dims, cfg.B, cfg.s, table.shape[1] * 64),
                         dtype=torch.uint8, device="cuda")
        if fp8:
            call = lambda: M.mla_decode_fp8(dims, q, codes, scales, bt, slt, cfg.s, lat, lse, ws)
            byts, flops, rows = algorithmic_fp8(cfg, sl, table.shape[1])
            row_bytes = 584
        else:
            call = lambda: M.mla_decode(dims, q, cache, bt, slt, cfg.s, lat, lse, ws)
            byts, flops, rows = algorithmic(cfg, sl, table.shape[1])
            row_bytes = 1152
        small = rows * row_bytes < L2_BYTES
        for _ in range(3):
            call()
        torch.cuda.synchronize()

        def timed(do_flush):
            ts = []
            for _ in range(iters):
                if do_flush:
                    flush.fill_(1)
                a, b = E(enable_timing=True), E(enable_timing=True)
                a.record()
                call()
                b.record()
                ts.append((a, b))
            torch.cuda.synchronize()
            return float(np.mean([x.elapsed_time(y) for x, y in ts])) / 1e3

        t = timed(small)
        hbm_t, tc_t = byts / (pk["hbm"] * 1e9), flops / (pk["tc"] * 1e12)
        r = {"workload": cfg.describe + (" (FP8 E4M3 cache)" if fp8 else ""), "us": t * 1e6,
             "cache_gbs": rows * row_bytes / t / 1e9,
             "gbs": byts / t / 1e9, "tflops": flops / t / 1e12,
             "bound": "hbm" if hbm_t >= tc_t else "tensor", "roofline_us": max(hbm_t, tc_t) * 1e6,
             "roofline_frac": max(hbm_t, tc_t) / t, "decode_ctas": M.mla_decode_ctas(dims, cfg.s),
             "l2": "flushed before each call" if small else "cache larger than L2"}
        if small:
            r["warm_l2_us"] = timed(False) * 1e6
        # the same call captured once as a CUDA graph and replayed, as a
        # serving loop would run it: on the small batches the eager time above
        # is mostly the host's launch cost
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            call()
            side.synchronize()
            with torch.cuda.graph(graph, stream=side):
                call()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        gts = []
        for _ in range(iters):
            if small:
                flush.fill_(1)
            a, b = E(enable_timing=True), E(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            gts.append((a, b))
        torch.cuda.synchronize()
        r["graph_us"] = float(np.mean([x.elapsed_time(y) for x, y in gts])) * 1e3
        del graph
        out[name] = r
        del cache, q, lat, lse, ws, bt, slt
        if fp8:
            del codes, scales
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------ expanded-form prefill
PREFILL_WORKLOADS = {
    "prompt4k": dict(B=1, s=4096, L=4096, H=128, seed=2001,
                     describe="DeepSeek-V2-shaped prompt prefill: B=1, s=L=4096, H=128"),
    "chunk1k_ctx8k": dict(B=1, s=1024, L=8192, H=128, seed=2002,
                          describe="chunked prefill: the last 1024 of 8192 tokens, H=128"),
    "v2lite_prompt4k": dict(B=4, s=4096, L=4096, H=16, seed=2003,
                            describe="DeepSeek-V2-Lite-shaped prompt prefill: B=4, s=L=4096, H=16"),
}


def prefill_flops(B, s, L, H, d_c=512, d_r=64, d_h=128):
    """(attention, expansion) flops of one mla_prefill call: 2 (d_h + d_r)
    for the logit and 2 d_h for the weighted sum per visible (query, key,
    head); 2 d_h d_c per row and head for each of K^C and V^C over the
    call's B * round_up(L, 128) expanded rows."""
    vis = s * (L - s) + s * (s + 1) // 2
    att = 2.0 * B * H * vis * ((d_h + d_r) + d_h)
    lpad = (L + 127) // 128 * 128
    exp_ = 2.0 * 2.0 * B * lpad * H * d_h * d_c
    return att, exp_


def prefill_bench(M, names=tuple(PREFILL_WORKLOADS), iters=10):
    """mla_prefill on each workload: CUDA-event time of the whole call
    (gather + two expansion GEMMs + attention; mean of `iters` calls after 3
    warm-ups, each call preceded by a 256 MB L2 flush), its TFLOP/s and the
    fraction of the measured dense bf16 peak (the call is tensor-bound).
    Inputs are seeded torch draws on the device with the workloads'
    distributions (cache, q^C, q^R N(0,1); U^K, U^V N(0,1/512)); the cache
    is paged through a random block permutation."""
    import torch
    out = {}
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    E = torch.cuda.Event
    for name in names:
        w = PREFILL_WORKLOADS[name]
        B, s, L, H = w["B"], w["s"], w["L"], w["H"]
        g = torch.Generator(device="cuda")
        g.manual_seed(w["seed"])
        nblk = (L + 63) // 64
        nphys = B * nblk
        cache = torch.randn((nphys, 64, 576), generator=g, device="cuda").to(torch.bfloat16)
        bt = torch.randperm(nphys, generator=g, device="cuda").to(torch.int32).view(B, nblk).contiguous()
        sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
        q_nope = torch.randn((B * s, H, 128), generator=g, device="cuda").to(torch.bfloat16)
        q_rope = torch.randn((B * s, H, 64), generator=g, device="cuda").to(torch.bfloat16)
        q_pos = (torch.arange(s, dtype=torch.int32, device="cuda") + (L - s)).repeat(B).contiguous()
        w_uk = (torch.randn((H, 128, 512), generator=g, device="cuda") * 512 ** -0.5).to(torch.bfloat16)
        w_uv = (torch.randn((H, 128, 512), generator=g, device="cuda") * 512 ** -0.5).to(torch.bfloat16)
        dims = M.dims(H)
        o = torch.empty((B * s, H, 128), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B * s, H), dtype=torch.float32, device="cuda")
        ws = torch.empty(M.mla_prefill_workspace_size(dims, B, s, L), dtype=torch.uint8, device="cuda")
        call = lambda: M.mla_prefill(dims, q_nope, q_rope, q_pos, w_uk, w_uv, cache, bt, sl, s, L, o, lse, ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        n0 = M.mla_kernel_launches()
        ts = []
        for _ in range(iters):
            flush.fill_(1)
            a, b = E(enable_timing=True), E(enable_timing=True)
            a.record()
            call()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        launches = (M.mla_kernel_launches() - n0) // iters
        t = float(np.mean([x.elapsed_time(y) for x, y in ts])) / 1e3
        att, exp_ = prefill_flops(B, s, L, H)
        achieved = (att + exp_) / t / 1e12
        out[name] = {"workload": w["describe"], "us": t * 1e6, "tokens_per_s": B * s / t,
                     "attention_gflop": att / 1e9, "expansion_gflop": exp_ / 1e9, "tflops": achieved,
                     "bound": "tensor", "peak_tflops": pk["tc"], "roofline_frac": achieved / pk["tc"],
                     "launches_per_call": int(launches), "l2": "flushed before each call",
                     "error_word": M.mla_decode_error(ws)}
        del cache, bt, sl, q_nope, q_rope, q_pos, w_uk, w_uv, o, lse, ws
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------- weight pre-absorption
def fold_bench(M, T=128, H=128, d_q=1536, d_model=5120, iters=20):
    """The query absorption and output projection of one decode step of the
    V2 shape (T tokens), two-step (mla_absorb_q from q^C, mla_up_v with W^O)
    against folded (mla_absorb_q_folded from c^Q, mla_up_out_folded), each
    call's CUDA-event time (mean of `iters` after 3 warm-ups, 256 MB L2 flush
    before each call) and the weight bytes it reads.  The two-step absorb
    takes q^C as given, so its time leaves out the W^UQ projection that
    produces q^C (a further 50 MB of weights at this shape)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(3001)
    dev = dict(device="cuda")
    rnd = lambda *shape, std=1.0: (torch.randn(shape, generator=g, **dev) * std).to(torch.bfloat16)
    dims = M.dims(H)
    c_q, q_c, q_r = rnd(T, d_q), rnd(T, H, 128), rnd(T, H, 64)
    q_pos = torch.arange(T, dtype=torch.int32, **dev)
    w_uq, w_uk, w_uv = rnd(H, 128, d_q, std=d_q ** -0.5), rnd(H, 128, 512, std=512 ** -0.5), rnd(H, 128, 512, std=512 ** -0.5)
    w_o = rnd(d_model, H * 128, std=(H * 128) ** -0.5)
    w_qk = torch.empty(H, 512, d_q, dtype=torch.bfloat16, **dev)
    w_ov = torch.empty(d_model, H * 512, dtype=torch.bfloat16, **dev)
    M.mla_fold_weights(dims, w_uq, w_uk, w_qk, w_o, w_uv, w_ov)
    lat = rnd(T, H, 512, std=0.125)
    q_abs = torch.empty(T, H, 576, dtype=torch.bfloat16, **dev)
    heads = torch.empty(T, H, 128, dtype=torch.bfloat16, **dev)
    u = torch.empty(T, d_model, dtype=torch.bfloat16, **dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, **dev)
    E = torch.cuda.Event

    def timed(call):
        for _ in range(3):
            call()
        ts = []
        for _ in range(iters):
            flush.fill_(1)
            a, b = E(enable_timing=True), E(enable_timing=True)
            a.record()
            call()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return float(np.mean([x.elapsed_time(y) for x, y in ts])) * 1e3

    out = {"workload": f"V2-shaped decode step: T={T}, H={H}, d_q={d_q}, d_model={d_model}",
           "absorb_two_step_us": timed(lambda: M.mla_absorb_q(dims, q_c, q_r, q_pos, w_uk, q_abs)),
           "absorb_folded_us": timed(lambda: M.mla_absorb_q_folded(dims, c_q, q_r, q_pos, w_qk, q_abs)),
           "out_two_step_us": timed(lambda: M.mla_up_v(dims, lat, w_uv, heads, w_o=w_o, out_model=u)),
           "out_folded_us": timed(lambda: M.mla_up_out_folded(dims, lat, w_ov, u)),
           "fold_weights_us": timed(lambda: M.mla_fold_weights(dims, w_uq, w_uk, w_qk, w_o, w_uv, w_ov)),
           "weight_bytes": {"U^K": H * 128 * 512 * 2, "W^UQ": H * 128 * d_q * 2, "W^QK": H * 512 * d_q * 2,
                            "U^V": H * 128 * 512 * 2, "W^O": d_model * H * 128 * 2, "W^OV": d_model * H * 512 * 2},
           "l2": "flushed before each call"}
    del flush, w_qk, w_ov, w_o
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------- CPU oracle (baseline)
def cpu_baseline(cfg: W.MLAConfig, budget_s: float = 10.0):
    """The fp64 expanded-form oracle, as it stands, on a bounded sample of the
    workload: (row 0, heads 0..k-1) at full context, k grown until the run
    takes about `budget_s`; tokens/s = 1 / (time per query row of H heads)."""
    import oracle
    d = W.make_decode_inputs(cfg.with_(B=1), with_cache_pages=True)
    f = oracle.bf16_to_f64
    args = (d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]), f(d["q_rope"]),
            f(d["w_uk"]), f(d["w_uv"]))
    k = max(1, min(cfg.H, oracle.num_threads()))
    while True:
        t = time.perf_counter()
        oracle.decode_expanded(*args, q_pos=d["q_pos"], rows=np.zeros(k, np.int32),
                               heads=np.arange(k, dtype=np.int32))
        el = time.perf_counter() - t
        if el >= budget_s / 3 or k >= cfg.H:
            break
        k = min(cfg.H, k * 2)
    per_row = el * cfg.H / k
    return {"value": 1.0 / per_row, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"expanded-form fp64 oracle on {k} of {cfg.H} heads of one query row at full "
                      f"context L={int(d['seq_lens'][0])}: {el:.2f} s, scaled to one row of all heads"}


# seconds the whole reference run (warm-up and timed steps) is sized to take
REFERENCE_BUDGET_S = 60.0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = W.CONFIGS[args.config]
    import oracle
    oracle._lib()
    k = max(1, min(cfg.H, oracle.num_threads()))
    L_full = int(W.seq_lens_of(cfg.with_(B=1))[0])

    def sample_step(L):
        # the expanded-form oracle on k heads of one query row over a context of
        # L tokens (its cost is linear in L: K/V expansion, scores, softmax, sum)
        d = W.make_decode_inputs(cfg.with_(B=1, L=L, seq_lens=None), with_cache_pages=True)
        f = oracle.bf16_to_f64
        a = (d["cache"], d["block_table"], d["seq_lens"], cfg.s, f(d["q_nope"]), f(d["q_rope"]),
             f(d["w_uk"]), f(d["w_uv"]))
        return lambda: oracle.decode_expanded(*a, q_pos=d["q_pos"], rows=np.zeros(k, np.int32),
                                              heads=np.arange(k, dtype=np.int32))

    # each step is sized so that the whole --warmup W --steps K run takes about
    # REFERENCE_BUDGET_S seconds: time a short context once, then pick the
    # context of every step's sample (a multiple of 64 tokens, at most L_full)
    per_step = REFERENCE_BUDGET_S / max(1, args.steps + args.warmup)
    L_cal = min(L_full, 512)
    cal = sample_step(L_cal)
    cal()
    t0 = time.perf_counter()
    cal()
    t_cal = max(time.perf_counter() - t0, 1e-6)
    L_s = int(min(L_full, max(64, L_cal * per_step / t_cal))) // 64 * 64
    L_s = max(64, min(L_full, L_s))
    step = sample_step(L_s)
    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = (time.perf_counter() - t) / args.steps
    # rows of all H heads at the workload's full context per second
    v = (k / cfg.H) * (L_s / L_full) / el
    sample = (f"each step: expanded-form fp64 oracle on {k} of {cfg.H} heads of one query row over "
              f"{L_s} of the workload's {L_full} context tokens; tokens/s = rows of all heads at full "
              f"context per second (cost linear in context)")
    print(json.dumps({
        "impl": "reference", "metric": "MLA decode tokens/s, latent-cache GB/s & TFLOP/s (H=128,B=128,L=4K) vs roofline",
        "value": v, "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": cfg.describe, "B": cfg.B, "s": cfg.s, "H": cfg.H},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="v2", choices=sorted(W.CONFIGS))
    ap.add_argument("--simple", action="store_true", help="force the CUDA-core decode kernel")
    ap.add_argument("--batch", type=int, default=0, help="override the number of sequences (profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip timing the decode of every workload")
    ap.add_argument("--no-prefill", action="store_true", help="skip timing the expanded-form prefill")
    ap.add_argument("--prefill-only", action="store_true", help="time only the prefill workloads")
    ap.add_argument("--decode-only", default="", help="comma-separated workloads: time only their decode calls")
    ap.add_argument("--fp8", action="store_true", help="with --decode-only: the FP8-cache decode")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps on the stream, not as a graph")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.decode_only:
        import torch
        import head_latent_attention_10_b200 as M
        M.load_library()
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        key = "per_config_fp8" if args.fp8 else "per_config"
        print(json.dumps({key: per_config(M, args.decode_only.split(","), fp8=args.fp8)}), flush=True)
    elif args.prefill_only:
        import torch
        import head_latent_attention_10_b200 as M
        M.load_library()
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps({"prefill": prefill_bench(M), "folded_weights": fold_bench(M)}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
