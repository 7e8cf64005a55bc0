"""Helpers shared by the GPU tests: upload a seeded workload, fill the paged
cache through the library's own cache writer, and compare with the oracle."""
from __future__ import annotations

import numpy as np

import mla_workloads as W


def torch_bits(a, dev="cuda"):
    """uint16 bf16 bits (numpy) -> torch bf16 tensor on the device."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def host_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def i32(a, dev="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)


class GpuWorkload:
    """A workload resident on the GPU, with its cache written by mla_append_latent."""

    def __init__(self, cfg: W.MLAConfig, d=None, chunk=1 << 20):
        import torch
        import head_latent_attention_10_b200 as M
        self.cfg = cfg
        self.d = d if d is not None else W.make_decode_inputs(cfg)
        d = self.d
        self.dims = M.dims(cfg.H)
        self.block_table = i32(d["block_table"])
        self.seq_lens = i32(d["seq_lens"])
        self.cache = torch.full((d["num_blocks"], cfg.block_size, cfg.d_c + cfg.d_r), float("nan"),
                                dtype=torch.bfloat16, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        N = d["tok_seq"].size
        for a in range(0, N, chunk):
            b = min(N, a + chunk)
            M.mla_append_latent(self.dims, torch_bits(d["c_kv"][a:b]), torch_bits(d["k_rope"][a:b]),
                                i32(d["tok_seq"][a:b]), i32(d["tok_pos"][a:b]), self.block_table,
                                self.cache, err_word=self.err)
        self.q_nope = torch_bits(d["q_nope"])
        self.q_rope = torch_bits(d["q_rope"])
        self.q_pos = i32(d["q_pos"])
        self.w_uk = torch_bits(d["w_uk"])
        self.w_uv = torch_bits(d["w_uv"])
        self.ws = torch.empty(M.mla_decode_workspace_size(self.dims, cfg.B, cfg.s,
                                                          d["block_table"].shape[1] * cfg.block_size),
                              dtype=torch.uint8, device="cuda")

    def absorb(self):
        import torch
        import head_latent_attention_10_b200 as M
        cfg = self.cfg
        q_abs = torch.empty(cfg.T, cfg.H, cfg.d_c + cfg.d_r, dtype=torch.bfloat16, device="cuda")
        M.mla_absorb_q(self.dims, self.q_nope, self.q_rope, self.q_pos, self.w_uk, q_abs)
        return q_abs

    def decode(self, q_abs, flags=0):
        import torch
        import head_latent_attention_10_b200 as M
        cfg = self.cfg
        lat = torch.empty(cfg.T, cfg.H, cfg.d_c, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device="cuda")
        M.mla_decode(self.dims, q_abs, self.cache, self.block_table, self.seq_lens, cfg.s, lat, lse,
                     self.ws, flags=flags)
        return lat, lse

    def up_v(self, lat):
        import torch
        import head_latent_attention_10_b200 as M
        cfg = self.cfg
        o = torch.empty(cfg.T, cfg.H, cfg.d_h, dtype=torch.bfloat16, device="cuda")
        M.mla_up_v(self.dims, lat, self.w_uv, o)
        return o


def rel_l2(g, r) -> float:
    g = np.asarray(g, np.float64); r = np.asarray(r, np.float64)
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))


def assert_parity(g, r, max_abs=2e-2, rel=1e-2, what=""):
    """The parity bar: max-abs <= 2e-2 and relative L2 <= 1e-2."""
    g = np.asarray(g, np.float64); r = np.asarray(r, np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    ma = float(np.max(np.abs(g - r))) if g.size else 0.0
    rl = rel_l2(g, r)
    assert ma <= max_abs and rl <= rel, f"{what}: max-abs {ma:.3e}, rel-L2 {rl:.3e}"
    return ma, rl
