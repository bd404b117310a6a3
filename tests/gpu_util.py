"""Test-side helpers: move seeded host inputs to the GPU and run the C ABI.

Nothing here computes any part of the ISD step; it only allocates buffers,
copies inputs and calls the library through its Python binding.
"""
from __future__ import annotations

import numpy as np
import torch

from speculative_verification_isd_b200 import inputs as I

# (label, counts) of every accept comparison in this session; printed by the
# terminal-summary hook in conftest.py so that near-threshold decisions and
# rounding-excused draws are reported, not only counted
PARITY_REPORT = []


def record_parity(label: str, rep: dict):
    PARITY_REPORT.append((label, dict(rep)))


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def i32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def f32_dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def row_stats_host(rs: torch.Tensor):
    r = rs.view(-1, 4).cpu()
    f = r.view(torch.float32).numpy()
    i = r.numpy()
    return f[:, 0].astype(np.float64), f[:, 1].astype(np.float64), i[:, 2].astype(np.int64)


class StepBuffers:
    """Device copies of one step's inputs plus output buffers for a config."""

    def __init__(self, isd, cfg: I.IsdConfig, inp: dict, mode: int = 0):
        self.isd = isd
        self.cfg = cfg
        self.inp = inp
        num_pages = inp["k_pool"].shape[0]
        self.dims = isd.make_dims(cfg.B, cfg.N, cfg.Hq, cfg.Hkv, cfg.D, cfg.V, cfg.page_size,
                                  num_pages, inp["page_table"].shape[1], cfg.lora_rank, mode)
        d = self.dims
        self.q = bf16_dev(inp["q"])
        self.k_new = bf16_dev(inp["k_new"])
        self.v_new = bf16_dev(inp["v_new"])
        self.k_pool = bf16_dev(inp["k_pool"])
        self.v_pool = bf16_dev(inp["v_pool"])
        self.page_table = i32_dev(inp["page_table"])
        self.kv_len = i32_dev(inp["kv_len"])
        self.n_clean = i32_dev(inp["n_clean"])
        self.clean_tok = i32_dev(inp["clean_tok"])
        self.W = bf16_dev(inp["W"])
        self.uniforms = f32_dev(inp["uniforms"])
        self.lora_A = bf16_dev(inp["lora_A"]) if cfg.lora_rank else None
        self.lora_B = bf16_dev(inp["lora_B"]) if cfg.lora_rank else None
        self.ws = isd.alloc_workspace(d)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        M, V, B, N = d.M, d.V, d.B, d.N
        self.hidden = torch.empty(M, d.H, dtype=torch.bfloat16, device="cuda")
        self.logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
        self.row_stats = torch.empty(M, 4, dtype=torch.int32, device="cuda")
        self.prev_logits = torch.empty(M, V, dtype=torch.float32, device="cuda")
        self.prev_row_stats = torch.empty(M, 4, dtype=torch.int32, device="cuda")
        self.accept_len = torch.empty(B, dtype=torch.int32, device="cuda")
        self.out_tok = torch.empty(B, N, dtype=torch.int32, device="cuda")
        self.next_n_clean = torch.empty(B, dtype=torch.int32, device="cuda")
        self.next_clean_tok = torch.empty(B, N, dtype=torch.int32, device="cuda")
        self.next_kv_len = torch.empty(B, dtype=torch.int32, device="cuda")
        self.ratio = torch.empty(B, max(N - 1, 1), dtype=torch.float32, device="cuda")

    def set_prev_logits(self, prev: np.ndarray):
        self.prev_logits.copy_(torch.from_numpy(prev.reshape(self.dims.M, -1)))
        self.isd.row_stats(self.dims, self.prev_logits, self.dims.M, self.prev_row_stats, self.ws)

    def attention(self):
        self.isd.attention(self.dims, self.q, self.k_new, self.v_new, self.k_pool, self.v_pool,
                           self.page_table, self.kv_len, self.n_clean, self.hidden, self.ws,
                           self.err)

    def lm_head(self, hidden=None):
        self.isd.lm_head(self.dims, self.hidden if hidden is None else hidden, self.W, self.logits,
                         self.row_stats, self.ws, self.lora_A, self.lora_B, self.err)

    def accept(self):
        self.isd.accept(self.dims, self.logits, self.row_stats, self.prev_logits,
                        self.prev_row_stats, self.n_clean, self.clean_tok, self.kv_len,
                        self.uniforms, self.accept_len, self.out_tok, self.next_n_clean,
                        self.next_clean_tok, self.next_kv_len, self.ws, self.ratio, self.err)

    def step(self):
        self.isd.step(self.dims, self.q, self.k_new, self.v_new, self.k_pool, self.v_pool,
                      self.page_table, self.kv_len, self.n_clean, self.clean_tok, self.W,
                      self.prev_logits, self.prev_row_stats, self.uniforms, self.logits,
                      self.row_stats, self.accept_len, self.out_tok, self.next_n_clean,
                      self.next_clean_tok, self.next_kv_len, self.ws, hidden=self.hidden,
                      ratio=self.ratio, lora_A=self.lora_A, lora_B=self.lora_B, err_flag=self.err)

    def outputs(self):
        torch.cuda.synchronize()
        return dict(accept_len=self.accept_len.cpu().numpy(), out_tok=self.out_tok.cpu().numpy(),
                    next_n_clean=self.next_n_clean.cpu().numpy(),
                    next_clean_tok=self.next_clean_tok.cpu().numpy(),
                    next_kv_len=self.next_kv_len.cpu().numpy(), ratio=self.ratio.cpu().numpy())
