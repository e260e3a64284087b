"""One HGA attention step (one layer, one active segment) over the C ABI.

Order of calls (every one a kernel launch in libhga.so):
  hga_block_summaries  -> resident per-block key summaries
  hga_select_topk      -> per query block, the top-K history blocks
  hga_attn_fwd         -> O, LSE over [selected history] U [causal segment]
  hga_attn_bwd         -> dQ, dK_seg, dV_seg (history detached)
This module only owns the output and scratch buffers (torch device memory).
"""
from __future__ import annotations

import torch

from ._binding import (Dims, hga_attn_bwd, hga_attn_bwd_workspace_size, hga_attn_fwd, hga_block_summaries,
                       hga_select_topk)


class AttentionStep:
    def __init__(self, dims: Dims, device: str | torch.device = "cuda"):
        self.dims = dims
        D = dims
        dt = D.torch_dtype
        self.summ = torch.empty((D.B, D.n_hist_blocks, D.Hkv, D.d), dtype=torch.float32, device=device)
        self.idx = torch.empty((D.B, D.Hkv, D.nqb, D.topk), dtype=torch.int32, device=device)
        self.o = torch.empty((D.B, D.S, D.Hq, D.d), dtype=dt, device=device)
        self.lse = torch.empty((D.B, D.Hq, D.S), dtype=torch.float32, device=device)
        self.dq = torch.empty((D.B, D.S, D.Hq, D.d), dtype=torch.float32, device=device)
        self.dk = torch.empty((D.B, D.S, D.Hkv, D.d), dtype=torch.float32, device=device)
        self.dv = torch.empty((D.B, D.S, D.Hkv, D.d), dtype=torch.float32, device=device)
        ws = hga_attn_bwd_workspace_size(D)
        self.ws = torch.empty((max(ws, 256),), dtype=torch.uint8, device=device)

    def select(self, q, k_hist, stream=None):
        D = self.dims
        if D.n_hist_blocks > 0:
            hga_block_summaries(D, k_hist, 0, D.n_hist_blocks, self.summ, stream)
        hga_select_topk(D, q, self.summ, self.idx, None, stream)
        return self.idx

    def forward(self, q, k_seg, v_seg, k_hist, v_hist, idx=None, n_kv_blocks=None, stream=None):
        D = self.dims
        nkv = D.n_hist_blocks if n_kv_blocks is None else n_kv_blocks
        hga_attn_fwd(D, q, k_seg, v_seg, k_hist, v_hist, nkv, self.idx if idx is None else idx, self.o, self.lse,
                     stream)
        return self.o, self.lse

    def backward(self, q, k_seg, v_seg, k_hist, v_hist, d_o, idx=None, n_kv_blocks=None, stream=None):
        D = self.dims
        nkv = D.n_hist_blocks if n_kv_blocks is None else n_kv_blocks
        hga_attn_bwd(D, q, k_seg, v_seg, k_hist, v_hist, nkv, self.idx if idx is None else idx, self.o, self.lse,
                     d_o, self.dq, self.dk, self.dv, self.ws, stream)
        return self.dq, self.dk, self.dv

    def run(self, q, k_seg, v_seg, k_hist, v_hist, d_o=None, stream=None):
        """summaries -> select -> forward (-> backward when d_o is given)."""
        self.select(q, k_hist, stream)
        self.forward(q, k_seg, v_seg, k_hist, v_hist, stream=stream)
        if d_o is not None:
            self.backward(q, k_seg, v_seg, k_hist, v_hist, d_o, stream=stream)
