"""Per-(layer, block) state for fb_step: the caller-owned cache buffers, the
workspace and the policy, allocated once with torch and reused every step.

Only allocation and marshalling live here; each step is one fb_step call.
"""

from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (FB_LOSA, FB_PER_HEAD, FB_SPARSE_RESIDUAL, FB_THRESHOLD, KV, fb_cache,
               fb_page_summary, fb_policy, fb_step, fb_workspace_size)

_MODES = {"threshold": FB_THRESHOLD, "per_head": FB_PER_HEAD, "losa": FB_LOSA,
          "sparse_residual": FB_SPARSE_RESIDUAL}


class BlockAttention:
    """Attention of one block across its denoise steps (FlashBlock / LoSA).

    mode: "threshold" (tau), "per_head" (gamma), "losa" (n_active, topk_pages) or
    "sparse_residual" (tau, topk_pages: pages selected per kv head).
    """

    def __init__(self, kv: KV, block: int, n_heads_q: int, mode: str, tau: int = 0,
                 gamma: float = 2.0, n_active: int = 0, topk_pages: int = 0,
                 scale: float = 1.0, device=None):
        self.kv, self.B, self.Hq, self.mode = kv, block, n_heads_q, mode
        dev = device or kv.k.device
        batch, d = kv.batch, kv.c.head_dim
        self.policy = fb_policy(_MODES[mode], tau, gamma, n_active, topk_pages, scale)
        f32 = dict(dtype=torch.float32, device=dev)
        self.a_out = torch.zeros(batch, block, n_heads_q, d, **f32)
        self.l_out = torch.zeros(batch, block, n_heads_q, **f32)
        self.t = {"a_out": self.a_out, "l_out": self.l_out}
        if mode == "per_head":
            self.t["a_out_prev"] = torch.zeros_like(self.a_out)
            self.t["head_mask"] = torch.ones(batch, n_heads_q, dtype=torch.uint8, device=dev)
            self.t["head_cos"] = torch.full((batch, n_heads_q), float("nan"), dtype=torch.float64,
                                            device=dev)
        self.page_min = self.page_max = None
        hkv = kv.c.n_heads_kv
        npg = kv.n_pages
        if mode in ("losa", "sparse_residual"):
            self.t["union_bitmap"] = torch.zeros(batch, hkv, -(-npg // 32), dtype=torch.int32,
                                                 device=dev)
            self.t["union_list"] = torch.zeros(batch, hkv, npg, dtype=torch.int32, device=dev)
            self.t["union_count"] = torch.zeros(batch, hkv, dtype=torch.int32, device=dev)
            self.page_min = torch.empty(batch, npg, hkv, d, dtype=kv.k.dtype, device=dev)
            self.page_max = torch.empty_like(self.page_min)
            fb_page_summary(kv, self.page_min, self.page_max)
        if mode == "losa":
            na = min(n_active, block)
            self.t["q_prev"] = torch.zeros(batch, block, n_heads_q, d, dtype=kv.k.dtype, device=dev)
            self.t["active_rows"] = torch.zeros(batch, max(na, 1), dtype=torch.int32, device=dev)
            self.t["row_scores"] = torch.zeros(batch, block, **f32)
        if mode == "sparse_residual":
            self.t["a_res"] = torch.zeros_like(self.a_out)
            self.t["l_res"] = torch.zeros_like(self.l_out)
            self.t["comp_list"] = torch.zeros(batch, hkv, npg, dtype=torch.int32, device=dev)
            self.t["comp_count"] = torch.zeros(batch, hkv, dtype=torch.int32, device=dev)
        if mode == "losa":
            ws = fb_workspace_size(kv, block, n_heads_q, n_active, topk_pages)
        elif mode == "sparse_residual":  # every row scored, every page a possible list entry
            ws = fb_workspace_size(kv, block, n_heads_q, block, npg)
        else:
            ws = fb_workspace_size(kv, block, n_heads_q)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        p = {k: v.data_ptr() for k, v in self.t.items()}
        self.cache = fb_cache(p.get("a_out"), p.get("l_out"), p.get("a_out_prev"), p.get("head_mask"),
                              p.get("head_cos"), p.get("q_prev"), p.get("active_rows"),
                              p.get("row_scores"), p.get("union_bitmap"), p.get("union_list"),
                              p.get("union_count"), 0, 0, p.get("a_res"), p.get("l_res"),
                              p.get("comp_list"), p.get("comp_count"))

    def reset(self) -> None:
        """Start a new block (the next step computes the prefix partial)."""
        self.cache.step = 0

    def step(self, q, k_in, v_in, a_full, l_full=None,
             m_updated: Optional[Sequence[int]] = None, stream=None) -> None:
        fb_step(self.policy, self.cache, q, k_in, v_in, self.kv, a_full, l_full, m_updated,
                self.page_min, self.page_max, self.workspace, stream)

    @property
    def step_index(self) -> int:
        return self.cache.step

    @property
    def recomputed(self) -> int:
        return self.cache.recomputed
