"""Per-(layer, block) state for fb_step: the caller-owned cache buffers, the
workspace and the policy, allocated once with torch and reused every step.

Only allocation and marshalling live here; each step is one fb_step call.
"""

from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (FB_LOSA, FB_PER_HEAD, FB_SPARSE_RESIDUAL, FB_THRESHOLD, KV, fb_cache,
               fb_page_summary, fb_policy, fb_step, fb_step_varlen, fb_workspace_size)

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


class VarlenBlockAttention:
    """Threshold (tau) reuse over packed block rows: the blocks (branches) of
    all sequences, of different sizes, in one launch per step.

    cu_rows: int32 [batch + 1] row offsets (host sequence or tensor); sequence
    b owns packed rows cu_rows[b] .. cu_rows[b+1]-1. Cache buffers are packed
    [total, Hq, d] like q; the workspace is sized for the longest block.
    """

    def __init__(self, kv: KV, cu_rows, n_heads_q: int, tau: int = 0, scale: float = 1.0,
                 device=None):
        dev = device or kv.k.device
        cu = [int(x) for x in (cu_rows.tolist() if hasattr(cu_rows, "tolist") else cu_rows)]
        if len(cu) != kv.batch + 1:
            raise ValueError("cu_rows needs batch + 1 offsets")
        self.kv, self.Hq = kv, n_heads_q
        self.total = cu[-1]
        self.max_rows = max(1, max(b - a for a, b in zip(cu[:-1], cu[1:])))
        self.cu = torch.tensor(cu, dtype=torch.int32, device=dev)
        d = kv.c.head_dim
        self.policy = fb_policy(FB_THRESHOLD, tau, 2.0, 0, 0, scale)
        self.a_out = torch.zeros(max(self.total, 1), n_heads_q, d, dtype=torch.float32, device=dev)
        self.l_out = torch.zeros(max(self.total, 1), n_heads_q, dtype=torch.float32, device=dev)
        self.workspace = torch.empty(fb_workspace_size(kv, self.max_rows, n_heads_q),
                                     dtype=torch.uint8, device=dev)
        self.cache = fb_cache(self.a_out.data_ptr(), self.l_out.data_ptr(), None, None, None, None,
                              None, None, None, None, None, 0, 0, None, None, None, None)

    def reset(self) -> None:
        self.cache.step = 0

    def step(self, q, k_in, v_in, a_full, l_full=None,
             m_updated: Optional[Sequence[int]] = None, stream=None) -> None:
        fb_step_varlen(self.policy, self.cache, q, k_in, v_in, self.cu, self.max_rows, self.kv,
                       a_full, l_full, m_updated, self.workspace, stream)

    @property
    def recomputed(self) -> int:
        return self.cache.recomputed


class HostBlockPipeline:
    """A block's denoise steps fed from pinned host memory and returned to it.

    Each step's q, k_in, v_in arrive as one packed host buffer (one copy in) and
    its A_full, L_full leave as one packed buffer (one copy out). Copies run on
    their own streams with `depth` device buffers in rotation, so the input copy
    of step s+1 and the output copy of step s-1 overlap the attention of step
    s; a step then costs about the larger of its copies and its attention. All
    work is enqueued on the current stream and two copy streams that fork from
    and join back into it, so a whole block can be captured in one CUDA graph.
    Attention itself is one fb_step call per step, as in BlockAttention.step.
    """

    def __init__(self, blk: BlockAttention, dtype, depth: int = 3):
        self.blk = blk
        self.depth = depth
        kv = blk.kv
        dev = kv.k.device
        batch, B, Hq, d = kv.batch, blk.B, blk.Hq, kv.c.head_dim
        hkv = kv.c.n_heads_kv
        self.q_shape = (batch, B, Hq, d)
        self.kv_shape = (batch, B, hkv, d)
        self.dtype = dtype
        esz = torch.empty((), dtype=dtype).element_size()
        self.nq = batch * B * Hq * d
        self.nkv = batch * B * hkv * d
        self.in_bytes = (self.nq + 2 * self.nkv) * esz
        self.nA = batch * B * Hq * d
        self.nL = batch * B * Hq
        self.dev_in = [torch.empty(self.in_bytes, dtype=torch.uint8, device=dev) for _ in range(depth)]
        self.dev_out = [torch.empty(self.nA + self.nL, dtype=torch.float32, device=dev)
                        for _ in range(depth)]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.in_done = [torch.cuda.Event() for _ in range(depth)]
        self.comp_done = [torch.cuda.Event() for _ in range(depth)]
        self.out_done = [torch.cuda.Event() for _ in range(depth)]

    @property
    def out_floats(self) -> int:
        return self.nA + self.nL

    def pack_inputs(self, q, k_in, v_in) -> torch.Tensor:
        """One pinned host buffer holding q, k_in, v_in (in that order)."""
        parts = [t.contiguous().view(torch.uint8).reshape(-1) for t in (q, k_in, v_in)]
        buf = torch.empty(self.in_bytes, dtype=torch.uint8).pin_memory()
        torch.cat(parts, out=buf)
        return buf

    def new_output(self) -> torch.Tensor:
        """A pinned host buffer for one step's A_full then L_full (float32)."""
        return torch.empty(self.out_floats, dtype=torch.float32).pin_memory()

    def unpack_output(self, out: torch.Tensor):
        return (out[: self.nA].view(*self.q_shape), out[self.nA:].view(*self.q_shape[:3]))

    def _views(self, slot):
        raw = self.dev_in[slot]
        esz = torch.empty((), dtype=self.dtype).element_size()
        q = raw[: self.nq * esz].view(self.dtype).view(*self.q_shape)
        k = raw[self.nq * esz: (self.nq + self.nkv) * esz].view(self.dtype).view(*self.kv_shape)
        v = raw[(self.nq + self.nkv) * esz:].view(self.dtype).view(*self.kv_shape)
        out = self.dev_out[slot]
        return q, k, v, out[: self.nA].view(*self.q_shape), out[self.nA:].view(*self.q_shape[:3])

    def enqueue_block(self, host_in: Sequence[torch.Tensor], host_out: Sequence[torch.Tensor],
                      m_updated: Optional[Sequence[Sequence[int]]] = None) -> None:
        """Enqueues every step of a block (step 0 starts the block)."""
        main = torch.cuda.current_stream()
        self.s_in.wait_stream(main)   # fork: the copy streams follow all prior work
        self.s_out.wait_stream(main)
        for s in range(len(host_in)):
            slot = s % self.depth
            with torch.cuda.stream(self.s_in):
                if s >= self.depth:  # the step that last read this input buffer is done
                    self.s_in.wait_event(self.comp_done[slot])
                self.dev_in[slot].copy_(host_in[s], non_blocking=True)
                self.in_done[slot].record(self.s_in)
            main.wait_event(self.in_done[slot])
            if s >= self.depth:  # the copy out of this output buffer is done
                main.wait_event(self.out_done[slot])
            q, k, v, A, L = self._views(slot)
            if s == 0:
                self.blk.reset()
            self.blk.step(q, k, v, A, L, m_updated=None if m_updated is None else m_updated[s])
            self.comp_done[slot].record(main)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.comp_done[slot])
                host_out[s].copy_(self.dev_out[slot], non_blocking=True)
                self.out_done[slot].record(self.s_out)
        main.wait_stream(self.s_in)  # join
        main.wait_stream(self.s_out)
